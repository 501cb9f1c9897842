"""KVzip query-agnostic KV importance scoring, global top-r selection and
per-head KV compaction on NVIDIA B200 (sm_100a).

Submodules (imported on first use):
  kvzip     ctypes binding of libkvzip (the CUDA path; no CPU fallback)
  pipeline  end-to-end scoring -> selection -> compaction over a whole context
  synth     seeded synthetic workloads (inputs only; no method arithmetic)
  build     nvcc build of libkvzip.so
"""
import importlib

__all__ = ["kvzip", "pipeline", "synth", "build"]


def __getattr__(name):
    if name in __all__:
        return importlib.import_module(f".{name}", __name__)
    raise AttributeError(name)
