"""The C ABI from a C program, without torch: host buffers in, packed cache out.

tests/c_abi_host_staging.c is compiled with gcc against include/kvzip.h,
libkvzip.so and the CUDA runtime.  It stages a small multi-chunk context
from page-locked host memory with cudaMemcpyAsync on one stream, calls
kvzip_score_chunk per chunk, kvzip_select and kvzip_compact on device
pointers, checks both workspaces' status words and copies the results back.
The same calls made through the Python binding on torch buffers must give the
same scores, offsets and packed K/V/positions bit for bit: the same kernels
run on the same inputs.
"""
import os
import shutil
import subprocess

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = "/usr/local/cuda"


def _compile(exe):
    from attention_score_reduction_b200 import build
    lib = build.build()
    libdir = os.path.dirname(lib)
    cc = shutil.which("gcc") or shutil.which("cc")
    assert cc, "no C compiler"
    cmd = [cc, "-O2", "-std=c11", "-Wall", "-Werror", "-I" + os.path.join(ROOT, "include"),
           "-I" + os.path.join(CUDA, "include"), os.path.join(ROOT, "tests", "c_abi_host_staging.c"),
           "-L" + libdir, "-lkvzip", "-Wl,-rpath," + libdir,
           "-L" + os.path.join(CUDA, "lib64"), "-lcudart", "-Wl,-rpath," + os.path.join(CUDA, "lib64"),
           "-o", exe]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr


def test_c_program_host_staging_matches_binding(tmp_path):
    from attention_score_reduction_b200 import kvzip as kz
    from attention_score_reduction_b200 import synth
    wl = synth.Workload("c_host", L=2, H=4, G=4, d=128, n_c=3000, m=700, r=(0.3,),
                        hi_frac=0.01, sinks=4, cfg_id=93)
    r = 0.3
    k_ctx, v = synth.context_kv(wl)
    chunks = [synth.chunk_qk(wl, c) for c in range(wl.n_chunks)]
    assert len(chunks) > 1 and chunks[-1][0].shape[2] != chunks[0][0].shape[2]   # ragged last
    B, G, d, n_c = wl.units, wl.G, wl.d, wl.n_c

    def raw(t):
        return t.contiguous().view(torch.int16).numpy().tobytes()

    src, dst, exe = tmp_path / "in.bin", tmp_path / "out.bin", str(tmp_path / "c_abi_host_staging")
    with open(src, "wb") as f:
        f.write(np.array([B, G, d, n_c, len(chunks)], dtype="<i8").tobytes())
        f.write(np.array([r], dtype="<f8").tobytes())
        f.write(np.array([q.shape[2] for q, _ in chunks], dtype="<i8").tobytes())
        f.write(raw(k_ctx))
        f.write(raw(v))
        for q, ks in chunks:
            f.write(raw(q))
            f.write(raw(ks))
    _compile(exe)
    run = subprocess.run([exe, str(src), str(dst)], capture_output=True, text=True, timeout=300)
    assert run.returncode == 0, run.stdout + run.stderr

    buf = dst.read_bytes()
    N = B * n_c
    k = int(np.frombuffer(buf, "<i8", 1)[0])
    o = 8
    scores = np.frombuffer(buf, "<f4", N, o); o += 4 * N
    offsets = np.frombuffer(buf, "<i8", B + 1, o); o += 8 * (B + 1)
    k_out = np.frombuffer(buf, "<i2", k * d, o); o += 2 * k * d
    v_out = np.frombuffer(buf, "<i2", k * d, o); o += 2 * k * d
    pos = np.frombuffer(buf, "<i4", k, o); o += 4 * k
    assert o == len(buf)

    # the same calls through the binding, on device-resident torch buffers
    dev = torch.device("cuda", 0)
    kd, vd = k_ctx.to(dev), v.to(dev)
    S = torch.zeros(B, n_c, device=dev)
    ws = kz.new_score_workspace(B, G, max(q.shape[2] for q, _ in chunks))
    for q, ks in chunks:
        kz.score_chunk(q.to(dev), kd, ks.to(dev), S, ws)
    assert kz.workspace_status(ws) == kz.OK
    assert k == kz.keep_count(r, N)
    keep, off, _ = kz.select(S.view(-1), k, B)
    ko, vo, po = kz.compact(kd, vd, keep, off, k)
    torch.cuda.synchronize()
    assert np.array_equal(scores.view(np.uint32), S.cpu().numpy().reshape(-1).view(np.uint32))
    assert np.array_equal(offsets, off.cpu().numpy())
    assert int(offsets[-1]) == k
    assert np.array_equal(k_out, ko.cpu().view(torch.int16).numpy().reshape(-1))
    assert np.array_equal(v_out, vo.cpu().view(torch.int16).numpy().reshape(-1))
    assert np.array_equal(pos, po.cpu().numpy())
