"""Host-only checks of the C ABI: the library loads, exports every function
include/kvzip.h declares, and rejects bad arguments before touching the GPU."""
import ctypes
import math
import os
import re

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kvzip.h")


@pytest.fixture(scope="module")
def kz():
    from attention_score_reduction_b200 import build
    build.build()
    from attention_score_reduction_b200 import kvzip
    return kvzip


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(kvzip_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("kvzip_score_chunk", "kvzip_select", "kvzip_compact",
                     "kvzip_score_workspace_size", "kvzip_select_workspace_size",
                     "kvzip_compact_workspace_size", "kvzip_keep_count", "kvzip_status_string",
                     "kvzip_workspace_status", "kvzip_set_wait_timeout_ns"):
        assert required in names


def test_library_exports_every_declared_symbol(kz):
    lib = ctypes.CDLL(kz.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(kz):
    for s in range(6):
        assert kz.status_string(s)
    assert kz.status_string(99) == "unknown status"


@pytest.mark.parametrize("r,N", [(0.3, 2048), (0.3, 4194304), (0.3, 33554432), (0.5, 33554432),
                                 (0.25, 47185920), (0.3, 66846720), (0.0, 10), (1.0, 10),
                                 (0.1, 10), (0.7, 123457)])
def test_keep_count_matches_oracle(kz, r, N):
    assert kz.keep_count(r, N) == oracle.keep_count(r, N)


def test_keep_count_rejects(kz):
    lib = kz.library()
    assert lib.kvzip_keep_count(-0.1, 10) == -1
    assert lib.kvzip_keep_count(1.5, 10) == -1
    assert lib.kvzip_keep_count(float("nan"), 10) == -1
    assert lib.kvzip_keep_count(0.5, -1) == -1


def test_workspace_sizes(kz):
    assert kz.score_workspace_size(256, 4, 2064) == 256 + 256 * (math.ceil(8256 / 768) * 768) * 4
    assert kz.select_workspace_size(33554432, 256) > 0
    assert kz.compact_workspace_size(256, 131072) > 0


FAKE = 1 << 20  # a well-aligned non-null address; never dereferenced on rejected calls


def _score(kz, **over):
    a = dict(dt=0, q=FAKE, k=FAKE, ks=FAKE, s=FAKE, B=2, G=4, n_in=100, n_c=1000, d=128,
             scale=0.0, ws=FAKE, ws_bytes=1 << 30, stream=None)
    a.update(over)
    return kz.library().kvzip_score_chunk(a["dt"], a["q"], a["k"], a["ks"], a["s"], a["B"], a["G"],
                                          a["n_in"], a["n_c"], a["d"], a["scale"], a["ws"],
                                          a["ws_bytes"], a["stream"])


def test_score_rejects_bad_arguments(kz):
    assert _score(kz, dt=7) == kz.ERR_INVALID_ARG
    assert _score(kz, q=None) == kz.ERR_INVALID_ARG
    assert _score(kz, k=None) == kz.ERR_INVALID_ARG
    assert _score(kz, ks=None) == kz.ERR_INVALID_ARG
    assert _score(kz, s=None) == kz.ERR_INVALID_ARG
    assert _score(kz, ws=None) == kz.ERR_INVALID_ARG
    assert _score(kz, d=64) == kz.ERR_UNSUPPORTED
    assert _score(kz, d=0) == kz.ERR_INVALID_ARG
    assert _score(kz, B=-1) == kz.ERR_INVALID_ARG
    assert _score(kz, q=FAKE + 8) == kz.ERR_INVALID_ARG        # not 16-byte aligned
    assert _score(kz, s=FAKE + 2) == kz.ERR_INVALID_ARG        # not 4-byte aligned
    assert _score(kz, ws=FAKE + 16) == kz.ERR_INVALID_ARG      # not 256-byte aligned
    assert _score(kz, ws_bytes=100) == kz.ERR_INVALID_ARG
    assert _score(kz, B=70000) == kz.ERR_UNSUPPORTED


def test_score_empty_is_noop(kz):
    for over in (dict(B=0), dict(G=0), dict(n_in=0), dict(n_c=0)):
        assert _score(kz, q=None, k=None, ks=None, s=None, ws=None, **over) == kz.OK


def _select(kz, **over):
    a = dict(s=FAKE, N=1000, k=300, H=10, keep=FAKE, off=FAKE, thr=None, ws=FAKE,
             ws_bytes=1 << 30)
    a.update(over)
    return kz.library().kvzip_select(a["s"], a["N"], a["k"], a["H"], a["keep"], a["off"], a["thr"],
                                     a["ws"], a["ws_bytes"], None)


def test_select_rejects_bad_arguments(kz):
    assert _select(kz, k=1001) == kz.ERR_INVALID_ARG
    assert _select(kz, k=-1) == kz.ERR_INVALID_ARG
    assert _select(kz, H=0) == kz.ERR_INVALID_ARG
    assert _select(kz, H=7) == kz.ERR_INVALID_ARG              # 1000 % 7 != 0
    assert _select(kz, s=None) == kz.ERR_INVALID_ARG
    assert _select(kz, keep=None) == kz.ERR_INVALID_ARG
    assert _select(kz, off=None) == kz.ERR_INVALID_ARG
    assert _select(kz, s=FAKE + 4) == kz.ERR_INVALID_ARG       # scores need 16-byte alignment
    assert _select(kz, off=FAKE + 4) == kz.ERR_INVALID_ARG
    assert _select(kz, ws_bytes=10) == kz.ERR_INVALID_ARG
    assert _select(kz, N=1 << 31, k=0, H=1) == kz.ERR_INVALID_ARG


def test_histogram_entry_points_reject_a_missing_histogram(kz):
    L = kz.library()
    assert L.kvzip_select_hist(FAKE, 1000, 300, 10, None, FAKE, FAKE, None, FAKE, 1 << 30,
                               None) == kz.ERR_INVALID_ARG
    assert L.kvzip_select_hist(FAKE, 1000, 300, 10, FAKE + 2, FAKE, FAKE, None, FAKE, 1 << 30,
                               None) == kz.ERR_INVALID_ARG        # 4-byte aligned counts
    assert L.kvzip_score_colmax_hist(kz.BF16, FAKE, FAKE, FAKE, FAKE, 2, 4, 64, 100, 128, 0.0,
                                     None, FAKE, 1 << 30, None) == kz.ERR_INVALID_ARG


def _compact(kz, **over):
    a = dict(k=FAKE, v=FAKE, keep=FAKE, off=FAKE, H=4, n_c=100, d=128, ko=FAKE, vo=FAKE, pos=None,
             ws=FAKE, ws_bytes=1 << 30)
    a.update(over)
    return kz.library().kvzip_compact(a["k"], a["v"], a["keep"], a["off"], a["H"], a["n_c"], a["d"],
                                      a["ko"], a["vo"], a["pos"], a["ws"], a["ws_bytes"], None)


def test_compact_rejects_bad_arguments(kz):
    assert _compact(kz, d=64) == kz.ERR_UNSUPPORTED
    assert _compact(kz, H=0) == kz.ERR_INVALID_ARG
    assert _compact(kz, k=None) == kz.ERR_INVALID_ARG
    assert _compact(kz, vo=None) == kz.ERR_INVALID_ARG
    assert _compact(kz, k=FAKE + 8) == kz.ERR_INVALID_ARG
    assert _compact(kz, pos=FAKE + 2) == kz.ERR_INVALID_ARG
    assert _compact(kz, ws_bytes=1) == kz.ERR_INVALID_ARG
    assert _compact(kz, n_c=0, k=None) == kz.OK


def test_head_scores_rejects_bad_arguments(kz):
    lib = kz.library()
    assert lib.kvzip_head_scores(None, 4, 10, FAKE, None) == kz.ERR_INVALID_ARG
    assert lib.kvzip_head_scores(FAKE, 0, 10, FAKE, None) == kz.ERR_INVALID_ARG
    assert lib.kvzip_head_scores(FAKE, 4, 0, FAKE, None) == kz.ERR_INVALID_ARG
    assert lib.kvzip_head_scores(FAKE + 2, 4, 10, FAKE, None) == kz.ERR_INVALID_ARG


def test_decode_rejects_bad_arguments(kz):
    lib = kz.library()
    f = lib.kvzip_decode_attention
    ok = dict(q=FAKE, k=FAKE, v=FAKE, rows=1000, off=FAKE, H=8, G=4, d=128, scale=0.0, out=FAKE,
              ws=FAKE, wsb=1 << 30)

    def call(**over):
        a = dict(ok)
        a.update(over)
        return f(a["q"], a["k"], a["v"], a["rows"], a["off"], a["H"], a["G"], a["d"], a["scale"],
                 a["out"], a["ws"], a["wsb"], None)
    assert call(G=3) == kz.ERR_UNSUPPORTED
    assert call(d=64) == kz.ERR_UNSUPPORTED
    assert call(H=0) == kz.ERR_INVALID_ARG
    assert call(q=None) == kz.ERR_INVALID_ARG
    assert call(k=None) == kz.ERR_INVALID_ARG           # k without v
    assert call(k=None, v=None) == kz.ERR_INVALID_ARG   # rows without buffers
    assert call(rows=-1) == kz.ERR_INVALID_ARG
    assert call(rows=1 << 31) == kz.ERR_INVALID_ARG
    assert call(q=FAKE + 8) == kz.ERR_INVALID_ARG
    assert call(wsb=16) == kz.ERR_INVALID_ARG
    assert kz.decode_workspace_size(8, 4, 128) > 0


def test_score_context_rejects_bad_arguments(kz):
    """kvzip_score_context validates its host arrays and the workspace before
    enqueueing anything (no GPU needed for any of these)."""
    lib = kz.library()
    vp = ctypes.c_void_p
    q = (vp * 2)(FAKE, FAKE)
    ks = (vp * 2)(FAKE, FAKE)
    n_in = (ctypes.c_int * 2)(16, 16)
    ws_ok = lib.kvzip_score_context_workspace_size(2, 4, 16)
    assert ws_ok == lib.kvzip_score_workspace_size(2, 4, 16)

    def call(n, qa=q, ka=ks, na=n_in, ws=ws_ok):
        return lib.kvzip_score_context(kz.BF16, n, qa, ka, na, FAKE, FAKE, 2, 4, 64, 128, 0.0,
                                       FAKE, ws, None)
    assert call(-1) == kz.ERR_INVALID_ARG
    assert call(0) == kz.OK                                  # nothing to score
    assert call(2, qa=None) == kz.ERR_INVALID_ARG
    assert call(2, ka=None) == kz.ERR_INVALID_ARG
    assert call(2, na=None) == kz.ERR_INVALID_ARG
    assert call(2, qa=(vp * 2)(FAKE, None)) == kz.ERR_INVALID_ARG
    assert call(2, na=(ctypes.c_int * 2)(16, 0)) == kz.ERR_INVALID_ARG
    assert call(2, ws=ws_ok - 1) == kz.ERR_INVALID_ARG       # workspace too small
    # the largest chunk sets the workspace: 16 and 1000 rows need the 1000-row size
    big = (ctypes.c_int * 2)(16, 1000)
    assert call(2, na=big) == kz.ERR_INVALID_ARG


def test_score_lse_layout(kz):
    """The row normalisers sit after the 256-byte status header, one row stride
    per unit, the stride being the unit's G * n_in rows rounded up to the pad;
    the workspace size covers exactly that."""
    for G, n_in in [(4, 2064), (5, 2064), (2, 1040), (1, 1), (4, 129)]:
        off, stride = kz.lse_layout(G, n_in)
        assert off == 256
        assert stride >= G * n_in and stride % 128 == 0 and stride - G * n_in < 768
        B = 7
        assert kz.score_workspace_size(B, G, n_in) == off + B * stride * 4
    lib = kz.library()
    o, s = ctypes.c_size_t(0), ctypes.c_int64(0)
    assert lib.kvzip_score_lse_layout(0, 10, ctypes.byref(o), ctypes.byref(s)) == kz.ERR_INVALID_ARG
    assert lib.kvzip_score_lse_layout(4, 10, None, ctypes.byref(s)) == kz.ERR_INVALID_ARG
    assert lib.kvzip_score_lse_layout(1 << 20, 1 << 20, ctypes.byref(o),
                                      ctypes.byref(s)) == kz.ERR_UNSUPPORTED


def test_c_caller_builds_against_header_and_library(tmp_path):
    """The torch-free C caller (tests/c_abi_host_staging.c, run on a GPU by
    test_gpu_c_abi_host.py) compiles with -Wall -Werror against include/kvzip.h
    and links against libkvzip.so and the CUDA runtime."""
    import shutil
    if not (shutil.which("gcc") or shutil.which("cc")):
        pytest.skip("no C compiler")
    from tests.test_gpu_c_abi_host import _compile
    exe = str(tmp_path / "c_abi_host_staging")
    _compile(exe)
    assert os.path.exists(exe)
