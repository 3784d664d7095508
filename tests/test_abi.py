"""The C ABI: libcq builds, loads and exports every symbol that include/cq.h
declares, and rejects bad arguments on the host before touching the GPU
(no GPU needed for any of this)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_symbols(header="cq.h"):
    with open(os.path.join(ROOT, "include", header)) as f:
        text = f.read()
    return sorted(set(re.findall(r"^\s*(?:CQ_API\s+)?(?:int|size_t|const char\s*\*)\s*(cq_\w+)\s*\(", text,
                                 re.M)))


@pytest.fixture(scope="module")
def lib():
    from bit_non_uniform_b200 import build
    build.build()
    import bit_non_uniform_b200 as cq
    return cq.lib()


def test_header_declares_the_boundary():
    syms = _declared_symbols()
    for s in ["cq_pack", "cq_decode", "cq_gemm", "cq_gemm_workspace_size",
              "cq_moe_grouped_gemm", "cq_moe_workspace_size", "cq_get_device_error",
              "cq_version", "cq_status_string"]:
        assert s in syms


def test_library_exports_every_declared_symbol(lib):
    for s in _declared_symbols():
        assert hasattr(lib, s), s


def test_hooks_are_declared_and_exported(lib):
    hooks = _declared_symbols("cq_hooks.h")
    assert hooks == ["cq_test_gemm_bounded", "cq_test_gemm_path",
                     "cq_test_gemm_path_workspace_size", "cq_trace_gemm"]
    for s in hooks:
        assert hasattr(lib, s), s


def test_version_and_status_strings(lib):
    assert lib.cq_version() >= 100
    for st in range(6):
        assert lib.cq_status_string(st)


FAKE = ctypes.c_void_p(0x1000)          # 16-byte aligned, never dereferenced
FAKE_ODD = ctypes.c_void_p(0x1008)      # 8-byte aligned only


def test_pack_rejects_bad_arguments(lib):
    assert lib.cq_pack(None, 4, 128, 4, FAKE, None) == 1
    assert lib.cq_pack(FAKE, -1, 128, 4, FAKE, None) == 1
    assert lib.cq_pack(FAKE, 4, 128, 9, FAKE, None) == 1
    assert lib.cq_pack(FAKE, 4, 3, 3, FAKE, None) == 2          # K*B not byte aligned


def test_decode_rejects_bad_arguments(lib):
    ok = (FAKE, FAKE, FAKE, 8, 512, 3, 128, 0, 0, FAKE, None)
    bad = [
        ((FAKE, FAKE, FAKE, 8, 512, 9, 128, 0, 0, FAKE, None), 2),   # B = 9
        ((FAKE, FAKE, FAKE, 8, 512, 1, 128, 1, 0, FAKE, None), 2),   # midtread needs B >= 2
        ((FAKE, FAKE, FAKE, 8, 512, 3, 100, 0, 0, FAKE, None), 2),   # G % 128
        ((FAKE, FAKE, FAKE, 8, 384, 3, 256, 0, 0, FAKE, None), 2),   # K % G
        ((FAKE, FAKE, FAKE, 8, 512, 3, 128, 7, 0, FAKE, None), 1),   # grid mode
        ((FAKE, FAKE, FAKE, 8, 512, 3, 128, 0, 9, FAKE, None), 1),   # dtype
        ((None, FAKE, FAKE, 8, 512, 3, 128, 0, 0, FAKE, None), 1),   # null
        ((FAKE_ODD, FAKE, FAKE, 8, 512, 3, 128, 0, 0, FAKE, None), 2),  # alignment
        ((FAKE, FAKE, FAKE, 8, 512, 3, 128, 0, 0, None, None), 1),   # null output
    ]
    for args, want in bad:
        assert lib.cq_decode(*args) == want, args
    assert ok  # the valid call needs a GPU and is exercised by the GPU tests


def test_gemm_rejects_bad_arguments(lib):
    def call(**kw):
        a = dict(x=FAKE, M=4, packed=FAKE, scales=FAKE, ab=FAKE, N=256, K=512, B=3, G=128,
                 mode=0, epi=0, dt=0, y=FAKE, ws=FAKE, wsb=1 << 30, s=None)
        a.update(kw)
        return lib.cq_gemm(a["x"], a["M"], a["packed"], a["scales"], a["ab"], a["N"], a["K"],
                           a["B"], a["G"], a["mode"], a["epi"], a["dt"], a["y"], a["ws"],
                           a["wsb"], a["s"])
    assert call(B=0) == 2                     # cq_gemm takes B in 1..8
    assert call(B=9) == 2
    assert call(B=1, mode=1) == 2             # the midtread grid needs B >= 2
    assert call(G=192) == 2
    assert call(K=640, G=256) == 2
    assert call(M=-1) == 1
    assert call(epi=3) == 1
    assert call(dt=2) == 1
    assert call(epi=1, N=200) == 2           # SwiGLU halves need N % 128 == 0
    assert call(M=0) == 0                     # empty problem is a no-op
    assert call(M=(1 << 24) + 1) == 2         # beyond the supported token count
    assert lib.cq_gemm_workspace_size((1 << 24) + 1, 256, 512, 3, 128, 0) == 0
    assert call(N=0) == 0


def test_gemm_host_rejects_bad_arguments_before_touching_the_gpu(lib):
    """The argument checks of cq_gemm_host run before any copy is queued:
    on a machine without a GPU these calls return their status."""
    f = lib.cq_gemm_host
    P = ctypes.c_void_p
    f.argtypes = [P, ctypes.c_int64, P, P, P, ctypes.c_int64, ctypes.c_int64, ctypes.c_int,
                  ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P, P, P,
                  ctypes.c_size_t, P]

    def call(**kw):
        a = dict(xh=FAKE, M=4, packed=FAKE, scales=FAKE, ab=FAKE, N=256, K=512, B=3, G=128,
                 mode=0, epi=0, dt=0, yh=FAKE, xd=FAKE, yd=FAKE, ws=FAKE, wsb=1 << 30, s=None)
        a.update(kw)
        return f(a["xh"], a["M"], a["packed"], a["scales"], a["ab"], a["N"], a["K"], a["B"],
                 a["G"], a["mode"], a["epi"], a["dt"], a["yh"], a["xd"], a["yd"], a["ws"],
                 a["wsb"], a["s"])
    assert call(B=9) == 2
    assert call(dt=2) == 1
    assert call(epi=3) == 1
    assert call(yd=None) == 1
    assert call(xd=FAKE_ODD) == 2
    assert call(M=-1) == 1
    assert call(epi=1, N=200) == 2
    assert call(M=0) == 0


def test_gemm_noalloc_rejects_bad_arguments_before_touching_the_gpu(lib):
    """Every check runs before the fixed array is looked up or cleared: on a
    machine without a GPU these calls return their status without a CUDA
    call failing first."""
    f = lib.cq_gemm_noalloc
    P = ctypes.c_void_p
    f.argtypes = [P, ctypes.c_int64, P, P, P, ctypes.c_int64, ctypes.c_int64, ctypes.c_int,
                  ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P]

    def call(**kw):
        a = dict(x=FAKE, M=4, packed=FAKE, scales=FAKE, ab=FAKE, N=256, K=512, B=3, G=128,
                 mode=0, epi=0, dt=0, y=FAKE, s=None)
        a.update(kw)
        return f(a["x"], a["M"], a["packed"], a["scales"], a["ab"], a["N"], a["K"], a["B"],
                 a["G"], a["mode"], a["epi"], a["dt"], a["y"], a["s"])
    assert call(B=9) == 2
    assert call(dt=2) == 1
    assert call(epi=3) == 1
    assert call(y=None) == 1
    assert call(x=FAKE_ODD) == 2
    assert call(M=(1 << 24) + 1) == 2
    assert call(epi=1, N=200) == 2
    assert call(M=0) == 0


def test_oracle_library_builds_and_loads():
    import oracle
    oracle.build()
    assert oracle.num_threads() >= 1
