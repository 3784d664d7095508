"""cq_gemm_noalloc: the GEMM entry point for callers that cannot allocate
device memory (it keeps its stream-K scratch in a fixed array inside libcq).

It must give the same results as cq_gemm with a caller workspace, also when
called twice in a row (the fixed array keeps the previous call's contents),
and must refuse a problem whose scratch would not fit.  This file is named so
that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import synthetic

pytestmark = pytest.mark.gpu

REL, ABS = 2e-3, 1e-6


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from bit_non_uniform_b200 import build
    build.build()
    import bit_non_uniform_b200 as cq
    L = cq.lib()
    f = L.cq_gemm_noalloc
    P = ctypes.c_void_p
    f.argtypes = [P, ctypes.c_int64, P, P, P, ctypes.c_int64, ctypes.c_int64, ctypes.c_int,
                  ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, P, P]
    f.restype = ctypes.c_int
    return cq, f


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def _noalloc(f, x, packed, s, ab, N, K, B, G, epi, out):
    st = f(_p(x), x.shape[0], _p(packed), _p(s), _p(ab), N, K, B, G, 0, epi, 0, _p(out),
           ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    return st


@pytest.mark.parametrize("M,N,K,B,G,epi", [(1, 7168, 3072, 3, 512, 0),
                                           (16, 1024, 2048, 2, 512, 1),
                                           (5, 640, 1536, 4, 128, 0)])
def test_noalloc_matches_workspace_gemm_twice(lib, M, N, K, B, G, epi):
    cq, f = lib
    codes, s, ab = synthetic.matrix(("noalloc", M, N, B), N, K, B, G)
    packed = cq.cq_pack(codes.cuda(), B)
    s, ab = s.cuda(), ab.cuda()
    w = cq.cq_decode(packed, s, ab, K, B, G, 0, cq.BF16).float()
    ncol = N // 2 if epi else N
    for call in range(2):
        x = synthetic.activations(900 + 17 * call + M, M, K).cuda()
        ref = cq.cq_gemm(x, packed, s, ab, N, K, B, G, epilogue=epi)
        out = torch.full((M, ncol), float("nan"), dtype=torch.float32, device="cuda")
        assert _noalloc(f, x, packed, s, ab, N, K, B, G, epi, out) == 0
        torch.cuda.synchronize()
        assert cq.device_error() == (0, 0)
        bound = (x.float().abs() @ w.abs().T).double()
        if epi == 0:
            tol = REL * bound + ABS
        else:
            # first-order propagation of the GEMM bound through h = silu(g) u
            yfull = cq.cq_gemm(x, packed, s, ab, N, K, B, G).double()
            g, u = yfull[:, :ncol], yfull[:, ncol:]
            eg, eu = REL * bound[:, :ncol] + ABS, REL * bound[:, ncol:] + ABS
            sig = torch.sigmoid(g)
            dsilu = (sig * (1 + g * (1 - sig))).abs()
            tol = dsilu * u.abs() * eg + (g * sig).abs() * eu + 1.1 * eg * eu + ABS
        err = (out.double() - ref.double()).abs()
        assert torch.all(err <= tol), float((err / tol).max())


def test_noalloc_rejects_problems_beyond_its_scratch(lib):
    cq, f = lib
    N, K, B, G, M = 7168, 3072, 3, 512, 256      # needs far more than 4 MiB of partials
    packed = torch.zeros((N, K * B // 8), dtype=torch.uint8, device="cuda")
    s = torch.ones((N, K // G), dtype=torch.float32, device="cuda")
    ab = torch.zeros((N, K // G, 2), dtype=torch.float16, device="cuda")
    x = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros((M, N), dtype=torch.float32, device="cuda")
    assert _noalloc(f, x, packed, s, ab, N, K, B, G, 0, out) == 5     # CQ_ERR_WORKSPACE
