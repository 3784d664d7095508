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


def _u16(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("M,N,K,B,G,epi", [(1, 7168, 3072, 3, 512, 0),
                                           (16, 1024, 2048, 2, 512, 1),
                                           (5, 640, 1536, 4, 128, 0)])
def test_noalloc_matches_workspace_gemm_twice(lib, M, N, K, B, G, epi):
    """Two calls in a row: each equals cq_gemm with a caller workspace bit
    for bit (both paths are run-to-run deterministic and run the same
    kernels), and the plain product is within the GEMM bound of the oracle."""
    import oracle
    cq, f = lib
    codes, s, ab = synthetic.matrix(("noalloc", M, N, B), N, K, B, G)
    packed = cq.cq_pack(codes.cuda(), B)
    sd, abd = s.cuda(), ab.cuda()
    ncol = N // 2 if epi else N
    po, so, ao = oracle.pack(codes.numpy(), B), s.numpy(), _u16(ab)
    for call in range(2):
        x = synthetic.activations(900 + 17 * call + M, M, K)
        xd = x.cuda()
        ref = cq.cq_gemm(xd, packed, sd, abd, N, K, B, G, epilogue=epi)
        out = torch.full((M, ncol), float("nan"), dtype=torch.float32, device="cuda")
        assert _noalloc(f, xd, packed, sd, abd, N, K, B, G, epi, out) == 0
        torch.cuda.synchronize()
        assert cq.device_error() == (0, 0)
        assert torch.equal(out, ref), f"call {call}: differs from cq_gemm"
        if epi == 0:
            yr, bd = oracle.gemm(_u16(x), po, so, ao, N, K, B, G)
            err = np.abs(out.double().cpu().numpy() - yr)
            assert np.all(err <= REL * bd + ABS), float(np.max(err / (REL * bd + ABS)))


def test_noalloc_rejects_problems_beyond_its_scratch(lib):
    cq, f = lib
    N, K, B, G, M = 7168, 3072, 3, 512, 256      # needs far more than 4 MiB of partials
    packed = torch.zeros((N, K * B // 8), dtype=torch.uint8, device="cuda")
    s = torch.ones((N, K // G), dtype=torch.float32, device="cuda")
    ab = torch.zeros((N, K // G, 2), dtype=torch.float16, device="cuda")
    x = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros((M, N), dtype=torch.float32, device="cuda")
    assert _noalloc(f, x, packed, s, ab, N, K, B, G, 0, out) == 5     # CQ_ERR_WORKSPACE
