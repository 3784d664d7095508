"""Failure detection on the GPU without a GPU fault: every wait of the
tensor-core engine is bounded.  A test hook withholds the first stage of
code and activation loads, so the waits for it can never complete; the
kernel must give up after the (short) limit, record CQ_ERR_TIMEOUT with the
site of the first wait that gave up, tear down (its other copies land, TMEM
is freed) and leave the context usable: a normal call right after is
checked against the oracle."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
import synthetic

pytestmark = pytest.mark.gpu

CQ_ERR_TIMEOUT = 4


@pytest.fixture(scope="module")
def cq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import bit_non_uniform_b200 as cq
    cq.lib()
    return cq


def u16(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def test_withheld_stage_times_out_and_context_survives(cq):
    M, N, K, B, G = 64, 256, 1024, 3, 256
    codes, s, ab = synthetic.matrix(("bounded", M), N, K, B, G)
    packed = cq.cq_pack(codes.cuda(), B)
    sd, abd = s.cuda(), ab.cuda()
    x = synthetic.activations(5, M, K).cuda()
    y = torch.zeros((M, N), dtype=torch.float32, device="cuda")
    assert cq.device_error() == (0, 0)
    ws = cq.gemm_workspace(M, N, K, B, G)
    L = cq.lib()
    fn = L.cq_test_gemm_bounded
    st = fn(cq._ptr(x), M, cq._ptr(packed), cq._ptr(sd), cq._ptr(abd), N, K, B, G,
            cq._ptr(y), cq._ptr(ws), ws.numel() * ws.element_size(),
            ctypes.c_uint64(20_000_000), 1, None)           # 20 ms limit, stage 0 withheld
    assert st == 0                                          # the launch itself succeeds
    status, site = cq.device_error()                        # synchronises, reads, clears
    assert status == CQ_ERR_TIMEOUT
    assert site > 0
    assert cq.device_error() == (0, 0)                      # cleared
    # the context is usable: an ordinary call with a fresh workspace is exact
    y2 = cq.cq_gemm(x, packed, sd, abd, N, K, B, G)
    torch.cuda.synchronize()
    assert cq.device_error() == (0, 0)
    yr, bd = oracle.gemm(u16(x), oracle.pack(codes.numpy(), B), s.numpy(), u16(ab), N, K, B, G)
    err = np.abs(y2.double().cpu().numpy() - yr)
    assert np.all(err <= 2e-3 * bd + 1e-6)
