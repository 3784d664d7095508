"""GPU parity of the Dynamic-A8 path (cq_quant_rows, cq_gemm_a8) against the
oracle's reading of "一份 checkpoint，同时服务 A16 与 Dynamic A8": INT8 carriers
RNE(127 sign(k) q(t)), activations quantized per row by their absmax, exact
integer dot products per group, FP32 group scaling.

Bars: the quantized activations bit-exact; the integer dot products bit-exact
(recovered from a single-group product whose scaling is exact enough to
round back); the output within 1e-5 of the bound sum |f xq carrier| (the only
errors are the FP32 scaling and sums)."""
import numpy as np
import pytest
import torch

import oracle
import synthetic

pytestmark = pytest.mark.gpu
REL = 1e-5            # FP32 group scaling, running sums and partial sums of exact INT32 dots


@pytest.fixture(scope="module")
def cq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import bit_non_uniform_b200 as cq
    cq.lib()
    return cq


def u16(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def test_quant_rows_bit_exact(cq):
    x = synthetic.activations(3, 7, 1000).float()
    x[2] = 0.0
    x[3] = torch.arange(-500, 500, dtype=torch.float32) % 255 - 127   # integers
    x[4, :509] = torch.arange(-254, 255, dtype=torch.float32)            # exact halves
    x[4, 509:] = 0.0
    xb = x.to(torch.bfloat16)
    xq, am = cq.cq_quant_rows(xb.cuda())
    rq, ra = oracle.quant_rows(u16(xb))
    np.testing.assert_array_equal(xq.cpu().numpy(), rq)
    np.testing.assert_array_equal(am.cpu().numpy(), ra)


CASES = [
    # M,   N,    K,    B, G,   mode, epi, dtype
    (3,   256,  512,  2, 128, 0, 0, 0),
    (16,  1000, 1536, 3, 256, 0, 0, 0),
    (40,  256,  768,  4, 128, 1, 0, 1),
    (64,  512,  1024, 3, 512, 0, 1, 0),
    (129, 384,  2048, 2, 512, 0, 0, 0),
    (300, 256,  1536, 4, 512, 0, 1, 1),
    (1,   7168, 3072, 3, 512, 0, 0, 0),
]


@pytest.mark.parametrize("M,N,K,B,G,mode,epi,dt", CASES)
def test_gemm_a8_matches_oracle(cq, M, N, K, B, G, mode, epi, dt):
    codes, s, ab = synthetic.matrix(("a8", M, N, K, B), N, K, B, G, mode)
    pk = cq.cq_pack(codes.cuda(), B)
    x = synthetic.activations(M * 3 + N, M, K)
    y = cq.cq_gemm_a8(x.cuda(), pk, s.cuda(), ab.cuda(), N, K, B, G, mode, epi, dt)
    assert cq.device_error() == (0, 0)
    xq, am = oracle.quant_rows(u16(x))
    po = oracle.pack(codes.numpy(), B)
    yr, bd = oracle.gemm_a8(xq, am, po, s.numpy(), u16(ab), N, K, B, G, mode)
    got = y.float().cpu().numpy().astype(np.float64)
    if epi == 0:
        tol = REL * bd + 1e-7
        if dt == 1:
            tol = tol + np.abs(yr) * 2.0 ** -8
        assert np.all(np.abs(got - yr) <= tol)
    else:
        h = N // 2
        g, u, bg, bu = yr[:, :h], yr[:, h:], bd[:, :h], bd[:, h:]
        sig = 1.0 / (1.0 + np.exp(-g))
        ref = g * sig * u
        eg, eu = REL * bg + 1e-7, REL * bu + 1e-7
        ds = np.abs(sig * (1.0 + g * (1.0 - sig)))
        tol = ds * np.abs(u) * eg + np.abs(g * sig) * eu + eg * eu + 1e-6 * np.abs(ref)
        if dt == 1:
            tol = tol + np.abs(ref) * 2.0 ** -8
        assert np.all(np.abs(got - ref) <= tol)


def test_gemm_a8_integer_dot_products_exact(cq):
    """One group per row (K = G = 128), every scale 1, and an activation row
    whose largest magnitude is 127 with integer entries: then xq = x, the
    output is acc / 127 with acc the group's integer dot product, and
    rint(127 y) recovers acc exactly (|acc| < 2^21, two FP32 roundings)."""
    N, K, B, G = 384, 128, 3, 128
    for mode in (0, 1):
        codes, _, ab = synthetic.matrix(("a8int", mode), N, K, B, G, mode)
        s = torch.ones((N, K // G), dtype=torch.float32)
        pk = cq.cq_pack(codes.cuda(), B)
        g = torch.Generator().manual_seed(5 + mode)
        x = torch.randint(-127, 128, (2, K), generator=g).float()
        x[:, 7] = 127.0
        xb = x.to(torch.bfloat16)
        y = cq.cq_gemm_a8(xb.cuda(), pk, s.cuda(), ab.cuda(), N, K, B, G, mode)
        assert cq.device_error() == (0, 0)
        xq, am = oracle.quant_rows(u16(xb))
        assert np.array_equal(xq.astype(np.float64), x.numpy()) and np.all(am == 127.0)
        yr, _ = oracle.gemm_a8(xq, am, oracle.pack(codes.numpy(), B), s.numpy(), u16(ab), N, K,
                               B, G, mode)
        acc_ref = np.rint(yr * 127.0)
        assert np.allclose(yr * 127.0, acc_ref, rtol=0, atol=1e-9)      # the oracle's integers
        acc_gpu = np.rint(y.double().cpu().numpy() * 127.0)
        assert np.array_equal(acc_gpu, acc_ref)
