"""GPU parity: the CUDA library (through its C ABI) against the CPU oracle on
the same seeded inputs.

Bars (from the build contract):
  * packed codes bit-exact;
  * decoded weights within 1 FP32 ulp of the oracle's level rounded to FP32
    (BF16 output: within 1 BF16 ulp);
  * GEMM outputs |y - y_ref| <= 2e-3 * sum_k |w_k x_k| + 1e-6 per element.
"""
import os

import numpy as np
import pytest
import torch

import oracle
import synthetic

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
REL, ABS = 2e-3, 1e-6


@pytest.fixture(scope="module")
def cq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import bit_non_uniform_b200 as cq
    cq.lib()
    return cq


def u16(t):
    """torch fp16/bf16/int16 tensor -> numpy uint16 bit patterns."""
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def make_matrix(tag, N, K, B, G, mode=0):
    codes, s, ab = synthetic.matrix(tag, N, K, B, G, mode)
    return codes, s, ab


def to_dev(codes, s, ab, B, cq):
    dc = codes.cuda()
    packed = cq.cq_pack(dc, B)
    return packed, s.cuda().contiguous(), ab.cuda().contiguous()


def oracle_inputs(codes, s, ab, B):
    packed = oracle.pack(codes.numpy(), B)
    return packed, s.numpy(), u16(ab)


def check_gemm(y_gpu, y_ref, bound, what=""):
    y = y_gpu.detach().float().cpu().numpy().astype(np.float64)
    err = np.abs(y - y_ref)
    tol = REL * bound + ABS
    bad = err > tol
    assert not bad.any(), (
        f"{what}: {bad.sum()} of {bad.size} outside tolerance; worst ratio "
        f"{np.max(err / tol):.3f}")
    return float(np.max(err / tol))


# --------------------------------------------------------------------------
# generator: CPU and GPU draws are bit-identical
# --------------------------------------------------------------------------

def test_generator_cpu_gpu_identical():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    for B, mode in [(2, 0), (3, 0), (4, 1)]:
        c0, s0, a0 = synthetic.matrix(("gen", B), 64, 1024, B, 128, mode)
        c1, s1, a1 = synthetic.matrix(("gen", B), 64, 1024, B, 128, mode, device="cuda")
        assert torch.equal(c0, c1.cpu())
        assert torch.equal(s0.view(torch.int32), s1.cpu().view(torch.int32))
        assert torch.equal(a0.view(torch.int16), a1.cpu().view(torch.int16))


# --------------------------------------------------------------------------
# pack / decode
# --------------------------------------------------------------------------

@pytest.mark.parametrize("B", [1, 2, 3, 4, 5, 6, 7, 8])
@pytest.mark.parametrize("N,K", [(1, 128), (37, 256), (300, 1536)])
def test_pack_bit_exact(cq, B, N, K):
    codes, _, _ = make_matrix(("pack", B, N), N, K, B, 128)
    got = cq.cq_pack(codes.cuda(), B).cpu().numpy()
    assert np.array_equal(got, oracle.pack(codes.numpy(), B))


@pytest.mark.parametrize("B,G,mode", [(2, 128, 0), (3, 512, 0), (4, 256, 0), (2, 128, 1),
                                      (3, 256, 1), (4, 128, 1),
                                      # the format tools also take 1 and 5..8 bits
                                      (1, 128, 0), (5, 256, 0), (6, 128, 1), (7, 512, 0),
                                      (8, 128, 0), (8, 256, 1)])
def test_decode_within_one_ulp(cq, B, G, mode):
    N, K = 203, 1024
    codes, s, ab = make_matrix(("dec", B, G, mode), N, K, B, G, mode)
    if mode == 1:      # include the unused code 2^B - 1 of the midtread grid
        codes[0, :16] = (1 << B) - 1
    pk, sd, abd = to_dev(codes, s, ab, B, cq)
    w32 = cq.cq_decode(pk, sd, abd, K, B, G, mode, cq.F32).cpu().numpy()
    w16 = u16(cq.cq_decode(pk, sd, abd, K, B, G, mode, cq.BF16))
    po, so, ao = oracle_inputs(codes, s, ab, B)
    r64, r32, r16 = oracle.decode(po, so, ao, N, K, B, G, mode)
    d32 = np.abs(w32.view(np.int32).astype(np.int64) - r32.view(np.int32).astype(np.int64))
    assert d32.max() <= 1
    d16 = np.abs(w16.astype(np.int64) - r16.astype(np.int64))
    assert d16.max() <= 1
    # in practice the FP64 level of both sides rounds to the same FP32 value
    assert (d32 == 0).mean() > 0.999


# --------------------------------------------------------------------------
# GEMM on small shapes: several tiles, ragged tails, every code path
# --------------------------------------------------------------------------

GEMM_CASES = [
    # M,   N,    K,    B, G,   mode, epi, dtype
    (1,   128,  128,  2, 128, 0, 0, 0),
    (1,   200,  1024, 3, 512, 0, 0, 0),
    (5,   384,  512,  4, 128, 0, 0, 0),
    (16,  1000, 1536, 3, 256, 0, 0, 0),
    (3,   256,  2048, 2, 512, 1, 0, 0),
    (24,  320,  1024, 4, 256, 1, 0, 0),
    (40,  256,  768,  2, 256, 0, 0, 1),
    (64,  512,  1024, 3, 512, 0, 1, 0),
    (100, 640,  512,  4, 128, 0, 0, 0),
    (129, 384,  1024, 2, 128, 0, 0, 0),
    (300, 256,  1536, 3, 512, 0, 1, 1),
    (17,  1152, 3072, 3, 512, 0, 1, 0),
    # 192-token tiles (two accumulator buffers beside a ring of two decoded
    # slices): two tiles with a ragged second one, one ragged tile under the
    # SwiGLU epilogue, and 128-token tiles where 192 would waste too much
    (380, 384,  1024, 3, 256, 0, 0, 0),
    (350, 256,  1024, 3, 512, 0, 1, 1),      # W3: two 176-token tiles, ragged, SwiGLU
    (190, 256,  2048, 4, 512, 1, 1, 1),
    (256, 384,  2048, 4, 256, 0, 0, 0),
    (600, 256,  1024, 3, 128, 1, 1, 1),
]


@pytest.mark.parametrize("M,N,K,B,G,mode,epi,dt", GEMM_CASES)
def test_gemm_small(cq, M, N, K, B, G, mode, epi, dt):
    codes, s, ab = make_matrix(("gemm", M, N, K, B), N, K, B, G, mode)
    pk, sd, abd = to_dev(codes, s, ab, B, cq)
    x = synthetic.activations(M * 7 + N, M, K)
    y = cq.cq_gemm(x.cuda(), pk, sd, abd, N, K, B, G, mode, epi, dt)
    po, so, ao = oracle_inputs(codes, s, ab, B)
    yr, bd = oracle.gemm(u16(x), po, so, ao, N, K, B, G, mode)
    if epi == 0:
        ref, tol_b = yr, bd
        if dt == 1:  # BF16 output: add the output rounding (half a BF16 ulp)
            tol_b = bd + np.abs(yr) * (2.0 ** -8) / REL
        check_gemm(y, ref, tol_b, "gemm")
    else:
        check_swiglu(y, yr, bd, dt)
    assert cq.device_error() == (0, 0)


# Decode-sized shapes (M <= 2 runs the GEMV kernel): every B, group sizes
# below, at and above one 512-code quad step, ragged N, N = 1, one group per
# row (quads that span four row blocks), SwiGLU and BF16 output.
GEMV_CASES = [
    # M, N,    K,    B, G,    mode, epi, dtype
    (1, 16,   128,  2, 128,  0, 0, 0),
    (1, 1,    512,  3, 512,  0, 0, 0),
    (2, 37,   1024, 3, 512,  0, 0, 0),
    (1, 300,  3072, 3, 512,  0, 0, 1),
    (2, 512,  2048, 4, 256,  1, 0, 0),
    (1, 256,  7168, 2, 512,  0, 1, 0),
    (2, 384,  1024, 2, 1024, 0, 1, 1),
    (1, 2048, 512,  4, 128,  1, 0, 0),
    (2, 4096, 256,  3, 256,  0, 0, 0),
]


@pytest.mark.parametrize("M,N,K,B,G,mode,epi,dt", GEMV_CASES)
def test_gemv_small(cq, M, N, K, B, G, mode, epi, dt):
    test_gemm_small(cq, M, N, K, B, G, mode, epi, dt)


# Code widths 1 and 5..8 ([CQ] "为什么只用两个形状参数？": the code stream is an
# ordinary 1..8-bit integer stream; the H200 crossover section measures W5 and
# W8): the engine's wide-code decoder at decode and prefill sizes, every width,
# both grids, ragged N and M, several groups per row, SwiGLU and BF16 output,
# the 128-byte swizzled rows of W8 and the unswizzled 80/96/112-byte rows.
WIDE_CASES = [
    # M,   N,    K,    B, G,   mode, epi, dtype
    (1,   256,  1024, 8, 128, 0, 0, 0),
    (2,   200,  1536, 5, 512, 0, 0, 0),
    (1,   384,  512,  1, 128, 0, 0, 0),
    (4,   512,  1024, 6, 256, 1, 1, 0),
    (16,  300,  2048, 7, 512, 0, 0, 1),
    (33,  256,  1024, 8, 256, 1, 0, 0),
    (64,  640,  768,  5, 128, 1, 0, 0),
    (130, 384,  1024, 6, 512, 0, 0, 0),
    (300, 256,  1536, 8, 512, 0, 1, 1),
    (200, 129,  512,  7, 128, 1, 0, 0),
    (17,  1152, 3072, 1, 512, 0, 1, 0),
]


@pytest.mark.parametrize("M,N,K,B,G,mode,epi,dt", WIDE_CASES)
def test_gemm_wide_codes(cq, M, N, K, B, G, mode, epi, dt):
    test_gemm_small(cq, M, N, K, B, G, mode, epi, dt)


@pytest.mark.parametrize("B,mode", [(5, 0), (6, 1), (7, 0), (8, 1), (1, 0)])
def test_wide_gemm_matches_decoded_bf16_matmul(cq, B, mode):
    """The wide-code decoder's operand is cq_decode's BF16 value: the GEMM
    equals a matmul of cq_decode's BF16 output up to FP32 summation order."""
    M, N, K, G = 40, 256, 1024, 256
    codes, s, ab = make_matrix(("wide_bf16mm", B, mode), N, K, B, G, mode)
    pk, sd, abd = to_dev(codes, s, ab, B, cq)
    x = synthetic.activations(23 + B, M, K).cuda()
    y = cq.cq_gemm(x, pk, sd, abd, N, K, B, G, mode).double()
    w = cq.cq_decode(pk, sd, abd, K, B, G, mode, cq.BF16).double()
    ref = x.double() @ w.T
    bound = x.double().abs() @ w.abs().T
    assert torch.all((y - ref).abs() <= 1e-5 * bound + 1e-7)
    assert cq.device_error() == (0, 0)


@pytest.mark.parametrize("M", [1, 2])
def test_gemv_is_deterministic_and_cleans_workspace(cq, M):
    N, K, B, G = 7168, 3072, 3, 512
    codes, s, ab = make_matrix(("gv_det", M), N, K, B, G)
    pk, sd, abd = to_dev(codes, s, ab, B, cq)
    x = synthetic.activations(13, M, K).cuda()
    ws = cq.gemm_workspace(M, N, K, B, G)
    y1 = cq.cq_gemm(x, pk, sd, abd, N, K, B, G, workspace=ws)
    y2 = cq.cq_gemm(x, pk, sd, abd, N, K, B, G, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    assert int(ws[:256].view(torch.int32).abs().sum()) == 0
    assert cq.device_error() == (0, 0)


@pytest.mark.parametrize("M,B,epi", [(1, 3, 0), (2, 2, 0), (1, 4, 0), (2, 3, 1)])
def test_gemv_matches_decoded_bf16_matmul(cq, M, B, epi):
    """Decode-sized GEMM = matmul of cq_decode's BF16 output up to FP32
    summation order (the operand is exactly that BF16 value)."""
    N, K, G = 1024, 3072, 512
    codes, s, ab = make_matrix(("gv_bf16mm", M, B), N, K, B, G)
    pk, sd, abd = to_dev(codes, s, ab, B, cq)
    x = synthetic.activations(17 + M, M, K).cuda()
    w = cq.cq_decode(pk, sd, abd, K, B, G, 0, cq.BF16).double()
    ref = x.double() @ w.T
    bound = x.double().abs() @ w.abs().T
    y = cq.cq_gemm(x, pk, sd, abd, N, K, B, G, epilogue=0).double()
    assert torch.all((y - ref).abs() <= 1e-5 * bound + 1e-7)
    if epi:
        h = cq.cq_gemm(x, pk, sd, abd, N, K, B, G, epilogue=cq.EPI_SWIGLU).double()
        g, u = ref[:, : N // 2], ref[:, N // 2:]
        href = g / (1 + torch.exp(-g)) * u
        assert torch.allclose(h, href, rtol=1e-4, atol=1e-5)


PATH_CASES = [
    # M,  N,    K,    B, G,   mode, epi
    (1,  7168, 3072, 3, 512, 0, 0),
    (2,  1000, 2048, 4, 256, 1, 0),
    (8,  512,  1536, 2, 128, 0, 1),
    (16, 384,  1024, 3, 512, 0, 0),
    (11, 257,  512,  2, 512, 0, 0),
]


@pytest.mark.parametrize("M,N,K,B,G,mode,epi", PATH_CASES)
def test_kernels_agree_on_the_decoded_bf16_operand(cq, M, N, K, B, G, mode, epi):
    """Every kernel that takes a problem (narrow-row for M <= 16, the GEMV for
    M <= 2, the tensor-core engine for any M) equals the matmul of cq_decode's
    BF16 weights up to FP32 summation order, and the narrow kernel is run to
    run deterministic."""
    codes, s, ab = make_matrix(("paths", M, N, B), N, K, B, G, mode)
    pk, sd, abd = to_dev(codes, s, ab, B, cq)
    x = synthetic.activations(31 + M, M, K).cuda()
    w = cq.cq_decode(pk, sd, abd, K, B, G, mode, cq.BF16).double()
    ref = x.double() @ w.T
    bound = x.double().abs() @ w.abs().T
    if epi:
        g, u = ref[:, : N // 2], ref[:, N // 2:]
        ref = g / (1 + torch.exp(-g)) * u
    ran = 0
    for path in (cq.PATH_NARROW, cq.PATH_GEMV, cq.PATH_ENGINE):
        try:
            y = cq.gemm_on_path(path, x, pk, sd, abd, N, K, B, G, mode, epi).double()
        except cq.CQError as e:
            assert e.status == 2 and (path != cq.PATH_ENGINE)
            continue
        ran += 1
        if epi:
            assert torch.allclose(y, ref, rtol=1e-4, atol=1e-5), f"path {path}"
        else:
            err = (y - ref).abs()
            assert torch.all(err <= 1e-5 * bound + 1e-7), f"path {path}: {float(err.max())}"
        if path == cq.PATH_NARROW:
            y2 = cq.gemm_on_path(path, x, pk, sd, abd, N, K, B, G, mode, epi).double()
            assert torch.equal(y, y2)
    assert ran >= 2
    torch.cuda.synchronize()
    assert cq.device_error() == (0, 0)


def check_swiglu(y_gpu, yr, bd, dt):
    n2 = yr.shape[1] // 2
    g, u = yr[:, :n2], yr[:, n2:]
    eg, eu = REL * bd[:, :n2] + ABS, REL * bd[:, n2:] + ABS
    sig = 1.0 / (1.0 + np.exp(-g))
    dsilu = np.abs(sig * (1.0 + g * (1.0 - sig)))
    h = g * sig * u
    tol = dsilu * np.abs(u) * eg + np.abs(g * sig) * eu + 1.1 * eg * eu + 1e-6 * np.abs(h) + ABS
    if dt == 1:
        tol = tol + np.abs(h) * 2.0 ** -8
    got = y_gpu.detach().float().cpu().numpy().astype(np.float64)
    err = np.abs(got - h)
    assert not (err > tol).any(), f"swiglu: worst ratio {np.max(err / tol):.3f}"


@pytest.mark.parametrize("M,N,K,B,G,epi,dt,pinned", [
    (1, 7168, 3072, 3, 512, 0, 0, True),
    (2, 512, 2048, 4, 256, 1, 1, True),
    (5, 640, 1024, 2, 512, 0, 0, False),
    (16, 384, 1024, 8, 128, 0, 1, True),
    (300, 256, 1536, 3, 512, 1, 0, True),
])
def test_gemm_host_buffers_equal_device_call(cq, M, N, K, B, G, epi, dt, pinned):
    """cq_gemm_host (x and y in host memory, copies queued on the stream)
    gives exactly cq_gemm's output: the kernels are run-to-run deterministic."""
    codes, s, ab = make_matrix(("host", M, N, B), N, K, B, G)
    pk, sd, abd = to_dev(codes, s, ab, B, cq)
    x = synthetic.activations(41 + M, M, K)
    ref = cq.cq_gemm(x.cuda(), pk, sd, abd, N, K, B, G, 0, epi, dt)
    xh = x.pin_memory() if pinned else x.clone()
    ncol = N // 2 if epi else N
    yh = torch.empty((M, ncol), dtype=torch.float32 if dt == 0 else torch.bfloat16)
    if pinned:
        yh = yh.pin_memory()
    st = torch.cuda.Stream()
    got = cq.cq_gemm_host(xh, pk, sd, abd, N, K, B, G, 0, epi, dt, y_host=yh, stream=st)
    st.synchronize()
    assert torch.equal(got, ref.cpu())
    assert cq.device_error() == (0, 0)


def test_gemm_is_deterministic_and_cleans_workspace(cq):
    M, N, K, B, G = 7, 896, 3072, 3, 512
    codes, s, ab = make_matrix(("det",), N, K, B, G)
    pk, sd, abd = to_dev(codes, s, ab, B, cq)
    x = synthetic.activations(11, M, K).cuda()
    ws = cq.gemm_workspace(M, N, K, B, G)
    y1 = cq.cq_gemm(x, pk, sd, abd, N, K, B, G, workspace=ws)
    y2 = cq.cq_gemm(x, pk, sd, abd, N, K, B, G, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    nt = cq.gemm_workspace_size(M, N, K, B, G)
    assert nt > 0
    # the tile counters at the head of the workspace are back to zero
    assert int(ws[:256].view(torch.int32).abs().sum()) == 0
    assert cq.device_error() == (0, 0)


def test_gemm_matches_decoded_bf16_matmul(cq):
    """The tensor path's operand is exactly BF16(decoded FP32 level): the GEMM
    equals a matmul of cq_decode's BF16 output up to FP32 summation order."""
    M, N, K, B, G = 64, 512, 2048, 4, 512
    codes, s, ab = make_matrix(("bf16mm",), N, K, B, G)
    pk, sd, abd = to_dev(codes, s, ab, B, cq)
    x = synthetic.activations(5, M, K).cuda()
    y = cq.cq_gemm(x, pk, sd, abd, N, K, B, G).double()
    w = cq.cq_decode(pk, sd, abd, K, B, G, 0, cq.BF16).double()
    ref = x.double() @ w.T
    bound = x.double().abs() @ w.abs().T
    assert torch.all((y - ref).abs() <= 1e-5 * bound + 1e-7)


# --------------------------------------------------------------------------
# full-size configurations
# --------------------------------------------------------------------------

def test_config1_fitted_w4_g128(cq):
    """256 x 1024 W4 G128 fitted by the oracle from Laplace(0, 0.02) weights
    (seed 0), M = 1, plus the same codes decoded with every group forced to
    a = 1, b = 0 (the uniform-INT special case)."""
    d = np.load(os.path.join(ROOT, "tests", "golden", "config1_w4g128.npz"))
    N, K, B, G = 256, 1024, 4, 128
    packed, s, ab = d["packed"], d["scales"], d["ab"]
    x = synthetic.activations(1, 1, K)
    for uniform in (False, True):
        abu = ab.copy()
        if uniform:
            abu[..., 0] = oracle.double_to_half(1.0)
            abu[..., 1] = 0
        yr, bd = oracle.gemm(u16(x), packed, s, abu, N, K, B, G)
        pk = torch.from_numpy(packed).cuda()
        sd = torch.from_numpy(s).cuda()
        abd = torch.from_numpy(abu.view(np.int16)).cuda()
        y = cq.cq_gemm(x.cuda(), pk, sd, abd, N, K, B, G)
        check_gemm(y, yr, bd, f"config1 uniform={uniform}")
        w32 = cq.cq_decode(pk, sd, abd, K, B, G, 0, cq.F32).cpu().numpy()
        _, r32, _ = oracle.decode(packed, s, abu, N, K, B, G)
        d32 = np.abs(w32.view(np.int32).astype(np.int64) - r32.view(np.int32).astype(np.int64))
        assert d32.max() <= 1


@pytest.mark.parametrize("M", [1, 4, 16])
def test_config2_w3_down_proj(cq, M):
    N, K, B, G = 7168, 3072, 3, 512
    codes, s, ab = make_matrix(("config2",), N, K, B, G)
    pk, sd, abd = to_dev(codes, s, ab, B, cq)
    x = synthetic.activations(200 + M, M, K)
    y = cq.cq_gemm(x.cuda(), pk, sd, abd, N, K, B, G)
    po, so, ao = oracle_inputs(codes, s, ab, B)
    yr, bd = oracle.gemm(u16(x), po, so, ao, N, K, B, G)
    check_gemm(y, yr, bd, f"config2 M={M}")


@pytest.mark.parametrize("M", [1, 16, 64])
def test_config3_w2_gate_up_swiglu(cq, M):
    N, K, B, G = 6144, 7168, 2, 512
    codes, s, ab = make_matrix(("config3",), N, K, B, G)
    pk, sd, abd = to_dev(codes, s, ab, B, cq)
    x = synthetic.activations(300 + M, M, K)
    po, so, ao = oracle_inputs(codes, s, ab, B)
    yr, bd = oracle.gemm(u16(x), po, so, ao, N, K, B, G)
    y = cq.cq_gemm(x.cuda(), pk, sd, abd, N, K, B, G, epilogue=cq.EPI_SWIGLU)
    check_swiglu(y, yr, bd, 0)
    y = cq.cq_gemm(x.cuda(), pk, sd, abd, N, K, B, G)
    check_gemm(y, yr, bd, f"config3 M={M} no epilogue")


def test_swiglu_wide_tiles_sampled_columns(cq):
    """The gate+up matrix with the SwiGLU epilogue at M = 4000: 192-token
    tiles (ragged last tile of 160 tokens), BF16 output; every token of a
    sample of output columns against the oracle's gate and up rows."""
    N, K, B, G, M = 6144, 7168, 2, 512, 4000
    codes, s, ab = make_matrix(("config3",), N, K, B, G)
    pk, sd, abd = to_dev(codes, s, ab, B, cq)
    x = synthetic.activations(4321, M, K)
    y = cq.cq_gemm(x.cuda(), pk, sd, abd, N, K, B, G, epilogue=cq.EPI_SWIGLU,
                   out_dtype=cq.BF16).cpu()
    torch.cuda.synchronize()
    assert cq.device_error() == (0, 0)
    n2 = N // 2
    cols = np.sort(np.random.default_rng(7).choice(n2, 24, replace=False))
    cols = np.unique(np.concatenate([cols, [0, 63, 64, n2 - 1]]))
    rows = np.concatenate([cols, cols + n2])
    po, so, ao = oracle_inputs(codes[rows], s[rows], ab[rows], B)
    yr, bd = oracle.gemm(u16(x), po, so, ao, len(rows), K, B, G)
    check_swiglu(y[:, cols], yr, bd, 1)


@pytest.mark.parametrize("cfg,M", [("config2", 256), ("config3", 1024), ("config2", 4096)])
def test_large_m_sampled_rows(cq, cfg, M):
    """M >= 256 on the full matrices: every output of a sample of weight rows
    (the oracle computes those rows one by one)."""
    if cfg == "config2":
        N, K, B, G = 7168, 3072, 3, 512
    else:
        N, K, B, G = 6144, 7168, 2, 512
    codes, s, ab = make_matrix((cfg,), N, K, B, G)
    pk, sd, abd = to_dev(codes, s, ab, B, cq)
    x = synthetic.activations(400 + M, M, K)
    y = cq.cq_gemm(x.cuda(), pk, sd, abd, N, K, B, G).cpu()
    rows = np.sort(np.random.default_rng(M).choice(N, 48, replace=False))
    rows = np.unique(np.concatenate([rows, [0, 127, 128, N - 1]]))
    po, so, ao = oracle_inputs(codes[rows], s[rows], ab[rows], B)
    yr, bd = oracle.gemm(u16(x), po, so, ao, len(rows), K, B, G)
    check_gemm(y[:, rows], yr, bd, f"{cfg} M={M}")
