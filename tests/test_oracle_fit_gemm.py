"""Pins of the oracle's GEMM, SwiGLU, MoE composition and data-free group
fitter (no GPU needed)."""
import itertools

import numpy as np
import pytest
import scipy.special

import oracle
import synthetic

RNG = np.random.default_rng(99)


def _rand_matrix(N, K, B, G, mode=oracle.MIDRISE, uniform=False, seed=0):
    rng = np.random.default_rng(seed)
    hi = (1 << B) if mode == oracle.MIDRISE else (1 << B) - 1
    codes = rng.integers(0, hi, size=(N, K), dtype=np.uint8)
    s = (np.abs(rng.normal(0, 0.02, size=(N, K // G))) + 1e-3).astype(np.float32)
    if uniform:
        a = np.full((N, K // G), 1.0, np.float16)
        b = np.zeros((N, K // G), np.float16)
    else:
        a = rng.uniform(0.3, 1.1, size=(N, K // G)).astype(np.float16)
        b = rng.uniform(-0.3, 0.3, size=(N, K // G)).astype(np.float16)
    ab = np.stack([a, b], -1).view(np.uint16)
    return codes, oracle.pack(codes, B), s, ab


def _bf16_act(M, K, seed=0):
    x = np.random.default_rng(seed).normal(0, 1, size=(M, K))
    return oracle.bf16_round(x)


# --------------------------------------------------------------------------
# GEMM
# --------------------------------------------------------------------------

@pytest.mark.parametrize("B,G,mode", [(2, 128, 0), (3, 256, 0), (4, 128, 1), (3, 512, 1)])
def test_gemm_equals_library_matmul_of_decoded(B, G, mode):
    N, K, M = 37, 1024, 5
    codes, packed, s, ab = _rand_matrix(N, K, B, G, mode, seed=B)
    x = _bf16_act(M, K, seed=B)
    w64, w32, _ = oracle.decode(packed, s, ab, N, K, B, G, mode)
    y, bound = oracle.gemm(x, packed, s, ab, N, K, B, G, mode)
    xf = oracle.bf16_bits_to_f64(x)
    assert np.allclose(y, xf @ w64.T, rtol=1e-12, atol=1e-12)
    assert np.allclose(bound, np.abs(xf) @ np.abs(w64).T, rtol=1e-12, atol=1e-12)
    assert np.array_equal(w32, w64.astype(np.float32))


@pytest.mark.parametrize("B,G,mode", [(2, 128, 0), (3, 512, 0), (4, 256, 1)])
def test_gemm_bf16_operand_is_matmul_of_decoded_bf16(B, G, mode):
    """operand="bf16" multiplies by the decode's BF16 weights (each level
    rounded to FP32, then to BF16), as a library matmul of cq's decode
    output does; the FP64-level product differs from it."""
    N, K, M = 29, 1024, 4
    codes, packed, s, ab = _rand_matrix(N, K, B, G, mode, seed=40 + B)
    x = _bf16_act(M, K, seed=41)
    _, _, w16 = oracle.decode(packed, s, ab, N, K, B, G, mode)
    wb = oracle.bf16_bits_to_f64(w16)
    y, bound = oracle.gemm(x, packed, s, ab, N, K, B, G, mode, operand="bf16")
    xf = oracle.bf16_bits_to_f64(x)
    assert np.allclose(y, xf @ wb.T, rtol=1e-12, atol=1e-12)
    assert np.allclose(bound, np.abs(xf) @ np.abs(wb).T, rtol=1e-12, atol=1e-12)
    y64, _ = oracle.gemm(x, packed, s, ab, N, K, B, G, mode)
    assert not np.allclose(y, y64, rtol=1e-9, atol=0)


def test_directed_rounding_helpers():
    v = np.concatenate([RNG.normal(size=2000) * 10.0 ** RNG.integers(-30, 30, size=2000),
                        [0.0, 1.0, -1.0, 1.0 + 2.0 ** -30, 3.0]])
    lo, hi = oracle.f32_down(v), oracle.f32_up(v)
    assert np.all(lo.astype(np.float64) <= v) and np.all(hi.astype(np.float64) >= v)
    # nothing representable in FP32 lies strictly between the result and v
    assert np.all(np.nextafter(lo, np.float32(np.inf)).astype(np.float64) > v)
    assert np.all(np.nextafter(hi, np.float32(-np.inf)).astype(np.float64) < v)
    exact = v.astype(np.float32).astype(np.float64) == v
    assert np.all(lo[exact] == hi[exact])
    # RNE FP32 -> BF16 agrees with the oracle's FP64 -> FP32 -> BF16 rounding on FP32 input
    f = (RNG.normal(size=5000) * 7).astype(np.float32)
    f = np.concatenate([f, np.float32([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8)])])
    assert np.array_equal(oracle.bf16_rne_of_f32(f),
                          oracle.bf16_bits_to_f64(oracle.bf16_round(f.astype(np.float64))))
    # smallest BF16 value >= v
    w = np.abs(RNG.normal(size=3000)) * 10.0 ** RNG.integers(-20, 20, size=3000)
    up = oracle.bf16_bits_to_f64(oracle.bf16_up_bits(w))
    assert np.all(up >= w)
    below = oracle.bf16_bits_to_f64(oracle.bf16_up_bits(w) - 1)
    assert np.all(below < w)


def _chain_layer(B=3, H=1024, I=512, E=3, seed=0):
    exps = []
    for e in range(E):
        _, pgu, sgu, agu = _rand_matrix(2 * I, H, B, 128, seed=seed + 10 * e)
        _, pdn, sdn, adn = _rand_matrix(H, I, B, 128, seed=seed + 10 * e + 5)
        exps.append(dict(B_gu=B, packed_gu=pgu, scales_gu=sgu, ab_gu=agu,
                         B_dn=B, packed_dn=pdn, scales_dn=sdn, ab_dn=adn))
    return exps


def _simulated_chain(x, ids, exps, H, I, G, operand, noise, rng, hround="rne", swap=False):
    """A stand-in for a kernel, on the CPU: the two products with errors of
    up to `noise` times their tolerance, h evaluated in FP32 and rounded to
    BF16 (or, to plant a mistake, truncated / with gate and up swapped)."""
    rel = 2e-3 if operand == "f64" else 2e-5
    T, k = ids.shape
    out = {}
    for r in range(T * k):
        ex = exps[int(ids[r // k, r % k])]
        gu, bgu = oracle.gemm(x[r // k:r // k + 1], ex["packed_gu"], ex["scales_gu"],
                              ex["ab_gu"], 2 * I, H, ex["B_gu"], G, operand=operand)
        gu = gu + noise * rng.uniform(-1, 1, gu.shape) * (rel * bgu + 1e-6)
        g, u = gu[0, :I].astype(np.float32), gu[0, I:].astype(np.float32)
        if swap:
            g, u = u, g
        hf = (g / (np.float32(1) + np.exp(-g)) * u).astype(np.float32)
        if hround == "rne":
            hb = oracle.bf16_round(hf.astype(np.float64))
        else:   # truncation toward zero
            hb = (hf.view(np.uint32) >> 16).astype(np.uint16)
        y, by = oracle.gemm(hb[None, :], ex["packed_dn"], ex["scales_dn"], ex["ab_dn"], H, I,
                            ex["B_dn"], G, operand=operand)
        out[r] = y[0] + noise * rng.uniform(-1, 1, H) * (rel * by[0] + 1e-6)
    return out


@pytest.mark.parametrize("operand", ["f64", "bf16"])
def test_moe_chain_tolerance_accepts_a_correct_chain_and_rejects_planted_mistakes(operand):
    """The chain tolerance of moe_routes: a CPU stand-in for a kernel whose
    products err by up to half their own tolerance (in either direction)
    and which rounds h to BF16 correctly passes; the same chain with h
    truncated instead of rounded (BF16-operand check), or with gate and up
    swapped, fails."""
    H, I, G, T, k, E = 1024, 512, 128, 3, 2, 3
    exps = _chain_layer(3, H, I, E, seed=300)
    x = _bf16_act(T, H, seed=301)
    ids, _ = synthetic.routing_uniform(302, T, E, k)
    ids = ids.numpy()
    rel, abs_ = (2e-3, 1e-6) if operand == "f64" else (2e-5, 1e-7)
    ref = oracle.moe_routes(x, ids, exps, H, I, G, rel=rel, abs_=abs_, operand=operand)
    rng = np.random.default_rng(303)

    def worst(sim):
        return max(float(np.max(np.abs(sim[r] - ref[r][0]) / ref[r][2])) for r in ref)

    assert worst(_simulated_chain(x, ids, exps, H, I, G, operand, 0.5, rng)) <= 1.0
    assert worst(_simulated_chain(x, ids, exps, H, I, G, operand, 0.0, rng, swap=True)) > 1.0
    if operand == "bf16":
        assert worst(_simulated_chain(x, ids, exps, H, I, G, operand, 0.0, rng,
                                      hround="trunc")) > 1.0
        # far tighter than the contract's bound on a typical element
        assert np.median(ref[0][2] / ref[0][1]) < 2e-3


@pytest.mark.parametrize("B", [2, 3, 4])
def test_gemm_uniform_case_is_integer_dequant_matmul(B):
    """With every group at a = 1, b = 0 the GEMM is the textbook symmetric
    uniform-integer dequantised matmul: w = s (2u - (2^B-1)) / (2^B-1)."""
    N, K, M, G = 20, 512, 3, 128
    codes, packed, s, ab = _rand_matrix(N, K, B, G, uniform=True, seed=7 + B)
    x = oracle.bf16_bits_to_f64(_bf16_act(M, K, seed=3))
    srow = np.repeat(s.astype(np.float64), G, axis=1)
    w = srow * (2.0 * codes - ((1 << B) - 1)) / ((1 << B) - 1)
    y, _ = oracle.gemm(oracle.bf16_round(x), packed, s, ab, N, K, B, G)
    assert np.allclose(y, x @ w.T, rtol=1e-12, atol=1e-13)


def test_silu_and_swiglu():
    g = np.linspace(-30, 30, 2001)
    assert np.allclose(oracle.silu(g), g * scipy.special.expit(g), rtol=1e-13, atol=1e-300)
    assert oracle.silu(0.0) == 0.0
    y = RNG.normal(size=(4, 10))
    h = oracle.swiglu(y)
    assert h.shape == (4, 5)
    assert np.allclose(h, y[:, :5] * scipy.special.expit(y[:, :5]) * y[:, 5:])


def test_moe_composition_tiny():
    """moe_routes / moe_combine against explicit per-route loops over
    decoded matrices (toy shapes of the family: hidden 512, moe_intermediate
    256, 8 experts, top-2)."""
    H, I, E, T, k, G = 512, 256, 8, 6, 2, 128
    experts = []
    for e in range(E):
        B = (2, 3, 4)[e % 3]
        _, pgu, sgu, agu = _rand_matrix(2 * I, H, B, G, seed=100 + e)
        _, pdn, sdn, adn = _rand_matrix(H, I, B, G, seed=200 + e)
        experts.append(dict(B_gu=B, packed_gu=pgu, scales_gu=sgu, ab_gu=agu,
                            B_dn=B, packed_dn=pdn, scales_dn=sdn, ab_dn=adn))
    x = _bf16_act(T, H, seed=5)
    ids, w = synthetic.routing_uniform(3, T, E, k)
    ids, w = ids.numpy(), w.numpy()
    routes = oracle.moe_routes(x, ids, experts, H, I, G)
    comb = oracle.moe_combine(routes, w)
    xf = oracle.bf16_bits_to_f64(x)
    for t in range(T):
        acc = np.zeros(H)
        for j in range(k):
            ex = experts[int(ids[t, j])]
            wgu, _, _ = oracle.decode(ex["packed_gu"], ex["scales_gu"], ex["ab_gu"], 2 * I, H,
                                      ex["B_gu"], G)
            wdn, _, _ = oracle.decode(ex["packed_dn"], ex["scales_dn"], ex["ab_dn"], H, I,
                                      ex["B_dn"], G)
            gu = wgu @ xf[t]
            h = gu[:I] * scipy.special.expit(gu[:I]) * gu[I:]
            hb = oracle.bf16_bits_to_f64(oracle.bf16_round(h))
            yr = wdn @ hb
            assert np.allclose(routes[t * k + j][0], yr, rtol=1e-11, atol=1e-12)
            acc += float(w[t, j]) * yr
        assert np.allclose(comb[t][0], acc, rtol=1e-11, atol=1e-12)


# --------------------------------------------------------------------------
# fitter  (section "从曲线到量化器：数据无关的组内拟合")
# --------------------------------------------------------------------------

def test_nearest_level_bruteforce():
    for _ in range(300):
        lv = np.sort(RNG.normal(size=RNG.integers(2, 17)))
        lv = np.unique(lv)
        vals = np.concatenate([RNG.normal(size=20) * 2, (lv[:-1] + lv[1:]) / 2, lv])
        for v in vals:
            assert oracle.nearest(lv, v) == oracle.nearest(lv, v, brute=True)


def _brute_optimal_sse(v, k):
    """Minimum SSE over all partitions of the sorted values into at most k
    contiguous clusters (exhaustive over cut points)."""
    v = np.sort(v)
    n = len(v)
    best = np.inf
    for kk in range(1, min(k, n) + 1):
        for cuts in itertools.combinations(range(1, n), kk - 1):
            parts = np.split(v, cuts)
            best = min(best, sum(float(np.sum((p - p.mean()) ** 2)) for p in parts))
    return best


def test_optimal_sse_dp_bruteforce():
    for _ in range(60):
        n = int(RNG.integers(1, 9))
        k = int(RNG.integers(1, 5))
        v = RNG.normal(size=n)
        assert oracle.optimal_sse(v, k) == pytest.approx(_brute_optimal_sse(v, k), abs=1e-12)


def _small_grids():
    a = np.arange(1, 41, dtype=np.float64) / 16.0
    b = np.arange(-32, 33, dtype=np.float64) / 16.0
    alpha = np.arange(30, 101, 2, dtype=np.float64) / 100.0
    return a, b, alpha


@pytest.mark.parametrize("B,mode", [(2, 0), (3, 0), (4, 0), (4, 1)])
def test_fit_error_bound_chain(B, mode):
    """Per group: optimal free scalar codebook <= Cubic <= optimal clipped
    uniform grid (the error bound of section "为什么只用两个形状参数？";
    the right inequality holds because (1, 0) is always a candidate)."""
    G = 128
    w = RNG.laplace(0, 0.02, size=16 * G)
    grids = _small_grids()
    cub = oracle.fit(w, G, B, mode, grids=grids)
    uni = oracle.fit(w, G, B, mode, uniform_only=True, grids=grids)
    nlev = (1 << B) if mode == 0 else (1 << B) - 1
    for g in range(16):
        grp = w[g * G:(g + 1) * G]
        assert cub["sse"][g] <= uni["sse"][g] * (1 + 1e-12)
        assert oracle.optimal_sse(grp, nlev) <= cub["sse"][g] * (1 + 1e-9)
        # uniform-only fit really is the clipped INT grid
        assert uni["ab"][g, 0] == oracle.double_to_half(1.0) and uni["ab"][g, 1] == 0


def test_fit_outputs_are_consistent():
    """Step (5): a, b are FP16 and s FP32; the codes are the nearest levels
    of the stored parameters and the reported SSE is recomputed from them."""
    G, B = 128, 3
    w = RNG.normal(0, 1, size=8 * G)
    r = oracle.fit(w, G, B, oracle.MIDRISE, grids=_small_grids())
    for g in range(8):
        assert oracle.is_monotone(int(r["ab"][g, 0]), int(r["ab"][g, 1]))
        lv = oracle.levels(B, oracle.MIDRISE, float(r["s"][g]), int(r["ab"][g, 0]),
                           int(r["ab"][g, 1]))
        grp = w[g * G:(g + 1) * G]
        codes = np.array([oracle.nearest(lv, v, brute=True) for v in grp])
        assert np.array_equal(codes, r["codes"][g])
        assert r["sse"][g] == pytest.approx(float(np.sum((grp - lv[codes]) ** 2)), rel=1e-12)
        assert r["clipped"][g] == int(np.sum(np.abs(grp) > r["s"][g]))


def test_fit_nrmse_table_w4_g128_midtread(golden):
    """The article's finite-group experiment (W4, G128, 15,360 samples per
    zero-mean distribution): the oracle's fitter in the sign-magnitude
    (midtread) grid reproduces the Cubic and optimal-clipped-INT4 columns to
    within sampling noise.  Tolerance 5% relative (seeds are not published)."""
    tab = golden["nrmse_w4_g128"]
    n, G = tab["samples"], tab["group"]
    rng = np.random.default_rng(2026)
    dists = {"uniform": rng.uniform(-1, 1, n), "gaussian": rng.normal(0, 1, n),
             "laplace": rng.laplace(0, 1, n)}
    for name, w in dists.items():
        cub = oracle.nrmse(oracle.fit(w, G, 4, oracle.MIDTREAD)["sse"], w)
        uni = oracle.nrmse(oracle.fit(w, G, 4, oracle.MIDTREAD, uniform_only=True)["sse"], w)
        ref = tab["rows"][name]
        assert abs(cub / ref["cubic"] - 1) < 0.05, (name, cub, ref["cubic"])
        assert abs(uni / ref["int4"] - 1) < 0.05, (name, uni, ref["int4"])
        assert cub < uni
