"""Pins of the oracle's Dynamic-A8 mode (the article's section "一份 checkpoint，
同时服务 A16 与 Dynamic A8"): the weight-side INT8 carrier, the per-row dynamic
activation quantization, the integer-dot-product GEMM with FP32 group scaling,
and the carrier-aware joint fit.

The article's formulas for the carrier and the joint objective were lost; the
reading pinned here is
  carrier(u) = RNE(127 sign(k) q(t)), saturated to [-127, 127];
  xq = RNE(x * 127 / absmax(row)), decided in FP32;
  y = sum_g (absmax / 127) (s_g / 127) sum_{k in g} xq carrier;
  fit objective L_C + lambda L_A8, codes of the nearest continuous level.

Pins: exact rational arithmetic (fractions), pure-Python brute force on small
cases, the case where the A8 product equals the A16 product exactly, and the
joint fit's exact invariants (the objective ordering between lambdas).
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
import synthetic


def _f16(h):
    return Fraction(float(np.array([h], dtype=np.uint16).view(np.float16)[0]))


def _f32(v):
    return Fraction(float(np.float32(v)))


def _coord(u, B, mode):
    """(sign, t) as exact rationals, from the grid definitions."""
    if mode == oracle.MIDRISE:
        k2 = 2 * u - ((1 << B) - 1)                      # 2k, never zero
        return (1 if k2 > 0 else -1), Fraction(abs(k2), (1 << B) - 1)
    Kc = (1 << (B - 1)) - 1
    k = u - Kc
    return (k > 0) - (k < 0), Fraction(abs(k), Kc)


def _exact_carrier(u, B, mode, a_h, b_h):
    """RNE of the exact rational 127 sign q(t); None when within 1e-9 of a tie
    (the FP64 evaluation may then take either side)."""
    sg, t = _coord(u, B, mode)
    a, b = _f16(a_h), _f16(b_h)
    v = 127 * sg * (a * t + b * t * t + (1 - a - b) * t * t * t)
    fl = v - (v.numerator // v.denominator)
    if abs(fl - Fraction(1, 2)) < Fraction(1, 10 ** 9):
        return None
    return max(-127, min(127, round(v)))                  # round(): ties to even


def _ab_pairs(n, seed):
    return synthetic.ab(synthetic.make_key("a8", seed), n).numpy().view(np.uint16).reshape(-1, 2)


@pytest.mark.parametrize("B", range(1, 9))
@pytest.mark.parametrize("mode", [oracle.MIDRISE, oracle.MIDTREAD])
def test_carrier_is_exact_rounding_of_the_rational_level(B, mode):
    if mode == oracle.MIDTREAD and B < 2:
        pytest.skip("the midtread grid needs B >= 2")
    pairs = [(0x3C00, 0x0000)] + [tuple(int(v) for v in p) for p in _ab_pairs(24, B)]
    used = (1 << B) if mode == oracle.MIDRISE else (1 << B) - 1
    skipped = 0
    for a_h, b_h in pairs:
        c = oracle.carriers(B, mode, a_h, b_h)
        for u in range(used):
            ref = _exact_carrier(u, B, mode, a_h, b_h)
            if ref is None:
                skipped += 1
                continue
            assert int(c[u]) == ref, (B, mode, hex(a_h), hex(b_h), u)
            assert oracle.carrier(u, B, mode, a_h, b_h) == ref
    assert skipped <= 1


@pytest.mark.parametrize("B", range(2, 9))
def test_carrier_special_cases(B):
    one, zero = 0x3C00, 0x0000
    # midtread, a = 1, b = 0: carrier = RNE(127 k / Kc); at B = 8 (Kc = 127) exactly k,
    # and the unused top code (t = 128/127) saturates
    Kc = (1 << (B - 1)) - 1
    c = oracle.carriers(B, oracle.MIDTREAD, one, zero)
    for u in range(2 * Kc + 1):
        assert int(c[u]) == round(Fraction(127 * (u - Kc), Kc))
    if B == 8:
        np.testing.assert_array_equal(c[:255], np.arange(255) - 127)
        assert c[255] == 127
    # every grid and shape: extreme codes at +-127, odd symmetry, non-decreasing
    for mode in (oracle.MIDRISE, oracle.MIDTREAD):
        used = (1 << B) if mode == oracle.MIDRISE else (1 << B) - 1
        for a_h, b_h in [(one, zero)] + [tuple(int(v) for v in p) for p in _ab_pairs(8, 100 + B)]:
            c = oracle.carriers(B, mode, a_h, b_h).astype(int)[:used]
            assert c[0] == -127 and c[-1] == 127
            np.testing.assert_array_equal(c, -c[::-1])
            assert np.all(np.diff(c) >= 0)
            if mode == oracle.MIDTREAD:
                assert c[Kc] == 0


def _bf16_bits(v):
    return (np.asarray(v, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


def _bf16_value(h):
    return float((np.asarray([h], dtype=np.uint32) << 16).view(np.float32)[0])


def test_quant_rows_properties():
    rng = np.random.default_rng(5)
    rows = [rng.normal(0, 1, 300), rng.normal(0, 1e-3, 300), rng.normal(0, 40, 300),
            rng.laplace(0, 0.5, 300), np.zeros(300), np.eye(1, 300, 17)[0] * -3.25]
    x = _bf16_bits(np.stack(rows))                       # truncation: still bf16 values
    xq, absmax = oracle.quant_rows(x)
    near_tie = 0
    for m in range(x.shape[0]):
        xv = [Fraction(_bf16_value(h)) for h in x[m]]
        mx = max(abs(v) for v in xv)
        assert Fraction(float(absmax[m])) == mx
        if mx == 0:
            assert not xq[m].any()
            continue
        for k, v in enumerate(xv):
            q = int(xq[m, k])
            assert -127 <= q <= 127
            if abs(v) == mx:
                assert q == (127 if v > 0 else -127)
            exact = v * 127 / mx
            fl = exact - (exact.numerator // exact.denominator)
            if abs(fl - Fraction(1, 2)) < Fraction(1, 10 ** 5):
                near_tie += 1                            # FP32 decides a near-tie
                assert q in (exact.numerator // exact.denominator,
                             exact.numerator // exact.denominator + 1)
                continue
            assert q == round(exact), (m, k)
    assert near_tie <= 3
    # negation symmetry
    xn, an = oracle.quant_rows(x ^ np.uint16(0x8000))
    np.testing.assert_array_equal(xn, -xq)
    np.testing.assert_array_equal(an, absmax)


def test_quant_rows_integer_rows_are_exact():
    rng = np.random.default_rng(6)
    v = rng.integers(-127, 128, size=(4, 256)).astype(np.float32)
    v[:, 3] = np.array([127, -127, 127, -127])
    xq, absmax = oracle.quant_rows(_bf16_bits(v))
    np.testing.assert_array_equal(absmax, 127.0)
    np.testing.assert_array_equal(xq, v.astype(np.int8))


def test_gemm_a8_equals_a16_when_both_are_exact():
    # B = 8 midtread with a = 1, b = 0: the carrier of code u is k = u - 127 exactly and
    # the continuous level is s k / 127, so the carrier reconstruction equals the level;
    # integer activations with absmax 127 quantize to themselves.  Then the A8 product
    # is the A16 product.
    rng = np.random.default_rng(7)
    N, K, G, B = 12, 512, 128, 8
    codes = rng.integers(0, 255, size=(N, K)).astype(np.uint8)
    packed = oracle.pack(codes, B)
    ng = K // G
    scales = rng.uniform(0.01, 2.0, size=(N, ng)).astype(np.float32)
    ab = np.tile(np.array([0x3C00, 0x0000], dtype=np.uint16), (N, ng, 1))
    v = rng.integers(-127, 128, size=(3, K)).astype(np.float32)
    v[:, 0] = 127
    x = _bf16_bits(v)
    xq, absmax = oracle.quant_rows(x)
    y8, b8 = oracle.gemm_a8(xq, absmax, packed, scales, ab, N, K, B, G, oracle.MIDTREAD)
    y16, b16 = oracle.gemm(x, packed, scales, ab, N, K, B, G, oracle.MIDTREAD)
    np.testing.assert_allclose(y8, y16, rtol=0, atol=1e-12 * b16.max())
    np.testing.assert_allclose(b8, b16, rtol=1e-12)


@pytest.mark.parametrize("B,mode", [(2, oracle.MIDRISE), (3, oracle.MIDRISE),
                                    (4, oracle.MIDTREAD), (3, oracle.MIDTREAD)])
def test_gemm_a8_bruteforce(B, mode):
    # every input drawn directly (xq, absmax, codes, s, a, b); the reference is the
    # definition in exact rational arithmetic with carriers rounded from the exact level
    rng = np.random.default_rng(10 + B + 7 * mode)
    M, N, K, G = 2, 3, 256, 128
    ng = K // G
    hi = (1 << B) if mode == oracle.MIDRISE else (1 << B) - 1
    codes = rng.integers(0, hi, size=(N, K)).astype(np.uint8)
    packed = oracle.pack(codes, B)
    scales = rng.uniform(0.001, 3.0, size=(N, ng)).astype(np.float32)
    ab = _ab_pairs(N * ng, 200 + B + mode).reshape(N, ng, 2)
    xq = rng.integers(-127, 128, size=(M, K)).astype(np.int8)
    absmax = rng.uniform(0.1, 10.0, size=M).astype(np.float32)
    y, bound = oracle.gemm_a8(xq, absmax, packed, scales, ab, N, K, B, G, mode)
    for m in range(M):
        for n in range(N):
            tot = Fraction(0)
            for g in range(ng):
                a_h, b_h = int(ab[n, g, 0]), int(ab[n, g, 1])
                acc = 0
                for k in range(g * G, (g + 1) * G):
                    c = _exact_carrier(int(codes[n, k]), B, mode, a_h, b_h)
                    assert c is not None
                    acc += int(xq[m, k]) * c
                tot += _f32(absmax[m]) / 127 * _f32(scales[n, g]) / 127 * acc
            assert abs(Fraction(float(y[m, n])) - tot) <= Fraction(1e-14) * Fraction(float(bound[m, n]))


GRIDS = (np.arange(1, 41, 2, dtype=np.float64) / 16.0,     # a: 1/16 .. 39/16 step 1/8
         np.arange(-32, 33, 2, dtype=np.float64) / 16.0,   # b: -2 .. 2 step 1/8
         np.round(np.arange(30, 101, 2, dtype=np.float64)) / 100.0)


@pytest.fixture(scope="module")
def weights():
    return synthetic.laplace_weights(41, 24 * 128, 0.02).double().numpy()


def test_joint_fit_lambda_zero_is_the_a16_fit(weights):
    for B, mode in [(3, oracle.MIDRISE), (2, oracle.MIDTREAD)]:
        f0 = oracle.fit(weights, 128, B, mode, grids=GRIDS)
        f1 = oracle.fit(weights, 128, B, mode, grids=GRIDS, lam=0.0)
        for key in ("codes", "s", "ab", "sse", "clipped"):
            np.testing.assert_array_equal(f0[key], f1[key])
        # the reported carrier error is that of the returned codes and carriers
        w = weights.reshape(-1, 128)
        for g in range(w.shape[0]):
            c = oracle.carriers(B, mode, int(f0["ab"][g, 0]), int(f0["ab"][g, 1])).astype(np.float64)
            rec = float(f0["s"][g]) * c[f0["codes"][g]] / 127.0
            assert f0["sse_a8"][g] == pytest.approx(np.sum((w[g] - rec) ** 2), rel=1e-12)


@pytest.mark.parametrize("B,mode", [(2, oracle.MIDRISE), (3, oracle.MIDRISE), (3, oracle.MIDTREAD)])
def test_joint_fit_trades_continuous_for_carrier_error(weights, B, mode):
    # over one candidate set, the minimiser of L_C + lam L_A8 has, per group,
    # L_C non-decreasing and L_A8 non-increasing in lam (exchange argument)
    fits = [oracle.fit(weights, 128, B, mode, grids=GRIDS, lam=lam) for lam in (0.0, 1.0, 1e6)]
    tol = 1e-12 * float(np.sum(weights ** 2))
    for lo, hi in zip(fits, fits[1:]):
        assert np.all(hi["sse"] >= lo["sse"] - tol)
        assert np.all(hi["sse_a8"] <= lo["sse_a8"] + tol)
    # the joint objective of the lam = 1 fit is the smallest over the three
    j = [f["sse"] + f["sse_a8"] for f in fits]
    assert np.all(j[1] <= j[0] + tol) and np.all(j[1] <= j[2] + tol)


def test_quant_rows_ties_go_to_even():
    # absmax 254 makes 127 / absmax = 1/2 exactly, so odd integers land on exact halves
    v = np.arange(-254, 255, dtype=np.float32)[None, :]
    xq, absmax = oracle.quant_rows(_bf16_bits(v))
    assert absmax[0] == 254.0
    np.testing.assert_array_equal(xq[0], [round(Fraction(int(t), 2)) for t in v[0]])


@pytest.mark.parametrize("lam", [0.25, 4.0])
def test_joint_fit_matches_bruteforce_search(weights, lam):
    # the joint fit over a small candidate set against a plain enumeration: every
    # (a, b, alpha), nearest continuous level per weight (ties to the lower code),
    # objective L_C + lam L_A8 with the candidate's own carriers; first minimum wins
    B, mode, G = 3, oracle.MIDRISE, 128
    a_grid = np.array([0.5, 0.75, 1.25], dtype=np.float64)
    b_grid = np.array([-0.5, 0.0, 0.25], dtype=np.float64)
    alpha = np.array([0.6, 0.8, 1.0], dtype=np.float64)
    w = weights.reshape(-1, G)[:6]
    fit = oracle.fit(w, G, B, mode, grids=(a_grid, b_grid, alpha), lam=lam)
    cands = [(1.0, 0.0)] + [(a, b) for a in a_grid for b in b_grid if (a, b) != (1.0, 0.0)]
    for g in range(w.shape[0]):
        mx = np.max(np.abs(w[g]))
        best = None
        for a, b in cands:
            a_h = int(np.array([a], dtype=np.float16).view(np.uint16)[0])
            b_h = int(np.array([b], dtype=np.float16).view(np.uint16)[0])
            if not oracle.is_monotone(a_h, b_h):
                continue
            car = oracle.carriers(B, mode, a_h, b_h).astype(np.float64)
            for al in alpha:
                s = float(np.float32(al * mx))
                lv = oracle.levels(B, mode, s, a_h, b_h)
                u = np.argmin(np.abs(w[g][:, None] - lv[None, :]), axis=1)   # first = lower code
                lc = np.sum((w[g] - lv[u]) ** 2)
                la = np.sum((w[g] - s * car[u] / 127.0) ** 2)
                j = lc + lam * la
                if best is None or j < best[0]:
                    best = (j, a_h, b_h, s, lc, la)
        _, a_h, b_h, s, lc, la = best
        assert (int(fit["ab"][g, 0]), int(fit["ab"][g, 1])) == (a_h, b_h)
        assert float(fit["s"][g]) == s
        assert fit["sse"][g] == pytest.approx(lc, rel=1e-12)
        assert fit["sse_a8"][g] == pytest.approx(la, rel=1e-12)
