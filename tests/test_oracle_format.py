"""Pins of the oracle's format and level arithmetic against what the
CubicQuant article and plain mathematics fix (no GPU needed)."""
import math

import numpy as np
import pytest
import torch

import oracle

RNG = np.random.default_rng(1234)


# --------------------------------------------------------------------------
# storage identity  (section "存储开销是透明的：B+64/G bit")
# --------------------------------------------------------------------------

def test_bits_per_weight_table(golden):
    for G, row in golden["bits_per_weight"]["rows"].items():
        G = int(G)
        assert oracle.bits_per_weight(0, G) == row["metadata"]
        for B in (2, 3, 4):
            assert oracle.bits_per_weight(B, G) == row[f"W{B}"]


def test_bytes_and_ratio_g512(golden):
    for name, row in golden["bytes_g512"]["rows"].items():
        B = int(name[1])
        bpw = oracle.bits_per_weight(B, 512) / 8
        assert bpw == row["bytes_per_weight"]
        assert round(2.0 / bpw, 2) == row["ratio_vs_bf16"]


def test_kimi_audit_arithmetic(golden):
    a = golden["kimi_audit"]
    n = sum(l["count"] for l in a["layers"])
    payload = sum(l["count"] * l["B"] for l in a["layers"]) / n
    meta = sum(l["count"] * (oracle.bits_per_weight(l["B"], l["G"]) - l["B"])
               for l in a["layers"]) / n
    assert round(payload, 4) == a["payload_bits"]
    assert round(meta, 4) == a["metadata_bits"]
    assert round(payload + meta, 4) == a["effective_bits"]


# --------------------------------------------------------------------------
# number conversions against numpy / torch (independent implementations)
# --------------------------------------------------------------------------

def test_half_to_double_all_patterns():
    bits = np.arange(65536, dtype=np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.half_to_double(int(b)) for b in bits])
    fin = np.isfinite(ref)
    assert np.array_equal(got[fin], ref[fin])
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    assert np.array_equal(np.isinf(got), np.isinf(ref))


def test_double_to_half_rne():
    xs = np.concatenate([RNG.normal(0, 1, 3000), RNG.normal(0, 1e-5, 1000),
                         RNG.uniform(-7e4, 7e4, 500),
                         # exact ties between neighbouring halves
                         (np.arange(1, 200, dtype=np.float64) + 0.5) / 1024.0,
                         np.array([0.0, -0.0, 65504.0, 65519.99, 65520.0, 6.0e-8, 2.98e-8])])
    for x in xs:
        with np.errstate(over="ignore"):
            ref = np.float16(x).view(np.uint16)
        assert oracle.double_to_half(float(x)) == int(ref), x


def test_float_to_bf16_rne():
    xs = np.concatenate([RNG.normal(0, 1, 5000), RNG.normal(0, 1e-30, 100)]).astype(np.float32)
    ref = torch.from_numpy(xs).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = np.array([oracle.float_to_bf16(float(x)) for x in xs], dtype=np.uint16)
    assert np.array_equal(got, ref)
    assert np.array_equal(oracle.bf16_round(xs.astype(np.float64)), ref)


# --------------------------------------------------------------------------
# bit stream: brute force over every code value at every bit phase
# --------------------------------------------------------------------------

def _pack_by_bitstring(codes, B):
    """Independent packing: build the row's bit string LSB-first, then bytes."""
    out = []
    for row in codes:
        bits = []
        for u in row:
            bits.extend(((int(u) >> j) & 1) for j in range(B))
        row_bytes = [sum(bits[8 * i + j] << j for j in range(8)) for i in range(len(bits) // 8)]
        out.append(row_bytes)
    return np.array(out, dtype=np.uint8)


# widths of the format tools (pack, decode): 1..8; the GEMM paths use 2..4
WIDTHS = [1, 2, 3, 4, 5, 6, 7, 8]


@pytest.mark.parametrize("B", WIDTHS)
def test_pack_exhaustive_small(B):
    K = 8 * (1 << B)             # every code value lands on every bit phase
    codes = np.array([[(k * 5 + r) % (1 << B) for k in range(K)] for r in range(3)],
                     dtype=np.uint8)
    packed = oracle.pack(codes, B)
    assert np.array_equal(packed, _pack_by_bitstring(codes, B))
    assert np.array_equal(oracle.unpack(packed, K, B), codes)


@pytest.mark.parametrize("B", WIDTHS)
def test_pack_roundtrip_random(B):
    codes = RNG.integers(0, 1 << B, size=(7, 384), dtype=np.uint16).astype(np.uint8)
    assert np.array_equal(oracle.unpack(oracle.pack(codes, B), 384, B), codes)


# --------------------------------------------------------------------------
# level arithmetic  (section "CubicQuant 核心")
# --------------------------------------------------------------------------

def _h(x):
    return oracle.double_to_half(x)


def _coord_closed_form(u, B, mode):
    """(signed integer numerator, denominator) of the signed coordinate
    k/Kc: midrise k/Kc = (2u-(2^B-1))/(2^B-1); midtread (u-Kc)/Kc."""
    if mode == oracle.MIDRISE:
        return 2 * u - ((1 << B) - 1), (1 << B) - 1
    Kc = (1 << (B - 1)) - 1
    return u - Kc, Kc


@pytest.mark.parametrize("B", WIDTHS)
@pytest.mark.parametrize("mode", [oracle.MIDRISE, oracle.MIDTREAD])
def test_basis_special_cases(B, mode):
    """q = t (a=1,b=0), q = t^2 (a=0,b=1), q = t^3 (a=0,b=0): each monomial
    of the cubic against the exact rational level sign(k)|k/Kc|^p."""
    if mode == oracle.MIDTREAD and B < 2:
        pytest.skip("the midtread grid needs B >= 2")
    s = 0.75
    ncodes = (1 << B) if mode == oracle.MIDRISE else (1 << B) - 1
    for (a, b, pw) in [(1.0, 0.0, 1), (0.0, 1.0, 2), (0.0, 0.0, 3)]:
        lv = oracle.levels(B, mode, s, _h(a), _h(b))
        for u in range(ncodes):
            num, den = _coord_closed_form(u, B, mode)
            exact = s * math.copysign(1.0, num) * (abs(num) / den) ** pw if num else 0.0
            assert lv[u] == pytest.approx(exact, rel=1e-15, abs=1e-300)


@pytest.mark.parametrize("B", WIDTHS)
def test_uniform_grid_midrise_is_linspace(B):
    """a = 1, b = 0 gives the symmetric uniform grid with 2^B levels spanning
    [-s, s] (section "CubicQuant 核心": the uniform integer grid is an exact
    special case)."""
    s = float(np.float32(0.0123))      # scales are FP32
    lv = oracle.levels(B, oracle.MIDRISE, s, _h(1.0), _h(0.0))
    assert np.allclose(lv, s * np.linspace(-1.0, 1.0, 1 << B), rtol=1e-14, atol=0)
    steps = np.diff(lv)
    assert np.allclose(steps, steps[0], rtol=1e-11)


@pytest.mark.parametrize("B", [2, 3, 4, 5, 6, 7, 8])
def test_uniform_grid_midtread_is_signed_integer(B):
    s = 1.5
    Kc = (1 << (B - 1)) - 1
    lv = oracle.levels(B, oracle.MIDTREAD, s, _h(1.0), _h(0.0))[: 2 * Kc + 1]
    assert np.allclose(lv, s * np.arange(-Kc, Kc + 1) / Kc, rtol=1e-15)


@pytest.mark.parametrize("B", WIDTHS)
@pytest.mark.parametrize("mode", [oracle.MIDRISE, oracle.MIDTREAD])
def test_exact_zero_and_endpoints(B, mode):
    """q(0) = 0 and q(1) = 1 exactly: the extreme codes decode to exactly
    -s and +s for every (a, b), and in midtread the middle code to 0."""
    if mode == oracle.MIDTREAD and B < 2:
        pytest.skip("the midtread grid needs B >= 2")
    for _ in range(200):
        a = float(np.float16(RNG.uniform(0.05, 2.5)))
        b = float(np.float16(RNG.uniform(-2, 2)))
        s = float(np.float32(abs(RNG.normal(0, 0.02)) + 1e-4))
        lv = oracle.levels(B, mode, s, _h(a), _h(b))
        top = (1 << B) - 1 if mode == oracle.MIDRISE else (1 << B) - 2
        assert lv[0] == -s and lv[top] == s
        if mode == oracle.MIDTREAD:
            assert lv[(1 << (B - 1)) - 1] == 0.0


def test_level_is_affine_in_shape_parameters():
    """L(a, b) = a L(1,0) + b L(0,1) + (1-a-b) L(0,0): the derived cubic
    coefficient is c = 1 - a - b."""
    for B in (2, 3, 4):
        for _ in range(50):
            a = float(np.float16(RNG.uniform(0.1, 2)))
            b = float(np.float16(RNG.uniform(-1, 1)))
            s = 0.3
            L = oracle.levels(B, oracle.MIDRISE, s, _h(a), _h(b))
            L10 = oracle.levels(B, oracle.MIDRISE, s, _h(1.0), _h(0.0))
            L01 = oracle.levels(B, oracle.MIDRISE, s, _h(0.0), _h(1.0))
            L00 = oracle.levels(B, oracle.MIDRISE, s, _h(0.0), _h(0.0))
            assert np.allclose(L, a * L10 + b * L01 + (1 - a - b) * L00, rtol=0, atol=1e-15)


# --------------------------------------------------------------------------
# monotonicity (q'(t) > 0 on [0,1])
# --------------------------------------------------------------------------

def _monotone_by_sampling(a, b, n=20001):
    t = np.linspace(0.0, 1.0, n)
    c = 1.0 - a - b
    return bool(np.all(a + 2 * b * t + 3 * c * t * t > 0))


def test_monotone_known_cases():
    assert oracle.is_monotone(_h(1.0), _h(0.0))
    assert not oracle.is_monotone(_h(0.0), _h(0.5))        # q'(0) = 0
    assert not oracle.is_monotone(_h(3.0), _h(-2.0))       # c = 0, q'(1) = -1
    assert oracle.is_monotone(_h(0.25), _h(0.0))           # q' = 1/4 + 9/4 t^2
    assert oracle.is_monotone(_h(0.25), _h(-1.0))          # interior minimum 0.06 > 0
    assert not oracle.is_monotone(_h(0.1), _h(-1.0))       # interior minimum < 0


def test_monotone_matches_dense_sampling():
    disagree = 0
    for _ in range(3000):
        a = float(np.float16(RNG.uniform(-0.5, 3.0)))
        b = float(np.float16(RNG.uniform(-3.0, 3.0)))
        exact = oracle.is_monotone(_h(a), _h(b))
        sampled = _monotone_by_sampling(a, b)
        if exact != sampled:
            # sampling can only miss a negative dip narrower than the grid
            assert not exact and sampled
            disagree += 1
    assert disagree <= 3


def test_monotone_implies_sorted_levels():
    for _ in range(500):
        a = float(np.float16(RNG.uniform(0.05, 2.5)))
        b = float(np.float16(RNG.uniform(-2, 2)))
        if not oracle.is_monotone(_h(a), _h(b)):
            continue
        for B in (2, 3, 4):
            lv = oracle.levels(B, oracle.MIDRISE, 1.0, _h(a), _h(b))
            assert np.all(np.diff(lv) > 0)


def test_synthetic_shape_parameters_are_increasing():
    """Every (a, b) the input generator emits passes the oracle's exact test,
    and the redraw rate matches the part of the box [0.3,1.5] x [-0.6,0.6]
    where q'(1) = 3 - 2a - b <= 0 (a triangle of area 0.09 out of 1.44)."""
    import synthetic
    ab = synthetic.ab(synthetic.make_key("pin"), 20000).view(torch.int16).numpy()
    ab = ab.view(np.uint16)
    assert all(oracle.is_monotone(int(a), int(b)) for a, b in ab)
    a = ab[:, 0].view(np.float16).astype(np.float64)
    b = ab[:, 1].view(np.float16).astype(np.float64)
    assert a.min() >= 0.3 - 1e-3 and a.max() <= 1.5 + 1e-3
    assert b.min() >= -0.6 - 1e-3 and b.max() <= 0.6 + 1e-3
    # first draws only: the acceptance test rejects ~6.25% of them
    key = synthetic.make_key("pin2")
    idx = torch.arange(40000, dtype=torch.int64) * 2
    ca = (synthetic._uniform24(key, idx) * 1.2 + 0.3).to(torch.float16)
    cb = (synthetic._uniform24(key, idx + 1) * 1.2 - 0.6).to(torch.float16)
    acc = synthetic._increasing(ca, cb).numpy()
    exact = np.array([oracle.is_monotone(int(x), int(y)) for x, y in
                      zip(ca.view(torch.int16).numpy().view(np.uint16),
                          cb.view(torch.int16).numpy().view(np.uint16))])
    assert np.array_equal(acc, exact)
    assert abs((1 - acc.mean()) - 0.09 / 1.44) < 0.006
