"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module holds no CubicQuant arithmetic: it only draws codes, scales,
shape parameters, activations and routings with the distributions of the
workloads (Kimi-K3 expert shapes: hidden 7168, moe_intermediate 3072, 896
experts, top-16).  Everything that is large (codes, per-group metadata) is
drawn from a counter-based hash so that the same function gives bit-identical
values on the CPU and on the GPU: the GPU generates full-size layers in place
and the oracle regenerates, on the CPU, only the experts or rows it samples.

The hash is SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom
number generators", OOPSLA 2014; the finaliser as published by Vigna):
    z = key + (i + 1) * 0x9E3779B97F4A7C15
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9
    z = (z ^ (z >> 27)) * 0x94D049BB133111EB
    z =  z ^ (z >> 31)
computed in torch int64 (two's-complement wrap-around) with logical shifts.

Recipes (one per tensor kind):
  codes   u = #{j : r >= T_j}, r the top 32 hash bits, T_j = 2^32 * F(j + 1/2
          - Kc) with F the Laplace(0, beta) CDF, beta = 2^B / 8 code steps:
          the rounded, clamped discretised Laplace centred on the grid middle.
  scales  s = |z| * 0.02 + 1e-3 in FP32, z the standard-normal quantile of the
          hash's top 16 bits ((i + 1/2) / 65536): a 65536-point |N(0, 0.02)|.
  a, b    a = fp16(0.3 + 1.2 u), b = fp16(-0.6 + 1.2 u'), u, u' = 24-bit
          uniforms, FP32 arithmetic then one rounding to FP16, redrawn (next
          counter value, up to 16 draws, else (1, 0)) until the cubic is
          increasing on [0, 1]: q'(t) = a + 2bt + 3ct^2 > 0 with c = 1-a-b,
          checked exactly on the FP16 values as integers.  About 6% of the
          box (2a + b >= 3, where q'(1) <= 0) is redrawn.
  x       torch.randn (CPU generator, seeded) rounded to BF16.
  routes  uniform distinct top-k, or Zipf(s) popularity with Gumbel-top-k;
          weights = softmax of N(0,1) logits over each token's k routes.
"""
from __future__ import annotations

import math
import statistics
from functools import lru_cache

import torch

_MASK64 = (1 << 64) - 1
_GOLDEN = 0x9E3779B97F4A7C15
_M1 = 0xBF58476D1CE4E5B9
_M2 = 0x94D049BB133111EB


def _s64(v: int) -> int:
    """unsigned 64-bit -> signed int64 with the same bits."""
    v &= _MASK64
    return v - (1 << 64) if v >= (1 << 63) else v


def splitmix64_py(key: int, i: int) -> int:
    """Reference (arbitrary-precision Python) SplitMix64 output number i."""
    z = (key + (i + 1) * _GOLDEN) & _MASK64
    z = ((z ^ (z >> 30)) * _M1) & _MASK64
    z = ((z ^ (z >> 27)) * _M2) & _MASK64
    return z ^ (z >> 31)


def _lsr(z: torch.Tensor, r: int) -> torch.Tensor:
    """Logical right shift of int64 bit patterns."""
    return (z >> r) & ((1 << (64 - r)) - 1)


def splitmix64(idx: torch.Tensor, key: int) -> torch.Tensor:
    """SplitMix64 of int64 counters idx under key (int64 bit patterns)."""
    z = idx.to(torch.int64) + 1
    z = z * _s64(_GOLDEN) + _s64(key)
    z = (z ^ _lsr(z, 30)) * _s64(_M1)
    z = (z ^ _lsr(z, 27)) * _s64(_M2)
    return z ^ _lsr(z, 31)


def make_key(*tags) -> int:
    """Mix integer / string tags into one 64-bit key."""
    k = 0x5EED
    for t in tags:
        if isinstance(t, (tuple, list)):
            t = make_key(*t)
        elif isinstance(t, str):
            t = int.from_bytes(t.encode(), "little") & _MASK64
        k = splitmix64_py(k ^ (int(t) & _MASK64), 0)
    return k


def _u32(key: int, start: int, n: int, device) -> torch.Tensor:
    idx = torch.arange(start, start + n, dtype=torch.int64, device=device)
    return _lsr(splitmix64(idx, key), 32)


# --------------------------------------------------------------------------
# codes
# --------------------------------------------------------------------------

def grid_half_range(B: int, mode: int) -> float:
    """Middle of the code range: (2^B-1)/2 for the midrise grid (mode 0),
    2^(B-1)-1 for the midtread grid (mode 1)."""
    return ((1 << B) - 1) / 2.0 if mode == 0 else float((1 << (B - 1)) - 1)


@lru_cache(maxsize=None)
def code_thresholds(B: int, mode: int) -> tuple:
    beta = (1 << B) / 8.0
    Kc = grid_half_range(B, mode)
    ncodes = (1 << B) if mode == 0 else (1 << B) - 1

    def F(x):  # Laplace(0, beta) CDF
        return 0.5 * math.exp(x / beta) if x < 0 else 1.0 - 0.5 * math.exp(-x / beta)

    return tuple(int(round(F(j + 0.5 - Kc) * 4294967296.0)) for j in range(ncodes - 1))


def codes(key: int, N: int, K: int, B: int, mode: int = 0, device="cpu",
          row0: int = 0) -> torch.Tensor:
    """uint8 [N][K] codes of rows row0 .. row0+N-1 of a K-wide matrix."""
    r = _u32(key, row0 * K, N * K, device)
    th = torch.tensor(code_thresholds(B, mode), dtype=torch.int64, device=device)
    # bucketize(right=True) counts the thresholds T_j <= r
    return torch.bucketize(r, th, right=True).to(torch.uint8).view(N, K)


# --------------------------------------------------------------------------
# per-group metadata
# --------------------------------------------------------------------------

@lru_cache(maxsize=None)
def _scale_table_list() -> tuple:
    nd = statistics.NormalDist()
    vals = []
    for i in range(65536):
        z = abs(nd.inv_cdf((i + 0.5) / 65536.0))
        vals.append(z * 0.02 + 1e-3)
    return tuple(vals)


def _scale_table(device) -> torch.Tensor:
    return torch.tensor(_scale_table_list(), dtype=torch.float64).to(torch.float32).to(device)


def scales(key: int, n_groups_total: int, device="cpu", start: int = 0) -> torch.Tensor:
    """FP32 scales of groups start .. start+n-1 (flat group index)."""
    idx = _lsr(splitmix64(torch.arange(start, start + n_groups_total, dtype=torch.int64,
                                       device=device), key), 48)
    return _scale_table(device)[idx]


def _uniform24(key: int, idx: torch.Tensor) -> torch.Tensor:
    return _lsr(splitmix64(idx, key), 40).to(torch.float32) * (2.0 ** -24)


def _increasing(a: torch.Tensor, b: torch.Tensor) -> torch.Tensor:
    """Input-recipe acceptance test: q'(t) = a + 2bt + 3ct^2 > 0 on [0, 1],
    c = 1 - a - b, for FP16 a, b.  FP16 values are multiples of 2^-24, so
    A = a 2^24, Bv = b 2^24 and C = 2^24 - A - Bv are exact integers and the
    test is exact: q'(0) > 0, q'(1) > 0, and a negative interior minimum
    (when c > 0 and 0 < -b < 3c) is excluded by Bv^2 < 3 A C."""
    one = 1 << 24
    A = torch.round(a.to(torch.float64) * one).to(torch.int64)
    Bv = torch.round(b.to(torch.float64) * one).to(torch.int64)
    C = one - A - Bv
    ok = (A > 0) & (3 * one - 2 * A - Bv > 0)
    interior = (C > 0) & (-Bv > 0) & (-Bv < 3 * C)
    return ok & ~(interior & (Bv * Bv >= 3 * A * C))


def ab(key: int, n_groups_total: int, device="cpu", start: int = 0,
       max_draws: int = 16) -> torch.Tensor:
    """FP16 [n][2] (a, b) of groups start .. start+n-1."""
    gidx = torch.arange(start, start + n_groups_total, dtype=torch.int64, device=device)
    a = torch.ones(n_groups_total, dtype=torch.float16, device=device)
    b = torch.zeros(n_groups_total, dtype=torch.float16, device=device)
    todo = torch.arange(n_groups_total, device=device)
    for draw in range(max_draws):
        if todo.numel() == 0:
            break
        idx = gidx[todo] * (2 * max_draws) + 2 * draw
        ca = (_uniform24(key, idx) * 1.2 + 0.3).to(torch.float16)
        cb = (_uniform24(key, idx + 1) * 1.2 - 0.6).to(torch.float16)
        ok = _increasing(ca, cb)
        a[todo[ok]] = ca[ok]
        b[todo[ok]] = cb[ok]
        todo = todo[~ok]
    return torch.stack([a, b], dim=-1)


def matrix(tag, N: int, K: int, B: int, G: int, mode: int = 0, device="cpu",
           row0: int = 0, nrows: int | None = None):
    """Codes [nrows][K] uint8, scales [nrows][K/G] f32, ab [nrows][K/G][2] f16
    for rows row0.. of the N x K matrix identified by tag (a tuple)."""
    nrows = N - row0 if nrows is None else nrows
    key = make_key(*tag)
    ng = K // G
    c = codes(make_key(key, "codes"), nrows, K, B, mode, device, row0)
    s = scales(make_key(key, "scales"), nrows * ng, device, row0 * ng).view(nrows, ng)
    a = ab(make_key(key, "ab"), nrows * ng, device, row0 * ng).view(nrows, ng, 2)
    return c, s, a


# --------------------------------------------------------------------------
# activations and routing
# --------------------------------------------------------------------------

def activations(seed: int, M: int, K: int) -> torch.Tensor:
    """BF16 [M][K] ~ N(0,1), drawn on the CPU."""
    g = torch.Generator().manual_seed(int(seed))
    return torch.randn(M, K, generator=g, dtype=torch.float32).to(torch.bfloat16)


def laplace_weights(seed: int, n: int, scale: float) -> torch.Tensor:
    """FP32 i.i.d. Laplace(0, scale) by inverse CDF of a seeded uniform."""
    g = torch.Generator().manual_seed(int(seed))
    u = torch.rand(n, generator=g, dtype=torch.float64) - 0.5
    w = -scale * torch.sign(u) * torch.log1p(-2.0 * torch.abs(u))
    return w.to(torch.float32)


def routing_uniform(seed: int, T: int, E: int, k: int):
    """k distinct experts per token, uniform; softmax(N(0,1)) weights."""
    g = torch.Generator().manual_seed(int(seed))
    keys = torch.rand(T, E, generator=g, dtype=torch.float64)
    ids = torch.topk(keys, k, dim=1).indices.to(torch.int32)
    logits = torch.randn(T, k, generator=g, dtype=torch.float32)
    return ids, torch.softmax(logits, dim=1)


def routing_zipf(seed: int, T: int, E: int, k: int, s: float = 1.1):
    """k distinct experts per token drawn without replacement with Zipf(s)
    popularity p_i ~ i^-s over ranks 1..E (ranks mapped to expert ids by a
    seeded permutation), via Gumbel-top-k; softmax(N(0,1)) weights."""
    g = torch.Generator().manual_seed(int(seed))
    perm = torch.randperm(E, generator=g)
    logp = -s * torch.log(torch.arange(1, E + 1, dtype=torch.float64))
    logp_e = torch.empty(E, dtype=torch.float64)
    logp_e[perm] = logp
    u = torch.rand(T, E, generator=g, dtype=torch.float64).clamp_min(1e-300)
    gumbel = -torch.log(-torch.log(u))
    ids = torch.topk(logp_e[None, :] + gumbel, k, dim=1).indices.to(torch.int32)
    logits = torch.randn(T, k, generator=g, dtype=torch.float32)
    return ids, torch.softmax(logits, dim=1)


def expert_bits(seed: int, E: int, probs=(0.6, 0.3, 0.1), widths=(2, 3, 4)):
    """Per-expert bit width drawn with the given probabilities."""
    g = torch.Generator().manual_seed(int(seed))
    u = torch.rand(E, generator=g, dtype=torch.float64)
    cum = torch.cumsum(torch.tensor(probs, dtype=torch.float64), 0)
    idx = torch.searchsorted(cum, u, right=True).clamp_max(len(widths) - 1)
    return torch.tensor(widths, dtype=torch.int32)[idx]
