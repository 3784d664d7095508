"""CPU oracle for CubicQuant weight-only GEMM -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the CUDA library and
its Python binding in ``bit_non_uniform_b200``) never does.

The arithmetic lives in ``cq_oracle.c`` (plain C, FP64, naive loops); this
module only marshals numpy arrays into it, and orchestrates the MoE layer as
the plain composition of those calls.  Source of the method: the ModelScope
article "CubicQuant：用三次曲线重塑低比特量化，Kimi K3 2.5Bit 模型首发实践"
(sections "CubicQuant 核心" for the format, "存储开销是透明的：B+64/G bit" for
the storage identity, "从曲线到量化器：数据无关的组内拟合" for the fitter and
"压缩权重必须“边解码、边计算”" for the A16 execution path).

Parity status: every function here is pinned by a not-gpu test in
``tests/test_oracle_*.py``.  The fitter is pinned by invariants (brute-force
nearest level, the exact 1-D optimum as a lower bound, the clipped-uniform
grid as an upper bound, consistency of its outputs) and, in midtread mode,
by the article's W4 G128 NRMSE table.  The fitter's *midrise* NRMSE
statistics: parity unpinned (the article prints none for that grid).

The Dynamic-A8 functions (``carrier``, ``quant_rows``, ``gemm_a8``, ``fit``
with ``lam > 0``) are pinned in ``tests/test_oracle_a8.py`` by exact rational
arithmetic, brute force on small cases, the special case where A8 equals the
A16 product exactly, and the joint fit's invariants.

The population analysis (``pop_*``, ``gap_recovery``: the error bound of
"为什么只用两个形状参数？" evaluated on the Gaussian and Laplace densities) is
pinned by quadrature, closed forms, the classical Lloyd-Max and optimum
uniform quantizer tables, the Panter-Dite limit, and the article's W4..W8
gap-recovery ranges (midtread grid) in ``tests/test_oracle_population.py``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

MIDRISE = 0
MIDTREAD = 1

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "cq_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile cq_oracle.c into liboracle.so (gcc, no FMA contraction)."""
    if force or not os.path.exists(_LIB_PATH) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    ):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-ffp-contract=off", "-fPIC", "-shared", "-pthread",
             _SRC, "-o", tmp, "-lm"]
        )
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is not None:
        return _lib
    build()
    lib = ctypes.CDLL(_LIB_PATH)
    P = ctypes.c_void_p
    i64, i32, dbl, flt = ctypes.c_int64, ctypes.c_int, ctypes.c_double, ctypes.c_float
    u16 = ctypes.c_uint16
    sig = {
        "cqo_half_to_double": (dbl, [u16]),
        "cqo_double_to_half": (u16, [dbl]),
        "cqo_float_to_bf16": (u16, [flt]),
        "cqo_bf16_to_double": (dbl, [u16]),
        "cqo_pack": (None, [P, i64, i64, i32, P]),
        "cqo_unpack": (None, [P, i64, i64, i32, P]),
        "cqo_q": (dbl, [dbl, dbl, dbl]),
        "cqo_level": (dbl, [i32, i32, i32, flt, u16, u16]),
        "cqo_levels": (None, [i32, i32, flt, u16, u16, P]),
        "cqo_is_monotone": (i32, [u16, u16]),
        "cqo_decode": (None, [P, P, P, i64, i64, i32, i32, i32, P, P, P]),
        "cqo_gemm": (None, [P, i64, P, P, P, i64, i64, i32, i32, i32, P, P, i32]),
        "cqo_gemm_ex": (None, [P, i64, P, P, P, i64, i64, i32, i32, i32, i32, P, P, i32]),
        "cqo_nearest": (i32, [P, i32, dbl]),
        "cqo_nearest_bruteforce": (i32, [P, i32, dbl]),
        "cqo_fit": (None, [P, i64, i32, i32, i32, P, i32, P, i32, P, i32, i32,
                           P, P, P, P, P, i32]),
        "cqo_fit_joint": (None, [P, i64, i32, i32, i32, P, i32, P, i32, P, i32, i32, dbl,
                                 P, P, P, P, P, P, i32]),
        "cqo_optimal_sse": (dbl, [P, i32, i32]),
        "cqo_carrier": (i32, [i32, i32, i32, u16, u16]),
        "cqo_carriers": (None, [i32, i32, u16, u16, P]),
        "cqo_quant_rows": (None, [P, i64, i64, P, P]),
        "cqo_gemm_a8": (None, [P, P, i64, P, P, P, i64, i64, i32, i32, i32, P, P]),
        "cqo_num_threads": (i32, [i32]),
        "cqo_pop_moments": (None, [i32, dbl, dbl, P]),
        "cqo_pop_mse": (dbl, [i32, P, i32]),
        "cqo_pop_lloyd_max": (dbl, [i32, i32, i32, dbl, P]),
        "cqo_pop_shape": (None, [i32, dbl, dbl, P]),
        "cqo_pop_monotone": (i32, [dbl, dbl]),
        "cqo_pop_best_scale": (dbl, [i32, P, i32, P]),
        "cqo_pop_cubic": (dbl, [i32, i32, P, P, P]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    _lib = lib
    return lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


# --------------------------------------------------------------------------
# number helpers
# --------------------------------------------------------------------------

def half_to_double(h: int) -> float:
    return _load().cqo_half_to_double(int(h))


def double_to_half(x: float) -> int:
    return int(_load().cqo_double_to_half(float(x)))


def float_to_bf16(x: float) -> int:
    return int(_load().cqo_float_to_bf16(float(x)))


def bf16_to_double(h: int) -> float:
    return _load().cqo_bf16_to_double(int(h))


def num_threads() -> int:
    return int(_load().cqo_num_threads(0))


# --------------------------------------------------------------------------
# format
# --------------------------------------------------------------------------

def bits_per_weight(B: int, G: int) -> float:
    """Storage per weight: G*B payload bits + 32 (FP32 s) + 32 (two FP16) per
    group, i.e. B + 64/G bits ("存储开销是透明的：B+64/G bit")."""
    return (G * B + 32 + 32) / G


def pack(codes: np.ndarray, B: int) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    N, K = codes.shape
    assert (K * B) % 8 == 0
    out = np.empty((N, K * B // 8), dtype=np.uint8)
    _load().cqo_pack(_ptr(codes), N, K, B, _ptr(out))
    return out


def unpack(packed: np.ndarray, K: int, B: int) -> np.ndarray:
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    N = packed.shape[0]
    out = np.empty((N, K), dtype=np.uint8)
    _load().cqo_unpack(_ptr(packed), N, K, B, _ptr(out))
    return out


def q(t: float, a: float, b: float) -> float:
    return _load().cqo_q(float(t), float(a), float(b))


def level(u: int, B: int, mode: int, s: float, a_h: int, b_h: int) -> float:
    return _load().cqo_level(int(u), B, mode, float(s), int(a_h), int(b_h))


def levels(B: int, mode: int, s: float, a_h: int, b_h: int) -> np.ndarray:
    out = np.empty(1 << B, dtype=np.float64)
    _load().cqo_levels(B, mode, float(s), int(a_h), int(b_h), _ptr(out))
    return out


def is_monotone(a_h: int, b_h: int) -> bool:
    return bool(_load().cqo_is_monotone(int(a_h), int(b_h)))


def decode(packed, scales, ab, N, K, B, G, mode=MIDRISE):
    """Returns (w64, w32, w16bits): exact FP64 levels, FP32 and BF16 roundings."""
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.float32)
    ab = np.ascontiguousarray(ab, dtype=np.uint16)
    w64 = np.empty((N, K), dtype=np.float64)
    w32 = np.empty((N, K), dtype=np.float32)
    w16 = np.empty((N, K), dtype=np.uint16)
    _load().cqo_decode(_ptr(packed), _ptr(scales), _ptr(ab), N, K, B, G, mode,
                       _ptr(w64), _ptr(w32), _ptr(w16))
    return w64, w32, w16


def gemm(x_bf16bits, packed, scales, ab, N, K, B, G, mode=MIDRISE, nthreads=0,
         operand="f64"):
    """y[m][n] = sum_k x[m][k] w[n][k] in FP64 and bound = sum_k |x w|.

    x_bf16bits: uint16 [M][K] (bfloat16 bit patterns).
    operand "f64": w is the exact level; "bf16": w is that level rounded to
    FP32 and then to BF16, the model-dtype operand of the A16 path
    ("压缩权重必须“边解码、边计算”")."""
    x = np.ascontiguousarray(x_bf16bits, dtype=np.uint16)
    M = x.shape[0]
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.float32)
    ab = np.ascontiguousarray(ab, dtype=np.uint16)
    y = np.empty((M, N), dtype=np.float64)
    bound = np.empty((M, N), dtype=np.float64)
    if operand not in ("f64", "bf16"):
        raise ValueError(operand)
    _load().cqo_gemm_ex(_ptr(x), M, _ptr(packed), _ptr(scales), _ptr(ab), N, K, B, G,
                        mode, int(operand == "bf16"), _ptr(y), _ptr(bound), nthreads)
    return y, bound


def silu(g):
    """silu(g) = g / (1 + exp(-g)), FP64."""
    g = np.asarray(g, dtype=np.float64)
    return g / (1.0 + np.exp(-g))


def swiglu(y: np.ndarray) -> np.ndarray:
    """SwiGLU over the two halves of the last axis: gate = first half,
    up = second half, h = silu(gate) * up (FP64)."""
    n2 = y.shape[-1] // 2
    return silu(y[..., :n2]) * y[..., n2:]


def bf16_round(v: np.ndarray) -> np.ndarray:
    """FP64 -> FP32 (RNE) -> BF16 (RNE); returns the uint16 bit patterns."""
    f = np.ascontiguousarray(np.asarray(v, dtype=np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    nan = (u & 0x7F800000) == 0x7F800000
    nan &= (u & 0x007FFFFF) != 0
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)
    r[nan] = 0x7FC0
    return r


def bf16_bits_to_f64(h: np.ndarray) -> np.ndarray:
    h = np.ascontiguousarray(h, dtype=np.uint16)
    return (h.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# --------------------------------------------------------------------------
# MoE layer: the composition gate/up -> SwiGLU -> down -> weighted combine
# --------------------------------------------------------------------------

def f32_down(v: np.ndarray) -> np.ndarray:
    """Largest FP32 value <= v (elementwise, FP64 in, FP32 out)."""
    v = np.asarray(v, dtype=np.float64)
    f = v.astype(np.float32)
    over = f.astype(np.float64) > v
    f[over] = np.nextafter(f[over], np.float32(-np.inf))
    return f


def f32_up(v: np.ndarray) -> np.ndarray:
    """Smallest FP32 value >= v (elementwise, FP64 in, FP32 out)."""
    v = np.asarray(v, dtype=np.float64)
    f = v.astype(np.float32)
    under = f.astype(np.float64) < v
    f[under] = np.nextafter(f[under], np.float32(np.inf))
    return f


def bf16_rne_of_f32(f: np.ndarray) -> np.ndarray:
    """FP32 -> BF16 round to nearest even; returns the BF16 values as FP64."""
    u = np.ascontiguousarray(f, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint32) << 16
    return r.view(np.float32).astype(np.float64)


def bf16_up_bits(v: np.ndarray) -> np.ndarray:
    """Bit patterns of the smallest BF16 value >= v, for finite v >= 0."""
    u = f32_up(v).view(np.uint32).astype(np.uint64)
    r = ((u + 0xFFFF) >> 16).astype(np.uint16)
    return r


def moe_routes(tokens_bf16bits, topk_ids, experts, H, I, G, mode=MIDRISE,
               routes=None, nthreads=0, rel=2e-3, abs_=1e-6, operand="f64"):
    """Per-route outputs of the routed-expert FFN, FP64.

    experts[e] = dict(B_gu, packed_gu [2I][H*B/8], scales_gu, ab_gu,
                      B_dn, packed_dn [H][I*B/8], scales_dn, ab_dn)
    (a callable e -> dict is accepted too, so large layers can be
    regenerated one expert at a time).
    Route r = (t, j) uses expert topk_ids[t][j]:
        gu = W_gu x_t (2I outputs), h = bf16(silu(gu[:I]) * gu[I:]),
        y_r = W_dn h (H outputs).
    h is rounded to BF16 because the chain keeps the activation between the
    two products in the model dtype ("压缩权重必须“边解码、边计算”").
    routes: optional list of flat route indices r = t*k + j to evaluate.
    operand: the weight operand of both products ("f64" exact levels, or
    "bf16" the model-dtype operand, see gemm()); rel, abs_: the per-product
    tolerance that is propagated (2e-3, 1e-6: the contract's GEMM bound for
    the exact levels; with the BF16 operand, the products differ from the
    kernel's only by the order of the FP32 sums).

    Returns dict r -> (y_r, bound_r, tol_r), all [H] float64:
      bound_r = sum_i |w_dn[n][i] h_i|;
      tol_r   = rel*bound_r + abs_ (the down product's own tolerance) plus
                (1 + rel) * sum_i |w_dn[n][i]| dh_i, the effect of the
                gate/up product's tolerance on h.  Each g, u may be off by
                e = rel*sum|w x| + abs_, which moves the unrounded h =
                silu(g) u by at most eh = |silu'(g)| |u| e_g + |silu(g)| e_u
                + e_g e_u (+ FP32 evaluation, 1e-6 |h|).  The GPU's h is the
                BF16 rounding of a value inside [h - eh, h + eh]; rounding is
                monotone, so it lies between the roundings of the interval's
                ends, and dh_i is the larger distance from the oracle's h_i to
                those two: zero wherever no BF16 rounding boundary falls
                inside the interval (then both sides round to the same h_i),
                one BF16 step where one does."""
    T, k = topk_ids.shape
    if routes is None:
        routes = range(T * k)
    by_expert: dict[int, list[int]] = {}
    for r in routes:
        e = int(topk_ids[r // k, r % k])
        by_expert.setdefault(e, []).append(int(r))
    get = experts if callable(experts) else (lambda e: experts[e])
    out = {}
    for e in sorted(by_expert):
        rs = by_expert[e]
        ex = get(e)
        xs = np.ascontiguousarray(tokens_bf16bits[[r // k for r in rs]])
        gu, bgu = gemm(xs, ex["packed_gu"], ex["scales_gu"], ex["ab_gu"], 2 * I, H,
                       ex["B_gu"], G, mode, nthreads, operand)
        hf = swiglu(gu)
        hb = bf16_round(hf)
        h = bf16_bits_to_f64(hb)
        g, u = gu[:, :I], gu[:, I:]
        eg, eu = rel * bgu[:, :I] + abs_, rel * bgu[:, I:] + abs_
        sig = 1.0 / (1.0 + np.exp(-g))
        dsilu = np.abs(sig * (1.0 + g * (1.0 - sig)))
        eh = dsilu * np.abs(u) * eg + np.abs(g * sig) * eu + eg * eu + 1e-6 * np.abs(hf)
        lo = bf16_rne_of_f32(f32_down(hf - eh))
        hi = bf16_rne_of_f32(f32_up(hf + eh))
        dh = np.maximum(np.maximum(h - lo, hi - h), 0.0)
        # one pass over W_dn: the rows of h give y and its bound; the rows of
        # dh (non-negative, rounded up to BF16) give sum_i |w_dn[n][i]| dh_i
        # from above as their bound
        xd = np.ascontiguousarray(np.concatenate([hb, bf16_up_bits(dh)]))
        yy, bb = gemm(xd, ex["packed_dn"], ex["scales_dn"], ex["ab_dn"], H, I,
                      ex["B_dn"], G, mode, nthreads, operand)
        n = len(rs)
        y, bnd, prop = yy[:n], bb[:n], bb[n:]
        for i, r in enumerate(rs):
            out[r] = (y[i], bnd[i], rel * bnd[i] + abs_ + (1.0 + rel) * prop[i])
    return out


def moe_combine(route_out, topk_w, tokens=None):
    """out[t] = sum_j w[t][j] * y_(t,j) in FP64 (j ascending); also returns
    the matching bound sum_j |w| * bound_(t,j)."""
    T, k = topk_w.shape
    tokens = range(T) if tokens is None else tokens
    res = {}
    for t in tokens:
        acc = None
        bnd = None
        for j in range(k):
            y, b = route_out[t * k + j][:2]
            w = float(topk_w[t, j])
            acc = w * y if acc is None else acc + w * y
            bnd = abs(w) * b if bnd is None else bnd + abs(w) * b
        res[t] = (acc, bnd)
    return res


# --------------------------------------------------------------------------
# fitter
# --------------------------------------------------------------------------

def default_grids():
    """Candidate grids of the data-free fitter (the article gives none):
    a in [1/16, 5/2] and b in [-2, 2], both in steps of 1/16 (all exact in
    FP16), clip ratio alpha in {0.30, 0.31, ..., 1.00}."""
    a = np.arange(1, 41, dtype=np.float64) / 16.0
    b = np.arange(-32, 33, dtype=np.float64) / 16.0
    alpha = np.round(np.arange(30, 101, dtype=np.float64)) / 100.0
    return a, b, alpha


def fit(w: np.ndarray, G: int, B: int, mode=MIDRISE, uniform_only=False,
        grids=None, nthreads=0, lam=0.0):
    """Fit every group of w (flattened, length multiple of G), minimising
    L_C + lam * L_A8 per group (lam = 0: the A16 fit; lam > 0: the A8
    carrier correction of "一份 checkpoint，同时服务 A16 与 Dynamic A8").

    Returns dict(codes [ng][G] uint8, s [ng] f32, ab [ng][2] fp16 bits,
    sse [ng] (L_C), sse_a8 [ng] (L_A8 of the same codes), clipped [ng])."""
    w = np.ascontiguousarray(np.asarray(w, dtype=np.float64).reshape(-1, G))
    ng = w.shape[0]
    a, b, alpha = grids if grids is not None else default_grids()
    a = np.ascontiguousarray(a, dtype=np.float64)
    b = np.ascontiguousarray(b, dtype=np.float64)
    alpha = np.ascontiguousarray(alpha, dtype=np.float64)
    codes = np.empty((ng, G), dtype=np.uint8)
    s = np.empty(ng, dtype=np.float32)
    ab = np.empty((ng, 2), dtype=np.uint16)
    sse = np.empty(ng, dtype=np.float64)
    clipped = np.empty(ng, dtype=np.int32)
    sse_a8 = np.empty(ng, dtype=np.float64)
    _load().cqo_fit_joint(_ptr(w), ng, G, B, mode, _ptr(a), len(a), _ptr(b), len(b),
                          _ptr(alpha), len(alpha), int(uniform_only), float(lam), _ptr(codes),
                          _ptr(s), _ptr(ab), _ptr(sse), _ptr(clipped), _ptr(sse_a8), nthreads)
    return dict(codes=codes, s=s, ab=ab, sse=sse, sse_a8=sse_a8, clipped=clipped)


def nrmse(sse: np.ndarray, w: np.ndarray) -> float:
    """Group reconstruction error normalised by source weight energy,
    sqrt(sum SSE / sum w^2) over the tensor."""
    return float(np.sqrt(np.sum(sse) / np.sum(np.asarray(w, dtype=np.float64) ** 2)))


def nearest(levels_sorted: np.ndarray, v: float, brute: bool = False) -> int:
    lv = np.ascontiguousarray(levels_sorted, dtype=np.float64)
    f = _load().cqo_nearest_bruteforce if brute else _load().cqo_nearest
    return int(f(_ptr(lv), len(lv), float(v)))


def optimal_sse(v: np.ndarray, nlev: int) -> float:
    v = np.ascontiguousarray(v, dtype=np.float64)
    return float(_load().cqo_optimal_sse(_ptr(v), len(v), nlev))


# --------------------------------------------------------------------------
# Dynamic A8 ("一份 checkpoint，同时服务 A16 与 Dynamic A8")
# --------------------------------------------------------------------------

def carrier(u: int, B: int, mode: int, a_h: int, b_h: int) -> int:
    """INT8 carrier of code u: RNE(127 sign(k) q(t)), saturated to +-127."""
    return int(_load().cqo_carrier(u, B, mode, a_h, b_h))


def carriers(B: int, mode: int, a_h: int, b_h: int) -> np.ndarray:
    out = np.empty(1 << B, dtype=np.int8)
    _load().cqo_carriers(B, mode, a_h, b_h, _ptr(out))
    return out


def quant_rows(x_bf16bits: np.ndarray):
    """Per-row dynamic INT8 quantization of bf16 activations [M][K]:
    returns (xq int8 [M][K], absmax f32 [M])."""
    x = np.ascontiguousarray(x_bf16bits, dtype=np.uint16)
    M, K = x.shape
    xq = np.empty((M, K), dtype=np.int8)
    absmax = np.empty(M, dtype=np.float32)
    _load().cqo_quant_rows(_ptr(x), M, K, _ptr(xq), _ptr(absmax))
    return xq, absmax


def gemm_a8(xq, absmax, packed, scales, ab, N, K, B, G, mode=MIDRISE):
    """Dynamic-A8 GEMM in FP64 from exact integer group sums: (y, bound),
    both f64 [M][N]."""
    xq = np.ascontiguousarray(xq, dtype=np.int8)
    absmax = np.ascontiguousarray(absmax, dtype=np.float32)
    packed = np.ascontiguousarray(packed, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.float32)
    ab = np.ascontiguousarray(ab, dtype=np.uint16)
    M = xq.shape[0]
    y = np.empty((M, N), dtype=np.float64)
    bound = np.empty((M, N), dtype=np.float64)
    _load().cqo_gemm_a8(_ptr(xq), _ptr(absmax), M, _ptr(packed), _ptr(scales), _ptr(ab),
                        N, K, B, G, mode, _ptr(y), _ptr(bound))
    return y, bound


# --------------------------------------------------------------------------
# population analysis (the error bound of "为什么只用两个形状参数？")
# --------------------------------------------------------------------------

GAUSS = 0      # N(0, 1)
LAPLACE = 1    # Laplace with unit variance


def pop_moments(dist: int, a: float, b: float) -> np.ndarray:
    """Integrals of x^j f(x) over [a, b], j = 0, 1, 2 (closed forms)."""
    m = np.zeros(3)
    _load().cqo_pop_moments(dist, float(a), float(b), _ptr(m))
    return m


def pop_mse(dist: int, levels: np.ndarray) -> float:
    """MSE of the nearest-level quantizer with these levels on the density."""
    lv = np.ascontiguousarray(np.sort(np.asarray(levels, dtype=np.float64)))
    return float(_load().cqo_pop_mse(dist, _ptr(lv), len(lv)))


def pop_lloyd_max(dist: int, n: int, max_iter: int = 100000, tol: float = 1e-13):
    """n-level Lloyd-Max quantizer of the density: (MSE, ascending levels)."""
    lv = np.zeros(n)
    mse = _load().cqo_pop_lloyd_max(dist, n, max_iter, tol, _ptr(lv))
    return float(mse), lv


def pop_shape(n: int, a: float, b: float) -> np.ndarray:
    """The n cubic levels on [-1, 1] (coordinate (2i - (n-1)) / (n-1))."""
    out = np.zeros(n)
    _load().cqo_pop_shape(n, float(a), float(b), _ptr(out))
    return out


def pop_monotone(a: float, b: float) -> bool:
    return bool(_load().cqo_pop_monotone(float(a), float(b)))


def pop_best_scale(dist: int, shape: np.ndarray):
    """min over s of the MSE of s * shape: (MSE, s)."""
    sh = np.ascontiguousarray(shape, dtype=np.float64)
    s = ctypes.c_double()
    mse = _load().cqo_pop_best_scale(dist, _ptr(sh), len(sh), ctypes.byref(s))
    return float(mse), s.value


def pop_uniform(dist: int, n: int):
    """Best clipped uniform (INT) quantizer with n levels: (MSE, s)."""
    return pop_best_scale(dist, pop_shape(n, 1.0, 0.0))


def pop_cubic(dist: int, n: int):
    """Best n-level cubic quantizer: (MSE, a, b, s)."""
    a, b, s = ctypes.c_double(), ctypes.c_double(), ctypes.c_double()
    mse = _load().cqo_pop_cubic(dist, n, ctypes.byref(a), ctypes.byref(b), ctypes.byref(s))
    return float(mse), a.value, b.value, s.value


def levels_of_width(B: int, mode: int) -> int:
    """Distinct levels a B-bit code carries: 2^B on the midrise grid, 2^B - 1
    on the midtread grid (its last code is unused)."""
    return (1 << B) if mode == MIDRISE else (1 << B) - 1


def gap_recovery(dist: int, B: int, mode: int) -> dict:
    """Share of the best-INT / Lloyd-Max MSE gap that the best cubic closes,
    (D_int - D_cubic) / (D_int - D_lloyd_max), all three with the same number
    of levels, on the density itself (no sample)."""
    n = levels_of_width(B, mode)
    d_lm, _ = pop_lloyd_max(dist, n)
    d_int, s_int = pop_uniform(dist, n)
    d_cu, a, b, s = pop_cubic(dist, n)
    return dict(n=n, lloyd_max=d_lm, int=d_int, int_s=s_int, cubic=d_cu, a=a, b=b, s=s,
                recovered=(d_int - d_cu) / (d_int - d_lm))

