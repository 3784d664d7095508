"""GPU parity of the grouped MoE layer (cq_moe_grouped_gemm) against the CPU
oracle's composition gate/up -> SwiGLU -> BF16 h -> down -> weighted combine.

Every route is checked twice (oracle.moe_routes):
  * the contract: exact FP64 levels in both products; the tolerance is the
    per-GEMM bound 2e-3 * sum|w h| + 1e-6 of the down product plus the
    effect on h of the gate/up product's own bound, through SwiGLU and |W_dn|
    (one BF16 step of h only where a BF16 rounding boundary lies within
    reach of the exact h);
  * the tight check: the model-dtype (BF16) operand the kernels multiply, so
    the oracle takes the BF16 rounding of h in the kernel's precision and the
    products differ from the kernel's only by the order of the FP32 sums
    (2e-5 * bound + 1e-7, twice the GEMM tests' decoded-BF16 allowance, as
    each route goes through two products).
Combined outputs use the weighted sum of the per-route tolerances.  The
large layers' codes are drawn on the GPU by the seeded generator (bit-equal
to its CPU draws, see test_gpu_parity) and packed on the host by the oracle.
"""
import os
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest
import torch

import oracle
import synthetic

pytestmark = pytest.mark.gpu

REL, ABS = 2e-3, 1e-6
TOL = {"f64": (REL, ABS), "bf16": (2e-5, 1e-7)}
_GEN_LOCK = threading.Lock()


@pytest.fixture(scope="module")
def cq():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import bit_non_uniform_b200 as cq
    cq.lib()
    return cq


def u16(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def expert_cpu(tag, e, B, H, I, G):
    """One expert's matrices on the CPU (codes, scales, ab)."""
    gu = synthetic.matrix((tag, "gu", e), 2 * I, H, B, G)
    dn = synthetic.matrix((tag, "dn", e), H, I, B, G)
    return gu, dn


def expert_gpu(cq, tag, e, B, H, I, G):
    gu = synthetic.matrix((tag, "gu", e), 2 * I, H, B, G, device="cuda")
    dn = synthetic.matrix((tag, "dn", e), H, I, B, G, device="cuda")
    return dict(B_gu=B, packed_gu=cq.cq_pack(gu[0], B), scales_gu=gu[1], ab_gu=gu[2],
                B_dn=B, packed_dn=cq.cq_pack(dn[0], B), scales_dn=dn[1], ab_dn=dn[2])


def expert_oracle(tag, e, B, H, I, G):
    (cg, sg, ag), (cd, sd, ad) = expert_cpu(tag, e, B, H, I, G)
    return dict(B_gu=B, packed_gu=oracle.pack(cg.numpy(), B), scales_gu=sg.numpy(), ab_gu=u16(ag),
                B_dn=B, packed_dn=oracle.pack(cd.numpy(), B), scales_dn=sd.numpy(), ab_dn=u16(ad))


def expert_oracle_from_device(tag, e, B, H, I, G):
    """One expert's matrices drawn on the GPU by the seeded generator, copied
    to the host and packed by the oracle."""
    with _GEN_LOCK:
        gu = [t.cpu() for t in synthetic.matrix((tag, "gu", e), 2 * I, H, B, G, device="cuda")]
        dn = [t.cpu() for t in synthetic.matrix((tag, "dn", e), H, I, B, G, device="cuda")]
    return dict(B_gu=B, packed_gu=oracle.pack(gu[0].numpy(), B), scales_gu=gu[1].numpy(),
                ab_gu=u16(gu[2]), B_dn=B, packed_dn=oracle.pack(dn[0].numpy(), B),
                scales_dn=dn[1].numpy(), ab_dn=u16(dn[2]))


def oracle_routes(x_u16, ids_np, get_expert, H, I, G, routes, tight_experts=None):
    """{"f64": {r: (y, bound, tol)}, "bf16": {...}} for the given routes,
    one expert per job on a thread pool (the C oracle runs outside the GIL).
    The tight (BF16-operand) reference is computed for every expert, or only
    for those in tight_experts."""
    k = ids_np.shape[1]
    by_e = {}
    for r in routes:
        by_e.setdefault(int(ids_np[r // k, r % k]), []).append(int(r))
    cores = os.cpu_count() or 8
    workers = max(1, min(len(by_e), cores // 2))

    def job(e):
        ex = get_expert(e)
        out = {}
        for op in ("f64", "bf16"):
            if op == "bf16" and tight_experts is not None and e not in tight_experts:
                continue
            rel, abs_ = TOL[op]
            out[op] = oracle.moe_routes(x_u16, ids_np, {e: ex}, H, I, G, routes=by_e[e],
                                        nthreads=2, rel=rel, abs_=abs_, operand=op)
        return out

    ref = {"f64": {}, "bf16": {}}
    with ThreadPoolExecutor(workers) as pool:
        for out in pool.map(job, sorted(by_e)):
            for op, d in out.items():
                ref[op].update(d)
    return ref


def check_routes(ro, ref, routes=None, what=""):
    """Every element of every route within its tolerance; returns (and
    prints) the worst error / tolerance ratio."""
    worst = 0.0
    rs = list(ref) if routes is None else [r for r in routes if r in ref]
    assert rs, "no route to check"
    got_all = ro.double().cpu().numpy()
    for r in rs:
        y, bnd, tol = ref[r]
        err = np.abs(got_all[r] - y)
        ratio = float(np.max(err / tol))
        worst = max(worst, ratio)
        assert ratio <= 1.0, f"{what} route {r}: worst ratio {ratio:.3f}"
    print(f"{what}: {len(rs)} routes, worst error/tolerance {worst:.4f}")
    return worst


def check_both(ro, ref, what):
    check_routes(ro, ref["f64"], what=f"{what} (contract)")
    check_routes(ro, ref["bf16"], what=f"{what} (BF16 operand)")


TOY = [
    # H,   I,   E, T,   k, G,   widths, routing
    (512, 256, 8, 37, 2, 128, (2, 3, 4), "uniform"),
    (512, 256, 4, 300, 2, 256, (3, 4), "uniform"),     # ~150 tokens per expert: several tiles
    (1024, 512, 16, 9, 4, 512, (2,), "zipf"),
    # few routes per expert: the decode-sized grouped path, mixed widths,
    # experts with one, two and more routes (chunks of two)
    (512, 256, 32, 24, 2, 128, (2, 3, 4), "uniform"),
    (1024, 512, 16, 24, 2, 512, (3, 4), "zipf"),
    # code widths 1 and 5..8 beside the table widths ([CQ] "为什么只用两个形状参数？":
    # an ordinary 1..8-bit code stream): the whole layer takes the engine's
    # wide-code decoder, at prefill and at decode sizes
    (512, 256, 8, 37, 2, 128, (5, 8, 2, 3), "uniform"),
    (512, 256, 16, 12, 2, 256, (1, 6, 7, 4), "uniform"),
]


@pytest.mark.parametrize("H,I,E,T,k,G,widths,routing", TOY)
def test_moe_toy_full_oracle(cq, H, I, E, T, k, G, widths, routing):
    tag = ("toy", H, E, T)
    Bs = [widths[e % len(widths)] for e in range(E)]
    experts = [expert_gpu(cq, tag, e, Bs[e], H, I, G) for e in range(E)]
    layer = cq.moe_prepare_layer(experts, H, I, G)
    x = synthetic.activations(T + 5, T, H)
    if routing == "uniform":
        ids, w = synthetic.routing_uniform(T, T, E, k)
    else:
        ids, w = synthetic.routing_zipf(T, T, E, k)
    ids[0, 0] = E + 3 if T > 1 else ids[0, 0]          # one dropped route
    ro, out = cq.cq_moe_grouped_gemm(x.cuda(), ids.cuda(), w.cuda(), layer, E, H, I, G)
    torch.cuda.synchronize()
    ids_np = ids.numpy()
    valid = [r for r in range(T * k) if 0 <= ids_np[r // k, r % k] < E]
    oexp = {e: expert_oracle(tag, e, Bs[e], H, I, G) for e in range(E)}
    refs = oracle_routes(u16(x), ids_np, lambda e: oexp[e], H, I, G, valid)
    check_both(ro, refs, f"toy {H}x{I} E={E} T={T}")
    assert torch.all(ro[0] == 0)                         # the dropped route's row is cleared
    check_combine(out, w, refs, T, k, range(T))


def check_combine(out, w, refs, T, k, tokens):
    """Combined outputs against the oracle's weighted sum over valid routes,
    within the weighted sum of the route tolerances (both references)."""
    wn = w.numpy().astype(np.float64)
    got = out.double().cpu().numpy()
    for op, ref in refs.items():
        for t in tokens:
            rs = [t * k + j for j in range(k) if t * k + j in ref]
            if not rs or len(rs) < sum(1 for j in range(k) if t * k + j in refs["f64"]):
                continue              # a token with routes outside this reference's sample
            H = len(ref[rs[0]][0])
            acc, tol, mag = np.zeros(H), np.zeros(H), np.zeros(H)
            for r in rs:
                acc += wn[r // k, r % k] * ref[r][0]
                tol += abs(wn[r // k, r % k]) * ref[r][2]
                mag += np.abs(wn[r // k, r % k] * ref[r][0])
            tol += 1e-6 * mag + 1e-7          # the kernel's FP32 sum over the k routes
            err = np.abs(got[t] - acc)
            assert np.all(err <= tol), f"{op} token {t}: worst {np.max(err / tol):.3f}"


def _full_layer(cq, tag, E, B_of, H, I, G):
    experts = [expert_gpu(cq, tag, e, int(B_of[e]), H, I, G) for e in range(E)]
    return experts, cq.moe_prepare_layer(experts, H, I, G)


def test_config4_decode_layer_every_route(cq):
    """896 experts with per-expert W2/W3/W4 (P = 0.6/0.3/0.1), G512, 64 tokens,
    uniform top-16: every output of every one of the 1,024 routes against the
    oracle (contract check on all of them, the BF16-operand check on the
    routes of one expert in eight), and every combined output."""
    H, I, E, T, k, G = 7168, 3072, 896, 64, 16, 512
    tag = ("config4",)
    Bs = synthetic.expert_bits(4, E)
    experts, layer = _full_layer(cq, tag, E, Bs, H, I, G)
    x = synthetic.activations(44, T, H)
    ids, w = synthetic.routing_uniform(4, T, E, k)
    ro, out = cq.cq_moe_grouped_gemm(x.cuda(), ids.cuda(), w.cuda(), layer, E, H, I, G)
    torch.cuda.synchronize()
    assert cq.device_error() == (0, 0)
    del experts, layer
    torch.cuda.empty_cache()
    ids_np = ids.numpy()
    active = sorted(set(ids_np.ravel().tolist()))
    tight = set(active[::8])
    refs = oracle_routes(u16(x), ids_np,
                         lambda e: expert_oracle_from_device(tag, e, int(Bs[e]), H, I, G),
                         H, I, G, range(T * k), tight_experts=tight)
    assert len(refs["f64"]) == T * k
    check_both(ro, refs, "config4")
    check_combine(out, w, {"f64": refs["f64"]}, T, k, range(T))


def test_config5_prefill_layer_four_routes_of_every_expert(cq):
    """896 W4 G512 experts, 8192 tokens, Zipf(1.1) top-16: four routes of
    every expert (all routes of those with fewer), the hottest and the
    coldest included, against the oracle (the BF16-operand check on one
    expert in eight); the combine of sampled tokens against the per-route
    outputs."""
    H, I, E, T, k, G = 7168, 3072, 896, 8192, 16, 512
    tag = ("config5",)
    Bs = np.full(E, 4)
    experts, layer = _full_layer(cq, tag, E, Bs, H, I, G)
    x = synthetic.activations(55, T, H)
    ids, w = synthetic.routing_zipf(5, T, E, k)
    ro, out = cq.cq_moe_grouped_gemm(x.cuda(), ids.cuda(), w.cuda(), layer, E, H, I, G)
    torch.cuda.synchronize()
    assert cq.device_error() == (0, 0)
    del experts, layer
    torch.cuda.empty_cache()
    ids_np = ids.numpy()
    flat = ids_np.ravel()
    counts = np.bincount(flat, minlength=E)
    assert counts.min() >= 1                     # every expert is active
    rng = np.random.default_rng(555)
    picks = []
    for e in range(E):
        rs = np.nonzero(flat == e)[0]
        if len(rs) > 4:
            rs = np.concatenate([[rs[0], rs[-1]], rng.choice(rs[1:-1], 2, replace=False)])
        picks += [int(r) for r in rs]
    tight = set(range(0, E, 8)) | {int(np.argmax(counts)), int(np.argmin(counts))}
    refs = oracle_routes(u16(x), ids_np,
                         lambda e: expert_oracle_from_device(tag, e, 4, H, I, G),
                         H, I, G, picks, tight_experts=tight)
    check_both(ro, refs, "config5")
    tk = [0, T // 2, T - 1]
    comb = (w[tk].double().cuda()[:, :, None] * ro.view(T, k, H)[tk].double()).sum(1)
    assert torch.allclose(out[tk].double(), comb, rtol=1e-6, atol=1e-6)


def test_moe_degenerate_layers(cq):
    """Degenerate routing: one expert with k = 1 (every token on it, the
    decode-sized path), every route dropped (all outputs zero), and an empty
    batch (nothing launched)."""
    H, I, G, B = 512, 256, 128, 3
    tag = ("degenerate",)
    experts = [expert_gpu(cq, tag, 0, B, H, I, G)]
    layer = cq.moe_prepare_layer(experts, H, I, G)
    # one expert, top-1, three tokens
    T = 3
    x = synthetic.activations(77, T, H)
    ids = torch.zeros((T, 1), dtype=torch.int32)
    w = torch.ones((T, 1), dtype=torch.float32)
    ro, out = cq.cq_moe_grouped_gemm(x.cuda(), ids.cuda(), w.cuda(), layer, 1, H, I, G)
    torch.cuda.synchronize()
    assert cq.device_error() == (0, 0)
    oexp = {0: expert_oracle(tag, 0, B, H, I, G)}
    refs = oracle_routes(u16(x), ids.numpy(), lambda e: oexp[e], H, I, G, list(range(T)))
    check_both(ro, refs, "one expert, top-1")
    assert torch.equal(out, ro)                       # weight 1: the combine is the route row
    # every route dropped (ids out of range): zero rows, zero combine
    bad = torch.full((T, 2), 5, dtype=torch.int32)
    w2 = torch.full((T, 2), 0.5, dtype=torch.float32)
    ro, out = cq.cq_moe_grouped_gemm(x.cuda(), bad.cuda(), w2.cuda(), layer, 1, H, I, G)
    torch.cuda.synchronize()
    assert cq.device_error() == (0, 0)
    assert torch.all(ro == 0) and torch.all(out == 0)
    # empty batch
    ro, out = cq.cq_moe_grouped_gemm(x[:0].cuda(), ids[:0].cuda(), w[:0].cuda(), layer, 1, H,
                                     I, G)
    torch.cuda.synchronize()
    assert ro.shape == (0, H) and out.shape == (0, H)


def test_expert_parallel_single_rank_is_the_grouped_gemm(cq):
    """The expert-parallel layer on one rank (no process group) hands every
    token row, in order, with its ids unchanged, to the same grouped GEMM:
    the output is bit-identical to calling cq_moe_grouped_gemm directly."""
    from bit_non_uniform_b200.ep import MoeExpertParallel, libcq_compute
    H, I, E, T, k, G = 512, 256, 8, 37, 2, 128
    tag = ("ep1", H, E, T)
    Bs = [(2, 3, 4)[e % 3] for e in range(E)]
    experts = [expert_gpu(cq, tag, e, Bs[e], H, I, G) for e in range(E)]
    layer = cq.moe_prepare_layer(experts, H, I, G)
    x = synthetic.activations(T + 9, T, H).cuda()
    ids, w = synthetic.routing_uniform(T + 9, T, E, k)
    ids, w = ids.cuda(), w.cuda()
    _, direct = cq.cq_moe_grouped_gemm(x, ids, w, layer, E, H, I, G)
    got = MoeExpertParallel(E, H, libcq_compute(layer, E, H, I, G)).forward(x, ids, w)
    torch.cuda.synchronize()
    assert cq.device_error() == (0, 0)
    assert got.dtype == torch.float32 and torch.equal(got, direct)
