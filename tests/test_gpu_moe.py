"""GPU parity of the grouped MoE layer (cq_moe_grouped_gemm) against the CPU
oracle's composition gate/up -> SwiGLU -> BF16 h -> down -> weighted combine.

Per-route outputs: |y - y_ref| <= the oracle's chain tolerance, i.e. the
per-GEMM bound 2e-3 * sum|w h| + 1e-6 of the down product plus the
first-order effect, through SwiGLU, the BF16 rounding of h and |W_dn|, of the
gate/up product's own 2e-3 * sum|w x| + 1e-6 bound.  Combined outputs use
the weighted sum of the per-route tolerances."""
import numpy as np
import pytest
import torch

import oracle
import synthetic

pytestmark = pytest.mark.gpu

REL, ABS = 2e-3, 1e-6


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


def check_routes(ro, ref, routes):
    for r in routes:
        y, bnd, tol = ref[r]
        got = ro[r].double().cpu().numpy()
        err = np.abs(got - y)
        assert np.all(err <= tol), f"route {r}: worst ratio {np.max(err / tol):.3f}"


TOY = [
    # H,   I,   E, T,   k, G,   widths, routing
    (512, 256, 8, 37, 2, 128, (2, 3, 4), "uniform"),
    (512, 256, 4, 300, 2, 256, (3, 4), "uniform"),     # ~150 tokens per expert: several tiles
    (1024, 512, 16, 9, 4, 512, (2,), "zipf"),
    # few routes per expert: the decode-sized grouped path, mixed widths,
    # experts with one, two and more routes (chunks of two)
    (512, 256, 32, 24, 2, 128, (2, 3, 4), "uniform"),
    (1024, 512, 16, 24, 2, 512, (3, 4), "zipf"),
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
    ref = oracle.moe_routes(u16(x), ids_np, oexp, H, I, G, routes=valid)
    check_routes(ro, ref, valid)
    assert torch.all(ro[0] == 0)                         # the dropped route's row is cleared
    # combined output against the oracle's weighted sum over valid routes
    wn = w.numpy().astype(np.float64)
    for t in range(T):
        acc = np.zeros(H)
        bnd = np.zeros(H)
        for j in range(k):
            r = t * k + j
            if r in ref:
                acc += wn[t, j] * ref[r][0]
                bnd += abs(wn[t, j]) * ref[r][2]
        err = np.abs(out[t].double().cpu().numpy() - acc)
        assert np.all(err <= bnd + 1e-6), f"token {t}"


def _full_layer(cq, tag, E, B_of, H, I, G):
    experts = [expert_gpu(cq, tag, e, int(B_of[e]), H, I, G) for e in range(E)]
    return experts, cq.moe_prepare_layer(experts, H, I, G)


def test_config4_decode_layer_sampled(cq):
    """896 experts with per-expert W2/W3/W4 (P = 0.6/0.3/0.1), G512, 64 tokens,
    uniform top-16: every output of sampled routes from each width against the
    oracle; the combine checked exactly against the per-route outputs."""
    H, I, E, T, k, G = 7168, 3072, 896, 64, 16, 512
    tag = ("config4",)
    Bs = synthetic.expert_bits(4, E)
    experts, layer = _full_layer(cq, tag, E, Bs, H, I, G)
    x = synthetic.activations(44, T, H)
    ids, w = synthetic.routing_uniform(4, T, E, k)
    ro, out = cq.cq_moe_grouped_gemm(x.cuda(), ids.cuda(), w.cuda(), layer, E, H, I, G)
    torch.cuda.synchronize()
    assert cq.device_error() == (0, 0)
    ids_np = ids.numpy()
    picks = []
    for want in (2, 3, 4):
        for r in range(T * k):
            if int(Bs[ids_np[r // k, r % k]]) == want:
                picks.append(r)
                break
    picks.append(T * k - 1)
    get = lambda e: expert_oracle(tag, e, int(Bs[e]), H, I, G)
    ref = oracle.moe_routes(u16(x), ids_np, get, H, I, G, routes=picks, nthreads=0)
    check_routes(ro, ref, picks)
    comb = (w.double().cuda()[:, :, None] * ro.double().view(T, k, H)).sum(1)
    assert torch.allclose(out.double(), comb, rtol=1e-6, atol=1e-6)
    del experts, layer


def test_config5_prefill_layer_sampled(cq):
    """896 W4 G512 experts, 8192 tokens, Zipf(1.1) top-16: routes of the
    hottest, the coldest and a median expert against the oracle."""
    H, I, E, T, k, G = 7168, 3072, 896, 8192, 16, 512
    tag = ("config5",)
    Bs = np.full(E, 4)
    experts, layer = _full_layer(cq, tag, E, Bs, H, I, G)
    x = synthetic.activations(55, T, H)
    ids, w = synthetic.routing_zipf(5, T, E, k)
    ro, out = cq.cq_moe_grouped_gemm(x.cuda(), ids.cuda(), w.cuda(), layer, E, H, I, G)
    torch.cuda.synchronize()
    assert cq.device_error() == (0, 0)
    ids_np = ids.numpy()
    counts = np.bincount(ids_np.ravel(), minlength=E)
    active = np.nonzero(counts)[0]
    order = active[np.argsort(counts[active])]
    sel_experts = [order[-1], order[0], order[len(order) // 2]]
    flat = ids_np.ravel()
    picks = []
    for e in sel_experts:
        rs = np.nonzero(flat == e)[0]
        picks += [int(rs[0]), int(rs[-1])]
    get = lambda e: expert_oracle(tag, e, 4, H, I, G)
    ref = oracle.moe_routes(u16(x), ids_np, get, H, I, G, routes=picks, nthreads=0)
    check_routes(ro, ref, picks)
    tk = [0, T - 1]
    comb = (w[tk].double().cuda()[:, :, None] * ro.view(T, k, H)[tk].double()).sum(1)
    assert torch.allclose(out[tk].double(), comb, rtol=1e-6, atol=1e-6)
    del experts, layer


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
    ref = oracle.moe_routes(u16(x), ids.numpy(), oexp, H, I, G, routes=list(range(T)))
    check_routes(ro, ref, range(T))
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
