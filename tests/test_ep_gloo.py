"""Expert parallelism of the MoE layer (bit_non_uniform_b200.ep) on CPU ranks
over gloo.

Each rank owns a contiguous block of experts and its own tokens.  The
exchange (dispatch all-to-all, local expert compute, combine all-to-all, sum
in rank order) is run with the oracle as every rank's expert compute, and
each rank's outputs are compared with the oracle's single-process layer over
all experts: the per-route outputs are the same numbers, so only the order of
the final FP64 sums differs."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

H, I, G, E, K_TOP = 256, 128, 128, 8, 4
WIDTHS = (2, 3, 4)


def _u16(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _experts():
    import oracle
    import synthetic
    out = []
    for e in range(E):
        B = WIDTHS[e % len(WIDTHS)]
        cg, sg, ag = synthetic.matrix(("ep", "gu", e), 2 * I, H, B, G)
        cd, sd, ad = synthetic.matrix(("ep", "dn", e), H, I, B, G)
        out.append(dict(B_gu=B, packed_gu=oracle.pack(cg.numpy(), B), scales_gu=sg.numpy(),
                        ab_gu=_u16(ag), B_dn=B, packed_dn=oracle.pack(cd.numpy(), B),
                        scales_dn=sd.numpy(), ab_dn=_u16(ad)))
    return out


def _inputs(rank, T):
    """This rank's tokens, ids and weights.  Rank 1 also drops a route and has
    a token whose routes all land on one rank."""
    import synthetic
    x = synthetic.activations(1000 + rank, T, H)
    ids, w = synthetic.routing_uniform(2000 + rank, T, E, K_TOP)
    if rank == 1 and T >= 2:
        ids[0, 1] = -1
        ids[1] = torch.tensor([0, 1, 2, 3], dtype=torch.int32)
    return x, ids, w


def oracle_compute(experts_local):
    """A rank's expert compute by the oracle: sum over the row's local routes
    of w * y, FP64."""
    import oracle

    def run(tokens, ids, w):
        n, k = ids.shape
        out = torch.zeros((n, H), dtype=torch.float64)
        if n == 0:
            return out
        ids_np = ids.numpy()
        routes = [r for r in range(n * k) if ids_np[r // k, r % k] >= 0]
        res = oracle.moe_routes(_u16(tokens), ids_np, experts_local, H, I, G, routes=routes)
        for i in range(n):
            for j in range(k):
                if ids_np[i, j] >= 0:
                    out[i] += float(w[i, j]) * torch.from_numpy(res[i * k + j][0])
        return out

    return run


def reference(x, ids, w, experts):
    import oracle
    k = ids.shape[1]
    ids_np = ids.numpy()
    routes = [r for r in range(ids_np.size) if ids_np[r // k, r % k] >= 0]
    res = oracle.moe_routes(_u16(x), ids_np, experts, H, I, G, routes=routes)
    ref = np.zeros((x.shape[0], H))
    for t in range(x.shape[0]):
        for j in range(k):
            if ids_np[t, j] >= 0:
                ref[t] += float(w[t, j]) * res[t * k + j][0]
    return ref


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, tokens_per_rank, q):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port),
                      RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        from bit_non_uniform_b200.ep import MoeExpertParallel, experts_per_rank
        experts = _experts()
        el = experts_per_rank(E, world)
        layer = MoeExpertParallel(E, H, oracle_compute(experts[rank * el:(rank + 1) * el]))
        T = tokens_per_rank[rank]
        x, ids, w = _inputs(rank, T)
        got = layer.forward(x, ids, w).numpy()
        ref = reference(x, ids, w, experts)
        err = float(np.max(np.abs(got - ref))) if T else 0.0
        scale = float(np.max(np.abs(ref))) if T else 1.0
        q.put((rank, got.shape, err, scale))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("tokens_per_rank", [(5, 6), (0, 4)])
def test_two_ranks_match_the_single_process_layer(tokens_per_rank):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.SimpleQueue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, tokens_per_rank, q))
             for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(300)
    codes = [p.exitcode for p in procs]
    for p in procs:
        if p.is_alive():
            p.kill()
    assert codes == [0, 0], codes
    for rank, shape, err, scale in sorted(q.get() for _ in range(world)):
        assert shape == (tokens_per_rank[rank], H)
        assert err <= 1e-12 * max(scale, 1.0), (rank, err, scale)


def test_single_process_layer_without_process_group():
    from bit_non_uniform_b200.ep import MoeExpertParallel
    experts = _experts()
    layer = MoeExpertParallel(E, H, oracle_compute(experts))
    x, ids, w = _inputs(1, 6)
    got = layer.forward(x, ids, w).numpy()
    np.testing.assert_allclose(got, reference(x, ids, w, experts), rtol=0, atol=1e-12)


def test_plan_sends_each_row_once_per_owner():
    from bit_non_uniform_b200.ep import MoeExpertParallel
    layer = MoeExpertParallel(8, 4, compute=None)
    layer.world, layer.E_local = 4, 2                 # the plan of rank-independent routing
    ids = torch.tensor([[0, 1, 6, -1],
                        [3, 2, 5, 4],
                        [7, 7, 9, 6]], dtype=torch.int32)   # id 9 is out of range: dropped
    rows, local = layer.plan(ids)
    assert [r.tolist() for r in rows] == [[0], [1], [1], [0, 2]]
    assert local[0].tolist() == [[0, 1, -1, -1]]
    assert local[1].tolist() == [[1, 0, -1, -1]]
    assert local[2].tolist() == [[-1, -1, 1, 0]]
    assert local[3].tolist() == [[-1, -1, 0, -1], [1, 1, -1, 0]]


def test_experts_must_split_evenly():
    from bit_non_uniform_b200.ep import experts_per_rank
    assert experts_per_rank(896, 8) == 112
    with pytest.raises(ValueError):
        experts_per_rank(10, 4)


def test_libcq_compute_calls_the_grouped_gemm(monkeypatch):
    # the product's expert compute hands the received rows to cq_moe_grouped_gemm with
    # the rank's own expert count, no per-route output and the combine on; a rank that
    # receives nothing makes no call
    import bit_non_uniform_b200 as cq
    from bit_non_uniform_b200.ep import libcq_compute
    seen = []

    def fake(tokens, ids, w, layer, E, H_, I_, G_, mode, out_dtype, route_out, combine):
        seen.append((tokens.shape, ids.shape, w.shape, layer, E, H_, I_, G_, mode, out_dtype,
                     route_out, combine))
        return None, torch.full((tokens.shape[0], H_), 2.0)

    monkeypatch.setattr(cq, "cq_moe_grouped_gemm", fake)
    run = libcq_compute("layer-table", 4, H, I, G, mode=1)
    x = torch.zeros((3, H), dtype=torch.bfloat16)
    ids = torch.zeros((3, K_TOP), dtype=torch.int32)
    w = torch.zeros((3, K_TOP), dtype=torch.float32)
    out = run(x, ids, w)
    assert torch.equal(out, torch.full((3, H), 2.0))
    assert seen == [((3, H), (3, K_TOP), (3, K_TOP), "layer-table", 4, H, I, G, 1, cq.F32,
                     None, True)]
    empty = run(x[:0], ids[:0], w[:0])
    assert empty.shape == (0, H) and empty.dtype == torch.float32 and len(seen) == 1
