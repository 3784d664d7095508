"""Expert parallelism of the MoE layer with the CUDA library as every rank's
expert compute: two ranks (processes) over gloo, both on cuda:0.

The exchange runs on the host (gloo all-to-alls of host tensors); each rank's
expert compute copies the rows it received to the GPU, runs
cq_moe_grouped_gemm over its own block of experts (the local ids made by the
plan, -1 for routes owned by the other rank, which the grouped GEMM drops)
and copies the combined partial rows back.  No kernel waits on another
process: the two ranks' launches are independent.  Each rank's outputs are
checked against the oracle's single-process layer over all experts, route by
route (the contract tolerance and the BF16-operand tight tolerance of
oracle.moe_routes), summed with the routing weights.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

H, I, G, E, K_TOP = 512, 256, 128, 8, 4
WIDTHS = (2, 3, 4)
TOL = {"f64": (2e-3, 1e-6), "bf16": (2e-5, 1e-7)}


def _u16(t):
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def _inputs(rank, T):
    """This rank's tokens, ids and weights; rank 1 also drops a route and has
    a token whose routes all land on one rank."""
    import synthetic
    x = synthetic.activations(3000 + rank, T, H)
    ids, w = synthetic.routing_uniform(4000 + rank, T, E, K_TOP)
    if rank == 1 and T >= 2:
        ids[0, 1] = -1
        ids[1] = torch.tensor([4, 5, 6, 7], dtype=torch.int32)
    return x, ids, w


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
        import bit_non_uniform_b200 as cq
        import synthetic
        from bit_non_uniform_b200.ep import MoeExpertParallel, experts_per_rank, libcq_compute
        torch.cuda.set_device(0)
        el = experts_per_rank(E, world)
        experts = []
        for e in range(rank * el, (rank + 1) * el):
            B = WIDTHS[e % len(WIDTHS)]
            cg, sg, ag = synthetic.matrix(("ep2", "gu", e), 2 * I, H, B, G, device="cuda")
            cd, sd, ad = synthetic.matrix(("ep2", "dn", e), H, I, B, G, device="cuda")
            experts.append(dict(B_gu=B, packed_gu=cq.cq_pack(cg, B), scales_gu=sg, ab_gu=ag,
                                B_dn=B, packed_dn=cq.cq_pack(cd, B), scales_dn=sd, ab_dn=ad))
        table = cq.moe_prepare_layer(experts, H, I, G)
        on_gpu = libcq_compute(table, el, H, I, G)

        def compute(tokens, ids, w):          # host rows in, host partial rows out
            return on_gpu(tokens.cuda(), ids.cuda(), w.cuda()).cpu()

        layer = MoeExpertParallel(E, H, compute)
        T = tokens_per_rank[rank]
        x, ids, w = _inputs(rank, T)
        got = layer.forward(x, ids, w).numpy()
        torch.cuda.synchronize()
        q.put((rank, got, cq.device_error()))
    finally:
        dist.destroy_process_group()


def _oracle_layer():
    import oracle
    import synthetic
    out = []
    for e in range(E):
        B = WIDTHS[e % len(WIDTHS)]
        cg, sg, ag = synthetic.matrix(("ep2", "gu", e), 2 * I, H, B, G)
        cd, sd, ad = synthetic.matrix(("ep2", "dn", e), H, I, B, G)
        out.append(dict(B_gu=B, packed_gu=oracle.pack(cg.numpy(), B), scales_gu=sg.numpy(),
                        ab_gu=_u16(ag), B_dn=B, packed_dn=oracle.pack(cd.numpy(), B),
                        scales_dn=sd.numpy(), ab_dn=_u16(ad)))
    return out


@pytest.mark.parametrize("tokens_per_rank", [(5, 6), (0, 4)])
def test_two_ranks_on_libcq_match_the_oracle_layer(tokens_per_rank):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import oracle
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
    results = sorted((q.get() for _ in range(world)), key=lambda r: r[0])
    experts = _oracle_layer()
    for rank, got, dev_err in results:
        T = tokens_per_rank[rank]
        assert got.shape == (T, H) and dev_err == (0, 0)
        if T == 0:
            continue
        x, ids, w = _inputs(rank, T)
        ids_np, wn = ids.numpy(), w.numpy().astype(np.float64)
        routes = [r for r in range(T * K_TOP) if ids_np[r // K_TOP, r % K_TOP] >= 0]
        for op, (rel, abs_) in TOL.items():
            ref = oracle.moe_routes(_u16(x), ids_np, experts, H, I, G, routes=routes, rel=rel,
                                    abs_=abs_, operand=op)
            for t in range(T):
                acc, tol, mag = np.zeros(H), np.zeros(H), np.zeros(H)
                for j in range(K_TOP):
                    r = t * K_TOP + j
                    if r in ref:
                        acc += wn[t, j] * ref[r][0]
                        tol += abs(wn[t, j]) * ref[r][2]
                        mag += np.abs(wn[t, j] * ref[r][0])
                # the rank-local FP32 sums and the FP32 sum of the two ranks' partials
                tol += 2e-6 * mag + 1e-7
                err = np.abs(got[t] - acc)
                assert np.all(err <= tol), (op, rank, t, float(np.max(err / tol)))
