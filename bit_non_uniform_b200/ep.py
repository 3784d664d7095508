"""Expert parallelism for the routed-expert MoE layer.

The article's reference deployment runs the quantized experts on one node of
8 GPUs with tensor and expert parallelism (sections "先看结论：这次发布了什么？"
and "快速部署：使用 vLLM Cubic 运行时", `--enable-expert-parallel`).  This module
is the expert-parallel exchange around `cq_moe_grouped_gemm`:

* the E experts are split over the W ranks of a process group in contiguous
  blocks (rank d owns experts [d E/W, (d+1) E/W));
* every rank brings its own tokens with their top-k ids and weights;
* **dispatch**: an all-to-all of row counts, then one all-to-all of packed
  rows sends each token row once to every rank that owns at least one of its
  experts, together with its top-k ids made local to that rank (ids of other
  ranks become -1, which the grouped GEMM drops) and the matching weights (0
  elsewhere): 2H + 8k bytes per row;
* **compute**: each rank runs the grouped GEMM over the rows it received and
  its own experts, combining the local routes of every row (FP32);
* **combine**: a second all-to-all returns the partial rows, and each token's
  output is the sum of its partials in rank order (deterministic).

The transfers go through `torch.distributed` (NCCL over NVLink on GPUs, gloo
on the host); the expert computation runs in libcq.  Every step takes the
same collectives in the same order on every rank, including ranks that send
or receive nothing.
"""
from __future__ import annotations

from typing import Callable

import torch
import torch.distributed as dist

Compute = Callable[[torch.Tensor, torch.Tensor, torch.Tensor], torch.Tensor]


def experts_per_rank(E: int, world: int) -> int:
    if world < 1 or E < world or E % world != 0:
        raise ValueError(f"{E} experts do not split evenly over {world} ranks")
    return E // world


def libcq_compute(layer: torch.Tensor, E_local: int, H: int, I: int, G: int,
                  mode: int = 0) -> Compute:
    """The rank's expert computation on the GPU: cq_moe_grouped_gemm over its
    E_local experts (`layer` from moe_prepare_layer), combined per row."""
    from . import F32, cq_moe_grouped_gemm

    def run(tokens: torch.Tensor, ids: torch.Tensor, w: torch.Tensor) -> torch.Tensor:
        if tokens.shape[0] == 0:
            return torch.zeros((0, H), dtype=torch.float32, device=tokens.device)
        _, out = cq_moe_grouped_gemm(tokens, ids, w, layer, E_local, H, I, G, mode, F32,
                                     route_out=None, combine=True)
        return out

    return run


def _a2a(out: torch.Tensor, inp: torch.Tensor, out_splits, in_splits, group) -> None:
    dist.all_to_all_single(out, inp, list(out_splits), list(in_splits), group=group)


class MoeExpertParallel:
    """One MoE layer's routed experts, sharded by expert over a process group.

    compute(tokens [n][H] bf16, ids [n][k] int32 (local, -1 = not here),
    w [n][k] float32) -> [n][H] partial outputs, the sum over j of
    w[i][j] * y_(i,j) for the row's local routes."""

    def __init__(self, E: int, H: int, compute: Compute, group=None):
        self.group = group
        self.world = dist.get_world_size(group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0
        self.E, self.H = E, H
        self.E_local = experts_per_rank(E, self.world)
        self.compute = compute

    def plan(self, topk_ids: torch.Tensor):
        """Per destination rank d: the local token rows sent to d (ascending)
        and their top-k ids made local to d (-1 for routes owned elsewhere
        and for dropped routes)."""
        valid = (topk_ids >= 0) & (topk_ids < self.E)
        dest = torch.where(valid, torch.div(topk_ids, self.E_local, rounding_mode="floor"),
                           torch.full_like(topk_ids, -1))
        rows, local_ids = [], []
        for d in range(self.world):
            mine = dest == d
            idx = torch.nonzero(mine.any(dim=1)).flatten()
            rows.append(idx)
            li = torch.where(mine[idx], topk_ids[idx] - d * self.E_local,
                             torch.full_like(topk_ids[idx], -1))
            local_ids.append(li.to(torch.int32))
        return rows, local_ids

    def forward(self, tokens: torch.Tensor, topk_ids: torch.Tensor,
                topk_w: torch.Tensor) -> torch.Tensor:
        T, k = topk_ids.shape
        H = self.H
        assert tokens.shape == (T, H) and tokens.dtype == torch.bfloat16
        dev = tokens.device
        rows, local_ids = self.plan(topk_ids)
        send_n = [int(r.numel()) for r in rows]
        # dispatch payload, one row per (token, destination): the token's 2H
        # bytes of BF16, then its k local ids and k weight bit patterns
        # (int32 each), all as bytes
        row_bytes = 2 * H + 8 * k
        send = torch.cat([
            torch.cat([tokens[r].view(torch.uint8).reshape(-1, 2 * H),
                       li.view(torch.uint8).reshape(-1, 4 * k),
                       torch.where(li >= 0, topk_w[r], torch.zeros_like(topk_w[r]))
                       .to(torch.float32).view(torch.uint8).reshape(-1, 4 * k)], dim=1)
            for r, li in zip(rows, local_ids)]).reshape(-1, row_bytes)
        if self.world == 1:
            recv_n = send_n
            recv = send
        else:
            cnt_out = torch.tensor(send_n, dtype=torch.int64, device=dev)
            cnt_in = torch.empty_like(cnt_out)
            _a2a(cnt_in, cnt_out, [1] * self.world, [1] * self.world, self.group)
            recv_n = [int(v) for v in cnt_in.tolist()]
            recv = torch.empty((sum(recv_n), row_bytes), dtype=torch.uint8, device=dev)
            _a2a(recv, send, recv_n, send_n, self.group)
        x_in = recv[:, :2 * H].contiguous().view(torch.bfloat16)
        ids_in = recv[:, 2 * H:2 * H + 4 * k].contiguous().view(torch.int32)
        w_in = recv[:, 2 * H + 4 * k:].contiguous().view(torch.float32)
        part = self.compute(x_in, ids_in, w_in)
        # combine: partials back to the token owners, summed in rank order
        if self.world == 1:
            back = part
        else:
            back = torch.empty((sum(send_n), H), dtype=part.dtype, device=dev)
            _a2a(back, part.contiguous(), send_n, recv_n, self.group)
        out = torch.zeros((T, H), dtype=part.dtype, device=dev)
        off = 0
        for r, n in zip(rows, send_n):
            out.index_add_(0, r, back[off:off + n])
            off += n
        return out
