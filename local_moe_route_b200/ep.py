"""Expert parallelism: one MoE layer whose experts are split over the ranks of
a process group.

The release history of the engine describes splitting a model over several
cards (kongchang.com release-history article, sections "第二步：把一张卡铺成一条
产品线" and "第三步"); on NVLink-connected B200s the natural split of an
expert layer is by expert.  Rank r of W owns experts [r E/W, (r+1) E/W) and
holds only their weights; every rank routes its own tokens.  One forward:

  1. slots s = (t, j) of the rank's tokens are ordered by the rank that owns
     their expert (the same counting sort as the expert grouping, with the
     owner rank as key), and the token row of every slot is gathered into
     that order;
  2. all-to-all: each rank sends its slot rows (and their local expert ids)
     to the owners and receives the rows routed to its own experts;
  3. the received rows are grouped by local expert and run through the
     grouped gate/up and down projections;
  4. the output rows return to received order and go back (all-to-all);
  5. each rank combines its tokens' k rows in slot order j = 0..k-1.

The exchange is `torch.distributed.all_to_all_single` (NCCL over NVLink on
GPUs, gloo on CPU); remote rows always land in this rank's memory before any
kernel reads them.  Every compute step goes through `ops`, an object with the
four methods below; `LibraryOps` binds them to this package's CUDA library.
"""

from __future__ import annotations

from typing import Any, List, Optional, Tuple

import torch
import torch.distributed as dist


def experts_per_rank(E: int, world: int) -> int:
    if world <= 0 or E % world:
        raise ValueError(f"{E} experts do not split evenly over {world} ranks")
    return E // world


def owner_of(expert: torch.Tensor, E: int, world: int) -> torch.Tensor:
    """Rank owning each expert id."""
    return torch.div(expert, experts_per_rank(E, world), rounding_mode="floor")


def _all_to_all_v(x: torch.Tensor, recv_counts: List[int], send_counts: List[int],
                  group=None) -> torch.Tensor:
    """Rows of x in send order (send_counts[r] rows for rank r) -> the rows
    every rank sent here, ordered by source rank."""
    out = x.new_empty((sum(recv_counts),) + tuple(x.shape[1:]))
    dist.all_to_all_single(out, x.contiguous(), recv_counts, send_counts, group=group)
    return out


class ExpertParallelMoE:
    """The expert-parallel forward of one layer on one rank.

    ops must provide
      group(keys[N] int32, nkeys) -> (counts[nkeys], offsets[nkeys+1],
            order[N] (position -> index), position[N] (index -> position)):
            stable counting sort of the indices by key;
      gather(src[N][...], index[M]) -> src[index];
      ffn(rows[R][d], order[R], offsets[El+1], rank) -> out[R][d]: the local
            experts' SwiGLU FFN of the grouped rows (row p of the output is
            for input row order[p], expert = the segment p falls in);
      combine(rows[S][d], w[T][k], position[S], T, k) -> y[T][d]:
            y[t] = sum_j w[t][j] * rows[position[t k + j]], j in order.
    """

    def __init__(self, E: int, k: int, ops: Any, group=None):
        self.E, self.k, self.ops, self.group = E, k, ops, group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.El = experts_per_rank(E, self.world)

    def forward(self, x: torch.Tensor, ids: torch.Tensor, w: torch.Tensor,
                stats: Optional[dict] = None) -> torch.Tensor:
        """x [T][d] this rank's tokens, ids / w [T][k] their routes (global
        expert ids, softmax weights) -> y [T][d]."""
        T, k = ids.shape
        if k != self.k:
            raise ValueError("route width differs from k")
        flat = ids.reshape(-1).to(torch.int32)
        dest = torch.div(flat, self.El, rounding_mode="floor").to(torch.int32)
        local = (flat - dest * self.El).to(torch.int32)
        # 1. slots in owner-rank order, their token rows and local expert ids
        send_counts, _, send_order, send_pos = self.ops.group(dest, self.world)
        x_send = self.ops.gather(x, torch.div(send_order, k, rounding_mode="floor"))
        le_send = self.ops.gather(local, send_order)
        # 2. exchange counts, then rows and expert ids
        sc = send_counts.to(torch.int64)
        rc = torch.empty_like(sc)
        dist.all_to_all_single(rc, sc, group=self.group)
        send_l: List[int] = sc.tolist()
        recv_l: List[int] = rc.tolist()
        x_recv = _all_to_all_v(x_send, recv_l, send_l, self.group)
        le_recv = _all_to_all_v(le_send, recv_l, send_l, self.group)
        R = int(sum(recv_l))
        # 3. grouped by local expert, through the local experts
        if R > 0:
            _, offsets_l, order_l, pos_l = self.ops.group(le_recv, self.El)
            out_g = self.ops.ffn(x_recv, order_l, offsets_l, self.rank)
            # 4. back to received order, back to the senders
            out_r = self.ops.gather(out_g, pos_l)
        else:
            out_r = x_recv.new_empty((0,) + tuple(self._row_shape(x)))
        out_back = _all_to_all_v(out_r, send_l, recv_l, self.group)
        if stats is not None:
            stats.update(sent=send_l, received=recv_l)
        # 5. combine in slot order
        return self.ops.combine(out_back, w, send_pos, T, k)

    def _row_shape(self, x: torch.Tensor) -> Tuple[int, ...]:
        return tuple(x.shape[1:])


class LibraryOps:
    """The four steps on the GPU through the CUDA library (device tensors).
    Weights are the full [E] tensors of the layer; a rank uses the slice of
    its own experts (a pointer offset, no copy)."""

    def __init__(self, weights: dict, dims: dict, world: int):
        import local_moe_route_b200 as sm
        self.sm = sm
        self.w = weights
        self.dims = dict(dims)
        self.El = experts_per_rank(dims["E"], world)

    def _local(self, name: str, rank: int):
        q, s = self.w[name + "_q"], self.w[name + "_s"]
        lo, hi = rank * self.El, (rank + 1) * self.El
        return q[lo:hi], s[lo:hi]

    def group(self, keys: torch.Tensor, nkeys: int):
        sm = self.sm
        N = keys.numel()
        dims = dict(self.dims, T=N, k=1, E=nkeys)
        counts = torch.empty(nkeys, dtype=torch.int32, device=keys.device)
        offsets = torch.empty(nkeys + 1, dtype=torch.int32, device=keys.device)
        order = torch.empty(max(N, 1), dtype=torch.int32, device=keys.device)
        pos = torch.empty(max(N, 1), dtype=torch.int32, device=keys.device)
        ws = sm.workspace(dims, keys.device)
        sm.check(sm.strata_moe_permute(keys.contiguous(), dims, counts, offsets, order, pos, ws),
                 "group")
        return counts, offsets, order[:N], pos[:N]

    def gather(self, src: torch.Tensor, index: torch.Tensor) -> torch.Tensor:
        sm = self.sm
        rows = index.numel()
        width = src[0].numel() if src.dim() > 1 else 1
        out = src.new_empty((rows,) + tuple(src.shape[1:]))
        if rows == 0:
            return out
        if src.element_size() == 2 and src.dim() == 2:
            sm.check(sm.strata_moe_gather_rows(src, index.to(torch.int32).contiguous(),
                                               src.shape[0], rows, width, out), "gather")
            return out
        return src.index_select(0, index.long())

    def ffn(self, rows: torch.Tensor, order: torch.Tensor, offsets: torch.Tensor,
            rank: int) -> torch.Tensor:
        sm = self.sm
        R = rows.shape[0]
        dims = dict(self.dims, T=R, k=1, E=self.El)
        n, d = dims["n"], dims["d"]
        ws = sm.workspace(dims, rows.device)
        h = torch.empty((R, n), dtype=torch.float16, device=rows.device)
        out = torch.empty((R, d), dtype=torch.float16, device=rows.device)
        sm.check(sm.strata_moe_expert_gemm_q4(sm.STRATA_OP_GATE_UP_SWIGLU, rows, order, offsets,
                                              self._local("gate", rank), self._local("up", rank),
                                              None, dims, h, ws), "gate_up")
        sm.check(sm.strata_moe_expert_gemm_q4(sm.STRATA_OP_DOWN, h, None, offsets,
                                              self._local("down", rank), None, None, dims, out,
                                              ws), "down")
        return out

    def combine(self, rows, w, position, T, k):
        sm = self.sm
        dims = dict(self.dims, T=T, k=k)
        y = torch.empty((T, dims["d"]), dtype=torch.bfloat16, device=rows.device)
        sm.check(sm.strata_moe_combine(rows, w.to(torch.float32).contiguous(),
                                       position.contiguous(), dims, y), "combine")
        return y
