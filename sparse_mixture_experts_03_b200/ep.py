"""Expert-parallel MoE layer over a process group.

Rank r of N holds the routed experts [r E_l, (r+1) E_l) (E_l = E / N) plus a
copy of the router and the shared experts ("大模型工程（一）：Transformer 到
MoE", section "混合专家：更多参数，相同 FLOPs": experts placed on different GPUs
and tokens exchanged by all-to-all over NVLink; its Mixtral / Qwen3-MoE /
DeepSeek-V3 comparison places expert groups per GPU).  One forward:

  1. dispatch   route this rank's tokens and copy each chosen (token, expert)
                row into expert order; expert order is destination-rank
                order, so the rows for rank q are one contiguous block
  2. exchange   all-to-all of the per-expert row counts, then of the rows and
                their gate weights (NCCL over NVLink on GPUs)
  3. experts    the received rows through this rank's experts, each result
                scaled by its gate weight, in the receive order
  4. return     all-to-all of the results back to the rows' owners
  5. combine    y[t] = shared experts(x_t) + the token's k rows, in top-k order

The shared experts (step 5's first term) depend only on the rank's own x, so
on a GPU they run on a side stream while steps 2-4 are in flight.

Every computing step is a call into the CUDA library (moe.dispatch,
moe.experts_forward, moe.shared_forward, moe.combine); this module only sizes
buffers, computes the exchange splits from the counts and issues the
collectives.  `ops` replaces those four calls (with the same signatures) so
the exchange logic can be exercised on CPU ranks; nothing here computes the
layer itself, and there is no CPU fallback.
"""
from __future__ import annotations

from typing import List, Optional, Sequence

import torch
import torch.distributed as dist

from . import moe


def rank_rows(counts: Sequence[int], n_ranks: int) -> List[int]:
    """Rows per destination rank from per-expert counts (experts in rank
    blocks of E / n_ranks)."""
    E = len(counts)
    if E % n_ranks:
        raise ValueError(f"{E} experts do not split over {n_ranks} ranks")
    E_l = E // n_ranks
    return [int(sum(counts[q * E_l:(q + 1) * E_l])) for q in range(n_ranks)]


class LibraryOps:
    """The four computing steps, on the CUDA library."""

    dispatch = staticmethod(moe.dispatch)
    experts_forward = staticmethod(moe.experts_forward)
    shared_forward = staticmethod(moe.shared_forward)
    combine = staticmethod(moe.combine)


class ExpertParallelMoE:
    """One rank of the expert-parallel layer.

    W_router [E, d] and W_shared (moe_forward layout, or None) are full
    copies; W_gate_up [E_l, 2 inter, d] and W_down [E_l, d, inter] are this
    rank's experts [rank E_l, (rank+1) E_l).  `group` is the process group of
    the n_ranks ranks (None: the default group); the phase methods work
    without one, for callers that run the exchanges themselves.
    """

    def __init__(self, W_router, W_gate_up, W_down, W_shared, k: int, n_group: int,
                 topk_group: int, inter: int, n_shared: int, rank: int, n_ranks: int,
                 group=None, out_dtype: torch.dtype = torch.float32, gate: str = "sigmoid",
                 expert_bias: Optional[torch.Tensor] = None, ops=None):
        self.W_router, self.W_gate_up, self.W_down, self.W_shared = (
            W_router, W_gate_up, W_down, W_shared)
        self.E, self.d = W_router.shape
        if self.E % n_ranks:
            raise ValueError(f"{self.E} experts do not split over {n_ranks} ranks")
        self.E_l = self.E // n_ranks
        if W_gate_up.shape[0] != self.E_l or W_down.shape[0] != self.E_l:
            raise ValueError("the local expert weights must hold E / n_ranks experts")
        self.k, self.n_group, self.topk_group = k, n_group, topk_group
        self.inter, self.n_shared = inter, n_shared
        self.rank, self.n_ranks, self.group = rank, n_ranks, group
        self.out_dtype, self.gate, self.expert_bias = out_dtype, gate, expert_bias
        self.ops = ops if ops is not None else LibraryOps()

    # ---- phases (each a library call)
    def dispatch(self, x: torch.Tensor) -> moe.Dispatched:
        return self.ops.dispatch(x, self.W_router, self.k, self.n_group, self.topk_group,
                                 gate=self.gate, expert_bias=self.expert_bias)

    def shared(self, x: torch.Tensor) -> Optional[torch.Tensor]:
        if self.n_shared == 0:
            return None
        return self.ops.shared_forward(x, self.W_shared, self.inter, self.n_shared)

    def experts(self, x_recv: torch.Tensor, w_recv: torch.Tensor,
                recv_counts: torch.Tensor) -> torch.Tensor:
        """recv_counts int32 [n_ranks, E_l]: rows from each source rank for
        each local expert, in the order the rows arrived."""
        return self.ops.experts_forward(x_recv, w_recv, recv_counts, self.W_gate_up, self.W_down,
                                        self.inter)

    def combine(self, rows_back: torch.Tensor, disp: moe.Dispatched,
                y_shared: Optional[torch.Tensor], T: int) -> torch.Tensor:
        return self.ops.combine(rows_back, disp.slot_row, y_shared, T, self.k, self.out_dtype)

    # ---- the whole forward with the collectives
    def forward(self, x: torch.Tensor) -> torch.Tensor:
        T, d = x.shape
        N, E_l = self.n_ranks, self.E_l
        disp = self.dispatch(x)
        side = None
        if x.is_cuda and self.n_shared:
            # the shared experts overlap the exchanges
            side = torch.cuda.Stream(device=x.device)
            side.wait_stream(torch.cuda.current_stream(x.device))
            with torch.cuda.stream(side):
                y_shared = self.shared(x)
        else:
            y_shared = self.shared(x)
        counts = disp.counts
        send = rank_rows(counts.tolist(), N)
        bad = sum(send) != T * self.k
        if bad:
            # a device error in the dispatch (its status word says which): this
            # rank announces no rows, takes the same exchange steps as every
            # other rank, and raises at the end
            counts = torch.zeros_like(counts)
            send = [0] * N
        recv_counts = torch.empty(N * E_l, dtype=counts.dtype, device=x.device)
        dist.all_to_all_single(recv_counts, counts, group=self.group)
        recv = rank_rows(recv_counts.tolist(), N)  # [src][e] blocks sum to rows per source
        recv_counts = recv_counts.view(N, E_l)
        R, n_send = sum(recv), sum(send)
        x_recv = torch.empty(R, d, dtype=disp.x_perm.dtype, device=x.device)
        w_recv = torch.empty(R, dtype=disp.w_perm.dtype, device=x.device)
        dist.all_to_all_single(x_recv, disp.x_perm[:n_send], recv, send, group=self.group)
        dist.all_to_all_single(w_recv, disp.w_perm[:n_send], recv, send, group=self.group)
        y_recv = self.experts(x_recv, w_recv, recv_counts.contiguous())
        rows_back = torch.empty(n_send, d, dtype=y_recv.dtype, device=x.device)
        dist.all_to_all_single(rows_back, y_recv, send, recv, group=self.group)
        if side is not None:
            torch.cuda.current_stream(x.device).wait_stream(side)
            y_shared.record_stream(torch.cuda.current_stream(x.device))
        if bad:
            raise RuntimeError("dispatch: the expert counts do not add up to T*k (a device "
                               "error; see moe.device_status of the dispatch workspace)")
        return self.combine(rows_back, disp, y_shared, T)

    __call__ = forward
