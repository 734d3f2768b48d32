"""Expert parallelism: one MoE layer with its E experts spread over G ranks.

"1.6 混合专家（MoE）" (llm.satori-ai.cn), expert parallelism: rank r holds experts
[r*El, (r+1)*El), El = E / G, and every rank routes its own tokens; the token rows travel to
the ranks that hold their experts (dispatch, an all-to-all), come back as expert outputs
(combine, a second all-to-all) and are summed there with the routing weights.  Every step
on the device runs in the library's kernels (moe_route, moe_permute, moe_ep_dispatch_rows,
moe_ep_recv_layout, moe_grouped_swiglu, moe_ep_return_rows, moe_combine); this module only
sequences them around the two exchanges.

The exchanges go through an ``exchange`` object with two collective calls, ``counts`` (the
[G, El] table of rows per destination expert) and ``rows`` (rows with uneven splits):
``NcclExchange`` runs them as torch.distributed all-to-all calls, one process per GPU (NCCL
over NVLink on a multi-GPU node; any backend works).  The row splits of an all-to-all are
host integers, so each layer call copies its expert offsets and the received counts to the
host once.

The layer call is also available in phases (``dispatch``, ``experts``, ``combine``) for
callers that run the exchanges themselves.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional

import torch

from . import (F32, combine, ep_dispatch_rows, ep_recv_layout, ep_return_rows,
               grouped_swiglu, permute, route)


def send_splits(offsets, G: int, El: int) -> List[int]:
    """Rows this rank sends to each rank: the expert-sorted rows of rank d's experts are
    [offsets[d*El], offsets[(d+1)*El]) (offsets [E+1], host integers)."""
    off = [int(v) for v in offsets]
    return [off[(d + 1) * El] - off[d * El] for d in range(G)]


class NcclExchange:
    """The two collectives of the layer as torch.distributed all-to-all calls on `group`
    (every rank of the group calls them in the same order)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group

    def counts(self, send: torch.Tensor) -> torch.Tensor:
        """send [G, El] int32: row d goes to rank d; returns [G, El], row s from rank s."""
        out = torch.empty_like(send)
        self.dist.all_to_all_single(out, send.contiguous(), group=self.group)
        return out

    def rows(self, send: torch.Tensor, send_splits: List[int],
             recv_splits: List[int]) -> torch.Tensor:
        """Rows [sum(send_splits), ...] split by destination; returns the received rows,
        source by source."""
        out = send.new_empty((sum(recv_splits),) + tuple(send.shape[1:]))
        self.dist.all_to_all_single(out, send.contiguous(), recv_splits, send_splits,
                                    group=self.group)
        return out


@dataclasses.dataclass
class DispatchState:
    """What one rank keeps between dispatch and combine."""
    T: int
    topk_idx: torch.Tensor        # [T, K] int32
    topk_w: torch.Tensor          # [T, K] fp32
    slot_to_row: torch.Tensor     # [T*K] int32
    shared_acc: Optional[torch.Tensor]  # [T, D] fp32 (shared expert, gated) or None
    x_sorted: torch.Tensor        # [T*K, D] bf16, expert-sorted rows to send
    send_counts: torch.Tensor     # [G, El] int32 rows per destination expert
    send_splits: List[int]        # rows per destination rank


class ExpertParallelLayer:
    """This rank's part of an MoE layer whose experts are spread over G ranks.

    w_router [E, D] and the shared expert are replicated on every rank; w_gate_up_local
    [El, 2f, D] and w_down_local [El, D, f] are the weights of this rank's experts
    [rank*El, (rank+1)*El)."""

    def __init__(self, rank: int, G: int, w_router, w_gate_up_local, w_down_local, K: int,
                 logit_bias=None, w_shared_gate=None, w_shared_gate_up=None,
                 w_shared_down=None):
        self.rank, self.G, self.K = rank, G, K
        self.E, self.D = w_router.shape
        self.El = w_gate_up_local.shape[0]
        if self.E != G * self.El:
            raise ValueError(f"{self.E} experts do not split into {G} ranks of {self.El}")
        self.f = w_gate_up_local.shape[1] // 2
        self.w_router, self.logit_bias = w_router, logit_bias
        self.w_gate_up, self.w_down = w_gate_up_local, w_down_local
        self.w_shared_gate = w_shared_gate
        self.w_shared_gate_up, self.w_shared_down = w_shared_gate_up, w_shared_down

    # ---------------------------------------------------------------- phases

    def dispatch(self, x) -> DispatchState:
        """Route and permute this rank's tokens; gather the rows in expert order; the shared
        expert runs here, on this rank's own tokens."""
        T = x.shape[0]
        idx, w, counts, sgate = route(x, self.w_router, self.K, self.logit_bias,
                                      self.w_shared_gate)
        pm = permute(idx, w, counts, self.E)
        x_sorted = ep_dispatch_rows(x, pm["sorted_token"], T * self.K)
        shared_acc = None
        if self.w_shared_gate_up is not None:
            shared_acc = torch.zeros((T, self.D), dtype=F32, device=x.device)
            off = torch.tensor([0, T], dtype=torch.int32, device=x.device)
            grouped_swiglu(x, None, off, sgate, self.w_shared_gate_up[None],
                           self.w_shared_down[None], T, out_acc=shared_acc)
        splits = send_splits(pm["offsets"].cpu(), self.G, self.El)
        return DispatchState(T, idx, w, pm["slot_to_row"], shared_acc, x_sorted,
                             counts.view(self.G, self.El), splits)

    def experts(self, recv_x, recv_counts) -> torch.Tensor:
        """This rank's experts over the rows it received (source by source, each source's
        rows in expert order; recv_counts [G, El] on the device): returns their outputs,
        unweighted, in the same order as recv_x."""
        n = recv_x.shape[0]
        if n == 0:
            return torch.empty((0, self.D), dtype=F32, device=recv_x.device)
        off, row = ep_recv_layout(recv_counts, n)
        y = torch.empty((n, self.D), dtype=F32, device=recv_x.device)
        grouped_swiglu(recv_x, row, off, None, self.w_gate_up, self.w_down, n, y_sorted=y)
        return ep_return_rows(y, row)

    def combine(self, st: DispatchState, y_back) -> torch.Tensor:
        """Sum the returned expert outputs (this rank's sorted order) with the routing
        weights, plus the shared expert: y [T, D] bf16."""
        return combine(st.T, self.D, self.K, out_acc=st.shared_acc, y_sorted=y_back,
                       slot_to_row=st.slot_to_row, topk_w=st.topk_w, device=y_back.device)

    # ---------------------------------------------------------------- whole layer

    def __call__(self, x, exchange) -> torch.Tensor:
        st = self.dispatch(x)
        recv_counts = exchange.counts(st.send_counts)
        recv_splits = [int(v) for v in recv_counts.sum(1).cpu()]
        recv_x = exchange.rows(st.x_sorted, st.send_splits, recv_splits)
        y_ret = self.experts(recv_x, recv_counts)
        y_back = exchange.rows(y_ret, recv_splits, st.send_splits)
        return self.combine(st, y_back)
