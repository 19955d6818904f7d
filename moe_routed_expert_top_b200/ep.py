"""Expert parallelism: the routed-experts forward with the experts split over
ranks. Rank r of `world` holds E_local = E / world experts (global ids
[r*E_local, (r+1)*E_local)) and its own tokens; one forward is (pypto-lib PR
#809 "predicate empty routed-expert stages": a dispatch step that produces the
per-rank expert counts and gathered rows, then routed stages that skip empty
local experts):

 1. dispatch, in this library's kernels: the destination rank of every
    (token, slot) pair is its expert // E_local (``moe_ep_split_ids``); the
    rank-level dispatch tables (``moe_route_permute`` with the ranks as the
    groups) order the pairs by destination, gather the rows to send
    (``x_send``, the hidden rows of the pairs) and give the count for every
    destination (``group_sizes``); the pairs' local expert ids follow their
    rows (``moe_gather_rows``);
 2. exchange: all-to-all of the counts, then of the rows and local ids;
 3. local experts, in this library's kernels: dispatch tables over the
    received rows (one pair per row), gate+up with the SwiGLU (or
    SwiGLU + FP8) epilogue, down with fp32 output, and the results gathered
    back into receive order (``moe_gather_rows``);
 4. exchange back: the reverse all-to-all of the fp32 results;
 5. combine (``moe_unpermute`` over the rank-level tables):
    out[t] = bf16(scale * sum_j w[t,j] * y[pair (t, j)]), summed in slot
    order, exactly as the one-GPU forward.

The exchange is pluggable. ``TorchDistExchange`` runs one process per rank
over ``torch.distributed`` (NCCL between GPUs, gloo on CPU);
``forward_emulated`` runs every rank's steps in one process on one device and
hands the buffers over directly: each rank's kernels run one after another and
nothing waits on another rank.
"""
from __future__ import annotations

import dataclasses

import torch

from . import (MOE_EPI_STORE_F32, MOE_EPI_SWIGLU, MOE_EPI_SWIGLU_FP8, make_problem,
               moe_ep_split_ids, moe_gather_rows, moe_get_tables_layout, moe_grouped_gemm,
               moe_quantize_weight_128x128, moe_route_permute, moe_unpermute)


@dataclasses.dataclass
class DispatchState:
    prob: object                  # moe_problem of this rank's tokens with the ranks as groups
    layout: dict
    tables: torch.Tensor          # rank-level dispatch tables
    status: torch.Tensor          # device status word (MOE_DEV_* flags)
    x_send: torch.Tensor          # [P, H] bf16, pairs in destination-rank order
    local_send: torch.Tensor      # [P] int32 local expert id of each sent row
    counts: torch.Tensor          # [world] int32 rows for each destination rank


class EPRank:
    """One rank's share of an expert-parallel routed-experts layer: its local
    experts' weights (w_gate_up_local [E_local, 2F, H], w_down_local
    [E_local, H, F], bf16) and the dispatch / local-expert / combine steps."""

    def __init__(self, w_gate_up_local: torch.Tensor, w_down_local: torch.Tensor, E: int,
                 top_k: int, world: int, rank: int, routed_scaling_factor: float = 1.0,
                 down_fp8: bool = False):
        E_local, two_f, H = w_gate_up_local.shape
        if E_local * world != E or not 0 <= rank < world:
            raise ValueError("need E == E_local * world and 0 <= rank < world")
        self.E, self.E_local, self.world, self.rank = E, E_local, world, rank
        self.F, self.H, self.top_k = two_f // 2, H, top_k
        self.scale = float(routed_scaling_factor)
        self.down_fp8 = bool(down_fp8)
        self.w_gate_up = w_gate_up_local.contiguous()
        self.w_down_scales = None
        if self.down_fp8:
            dev = w_down_local.device
            q = torch.empty(E_local, H, self.F, dtype=torch.uint8, device=dev)
            s = torch.empty(E_local, H // 128, self.F // 128, dtype=torch.float32, device=dev)
            moe_quantize_weight_128x128(E_local, H, self.F, w_down_local.contiguous(), q, s)
            self.w_down, self.w_down_scales = q, s
        else:
            self.w_down = w_down_local.contiguous()
        self.dispatch_status = None   # device status words of the last dispatch / compute
        self.local_status = None

    # -- step 1 -------------------------------------------------------------
    def dispatch(self, hidden: torch.Tensor, topk_ids: torch.Tensor) -> DispatchState:
        T, k = topk_ids.shape
        P = T * k
        dev = hidden.device
        prob = make_problem(T=T, H=self.H, F=self.F, E=self.world, top_k=k)
        L = moe_get_tables_layout(prob)
        tables = torch.zeros(max(L["total_int32"], 1), dtype=torch.int32, device=dev)
        status = torch.zeros(1, dtype=torch.int32, device=dev)
        x_send = torch.empty(P, self.H, dtype=torch.bfloat16, device=dev)
        local_send = torch.empty(P, dtype=torch.int32, device=dev)
        if P == 0:
            counts = torch.zeros(self.world, dtype=torch.int32, device=dev)
            return DispatchState(prob, L, tables, status, x_send, local_send, counts)
        ids = topk_ids.contiguous()
        rank_ids = torch.empty_like(ids)
        local_ids = torch.empty_like(ids)
        moe_ep_split_ids(P, self.E_local, self.world, ids, rank_ids, local_ids)
        moe_route_permute(prob, None, rank_ids, None, hidden.contiguous(), x_send, tables, status)
        por = tables[L["pair_of_row"]:L["pair_of_row"] + P]
        moe_gather_rows(P, P, 4, por, local_ids, local_send, status)
        counts = tables[L["group_sizes"]:L["group_sizes"] + self.world]
        self.dispatch_status = status
        return DispatchState(prob, L, tables, status, x_send, local_send, counts)

    # -- step 3 -------------------------------------------------------------
    def compute(self, recv_x: torch.Tensor, recv_local: torch.Tensor) -> torch.Tensor:
        """fp32 expert outputs [R, H] of the received rows, in receive order."""
        R = recv_x.shape[0]
        dev = recv_x.device
        H, F = self.H, self.F
        y_back = torch.empty(R, H, dtype=torch.float32, device=dev)
        self.local_status = torch.zeros(1, dtype=torch.int32, device=dev)
        if R == 0:
            return y_back
        st = self.local_status
        prob = make_problem(T=R, H=H, F=F, E=self.E_local, top_k=1, down_fp8=self.down_fp8)
        L = moe_get_tables_layout(prob)
        tables = torch.empty(L["total_int32"], dtype=torch.int32, device=dev)
        x_perm = torch.empty(R, H, dtype=torch.bfloat16, device=dev)
        moe_route_permute(prob, None, recv_local.reshape(R, 1).contiguous(), None,
                          recv_x.contiguous(), x_perm, tables, st)
        y_perm = torch.empty(R, H, dtype=torch.float32, device=dev)
        if self.down_fp8:
            h = torch.empty(R, F, dtype=torch.uint8, device=dev)
            hs = torch.empty(R, F // 128, dtype=torch.float32, device=dev)
            moe_grouped_gemm(prob, 0, 2 * F, H, x_perm, None, self.w_gate_up, None, tables,
                             MOE_EPI_SWIGLU_FP8, h, hs, None, st)
            moe_grouped_gemm(prob, 0, H, F, h, hs, self.w_down, self.w_down_scales, tables,
                             MOE_EPI_STORE_F32, y_perm, None, None, st)
        else:
            h = torch.empty(R, F, dtype=torch.bfloat16, device=dev)
            moe_grouped_gemm(prob, 0, 2 * F, H, x_perm, None, self.w_gate_up, None, tables,
                             MOE_EPI_SWIGLU, h, None, None, st)
            moe_grouped_gemm(prob, 0, H, F, h, None, self.w_down, None, tables,
                             MOE_EPI_STORE_F32, y_perm, None, None, st)
        rop = tables[L["row_of_pair"]:L["row_of_pair"] + R]
        moe_gather_rows(R, R, 4 * H, rop, y_perm, y_back, st)
        return y_back

    # -- step 5 -------------------------------------------------------------
    def combine(self, state: DispatchState, y_ret: torch.Tensor, topk_weights: torch.Tensor,
                out: torch.Tensor | None = None) -> torch.Tensor:
        T = topk_weights.shape[0]
        if out is None:
            out = torch.empty(T, self.H, dtype=torch.bfloat16, device=y_ret.device)
        if T:
            moe_unpermute(state.prob, y_ret.contiguous(), state.tables, topk_weights.contiguous(),
                          self.scale, None, out)
        return out


class TorchDistExchange:
    """All-to-all over torch.distributed (one process per rank)."""

    def __init__(self, group=None):
        self.group = group

    def counts(self, send_counts: torch.Tensor):
        import torch.distributed as dist
        send = send_counts.to(torch.int64)
        recv = torch.empty_like(send)
        dist.all_to_all_single(recv, send, group=self.group)
        return send.tolist(), recv.tolist()

    def rows(self, send: torch.Tensor, send_splits, recv_splits) -> torch.Tensor:
        import torch.distributed as dist
        out = send.new_empty((sum(recv_splits),) + tuple(send.shape[1:]))
        dist.all_to_all_single(out, send.contiguous(), list(recv_splits), list(send_splits),
                               group=self.group)
        return out


def forward(rank: EPRank, hidden: torch.Tensor, topk_ids: torch.Tensor,
            topk_weights: torch.Tensor, exchange: TorchDistExchange) -> torch.Tensor:
    """One expert-parallel forward of this rank's tokens (every rank calls it
    with the same exchange sequence)."""
    st = rank.dispatch(hidden, topk_ids)
    send_splits, recv_splits = exchange.counts(st.counts)
    recv_x = exchange.rows(st.x_send, send_splits, recv_splits)
    recv_local = exchange.rows(st.local_send, send_splits, recv_splits)
    y_back = rank.compute(recv_x, recv_local)
    y_ret = exchange.rows(y_back, recv_splits, send_splits)
    return rank.combine(st, y_ret, topk_weights)


def _route(bufs, counts):
    """bufs[src] holds rows ordered by destination with counts[src][dst] rows
    each; returns, for every destination, the rows it receives (sources in
    rank order) and its receive counts per source."""
    world = len(bufs)
    out, recv = [], []
    for dst in range(world):
        parts, c = [], []
        for src in range(world):
            off = sum(counts[src][:dst])
            n = counts[src][dst]
            parts.append(bufs[src][off:off + n])
            c.append(n)
        out.append(torch.cat(parts) if parts else bufs[dst][:0])
        recv.append(c)
    return out, recv


def forward_emulated(ranks, hiddens, topk_ids, topk_weights):
    """All ranks of one expert-parallel forward in one process on one device:
    the same steps as ``forward``, with the all-to-alls done by handing the
    buffers over."""
    states = [r.dispatch(h, i) for r, h, i in zip(ranks, hiddens, topk_ids)]
    counts = [s.counts.tolist() for s in states]
    recv_x, recv_counts = _route([s.x_send for s in states], counts)
    recv_local, _ = _route([s.local_send for s in states], counts)
    y_back = [r.compute(x, l) for r, x, l in zip(ranks, recv_x, recv_local)]
    y_ret, _ = _route(y_back, recv_counts)
    return [r.combine(s, y, w) for r, s, y, w in zip(ranks, states, y_ret, topk_weights)]
