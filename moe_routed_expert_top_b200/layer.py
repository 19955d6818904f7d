"""Layer objects around the C entry points: ``RoutedExperts``
(``moe_experts_forward``), ``SharedExpert`` (``moe_shared_expert_forward``,
one tensor-parallel rank) and ``SharedFusedMoE`` (both, with the partial
output contract).

Each owns its weights (device tensors) and a workspace buffer sized by the
library; ``forward`` only marshals pointers into the C entry points. FP8 down
weights are prepared once with ``moe_quantize_weight_128x128`` when
``down_fp8`` is set.
"""
from __future__ import annotations

import torch

from . import (make_problem, moe_experts_forward, moe_quantize_weight_128x128,
               moe_route_topk, moe_shared_expert_forward, moe_shared_workspace_bytes,
               moe_workspace_bytes)


class RoutedExperts:
    def __init__(self, w_gate_up: torch.Tensor, w_down: torch.Tensor, top_k: int,
                 score_fn: str = "softmax", renormalize: bool = True,
                 routed_scaling_factor: float = 1.0, down_fp8: bool = False,
                 ws_gate_up: torch.Tensor | None = None, ws_down: torch.Tensor | None = None,
                 padding_M: int = 128):
        E, two_f, H = w_gate_up.shape
        self.E, self.F, self.H = E, two_f // 2, H
        self.top_k = top_k
        self.score_fn = score_fn
        self.renormalize = renormalize
        self.scale = float(routed_scaling_factor)
        self.down_fp8 = bool(down_fp8)
        self.F_shared = 0 if ws_gate_up is None else ws_gate_up.shape[0] // 2
        self.padding_M = padding_M
        self.w_gate_up = w_gate_up.contiguous()
        self.ws_gate_up = None if ws_gate_up is None else ws_gate_up.contiguous()
        self.ws_down = None if ws_down is None else ws_down.contiguous()
        self.w_down_scales = None
        if self.down_fp8:
            q = torch.empty(E, H, self.F, dtype=torch.uint8, device=w_down.device)
            s = torch.empty(E, H // 128, self.F // 128, dtype=torch.float32, device=w_down.device)
            moe_quantize_weight_128x128(E, H, self.F, w_down.contiguous(), q, s)
            self.w_down, self.w_down_scales = q, s
        else:
            self.w_down = w_down.contiguous()
        self._ws = None

    def problem(self, T: int):
        return make_problem(T=T, H=self.H, F=self.F, E=self.E, top_k=self.top_k,
                            padding_M=self.padding_M, score_fn=self.score_fn,
                            renormalize=self.renormalize,
                            routed_scaling_factor=self.scale, down_fp8=self.down_fp8,
                            F_shared=self.F_shared)

    def workspace(self, T: int, device) -> torch.Tensor:
        need = moe_workspace_bytes(self.problem(T))
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(max(need, 1024), dtype=torch.uint8, device=device)
        return self._ws

    def route(self, logits: torch.Tensor):
        T = logits.shape[0]
        ids = torch.empty(T, self.top_k, dtype=torch.int32, device=logits.device)
        w = torch.empty(T, self.top_k, dtype=torch.float32, device=logits.device)
        moe_route_topk(self.problem(T), logits, ids, w)
        return ids, w

    def forward(self, hidden: torch.Tensor, topk_ids: torch.Tensor, topk_weights: torch.Tensor,
                out: torch.Tensor | None = None) -> torch.Tensor:
        T = hidden.shape[0]
        if out is None:
            out = torch.empty(T, self.H, dtype=torch.bfloat16, device=hidden.device)
        ws = self.workspace(T, hidden.device)
        moe_experts_forward(self.problem(T), hidden, topk_ids, topk_weights, self.w_gate_up,
                            self.w_down, self.w_down_scales, self.ws_gate_up, self.ws_down,
                            self.scale, out, ws)
        return out

    def device_status(self) -> int:
        """The device status word of the last forward (synchronises)."""
        return int(self._ws[:4].view(torch.int32).item())


class SharedExpert:
    """One tensor-parallel rank's share of the shared expert (TileOPs PR #778
    "SharedFusedMoE with native shared expert kernel and TP support": TP split
    convention, Partial output contract). It takes the COMPLETE weights
    w_gate_up [2*F_s, H] (gate rows, then up rows) and w_down [H, F_s]; the
    library reads rank r's F_s / tp_size columns in place (column-parallel
    gate/up rows, row-parallel down columns), with no slice copies.
    ``forward`` returns this rank's partial output [T, H]: with tp_size > 1
    the caller all-reduces it over the ranks (``SharedFusedMoE.combine``)."""

    def __init__(self, w_gate_up: torch.Tensor, w_down: torch.Tensor, tp_size: int = 1,
                 tp_rank: int = 0):
        two_fs, H = w_gate_up.shape
        self.F_s, self.H = two_fs // 2, H
        if w_down.shape != (H, self.F_s):
            raise ValueError("w_down must be [H, F_s]")
        if tp_size < 1 or not 0 <= tp_rank < tp_size or self.F_s % tp_size:
            raise ValueError("need 0 <= tp_rank < tp_size and F_s % tp_size == 0")
        self.tp_size, self.tp_rank = tp_size, tp_rank
        self.w_gate_up = w_gate_up.contiguous()
        self.w_down = w_down.contiguous()
        self._ws = None

    def forward(self, hidden: torch.Tensor, out: torch.Tensor | None = None,
                out_f32: bool = True) -> torch.Tensor:
        T = hidden.shape[0]
        if out is None:
            out = torch.empty(T, self.H, dtype=torch.float32 if out_f32 else torch.bfloat16,
                              device=hidden.device)
        need = moe_shared_workspace_bytes(T, self.H, self.F_s, self.tp_size)
        if self._ws is None or self._ws.numel() < need:
            self._ws = torch.empty(max(need, 1024), dtype=torch.uint8, device=hidden.device)
        moe_shared_expert_forward(T, self.H, self.F_s, self.tp_size, self.tp_rank, hidden,
                                  self.w_gate_up, self.w_down, out.dtype == torch.float32, out,
                                  self._ws)
        return out

    def device_status(self) -> int:
        return int(self._ws[:4].view(torch.int32).item())


class SharedFusedMoE:
    """Routed experts plus a tensor-parallel shared expert, with the pages'
    partial output contract (TileOPs PR #778): ``forward`` returns
    ``(shared_partial, routed_out)``; the routed path is not sharded. With
    tp_size > 1 the caller all-reduces ``shared_partial`` and adds
    ``routed_out`` (``combine`` does both)."""

    def __init__(self, routed: RoutedExperts, shared: SharedExpert | None):
        if routed.F_shared:
            raise ValueError("the routed layer must not carry the shared expert as well")
        self.routed, self.shared = routed, shared

    def forward(self, hidden: torch.Tensor, topk_ids: torch.Tensor, topk_weights: torch.Tensor):
        routed_out = self.routed.forward(hidden, topk_ids, topk_weights)
        shared_partial = None if self.shared is None else self.shared.forward(hidden)
        return shared_partial, routed_out

    @staticmethod
    def combine(shared_partial: torch.Tensor | None, routed_out: torch.Tensor, group=None,
                world_size: int = 1) -> torch.Tensor:
        """bf16(all_reduce_sum(shared_partial) + routed_out): the caller's side
        of the contract (``group``/``world_size`` of the tensor-parallel ranks;
        no collective when world_size == 1).

        Rounding: ``routed_out`` is already one bf16 rounding of the routed sum
        (moe_experts_forward's output), and this add rounds once more, as the
        pages' contract adds two tensors (TileOPs PR #778, Partial output
        contract). The one-GPU path with ``F_shared > 0`` instead adds the
        shared expert in fp32 before its single cast. The two differ by at
        most one bf16 rounding of the routed part (2**-9 relative), inside the
        forward's tolerance."""
        if shared_partial is None:
            return routed_out
        if world_size > 1:
            import torch.distributed as dist
            dist.all_reduce(shared_partial, op=dist.ReduceOp.SUM, group=group)
        return (shared_partial.float() + routed_out.float()).to(torch.bfloat16)
