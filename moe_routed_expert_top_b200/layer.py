"""A routed-experts layer object around ``moe_experts_forward``.

It owns the weights (device tensors), the problem description and a
workspace buffer sized by ``moe_workspace_bytes``; ``forward`` only marshals
pointers into the C entry point. FP8 down weights are prepared once with
``moe_quantize_weight_128x128`` when ``down_fp8`` is set.
"""
from __future__ import annotations

import torch

from . import (make_problem, moe_experts_forward, moe_quantize_weight_128x128,
               moe_route_topk, moe_workspace_bytes)


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
