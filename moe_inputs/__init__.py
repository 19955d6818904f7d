"""Seeded synthetic inputs for the routed mixture-of-experts expert forward.

This module is shared by the CPU oracle's tests, the CUDA path's tests and the
benchmark. It only draws random numbers and shapes tensors: it holds none of
the method's arithmetic (no routing, no tables, no GEMM, no quantisation).

Workloads (shapes after the TileOPs PR #1580 "Grouped-GEMM TMA OOB zero-fill +
unpermute out=" §Effect table, which names Qwen3- and DeepSeek-style decode and
prefill experts-forward runs, and the TileLang tutorial "Example 07: MoE
dispatch contract and quantised GEMM" §1 for the tiny case):

  tiny            T=9    E=4   k=2 H=128  F=64   softmax, s=1.0
  qwen3_decode    T=512  E=128 k=8 H=2048 F=768  softmax over U[0,1) logits
  qwen3_prefill   T=4096 E=128 k=8 H=2048 F=768  softmax over U[0,1) logits
  dsv3_prefill    T=4096 E=256 k=8 H=7168 F=2048 sigmoid, s=2.5, shared F_s=2048
  dsv3_decode_fp8 T=512  E=256 k=8 H=7168 F=2048 sigmoid, s=2.5, Zipf-skewed
                  routing (30% of experts empty), FP8 1x128 activations and
                  128x128 block-scaled FP8 down weights

Value distributions: hidden ~ N(0,1) bf16; weights ~ N(0, 0.02) bf16; router
logits from NumPy's PCG64 ``default_rng(seed)`` (host), so the routing input is
identical on every machine. Large tensors (hidden, weights) come from torch's
generator on the device they are created on; a CPU-made and a CUDA-made tensor
with the same seed differ, so every consumer receives the very same tensor
(copied), never a regenerated one.
"""
from __future__ import annotations

import dataclasses

import numpy as np
import torch

__all__ = ["MoeConfig", "CONFIGS", "get_config", "make_logits", "make_hidden",
           "make_weights", "make_inputs", "zipf_logits"]


@dataclasses.dataclass(frozen=True)
class MoeConfig:
    name: str
    T: int
    E: int
    top_k: int
    H: int
    F: int
    padding_M: int = 128
    score_fn: str = "softmax"          # "softmax" | "sigmoid"
    renormalize: bool = True
    routed_scaling_factor: float = 1.0
    logits: str = "normal"             # "normal" | "uniform" | "zipf"
    F_shared: int = 0
    down_fp8: bool = False
    seed: int = 0
    zipf_s: float = 1.2
    zipf_empty_frac: float = 0.30

    @property
    def P(self) -> int:
        return self.T * self.top_k

    def replace(self, **kw) -> "MoeConfig":
        return dataclasses.replace(self, **kw)


CONFIGS = {
    "tiny": MoeConfig("tiny", T=9, E=4, top_k=2, H=128, F=64, padding_M=128,
                      score_fn="softmax", logits="normal", seed=0),
    "qwen3_decode": MoeConfig("qwen3_decode", T=512, E=128, top_k=8, H=2048, F=768,
                              score_fn="softmax", logits="uniform", seed=1),
    "qwen3_prefill": MoeConfig("qwen3_prefill", T=4096, E=128, top_k=8, H=2048, F=768,
                               score_fn="softmax", logits="uniform", seed=2),
    "dsv3_prefill": MoeConfig("dsv3_prefill", T=4096, E=256, top_k=8, H=7168, F=2048,
                              score_fn="sigmoid", logits="normal",
                              routed_scaling_factor=2.5, F_shared=2048, seed=3),
    "dsv3_decode_fp8": MoeConfig("dsv3_decode_fp8", T=512, E=256, top_k=8, H=7168, F=2048,
                                 score_fn="sigmoid", logits="zipf",
                                 routed_scaling_factor=2.5, down_fp8=True, seed=4),
    # Kimi-K2-scale layer with its large shared expert (TileOPs PR #778
    # "SharedFusedMoE with native shared expert kernel and TP support",
    # Benchmark: E=384, top-8, H=7168, F=2048, F_s=18432, sigmoid, tokens
    # 1..4096); routed_scaling_factor 2.827 as in the end-to-end linearity check
    # of TileOPs PR #1580 (Test Plan)
    "kimi_k2": MoeConfig("kimi_k2", T=512, E=384, top_k=8, H=7168, F=2048,
                         score_fn="sigmoid", logits="normal", routed_scaling_factor=2.827,
                         F_shared=18432, seed=5),
}


def get_config(config_name: str, **overrides) -> MoeConfig:
    """A named workload, optionally with fields replaced (``name`` included)."""
    cfg = CONFIGS[config_name]
    return cfg.replace(**overrides) if overrides else cfg


def zipf_logits(T: int, E: int, s: float, empty_frac: float,
                rng: np.random.Generator) -> np.ndarray:
    """Skewed router logits: a seeded 30% of experts are masked to -inf; each
    other expert gets a distinct popularity rank r in 1..E' and every token's
    logit for it is ``-s*ln(r) + Gumbel(0,1)``. Taking the top-k of such logits
    samples k experts without replacement with probability proportional to
    r**-s (the Gumbel-top-k construction of Plackett-Luce sampling)."""
    n_masked = int(round(empty_frac * E))
    perm = rng.permutation(E)
    masked = perm[:n_masked]
    live = perm[n_masked:]
    ranks = np.empty(E, dtype=np.float64)
    ranks[live] = rng.permutation(len(live)) + 1.0
    gumbel = rng.gumbel(size=(T, E))
    out = np.empty((T, E), dtype=np.float64)
    out[:, live] = -s * np.log(ranks[live])[None, :] + gumbel[:, live]
    out[:, masked] = -np.inf
    return out.astype(np.float32)


def make_logits(cfg: MoeConfig) -> np.ndarray:
    """Router logits, fp32 [T, E], from PCG64 seeded with ``cfg.seed``."""
    rng = np.random.default_rng(cfg.seed)
    if cfg.logits == "normal":
        return rng.standard_normal((cfg.T, cfg.E)).astype(np.float32)
    if cfg.logits == "uniform":
        return rng.random((cfg.T, cfg.E)).astype(np.float32)
    if cfg.logits == "zipf":
        return zipf_logits(cfg.T, cfg.E, cfg.zipf_s, cfg.zipf_empty_frac, rng)
    raise ValueError(cfg.logits)


def _gen(device: str | torch.device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def make_hidden(cfg: MoeConfig, device="cpu") -> torch.Tensor:
    """hidden ~ N(0,1), bf16 [T, H]."""
    g = _gen(device, 1000 + cfg.seed)
    return torch.randn(cfg.T, cfg.H, generator=g, device=device,
                       dtype=torch.float32).to(torch.bfloat16)


def _normal_bf16(shape, std, g, device) -> torch.Tensor:
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    # draw in fp32 chunks of at most 2**28 elements to bound the temporary
    flat = out.view(-1)
    n = flat.numel()
    step = 1 << 28
    for i in range(0, n, step):
        j = min(n, i + step)
        flat[i:j] = (torch.randn(j - i, generator=g, device=device,
                                 dtype=torch.float32) * std).to(torch.bfloat16)
    return out


def make_weights(cfg: MoeConfig, device="cpu", std: float = 0.02) -> dict:
    """Expert weights ~ N(0, std) bf16.

    w_gate_up [E, 2F, H]: rows [0, F) are the gate projection, [F, 2F) the up
    projection; w_down [E, H, F]. With ``cfg.F_shared`` > 0 also the shared
    expert's ws_gate_up [2F_s, H] and ws_down [H, F_s]."""
    g = _gen(device, 2000 + cfg.seed)
    w = {
        "w_gate_up": _normal_bf16((cfg.E, 2 * cfg.F, cfg.H), std, g, device),
        "w_down": _normal_bf16((cfg.E, cfg.H, cfg.F), std, g, device),
    }
    if cfg.F_shared:
        w["ws_gate_up"] = _normal_bf16((2 * cfg.F_shared, cfg.H), std, g, device)
        w["ws_down"] = _normal_bf16((cfg.H, cfg.F_shared), std, g, device)
    return w


def make_inputs(cfg: MoeConfig, device="cpu") -> dict:
    """All inputs of one experts-forward call for ``cfg``."""
    d = {"logits": make_logits(cfg), "hidden": make_hidden(cfg, device)}
    d.update(make_weights(cfg, device))
    return d


def ceil_div(a: int, b: int) -> int:
    return -(-a // b)


def zipf_expected_empty(cfg: MoeConfig) -> int:
    return int(round(cfg.zipf_empty_frac * cfg.E))

