"""Helpers shared by the GPU parity tests: call the CUDA path through the
C-ABI binding and compare with the CPU oracle."""
from __future__ import annotations

import numpy as np
import torch

import moe_routed_expert_top_b200 as M
from moe_inputs import MoeConfig
from oracle import moe_oracle as O

DEV = "cuda"
RTOL = 1e-2
ATOL = 1e-2


def ensure_built():
    from moe_routed_expert_top_b200 import build
    build.build()
    M.lib()


def problem(cfg: MoeConfig, **kw) -> M.Problem:
    d = dict(T=cfg.T, H=cfg.H, F=cfg.F, E=cfg.E, top_k=cfg.top_k, padding_M=cfg.padding_M,
             score_fn=cfg.score_fn, renormalize=cfg.renormalize,
             routed_scaling_factor=cfg.routed_scaling_factor, down_fp8=cfg.down_fp8,
             F_shared=cfg.F_shared)
    d.update(kw)
    return M.make_problem(**d)


def score_code(cfg) -> int:
    return O.SOFTMAX if cfg.score_fn == "softmax" else O.SIGMOID


def assert_within_tol(gpu, ref, what="", rtol=RTOL, atol=ATOL):
    """max |gpu - ref| <= atol + rtol*|ref| element by element."""
    g = np.asarray(gpu, dtype=np.float64)
    r = np.asarray(ref, dtype=np.float64)
    assert g.shape == r.shape, (what, g.shape, r.shape)
    err = np.abs(g - r)
    bound = atol + rtol * np.abs(r)
    bad = err > bound
    if np.any(bad):
        i = np.unravel_index(np.argmax(err - bound), err.shape)
        raise AssertionError(f"{what}: {bad.sum()} of {bad.size} outside tolerance; worst at {i}: "
                             f"gpu={g[i]!r} ref={r[i]!r} err={err[i]:.3e} bound={bound[i]:.3e}")


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def gpu_route(cfg, logits_np, renormalize=None):
    prob = problem(cfg) if renormalize is None else problem(cfg, renormalize=renormalize)
    logits = torch.from_numpy(logits_np).to(DEV)
    ids = torch.empty(cfg.T, cfg.top_k, dtype=torch.int32, device=DEV)
    w = torch.empty(cfg.T, cfg.top_k, dtype=torch.float32, device=DEV)
    M.moe_route_topk(prob, logits, ids, w)
    torch.cuda.synchronize()
    return ids.cpu().numpy(), w.cpu().numpy()


def gpu_tables(cfg, ids_np, hidden=None, padding_M=None):
    prob = problem(cfg) if padding_M is None else problem(cfg, padding_M=padding_M)
    L = M.moe_get_tables_layout(prob)
    ids = torch.from_numpy(np.ascontiguousarray(ids_np, dtype=np.int32)).to(DEV)
    tables = torch.full((L["total_int32"],), -7, dtype=torch.int32, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    x_perm = None
    if hidden is not None:
        x_perm = torch.empty(L["P"], cfg.H, dtype=torch.bfloat16, device=DEV)
    M.moe_route_permute(prob, None, ids, None, hidden, x_perm, tables, status)
    torch.cuda.synchronize()
    return L, tables, status, x_perm


def split_tables(L, tables: torch.Tensor, E: int) -> dict:
    t = tables.cpu().numpy()
    P = L["P"]
    return {
        "group_sizes": t[L["group_sizes"]:L["group_sizes"] + E],
        "group_offsets": t[L["group_offsets"]:L["group_offsets"] + E + 1],
        "group_padded_offsets": t[L["group_padded_offsets"]:L["group_padded_offsets"] + E + 1],
        "group_idx_for_bx": t[L["group_idx_for_bx"]:L["group_idx_for_bx"] + L["M_blk"]],
        "row_of_pair": t[L["row_of_pair"]:L["row_of_pair"] + P],
        "pair_of_row": t[L["pair_of_row"]:L["pair_of_row"] + P],
    }


def random_ids(T, E, k, rng, sizes=None):
    """Routing with no repeated expert per token. With ``sizes`` (rows per
    expert, summing to T*k and each <= T) the ids are built to give exactly
    those group sizes."""
    if sizes is None:
        return np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    sizes = np.asarray(sizes)
    assert sizes.sum() == T * k and sizes.max() <= T
    ids = np.full((T, k), -1, dtype=np.int64)
    order = np.argsort(-sizes, kind="stable")
    fill = np.zeros(T, dtype=np.int64)
    for e in order:
        # give expert e to the tokens with the most free slots
        cand = np.argsort(fill, kind="stable")[:sizes[e]]
        for t in cand:
            ids[t, fill[t]] = e
            fill[t] += 1
    assert np.all(fill == k)
    for t in range(T):
        rng.shuffle(ids[t])
    return ids.astype(np.int32)
