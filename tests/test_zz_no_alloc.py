"""GPU test of moe_experts_forward_noalloc, the forward for callers that cannot
allocate device memory (its workspace is a fixed 64 MiB array inside the
library). Called through the C ABI twice in a row, its output must match the
CPU oracle (every element of the small case, seeded token samples of the
decode workload) and the regular moe_experts_forward (caller-supplied
workspace), within the bf16 tolerance used by every forward test; its status
word, read back with moe_noalloc_read_status, is 0 after a clean call and
carries MOE_DEV_BAD_EXPERT_ID after a call with an out-of-range expert id; a
problem too large for the array is rejected before anything runs. Collected
last so a failure here comes after every other test has run; it also passes
alone in a fresh process."""
import ctypes

import numpy as np
import pytest
import torch

from moe_inputs import get_config, make_hidden, make_logits, make_weights
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu

CASES = [
    get_config("tiny", name="noalloc_small", T=200, E=8, top_k=2, H=256, F=384, seed=41),
    get_config("qwen3_decode"),
]


def _noalloc(M, prob, hidden, ids, w, wgu, wd, scale, out):
    L = M.lib()
    return L.moe_experts_forward_noalloc(ctypes.byref(prob), hidden.data_ptr(), ids.data_ptr(),
                                         w.data_ptr(), wgu.data_ptr(), wd.data_ptr(), None, None,
                                         None, ctypes.c_float(scale), out.data_ptr(),
                                         torch.cuda.current_stream().cuda_stream)


def _oracle(cfg, hidden, ids, w, weights, tokens):
    loader = lambda name, e: weights[name][e].float().cpu()
    return O.experts_forward(hidden.float().cpu(), ids, w, None, None,
                             cfg.routed_scaling_factor, tokens=tokens, weight_loader=loader)


@pytest.mark.parametrize("cfg", CASES, ids=[c.name for c in CASES])
def test_noalloc_matches_oracle_and_workspace_forward_twice(cfg):
    from moe_routed_expert_top_b200 import build
    build.build()
    import moe_routed_expert_top_b200 as M
    from tests.gpu_util import assert_within_tol, problem
    prob = problem(cfg)
    assert M.moe_workspace_bytes(prob) <= 64 * 1024 * 1024
    weights = make_weights(cfg, "cuda")
    hidden = make_hidden(cfg, "cuda")
    ids_np, w_np = O.route_topk(make_logits(cfg), cfg.top_k,
                                O.SOFTMAX if cfg.score_fn == "softmax" else O.SIGMOID, True)
    ids = torch.from_numpy(ids_np).cuda()
    w = torch.from_numpy(w_np).cuda()
    # the oracle on every token of the small case, on a seeded sample of the decode one
    if cfg.T <= 256:
        tokens = np.arange(cfg.T)
    else:
        tokens = np.unique(np.concatenate([[0, cfg.T - 1], np.random.default_rng(3).choice(
            cfg.T, 64, replace=False)]))
    oracle = _oracle(cfg, hidden, ids_np, w_np, weights, tokens)
    ref = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(M.moe_workspace_bytes(prob), dtype=torch.uint8, device="cuda")
    M.moe_experts_forward(prob, hidden, ids, w, weights["w_gate_up"], weights["w_down"], None,
                          None, None, cfg.routed_scaling_factor, ref, ws)
    torch.cuda.synchronize()
    ref_np = ref.double().cpu().numpy()
    for _ in range(2):
        out = torch.full((cfg.T, cfg.H), float("nan"), dtype=torch.bfloat16, device="cuda")
        st = _noalloc(M, prob, hidden, ids, w, weights["w_gate_up"], weights["w_down"],
                      cfg.routed_scaling_factor, out)
        assert st == 0, M.moe_status_string(st)
        torch.cuda.synchronize()
        got = out.double().cpu().numpy()
        assert np.isfinite(got).all()
        assert_within_tol(got[tokens], oracle, f"noalloc vs oracle {cfg.name}")
        assert_within_tol(got, ref_np, f"noalloc vs workspace forward {cfg.name}")
        assert M.moe_noalloc_read_status() == 0


def test_noalloc_status_word_reports_bad_expert_id():
    from moe_routed_expert_top_b200 import build
    build.build()
    import moe_routed_expert_top_b200 as M
    from tests.gpu_util import problem, random_ids
    cfg = get_config("tiny", name="noalloc_flag", T=64, E=8, top_k=2, H=256, F=128, seed=42)
    prob = problem(cfg)
    weights = make_weights(cfg, "cuda")
    hidden = make_hidden(cfg, "cuda")
    ids_np = random_ids(cfg.T, cfg.E, cfg.top_k, np.random.default_rng(6))
    w = torch.full((cfg.T, cfg.top_k), 0.5, dtype=torch.float32, device="cuda")
    out = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device="cuda")
    bad = ids_np.copy()
    bad[5, 1] = cfg.E          # one pair routed outside [0, E): skipped and flagged
    for ids_case, flag in ((bad, M.MOE_DEV_BAD_EXPERT_ID), (ids_np, 0)):
        ids = torch.from_numpy(ids_case).cuda()
        st = _noalloc(M, prob, hidden, ids, w, weights["w_gate_up"], weights["w_down"], 1.0, out)
        assert st == 0, M.moe_status_string(st)
        assert M.moe_noalloc_read_status() == flag


def test_noalloc_rejects_problem_larger_than_its_scratch():
    from moe_routed_expert_top_b200 import build
    build.build()
    import moe_routed_expert_top_b200 as M
    from tests.gpu_util import problem
    cfg = get_config("qwen3_prefill")
    prob = problem(cfg)
    assert M.moe_workspace_bytes(prob) > 64 * 1024 * 1024
    dummy = torch.empty(16, dtype=torch.uint8, device="cuda")
    L = M.lib()
    st = L.moe_experts_forward_noalloc(ctypes.byref(prob), dummy.data_ptr(), dummy.data_ptr(),
                                       dummy.data_ptr(), dummy.data_ptr(), dummy.data_ptr(), None,
                                       None, None, ctypes.c_float(1.0), dummy.data_ptr(),
                                       torch.cuda.current_stream().cuda_stream)
    assert st == M.MOE_ERR_WORKSPACE
