"""GPU test of moe_experts_forward_noalloc, the forward for callers that cannot
allocate device memory (its workspace is a fixed 64 MiB array inside the
library). Called through the C ABI twice in a row, its output must match the
regular moe_experts_forward (caller-supplied workspace) within the bf16
tolerance used by every forward test; a problem too large for the array is
rejected before anything runs. Collected last so a failure here comes after
every other test has run; it also passes alone in a fresh process."""
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


@pytest.mark.parametrize("cfg", CASES, ids=[c.name for c in CASES])
def test_noalloc_matches_workspace_forward_twice(cfg):
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
        assert_within_tol(out.double().cpu().numpy(), ref_np, f"noalloc {cfg.name}")
        assert np.isfinite(out.double().cpu().numpy()).all()


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
