"""GPU parity of expert parallelism (moe_routed_expert_top_b200.ep): experts
split over `world` ranks, tokens dispatched to the ranks owning their experts
and combined back (pypto-lib PR #809). The ranks run emulated in one process on
the one GPU (every kernel is the library's; the all-to-alls hand buffers over),
so the whole dispatch / local-expert / combine data path runs for world 1, 2
and 4, with ragged token counts per rank, a rank without tokens, and the FP8
down path. Each rank's bf16 output is checked against the oracle's forward of
its tokens with all experts (|err| <= 1e-2 + 1e-2*|ref|) and against the
one-GPU forward of the same tokens."""
import numpy as np
import pytest
import torch

from moe_inputs import get_config, make_logits, make_weights
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from tests.gpu_util import ensure_built
    ensure_built()


def _gu():
    from tests import gpu_util
    return gpu_util


def _run(world, T_ranks, E, k, H, F, seed, fp8=False, bad_id=False):
    gu = _gu()
    from moe_routed_expert_top_b200.ep import EPRank, forward_emulated
    from moe_routed_expert_top_b200.layer import RoutedExperts
    T = sum(T_ranks)
    cfg = get_config("tiny", name=f"ep{world}", T=T, E=E, top_k=k, H=H, F=F,
                     score_fn="sigmoid", routed_scaling_factor=2.5, down_fp8=fp8, seed=seed)
    w = make_weights(cfg, "cuda")
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    hidden = torch.randn(T, H, generator=g, device="cuda").to(torch.bfloat16)
    ids, wt = O.route_topk(make_logits(cfg), k, O.SIGMOID, True)
    if bad_id:
        ids = ids.copy()
        ids[0, 0] = E                                        # no rank owns it
    El = E // world
    ranks = [EPRank(w["w_gate_up"][r * El:(r + 1) * El], w["w_down"][r * El:(r + 1) * El], E, k,
                    world, r, 2.5, fp8) for r in range(world)]
    cuts = np.cumsum([0] + list(T_ranks))
    hs = [hidden[cuts[r]:cuts[r + 1]] for r in range(world)]
    ids_r = [torch.from_numpy(ids[cuts[r]:cuts[r + 1]]).cuda() for r in range(world)]
    wt_r = [torch.from_numpy(wt[cuts[r]:cuts[r + 1]]).cuda() for r in range(world)]
    outs = forward_emulated(ranks, hs, ids_r, wt_r)
    torch.cuda.synchronize()
    return cfg, w, hidden, ids, wt, ranks, outs, cuts


@pytest.mark.parametrize("world,T_ranks", [(1, [150]), (2, [100, 37]), (4, [64, 0, 91, 5])])
@pytest.mark.parametrize("fp8", [False, True])
def test_ep_emulated_matches_oracle_and_one_gpu(world, T_ranks, fp8):
    gu = _gu()
    from moe_routed_expert_top_b200.layer import RoutedExperts
    E, k, H, F = 16, 4, 256, 256
    cfg, w, hidden, ids, wt, ranks, outs, cuts = _run(world, T_ranks, E, k, H, F,
                                                      7 + world, fp8)
    for r in ranks:
        assert int(r.dispatch_status.item()) == 0 if r.dispatch_status is not None else True
        assert int(r.local_status.item()) == 0
    out = torch.cat(outs)
    assert out.shape == (sum(T_ranks), H)

    def loader(name, e):
        return None if name in ("w_down_q", "w_down_s") else w[name][e].float().cpu()

    ref = O.experts_forward(hidden.float().cpu(), ids, wt, None, None, 2.5, fp8=fp8,
                            weight_loader=loader)
    gu.assert_within_tol(gu.f64(out), ref, f"ep world {world}")
    one = RoutedExperts(w["w_gate_up"], w["w_down"], k, "sigmoid", True, 2.5, fp8)
    single = one.forward(hidden, torch.from_numpy(ids).cuda(), torch.from_numpy(wt).cuda())
    torch.cuda.synchronize()
    gu.assert_within_tol(gu.f64(out), gu.f64(single), "ep vs one-GPU forward")


def test_ep_flags_an_id_no_rank_owns():
    import moe_routed_expert_top_b200 as M
    _, _, _, _, _, ranks, outs, _ = _run(2, [40, 40], 8, 2, 128, 128, 3, bad_id=True)
    assert int(ranks[0].dispatch_status.item()) & M.MOE_DEV_BAD_EXPERT_ID
    assert int(ranks[1].dispatch_status.item()) == 0


def test_gather_rows_and_split_ids():
    import moe_routed_expert_top_b200 as M
    src = torch.arange(40, dtype=torch.float32, device="cuda").reshape(10, 4)
    mp = torch.tensor([3, -1, 9, 0, 12], dtype=torch.int32, device="cuda")
    dst = torch.full((5, 4), 7.0, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    M.moe_gather_rows(5, 10, 16, mp, src, dst, st)
    torch.cuda.synchronize()
    want = torch.stack([src[3], torch.zeros(4, device="cuda"), src[9], src[0],
                        torch.zeros(4, device="cuda")])
    assert torch.equal(dst, want) and int(st.item()) & M.MOE_DEV_BAD_TABLES
    ids = torch.tensor([0, 5, 11, 12, -1, 7], dtype=torch.int32, device="cuda")
    rk, lo = torch.empty_like(ids), torch.empty_like(ids)
    M.moe_ep_split_ids(6, 4, 3, ids, rk, lo)
    torch.cuda.synchronize()
    assert rk.tolist() == [0, 1, 2, 3, 3, 1] and lo.tolist() == [0, 1, 3, 0, 0, 3]
