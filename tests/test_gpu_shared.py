"""GPU parity of moe_shared_expert_forward: the shared expert of one
tensor-parallel rank, reading its shard of the complete weights in place
(TileOPs PR #778, TP split convention and Partial output contract). Every rank
of tp_size is run in turn on the one GPU; each partial is compared with the
oracle's partial of that rank, and the sum of the partials with the unsharded
shared expert. Tolerance |err| <= 1e-2 + 1e-2*|ref| (the forward's bound: h is
rounded to bf16 on both sides, so a rounding-boundary flip of one h element
moves the output by up to one bf16 ulp of that term)."""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from tests.gpu_util import ensure_built
    ensure_built()


def _gu():
    from tests import gpu_util
    return gpu_util


def _weights(T, H, F_s, seed, std=0.05):
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    hidden = torch.randn(T, H, generator=g, device="cuda").to(torch.bfloat16)
    wgu = (torch.randn(2 * F_s, H, generator=g, device="cuda") * std).to(torch.bfloat16)
    wd = (torch.randn(H, F_s, generator=g, device="cuda") * std).to(torch.bfloat16)
    return hidden, wgu, wd


@pytest.mark.parametrize("T,H,F_s,tp", [(200, 256, 512, 1), (200, 256, 512, 2),
                                        (300, 512, 1024, 4), (1, 256, 256, 2),
                                        (37, 256, 768, 3), (130, 512, 1024, 8)])
def test_shared_partials_and_their_sum(T, H, F_s, tp):
    gu = _gu()
    from moe_routed_expert_top_b200.layer import SharedExpert
    hidden, wgu, wd = _weights(T, H, F_s, 11 * tp + T)
    full = O.dense_swiglu_mlp(hidden.cpu(), wgu.cpu(), wd.cpu())
    total = torch.zeros(T, H, dtype=torch.float64)
    for r in range(tp):
        layer = SharedExpert(wgu, wd, tp, r)
        p32 = layer.forward(hidden, out_f32=True)
        p16 = layer.forward(hidden, out_f32=False)
        torch.cuda.synchronize()
        assert layer.device_status() == 0
        ref = O.shared_expert_partial(hidden.cpu(), wgu.cpu(), wd.cpu(), tp, r)
        gu.assert_within_tol(gu.f64(p32), ref, f"partial {r}/{tp} fp32")
        gu.assert_within_tol(gu.f64(p16), O.bf16_round(ref), f"partial {r}/{tp} bf16")
        # the bf16 output is the fp32 one, rounded once
        assert torch.equal(p16, p32.to(torch.bfloat16))
        total += p32.double().cpu()
    gu.assert_within_tol(total.numpy(), full, f"sum of {tp} partials")


def test_shared_kimi_k2_scale_shard():
    """One rank of tp_size 8 at the Kimi-K2 shared-expert size (H=7168,
    F_s=18432; TileOPs PR #778, Benchmark)."""
    gu = _gu()
    from moe_routed_expert_top_b200.layer import SharedExpert
    T, H, F_s, tp, r = 64, 7168, 18432, 8, 5
    hidden, wgu, wd = _weights(T, H, F_s, 99, std=0.02)
    out = SharedExpert(wgu, wd, tp, r).forward(hidden)
    torch.cuda.synchronize()
    ref = O.shared_expert_partial(hidden.cpu(), wgu.cpu(), wd.cpu(), tp, r)
    gu.assert_within_tol(gu.f64(out), ref, "kimi-k2 shard")


def test_shared_rejects():
    import moe_routed_expert_top_b200 as M
    T, H, F_s = 16, 256, 512
    hidden, wgu, wd = _weights(T, H, F_s, 3)
    out = torch.empty(T, H, dtype=torch.float32, device="cuda")
    ws = torch.empty(M.moe_shared_workspace_bytes(T, H, F_s, 2), dtype=torch.uint8,
                     device="cuda")

    def status_of(*args, ws_bytes=None):
        try:
            M.moe_shared_expert_forward(*args, out, ws, ws_bytes=ws_bytes)
        except M.MoeError as e:
            return e.status
        return M.MOE_OK

    assert status_of(T, H, F_s, 2, 2, hidden, wgu, wd, 1) == M.MOE_ERR_INVALID_ARG  # rank
    assert status_of(T, H, F_s, 3, 0, hidden, wgu, wd, 1) == M.MOE_ERR_INVALID_ARG  # F_s % tp
    assert status_of(T, H, 384, 2, 0, hidden, wgu, wd, 1) == M.MOE_ERR_UNSUPPORTED  # F_p % 128
    assert status_of(T, H, F_s, 2, 0, hidden, wgu, wd, 1, ws_bytes=16) == M.MOE_ERR_WORKSPACE
    assert status_of(0, H, F_s, 2, 0, hidden, wgu, wd, 1) == M.MOE_OK              # no tokens
    assert M.moe_last_launch_count() == 0
