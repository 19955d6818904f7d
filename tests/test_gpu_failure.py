"""Failure detection on the GPU without a fault: a bounded pipeline wait that
runs out. moe_selftest_bounded_wait runs the kernels' own mbarrier wait on
barriers that nothing arrives on, with a 2 ms limit in place of the 4 s
production limit. The wait must give up (never hang), OR MOE_DEV_TIMEOUT into
the status word, stop the CTA's other waiting thread through the abort flag,
finish its deadline-bounded drain and free its tensor memory, leaving the
CUDA context usable; the host maps the flag to MOE_ERR_TIMEOUT."""
import pytest
import torch

pytestmark = pytest.mark.gpu

LIMIT_NS = 2_000_000  # 2 ms


@pytest.fixture(scope="module", autouse=True)
def _built():
    from tests.gpu_util import ensure_built
    ensure_built()


def test_bounded_wait_runs_out_and_reports_timeout():
    import moe_routed_expert_top_b200 as M
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    result = torch.full((6,), -1, dtype=torch.int64, device="cuda")
    M.moe_selftest_bounded_wait(LIMIT_NS, status, result)
    torch.cuda.synchronize()
    ok0, t0, ok1, t1, drained, t_drain = (int(v) for v in result.cpu())
    st = int(status.item())
    assert st & M.MOE_DEV_TIMEOUT
    assert M.moe_decode_device_status(st) == M.MOE_ERR_TIMEOUT
    # the lonely wait gave up after its limit, and not much later
    assert ok0 == 0 and LIMIT_NS <= t0 < 50 * LIMIT_NS, t0
    # the second thread saw the abort flag instead of running to its own 10x limit
    assert ok1 == 0 and t1 < 10 * LIMIT_NS, t1
    # the teardown drain is bounded by its shared deadline
    assert drained == 0 and LIMIT_NS <= t_drain < 50 * LIMIT_NS, t_drain


def test_context_usable_after_a_timeout():
    """After the timed-out kernel returns, the device still runs work (the
    tensor memory it held was freed: a second self-test allocates it again)."""
    import moe_routed_expert_top_b200 as M
    for _ in range(2):
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        result = torch.full((6,), -1, dtype=torch.int64, device="cuda")
        M.moe_selftest_bounded_wait(LIMIT_NS, status, result)
        torch.cuda.synchronize()
        assert int(status.item()) == M.MOE_DEV_TIMEOUT
    x = torch.arange(1024, device="cuda", dtype=torch.float32)
    assert float((x * 2).sum().item()) == 2.0 * 1023 * 1024 / 2
