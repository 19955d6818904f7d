"""GPU parity of the training-side FP8 kernels (XTuner PR #2089, Changes):
dual-layout quantisation (forward 1x128 rows + transposed expert-padded copy
with per-block or per-tile scales), its SwiGLU-fused form, and the SwiGLU
backward. Codes and scales are bit-exact against the oracle (for the fused
SwiGLU form: from the kernel's own fp32 h, which is itself checked against the
oracle's h); the backward's bf16 output within 4e-3*|ref| + 1e-4."""
import numpy as np
import pytest
import torch

from moe_inputs import get_config
from oracle import moe_oracle as O

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from tests.gpu_util import ensure_built
    ensure_built()


def _gu():
    from tests import gpu_util
    return gpu_util


def _grouped(M, E, sizes, seed):
    """Tables for M rows routed one expert each (top_k 1) with given sizes."""
    gu = _gu()
    cfg = get_config("tiny", T=M, E=E, top_k=1, H=128, F=128)
    ids = gu.random_ids(M, E, 1, np.random.default_rng(seed), sizes=sizes)
    L, tables, status, _ = gu.gpu_tables(cfg, ids)
    assert int(status.item()) == 0
    tab = O.dispatch_tables(ids, E, 128)
    return gu.problem(cfg), L, tables, tab


def _outputs(M, K, M_blk, per_block):
    dev = "cuda"
    q = torch.full((M, K), 0x55, dtype=torch.uint8, device=dev)
    s = torch.full((M, K // 128), -1.0, device=dev)
    qT = torch.full((K, 128 * M_blk), 0x55, dtype=torch.uint8, device=dev)
    sT = torch.full((K // 128, M_blk) if per_block else (K, M_blk), -1.0, device=dev)
    return q, s, qT, sT


def _compare(x32, cols, M_blk, per_block, q, s, qT, sT):
    rq, rs, rqT, rsT = O.quant_dual(x32, cols, 128 * M_blk, per_block)
    assert np.array_equal(q.cpu().numpy(), rq)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), rs.view(np.uint32))
    assert np.array_equal(qT.cpu().numpy(), rqT)
    assert np.array_equal(sT.cpu().numpy().view(np.uint32), rsT.view(np.uint32))


CASES = [
    # M, E, sizes, K
    (260, 8, None, 256),
    (1100, 8, [0, 1, 127, 128, 129, 0, 255, 460], 256),
    (700, 9, None, 384),
    (1000, 3, [1000, 0, 0], 128),
]


def _sizes(M, E, sizes, rng):
    if sizes is not None and sum(sizes) == M and min(sizes) >= 0:
        return sizes
    p = rng.dirichlet(np.ones(E))
    s = np.floor(p * M).astype(int)
    s[0] += M - s.sum()
    return list(s)


@pytest.mark.parametrize("per_block", [True, False])
@pytest.mark.parametrize("M,E,sizes,K", CASES)
def test_quant_dual_grouped_bit_exact(M, E, sizes, K, per_block):
    import moe_routed_expert_top_b200 as Mo
    rng = np.random.default_rng(M + K)
    sizes = _sizes(M, E, sizes, rng)
    prob, L, tables, tab = _grouped(M, E, sizes, M)
    M_blk = Mo.moe_dual_blocks(prob, M)
    assert M_blk == L["M_blk"]
    x = (torch.randn(M, K, device="cuda") * torch.rand(M, 1, device="cuda") * 4).to(torch.bfloat16)
    x[::7, :128] = 0                                   # all-zero row tiles
    q, s, qT, sT = _outputs(M, K, M_blk, per_block)
    mode = Mo.MOE_TRANS_PER_BLOCK if per_block else Mo.MOE_TRANS_PER_TILE
    Mo.moe_quant_dual(prob, tables, M, K, x, mode, q, s, qT, sT)
    torch.cuda.synchronize()
    _compare(x.float().cpu().numpy(), O.padded_columns(tab), M_blk, per_block, q, s, qT, sT)


@pytest.mark.parametrize("per_block", [True, False])
@pytest.mark.parametrize("M", [1, 128, 129, 300])
def test_quant_dual_dense_bit_exact(M, per_block):
    import moe_routed_expert_top_b200 as Mo
    K = 256
    M_blk = Mo.moe_dual_blocks(None, M)
    assert M_blk == -(-M // 128)
    x = torch.randn(M, K, device="cuda").to(torch.bfloat16)
    q, s, qT, sT = _outputs(M, K, M_blk, per_block)
    mode = Mo.MOE_TRANS_PER_BLOCK if per_block else Mo.MOE_TRANS_PER_TILE
    Mo.moe_quant_dual(None, None, M, K, x, mode, q, s, qT, sT)
    torch.cuda.synchronize()
    _compare(x.float().cpu().numpy(), np.arange(M), M_blk, per_block, q, s, qT, sT)


def _midpoint_tile_values(rng, n, scale):
    """bf16 values x = scale * m for E4M3 rounding midpoints m (exact in bf16),
    and their one-bf16-ulp neighbours: x / scale is exactly a tie, or just off
    one, so a quotient one fp32 ulp wrong changes the code."""
    v = np.unique(np.abs(O.e4m3_decode_table()[np.isfinite(O.e4m3_decode_table())]))
    mids = (v[:-1] + v[1:]) / 2
    x = scale * rng.choice(mids, size=n) * rng.choice([-1.0, 1.0], size=n)
    xb = np.asarray(O.bf16_round(x))
    bits = O.bf16_bits(xb).astype(np.int32) + rng.choice([-1, 0, 0, 1], size=n)
    return O.bf16_from_bits(bits.astype(np.uint16))


@pytest.mark.parametrize("per_block", [True, False])
def test_quant_dual_division_at_e4m3_midpoints(per_block):
    import moe_routed_expert_top_b200 as Mo
    rng = np.random.default_rng(12)
    K = 256
    groups = [(672.0, 1.5), (560.0, 1.25), (784.0, 1.75),
              (672.0 * 2.0 ** -80, 1.5 * 2.0 ** -80),    # fast path, tiny scale
              (672.0 * 2.0 ** -100, 1.5 * 2.0 ** -100)]  # below 2^-90: plain division
    rows = []
    for amax, s in groups:
        blk = _midpoint_tile_values(rng, 128 * K, s).reshape(128, K)
        blk[0, :] = amax          # every row tile, column tile and block has this amax
        blk[:, 0] = amax
        blk[:, 128] = amax
        rows.append(blk)
    x32 = np.concatenate(rows).astype(np.float32)
    M = x32.shape[0]
    x = torch.from_numpy(x32).to(torch.bfloat16).cuda()
    assert np.array_equal(x.float().cpu().numpy(), x32)       # exact in bf16
    M_blk = Mo.moe_dual_blocks(None, M)
    q, s, qT, sT = _outputs(M, K, M_blk, per_block)
    mode = Mo.MOE_TRANS_PER_BLOCK if per_block else Mo.MOE_TRANS_PER_TILE
    Mo.moe_quant_dual(None, None, M, K, x, mode, q, s, qT, sT)
    torch.cuda.synchronize()
    _compare(x32, np.arange(M), M_blk, per_block, q, s, qT, sT)


@pytest.mark.parametrize("per_block", [True, False])
def test_swiglu_quant_dual(per_block):
    import moe_routed_expert_top_b200 as Mo
    M, E, F = 600, 7, 256
    rng = np.random.default_rng(5)
    prob, L, tables, tab = _grouped(M, E, _sizes(M, E, None, rng), 5)
    M_blk = Mo.moe_dual_blocks(prob, M)
    gate_up = (torch.randn(M, 2 * F, device="cuda") * 2).to(torch.bfloat16)
    q, s, qT, sT = _outputs(M, F, M_blk, per_block)
    h = torch.empty(M, F, device="cuda")
    mode = Mo.MOE_TRANS_PER_BLOCK if per_block else Mo.MOE_TRANS_PER_TILE
    Mo.moe_swiglu_quant_dual(prob, tables, M, F, gate_up, mode, q, s, qT, sT, h)
    torch.cuda.synchronize()
    # the kernel's fp32 h against the oracle's SwiGLU, then every code from it
    gu = _gu()
    gu.assert_within_tol(gu.f64(h), O.swiglu(gu.f64(gate_up), F), "h", rtol=1e-5, atol=1e-6)
    _compare(h.cpu().numpy(), O.padded_columns(tab), M_blk, per_block, q, s, qT, sT)


@pytest.mark.parametrize("M,F", [(1, 8), (333, 136), (2048, 1024)])
def test_swiglu_backward(M, F):
    import moe_routed_expert_top_b200 as Mo
    gate_up = (torch.randn(M, 2 * F, device="cuda") * 2).to(torch.bfloat16)
    gate_up[0, :4] = torch.tensor([0.0, -1.2785, 30.0, -30.0])     # dSiLU zero crossing, saturation
    grad_h = torch.randn(M, F, device="cuda").to(torch.bfloat16)
    out = torch.full((M, 2 * F), float("nan"), dtype=torch.bfloat16, device="cuda")
    Mo.moe_swiglu_backward(M, F, gate_up, grad_h, out)
    torch.cuda.synchronize()
    gu = _gu()
    ref = O.swiglu_backward(gu.f64(gate_up), gu.f64(grad_h))
    gu.assert_within_tol(gu.f64(out), ref, "grad_gate_up", rtol=4e-3, atol=1e-4)


def test_full_size_sampled_blocks():
    """The pages' benchmark shape: x [131072, 6144] over 256 experts; rows and
    transposed blocks sampled, each recomputed by the oracle from its own
    rows (a block depends only on them)."""
    import moe_routed_expert_top_b200 as Mo
    M, E, K = 131072, 256, 6144
    rng = np.random.default_rng(9)
    prob, L, tables, tab = _grouped(M, E, _sizes(M, E, None, rng), 9)
    M_blk = Mo.moe_dual_blocks(prob, M)
    x = torch.randn(M, K, device="cuda").to(torch.bfloat16)
    for per_block in (True, False):
        q, s, qT, sT = _outputs(M, K, M_blk, per_block)
        mode = Mo.MOE_TRANS_PER_BLOCK if per_block else Mo.MOE_TRANS_PER_TILE
        Mo.moe_quant_dual(prob, tables, M, K, x, mode, q, s, qT, sT)
        torch.cuda.synchronize()
        rows = rng.choice(M, 16, replace=False)
        rq, rs = O.quant_1x128(x[torch.from_numpy(rows).cuda()].float().cpu().numpy())
        assert np.array_equal(q[torch.from_numpy(rows).cuda()].cpu().numpy(), rq)
        assert np.array_equal(s[torch.from_numpy(rows).cuda()].cpu().numpy(), rs)
        for bx in rng.choice(int(tab["group_padded_offsets"][-1]) // 128, 6, replace=False):
            _, m0, n = O.block_rows(tab, int(bx), 128)
            kb = int(rng.integers(K // 128))
            blk = x[m0:m0 + n, kb * 128:(kb + 1) * 128].float().cpu().numpy()
            bq, bs = O.quant_transposed(blk, np.arange(n), 128, per_block)
            got = qT[kb * 128:(kb + 1) * 128, bx * 128:(bx + 1) * 128].cpu().numpy()
            assert np.array_equal(got, bq)
            if per_block:
                assert sT[kb, bx].item() == bs[0, 0]
            else:
                assert np.array_equal(sT[kb * 128:(kb + 1) * 128, bx].cpu().numpy(), bs[:, 0])


def test_more_tiles_than_the_rows_table_holds():
    """Dense x [20000037, 128]: 156251 128x128 tiles, more per persistent CTA
    than the kernel's precomputed table of tile rows holds (512), so the last
    tiles of every CTA take their rows from the tables as they go, and the
    row and column offsets pass 2^31 bytes. Sampled rows and blocks, the
    ragged last block among them, against the oracle."""
    import moe_routed_expert_top_b200 as Mo
    M, K = 20000037, 128
    rng = np.random.default_rng(31)
    M_blk = Mo.moe_dual_blocks(None, M)
    assert M_blk == (M + 127) // 128
    torch.manual_seed(31)
    x = torch.randn(M, K, device="cuda", dtype=torch.bfloat16)
    for per_block in (True, False):
        q, s, qT, sT = _outputs(M, K, M_blk, per_block)
        mode = Mo.MOE_TRANS_PER_BLOCK if per_block else Mo.MOE_TRANS_PER_TILE
        Mo.moe_quant_dual(None, None, M, K, x, mode, q, s, qT, sT)
        torch.cuda.synchronize()
        rows = np.concatenate([rng.choice(M, 8, replace=False), [M - 1, M - 37, 19_500_000]])
        ridx = torch.from_numpy(rows).cuda()
        rq, rs = O.quant_1x128(x[ridx].float().cpu().numpy())
        assert np.array_equal(q[ridx].cpu().numpy(), rq)
        assert np.array_equal(s[ridx].cpu().numpy(), rs)
        for bx in list(rng.integers(152_000, M_blk - 1, 4)) + [0, M_blk - 1]:
            m0 = int(bx) * 128
            n = min(128, M - m0)
            blk = x[m0:m0 + n].float().cpu().numpy()
            bq, bs = O.quant_transposed(blk, np.arange(n), 128, per_block)
            got = qT[:, int(bx) * 128:(int(bx) + 1) * 128].cpu().numpy()
            assert np.array_equal(got, bq)
            if per_block:
                assert sT[0, int(bx)].item() == bs[0, 0]
            else:
                assert np.array_equal(sT[:, int(bx)].cpu().numpy(), bs[:, 0])
        del q, s, qT, sT
        torch.cuda.empty_cache()


def test_train_fp8_rejects():
    import moe_routed_expert_top_b200 as Mo
    x = torch.zeros(8, 128, dtype=torch.bfloat16, device="cuda")
    q, s, qT, sT = _outputs(8, 128, 1, True)

    def st(call):
        try:
            call()
        except Mo.MoeError as e:
            return e.status
        return Mo.MOE_OK

    assert st(lambda: Mo.moe_quant_dual(None, None, 8, 64, x, 0, q, s, qT, sT)) == \
        Mo.MOE_ERR_INVALID_ARG                                     # K % 128
    assert st(lambda: Mo.moe_quant_dual(None, None, 8, 128, x, 2, q, s, qT, sT)) == \
        Mo.MOE_ERR_INVALID_ARG                                     # trans mode
    assert st(lambda: Mo.moe_quant_dual(None, None, 0, 128, x, 0, q, s, qT, sT)) == Mo.MOE_OK
    assert st(lambda: Mo.moe_swiglu_backward(8, 12, x, x, x)) == Mo.MOE_ERR_INVALID_ARG
