"""GPU parity of the down GEMM with the routing weight folded into its epilogue
(moe_down_gemm_weighted) and of the combine that follows (moe_combine),
element by element against the oracle's ``weighted_rows`` and ``combine``.

Shapes span several tiles, ragged expert tails, empty experts, experts just
past one token tile, pairs routed to an invalid expert (no permuted row: never
written, never summed), bf16 and FP8 block-scaled operands, and every tiling
(token-row tiles refuse the weighted store), weighted rows in bf16 and in
fp32. Tolerance: bf16 outputs |err| <= 1e-2 + 1e-2*|ref|, fp32 rows 1e-4 +
1e-4*|ref|. The combine is also checked bit for bit against fp32 sums in slot
order, its stated arithmetic, for bf16 and fp32 inputs."""
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


TILINGS = [0x00, 0x20, 0x30]   # MOE_TILE_AUTO, MOE_TILE_WEIGHT_ROWS, MOE_TILE_WEIGHT_ROWS_PAIR

CASES = [
    # T, E, k, K, N, sizes (rows per expert) or None, invalid-id fraction
    (9, 4, 2, 64, 128, None, 0.0),
    (260, 8, 3, 384, 256, [0, 1, 127, 128, 129, 0, 255, 140], 0.0),
    (546, 8, 4, 256, 512, [257, 288, 289, 517, 544, 256, 0, 33], 0.0),
    (300, 16, 4, 256, 768, None, 0.05),
    (2048, 16, 4, 512, 512, None, 0.0),
]


def _routing(T, E, k, sizes, bad, rng):
    ids = _gu().random_ids(T, E, k, rng, sizes=sizes)
    if bad:
        mask = rng.random(ids.shape) < bad
        ids = np.where(mask, E, ids).astype(np.int32)   # expert E does not exist
    w = rng.random((T, k)).astype(np.float32) + 0.05
    return ids, w


def _oracle_tables(ids, E):
    """The oracle's tables for a routing that may hold ids outside [0, E):
    those pairs get no row. Computed as the tables of E + 1 experts with every
    invalid id sent to the extra last expert, whose rows (after all valid ones
    in expert order) are then dropped."""
    ids = np.asarray(ids)
    t = O.dispatch_tables(np.where((ids < 0) | (ids >= E), E, ids), E + 1, 128)
    nvalid = int(t["group_offsets"][E])
    rop = np.array(t["row_of_pair"])
    por = np.array(t["pair_of_row"])
    rop[rop >= nvalid] = -1
    por[nvalid:] = -1
    return {"group_offsets": np.asarray(t["group_offsets"])[:E + 1], "row_of_pair": rop,
            "pair_of_row": por}


def _rows(A_np, N, ref, E, W_np=None, fp8=None):
    """Oracle down rows over each expert's permuted rows (float64): bf16
    operands A @ W[e]^T, or the FP8 block-scaled product of ``fp8``."""
    P = A_np.shape[0]
    out = np.zeros((P, N))
    for e in range(E):
        a, b = ref["group_offsets"][e], ref["group_offsets"][e + 1]
        if b > a:
            if fp8 is None:
                out[a:b] = A_np[a:b] @ W_np[e].T
            else:
                qa, sa, wq, ws = fp8
                out[a:b] = O.fp8_block_scaled_matmul(qa[a:b], sa[a:b], wq[e], ws[e])
    return out


@pytest.mark.parametrize("f32", [False, True])
@pytest.mark.parametrize("tiling", TILINGS + [0x10])
@pytest.mark.parametrize("T,E,k,K,N,sizes,bad", CASES)
def test_down_gemm_weighted_bf16(T, E, k, K, N, sizes, bad, tiling, f32):
    gu = _gu()
    import moe_routed_expert_top_b200 as M
    rng = np.random.default_rng(T + N)
    ids, w = _routing(T, E, k, sizes, bad, rng)
    cfg = get_config("tiny", T=T, E=E, top_k=k, H=K, F=64)
    g = torch.Generator(device="cuda")
    g.manual_seed(T)
    hidden = torch.randn(T, K, generator=g, device="cuda").to(torch.bfloat16)
    L, tables, status, x_perm = gu.gpu_tables(cfg, ids, hidden=hidden)
    status.zero_()
    ref = _oracle_tables(ids, E)
    W = (torch.randn(E, N, K, generator=g, device="cuda") * 0.05).to(torch.bfloat16)
    y_w = torch.full((L["P"], N), float("nan"), dtype=torch.float32 if f32 else torch.bfloat16,
                     device="cuda")
    wt = torch.from_numpy(w).cuda()
    epi = (M.MOE_EPI_STORE_F32 if f32 else M.MOE_EPI_STORE) | tiling
    call = lambda: M.moe_down_gemm_weighted(gu.problem(cfg), N, K, x_perm, None, W, None, tables,
                                            wt, 2.5, epi, y_w, status)
    if tiling == 0x10 or (tiling == 0x30 and N % 256 != 0):
        with pytest.raises(M.MoeError) as ei:
            call()
        assert ei.value.status == M.MOE_ERR_UNSUPPORTED
        return
    call()
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    A = O.permute(gu.f64(hidden), ref["pair_of_row"], k)
    rows = _rows(A, N, ref, E, W_np=gu.f64(W))
    want, written = O.weighted_rows(rows, ref["pair_of_row"], w, 2.5, round_output=not f32)
    got = gu.f64(y_w)
    assert np.isfinite(got[written]).all()
    assert np.isnan(got[~written]).all()            # pairs without a row are not written
    if f32:
        gu.assert_within_tol(got[written], want[written], "weighted down rows f32",
                             rtol=1e-4, atol=1e-4)
    else:
        gu.assert_within_tol(got[written], want[written], "weighted down rows")


@pytest.mark.parametrize("f32", [False, True])
@pytest.mark.parametrize("tiling", [0x00, 0x20, 0x30])
@pytest.mark.parametrize("T,E,k,H,F,sizes,bad", [(200, 8, 2, 256, 384, None, 0.0),
                                                (260, 8, 3, 512, 256,
                                                 [0, 1, 127, 128, 129, 0, 255, 140], 0.0),
                                                (150, 6, 2, 384, 512, None, 0.1)])
def test_down_gemm_weighted_fp8(T, E, k, H, F, sizes, bad, tiling, f32):
    gu = _gu()
    import moe_routed_expert_top_b200 as M
    rng = np.random.default_rng(7 + T)
    ids, w = _routing(T, E, k, sizes, bad, rng)
    cfg = get_config("tiny", T=T, E=E, top_k=k, H=H, F=F)
    L, tables, status, _ = gu.gpu_tables(cfg, ids)
    status.zero_()
    ref = _oracle_tables(ids, E)
    P = L["P"]
    h = (rng.standard_normal((P, F)) * rng.uniform(0.1, 3, (P, 1))).astype(np.float32)
    qa, sa = O.quant_1x128(h)
    wd = (rng.standard_normal((E, H, F)) * 0.05).astype(np.float32)
    wq, ws = zip(*[O.quant_weight_128x128(wd[e]) for e in range(E)])
    wq, ws = np.stack(wq), np.stack(ws)
    y_w = torch.full((P, H), float("nan"), dtype=torch.float32 if f32 else torch.bfloat16,
                     device="cuda")
    epi = (M.MOE_EPI_STORE_F32 if f32 else M.MOE_EPI_STORE) | tiling
    call = lambda: M.moe_down_gemm_weighted(
        gu.problem(cfg), H, F, torch.from_numpy(qa).cuda(), torch.from_numpy(sa).cuda(),
        torch.from_numpy(wq).cuda(), torch.from_numpy(ws).cuda(), tables,
        torch.from_numpy(w).cuda(), 2.5, epi, y_w, status)
    if tiling == 0x30:   # the pair tiling is bf16 only
        with pytest.raises(M.MoeError) as ei:
            call()
        assert ei.value.status == M.MOE_ERR_UNSUPPORTED
        return
    call()
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    rows = _rows(qa, H, ref, E, fp8=(qa, sa, wq, ws))
    want, written = O.weighted_rows(rows, ref["pair_of_row"], w, 2.5, round_output=not f32)
    got = gu.f64(y_w)
    assert np.isnan(got[~written]).all()
    if f32:
        gu.assert_within_tol(got[written], want[written], "fp8 weighted down rows f32",
                             rtol=1e-4, atol=1e-4)
    else:
        gu.assert_within_tol(got[written], want[written], "fp8 weighted down rows")


def _fp32_slot_order(y_w_f32, rop, k, addend):
    """The combine's stated arithmetic: fp32 sums in slot order, then the addend."""
    P, H = y_w_f32.shape
    T = P // k
    acc = np.zeros((T, H), dtype=np.float32)
    for j in range(k):
        has = rop[j::k] >= 0
        acc[has] = (acc[has] + y_w_f32[j::k][has]).astype(np.float32)
    if addend is not None:
        acc = (acc + addend).astype(np.float32)
    return O.bf16_round(acc.astype(np.float64))


@pytest.mark.parametrize("f32", [False, True])
@pytest.mark.parametrize("T,E,k,H,addend,bad", [(9, 4, 2, 128, False, 0.0),
                                               (300, 16, 8, 2048, True, 0.0),
                                               (77, 7, 3, 7168, True, 0.2),
                                               (1, 8, 8, 256, False, 0.0),
                                               (40, 40, 32, 128, True, 0.1)])
def test_combine(T, E, k, H, addend, bad, f32):
    gu = _gu()
    import moe_routed_expert_top_b200 as M
    rng = np.random.default_rng(100 + T)
    ids, _ = _routing(T, E, k, None, bad, rng)
    cfg = get_config("tiny", T=T, E=E, top_k=k, H=H, F=64)
    L, tables, status, _ = gu.gpu_tables(cfg, ids)
    ref_t = _oracle_tables(ids, E)
    rop = np.asarray(ref_t["row_of_pair"])
    y_w = torch.from_numpy((rng.standard_normal((T * k, H)) * 0.7).astype(np.float32)).cuda()
    if not f32:
        y_w = y_w.to(torch.bfloat16)
    add = (rng.standard_normal((T, H)) * 0.5).astype(np.float32) if addend else None
    out = torch.full((T, H), float("nan"), dtype=torch.bfloat16, device="cuda")
    M.moe_combine(gu.problem(cfg), y_w, tables, torch.from_numpy(add).cuda() if addend else None,
                  out)
    torch.cuda.synchronize()
    yw = gu.f64(y_w)
    gu.assert_within_tol(gu.f64(out), O.combine(yw, rop, k, addend=add), "combine")
    exact = _fp32_slot_order(yw.astype(np.float32), rop, k, add)
    assert np.array_equal(gu.f64(out), exact)


def test_combine_rejects():
    gu = _gu()
    import moe_routed_expert_top_b200 as M
    cfg = get_config("tiny", T=4, E=4, top_k=2, H=100, F=64)
    t = torch.zeros(4096, dtype=torch.int32, device="cuda")
    y = torch.zeros(8, 104, dtype=torch.bfloat16, device="cuda")
    out = torch.zeros(4, 104, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(M.MoeError) as ei:        # H % 8 != 0
        M.moe_combine(gu.problem(cfg), y, t, None, out)
    assert ei.value.status == M.MOE_ERR_INVALID_ARG
    cfg = get_config("tiny", T=4, E=4, top_k=2, H=128, F=64)
    with pytest.raises(M.MoeError) as ei:        # no tables
        M.moe_combine(gu.problem(cfg), y, None, None, out)
    assert ei.value.status == M.MOE_ERR_INVALID_ARG


@pytest.mark.parametrize("f32", [True, False])
def test_weighted_then_combine_is_the_forward(f32):
    """gate+up, the weighted down GEMM and the combine chained give the
    layer's output: against the oracle's forward within the output tolerance,
    and within the same tolerance of moe_experts_forward (which keeps the
    unweighted rows in the f16e format and sums them in the unpermute)."""
    gu = _gu()
    import moe_routed_expert_top_b200 as M
    from moe_inputs import make_hidden, make_logits, make_weights
    cfg = get_config("tiny", name="chain", T=200, E=8, top_k=2, H=256, F=256, seed=41,
                     routed_scaling_factor=1.7)
    prob = gu.problem(cfg)
    wts = make_weights(cfg, "cuda")
    hidden = make_hidden(cfg, "cuda")
    ids_np, w_np = O.route_topk(make_logits(cfg), cfg.top_k, gu.score_code(cfg), True)
    ids = torch.from_numpy(ids_np).cuda()
    w = torch.from_numpy(w_np).cuda()
    ws = torch.empty(M.moe_workspace_bytes(prob), dtype=torch.uint8, device="cuda")
    fwd = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device="cuda")
    M.moe_experts_forward(prob, hidden, ids, w, wts["w_gate_up"], wts["w_down"], None, None, None,
                          cfg.routed_scaling_factor, fwd, ws)
    L, tables, status, x_perm = gu.gpu_tables(cfg, ids_np, hidden=hidden)
    P = L["P"]
    h = torch.empty(P, cfg.F, dtype=torch.bfloat16, device="cuda")
    M.moe_grouped_gemm(prob, 0, 2 * cfg.F, cfg.H, x_perm, None, wts["w_gate_up"], None, tables,
                       M.MOE_EPI_SWIGLU, h, None, None, status)
    y_w = torch.empty(P, cfg.H, dtype=torch.float32 if f32 else torch.bfloat16, device="cuda")
    M.moe_down_gemm_weighted(prob, cfg.H, cfg.F, h, None, wts["w_down"], None, tables, w,
                             cfg.routed_scaling_factor,
                             M.MOE_EPI_STORE_F32 if f32 else M.MOE_EPI_STORE, y_w, status)
    out = torch.empty_like(fwd)
    M.moe_combine(prob, y_w, tables, None, out)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref = O.experts_forward(gu.f64(hidden), ids_np, w_np, gu.f64(wts["w_gate_up"]),
                            gu.f64(wts["w_down"]), cfg.routed_scaling_factor)
    gu.assert_within_tol(gu.f64(out), ref, "weighted down + combine")
    gu.assert_within_tol(gu.f64(out), gu.f64(fwd), "weighted down + combine vs the forward")


def test_weighted_down_needs_a_weight_row_tiling():
    """H = 192 (not a multiple of 128): no weight-row tiling takes N, so the
    weighted down GEMM refuses; the layer's forward (fp32 rows + unpermute)
    still runs and matches the oracle."""
    gu = _gu()
    import moe_routed_expert_top_b200 as M
    from moe_inputs import make_hidden, make_logits, make_weights
    cfg = get_config("tiny", name="h192", T=130, E=6, top_k=2, H=192, F=128, seed=42,
                     routed_scaling_factor=1.3)
    prob = gu.problem(cfg)
    wts = make_weights(cfg, "cuda")
    hidden = make_hidden(cfg, "cuda")
    ids_np, w_np = O.route_topk(make_logits(cfg), cfg.top_k, gu.score_code(cfg), True)
    L, tables, status, _ = gu.gpu_tables(cfg, ids_np)
    h = torch.zeros(L["P"], cfg.F, dtype=torch.bfloat16, device="cuda")
    y_w = torch.empty(L["P"], cfg.H, dtype=torch.float32, device="cuda")
    with pytest.raises(M.MoeError) as ei:
        M.moe_down_gemm_weighted(prob, cfg.H, cfg.F, h, None, wts["w_down"], None, tables,
                                 torch.from_numpy(w_np).cuda(), 1.0, M.MOE_EPI_STORE_F32, y_w,
                                 status)
    assert ei.value.status == M.MOE_ERR_UNSUPPORTED
    ws = torch.empty(M.moe_workspace_bytes(prob), dtype=torch.uint8, device="cuda")
    out = torch.empty(cfg.T, cfg.H, dtype=torch.bfloat16, device="cuda")
    M.moe_experts_forward(prob, hidden, torch.from_numpy(ids_np).cuda(),
                          torch.from_numpy(w_np).cuda(), wts["w_gate_up"], wts["w_down"], None,
                          None, None, cfg.routed_scaling_factor, out, ws)
    torch.cuda.synchronize()
    ref = O.experts_forward(gu.f64(hidden), ids_np, w_np, gu.f64(wts["w_gate_up"]),
                            gu.f64(wts["w_down"]), cfg.routed_scaling_factor)
    gu.assert_within_tol(gu.f64(out), ref, "forward H=192")


@pytest.mark.parametrize("name,f32", [("qwen3_prefill", True), ("qwen3_prefill", False),
                                      ("dsv3_decode_fp8", True)])
def test_weighted_chain_full_size_sampled(name, f32):
    """Full-size workloads: tables, gate+up (SwiGLU, or SwiGLU + FP8 1x128),
    the weighted down GEMM (bf16 or FP8 block-scaled) and the combine, against
    the oracle's forward on seeded token samples (including the tokens of the
    most and the least loaded experts)."""
    gu = _gu()
    import moe_routed_expert_top_b200 as M
    from moe_routed_expert_top_b200.layer import RoutedExperts
    from tests.test_gpu_forward import _inputs, _oracle
    cfg = get_config(name)
    hidden, ids, w, weights = _inputs(cfg)
    layer = RoutedExperts(weights["w_gate_up"], weights["w_down"], cfg.top_k, cfg.score_fn,
                          cfg.renormalize, cfg.routed_scaling_factor, cfg.down_fp8)
    prob = layer.problem(cfg.T)
    L, tables, status, x_perm = gu.gpu_tables(cfg, ids, hidden=hidden)
    P, H, F = L["P"], cfg.H, cfg.F
    if cfg.down_fp8:
        h = torch.empty(P, F, dtype=torch.uint8, device="cuda")
        hs = torch.empty(P, F // 128, dtype=torch.float32, device="cuda")
        epi = M.MOE_EPI_SWIGLU_FP8
    else:
        h = torch.empty(P, F, dtype=torch.bfloat16, device="cuda")
        hs, epi = None, M.MOE_EPI_SWIGLU
    M.moe_grouped_gemm(prob, 0, 2 * F, H, x_perm, None, layer.w_gate_up, None, tables, epi, h,
                       hs, None, status)
    y_w = torch.full((P, H), float("nan"), dtype=torch.float32 if f32 else torch.bfloat16,
                     device="cuda")
    M.moe_down_gemm_weighted(prob, H, F, h, hs, layer.w_down, layer.w_down_scales, tables,
                             torch.from_numpy(w).cuda(), cfg.routed_scaling_factor,
                             M.MOE_EPI_STORE_F32 if f32 else M.MOE_EPI_STORE, y_w, status)
    out = torch.empty(cfg.T, H, dtype=torch.bfloat16, device="cuda")
    M.moe_combine(prob, y_w, tables, None, out)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.isfinite(y_w.float()).all()          # every pair row written
    rng = np.random.default_rng(8)
    sizes = np.bincount(ids.reshape(-1), minlength=cfg.E)
    big = int(np.argmax(sizes))
    small = int(np.argmin(np.where(sizes > 0, sizes, 1 << 30)))
    t_big = int(np.nonzero((ids == big).any(1))[0][0])
    t_small = int(np.nonzero((ids == small).any(1))[0][0])
    n = 8 if cfg.H > 4096 else 24
    tokens = np.unique(np.concatenate([[0, cfg.T - 1, t_big, t_small],
                                       rng.choice(cfg.T, n, replace=False)]))
    ref = _oracle(cfg, hidden, ids, w, weights, tokens=tokens)
    gu.assert_within_tol(gu.f64(out[torch.from_numpy(tokens).cuda()]), ref,
                         f"{name} weighted chain")
