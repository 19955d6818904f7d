"""GPU parity: a4/a6 grouped GEMM (bf16 and FP8 block-scaled), the SwiGLU
and SwiGLU+FP8 epilogues, the standalone SwiGLU/quant kernel and the 128x128
weight quantiser, element by element against the oracle.

Shapes span several M-, N- and K-tiles, ragged expert tails, empty experts and
experts of 1/127/128/129 rows. Tolerance for bf16 outputs: |err| <= 1e-2 +
1e-2*|ref|; fp32 outputs 1e-4 + 1e-4*|ref|. FP8 codes and scales: bit-exact
against the oracle when the oracle's fp32 h is fed to the quantiser; the fused
epilogue's codes and scales bit for bit against the oracle's quantiser fed the
kernel's own fp32 h (also at the full DeepSeek-V3 decode size, in the launch
configuration the benchmark times), and against the oracle's h by the E4M3
error bound."""
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


def _setup(T, E, k, H, F, seed, sizes=None, std=0.05):
    """Tables from a routing (oracle-built ids), GPU tables, permuted rows."""
    gu = _gu()
    cfg = get_config("tiny", T=T, E=E, top_k=k, H=H, F=F)
    rng = np.random.default_rng(seed)
    ids = gu.random_ids(T, E, k, rng, sizes=sizes)
    g = torch.Generator(device="cuda")
    g.manual_seed(seed)
    hidden = torch.randn(T, H, generator=g, device="cuda").to(torch.bfloat16)
    L, tables, status, x_perm = gu.gpu_tables(cfg, ids, hidden=hidden)
    ref = O.dispatch_tables(ids, E, 128)
    wgu = (torch.randn(E, 2 * F, H, generator=g, device="cuda") * std).to(torch.bfloat16)
    wd = (torch.randn(E, H, F, generator=g, device="cuda") * std).to(torch.bfloat16)
    return cfg, ids, hidden, L, tables, status, x_perm, ref, wgu, wd


def _oracle_rows_gemm(hidden, W, ref, E, k):
    """Oracle C = A @ B[e]^T over each expert's rows (float64), A = the
    oracle's own permutation of hidden."""
    A = O.permute(_gu().f64(hidden), ref["pair_of_row"], k)
    out = np.zeros((A.shape[0], W.shape[1]))
    Wf = _gu().f64(W)
    for e in range(E):
        a, b = ref["group_offsets"][e], ref["group_offsets"][e + 1]
        if b > a:
            out[a:b] = O.gate_up_rows(A[a:b], Wf[e])
    return out


GEMM_CASES = [
    # T, E, k, H, F, sizes
    (9, 4, 2, 128, 64, None),
    (200, 8, 2, 256, 384, None),
    (260, 8, 3, 512, 128, [0, 1, 127, 128, 129, 0, 255, 140]),
    (300, 5, 1, 192, 256, [0, 0, 300, 0, 0]),
    # more tiles than resident CTAs: every persistent loop wraps
    (2048, 16, 4, 512, 512, None),
    # experts just past one or two token tiles (the pair tiling splits them
    # evenly over their tiles): 256-token tiles, then 64-token ones
    (546, 8, 4, 256, 256, [257, 288, 289, 517, 544, 256, 0, 33]),
    (256, 8, 2, 256, 256, [65, 96, 97, 160, 64, 0, 1, 29]),
    # experts averaging <= 160 rows take 192-token pair tiles (96-row token
    # boxes): one tile up to 192 rows, two above
    (300, 8, 4, 256, 256, [192, 193, 0, 150, 129, 300, 96, 140]),
]


# MOE_TILE_TOKEN_ROWS, MOE_TILE_WEIGHT_ROWS, MOE_TILE_WEIGHT_ROWS_PAIR
TILINGS = [0x10, 0x20, 0x30]
PAIR = 0x30


def _pair_unsupported(tiling, N, fp8=False):
    """The pair tiling takes bf16 operands with N % 256 == 0 only."""
    return tiling == PAIR and (fp8 or N % 256 != 0)


def _expect_unsupported(call):
    import moe_routed_expert_top_b200 as M
    with pytest.raises(M.MoeError) as ei:
        call()
    assert ei.value.status == M.MOE_ERR_UNSUPPORTED


@pytest.mark.parametrize("tiling", TILINGS)
@pytest.mark.parametrize("f32", [False, True])
@pytest.mark.parametrize("T,E,k,H,F,sizes", GEMM_CASES)
def test_grouped_gemm_store(T, E, k, H, F, sizes, f32, tiling):
    gu = _gu()
    import moe_routed_expert_top_b200 as M
    cfg, ids, hidden, L, tables, status, x_perm, ref, wgu, wd = _setup(T, E, k, H, F, 1, sizes)
    prob = gu.problem(cfg)
    C = torch.full((L["P"], 2 * F), float("nan"), dtype=torch.float32 if f32 else torch.bfloat16,
                   device="cuda")
    call = lambda: M.moe_grouped_gemm(prob, 0, 2 * F, H, x_perm, None, wgu, None, tables,
                                      (M.MOE_EPI_STORE_F32 if f32 else M.MOE_EPI_STORE) | tiling,
                                      C, None, None, status)
    if _pair_unsupported(tiling, 2 * F):
        _expect_unsupported(call)
        return
    call()
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    refC = _oracle_rows_gemm(hidden, wgu, ref, E, k)
    if f32:
        # the unrounded accumulator: far inside the bf16 tolerance
        gu.assert_within_tol(gu.f64(C), refC, "gate_up store f32", rtol=1e-4, atol=1e-4)
    else:
        gu.assert_within_tol(gu.f64(C), refC, "gate_up store")


@pytest.mark.parametrize("tiling", TILINGS)
@pytest.mark.parametrize("T,E,k,H,F,sizes", GEMM_CASES)
def test_grouped_gemm_swiglu(T, E, k, H, F, sizes, tiling):
    gu = _gu()
    import moe_routed_expert_top_b200 as M
    cfg, ids, hidden, L, tables, status, x_perm, ref, wgu, wd = _setup(T, E, k, H, F, 2, sizes)
    prob = gu.problem(cfg)
    h = torch.full((L["P"], F), float("nan"), dtype=torch.bfloat16, device="cuda")
    call = lambda: M.moe_grouped_gemm(prob, 0, 2 * F, H, x_perm, None, wgu, None, tables,
                                      M.MOE_EPI_SWIGLU | tiling, h, None, None, status)
    if _pair_unsupported(tiling, 2 * F):
        _expect_unsupported(call)
        return
    call()
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    G = _oracle_rows_gemm(hidden, wgu, ref, E, k)
    gu.assert_within_tol(gu.f64(h), O.bf16_round(O.swiglu(G, F)), "swiglu epilogue")


@pytest.mark.parametrize("epi", ["store_f32", "swiglu"])
@pytest.mark.parametrize("T,E,k,H,F,sizes", [c for c in GEMM_CASES if c[4] % 128 == 0])
def test_grouped_gemm_gather(T, E, k, H, F, sizes, epi):
    """The permutation fused into the gate+up GEMM (MOE_A_GATHER): A is the
    hidden states and row r is hidden[pair_of_row[r] / k]. Against the oracle
    (which permutes on its own), and bit-identical to the same tiling fed the
    explicitly permuted rows."""
    gu = _gu()
    import moe_routed_expert_top_b200 as M
    cfg, ids, hidden, L, tables, status, x_perm, ref, wgu, wd = _setup(T, E, k, H, F, 5, sizes)
    prob = gu.problem(cfg)
    P = L["P"]
    f32 = epi == "store_f32"
    flag = M.MOE_EPI_STORE_F32 if f32 else M.MOE_EPI_SWIGLU
    shape = (P, 2 * F) if f32 else (P, F)
    dt = torch.float32 if f32 else torch.bfloat16
    out_g = torch.full(shape, float("nan"), dtype=dt, device="cuda")
    out_x = torch.full(shape, float("nan"), dtype=dt, device="cuda")
    for tiling in (M.MOE_TILE_AUTO, PAIR):
        M.moe_grouped_gemm(prob, 0, 2 * F, H, hidden, None, wgu, None, tables,
                           flag | tiling | M.MOE_A_GATHER, out_g, None, None, status)
        M.moe_grouped_gemm(prob, 0, 2 * F, H, x_perm, None, wgu, None, tables, flag | PAIR,
                           out_x, None, None, status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert torch.equal(out_g.view(torch.int32 if f32 else torch.int16),
                           out_x.view(torch.int32 if f32 else torch.int16))
    G = _oracle_rows_gemm(hidden, wgu, ref, E, k)
    if f32:
        gu.assert_within_tol(gu.f64(out_g), G, "gathered gate_up f32", rtol=1e-4, atol=1e-4)
    else:
        gu.assert_within_tol(gu.f64(out_g), O.bf16_round(O.swiglu(G, F)), "gathered swiglu")


def test_grouped_gemm_gather_rejects():
    gu = _gu()
    import moe_routed_expert_top_b200 as M
    T, E, k, H, F = 200, 8, 2, 256, 384
    cfg, ids, hidden, L, tables, status, x_perm, ref, wgu, wd = _setup(T, E, k, H, F, 6)
    prob = gu.problem(cfg)
    h = torch.empty(L["P"], F, dtype=torch.bfloat16, device="cuda")
    # another tiling
    _expect_unsupported(lambda: M.moe_grouped_gemm(
        prob, 0, 2 * F, H, hidden, None, wgu, None, tables,
        M.MOE_EPI_SWIGLU | M.MOE_TILE_WEIGHT_ROWS | M.MOE_A_GATHER, h, None, None, status))
    # no tables to gather through; K other than H
    for call in (lambda: M.moe_grouped_gemm(None, T, 2 * F, H, hidden, None, wgu, None, None,
                                            M.MOE_EPI_SWIGLU | M.MOE_A_GATHER, h, None, None,
                                            status),
                 lambda: M.moe_grouped_gemm(prob, 0, 2 * F, H - 64, hidden, None, wgu, None,
                                            tables, M.MOE_EPI_SWIGLU | M.MOE_A_GATHER, h, None,
                                            None, status)):
        with pytest.raises(M.MoeError) as ei:
            call()
        assert ei.value.status == M.MOE_ERR_INVALID_ARG


@pytest.mark.parametrize("T,E,k,H,F,sizes", [c for c in GEMM_CASES if c[4] % 128 == 0])
def test_grouped_gemm_swiglu_fp8_epilogue(T, E, k, H, F, sizes):
    gu = _gu()
    import moe_routed_expert_top_b200 as M
    cfg, ids, hidden, L, tables, status, x_perm, ref, wgu, wd = _setup(T, E, k, H, F, 3, sizes)
    prob = gu.problem(cfg)
    P = L["P"]
    q = torch.zeros(P, F, dtype=torch.uint8, device="cuda")
    s = torch.zeros(P, F // 128, dtype=torch.float32, device="cuda")
    dh = torch.zeros(P, F, dtype=torch.float32, device="cuda")
    M.moe_grouped_gemm(prob, 0, 2 * F, H, x_perm, None, wgu, None, tables, M.MOE_EPI_SWIGLU_FP8,
                       q, s, dh, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    # against the oracle: the fused fp32 h, the scales and the dequantised codes
    G = _oracle_rows_gemm(hidden, wgu, ref, E, k)
    h_ref = O.swiglu(G, F)
    h32 = dh.cpu().numpy().astype(np.float64)
    gu.assert_within_tol(h32, h_ref, "fused h", rtol=1e-3, atol=1e-4)
    amax = np.abs(h_ref).reshape(P, F // 128, 128).max(2)
    gu.assert_within_tol(s.cpu().numpy(), amax / 448, "scales", rtol=1e-3, atol=1e-7)
    deq = O.e4m3_value(q.cpu().numpy()) * np.repeat(s.cpu().numpy().astype(np.float64), 128, 1)
    bound = np.abs(h_ref) * (2.0 ** -4 + 2e-3) + np.repeat(amax / 448, 128, 1) * (2.0 ** -9 + 1e-3)
    assert np.all(np.abs(deq - h_ref) <= bound)
    # bit for bit against the oracle's quantiser fed the kernel's own fp32 h
    # (XTuner PR #2089 review thread: bitwise tests of the fused kernel)
    q_ref, s_ref = O.quant_1x128(dh.cpu().numpy())
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    # the fused epilogue and the standalone quantiser agree byte for byte on the
    # same fp32 h
    q2 = torch.zeros_like(q)
    s2 = torch.zeros_like(s)
    M.moe_swiglu_quant(P, F, None, dh, 1, q2, s2)
    torch.cuda.synchronize()
    assert torch.equal(q2, q) and torch.equal(s2.view(torch.int32), s.view(torch.int32))


@pytest.mark.parametrize("T,E,k,H,F,sizes", [(200, 8, 2, 256, 384, None),
                                            (260, 8, 3, 512, 256, [0, 1, 127, 128, 129, 0, 255, 140])])
@pytest.mark.parametrize("tiling", TILINGS)
def test_grouped_gemm_fp8_block_scaled(T, E, k, H, F, sizes, tiling):
    gu = _gu()
    import moe_routed_expert_top_b200 as M
    cfg, ids, hidden, L, tables, status, x_perm, ref, wgu, wd = _setup(T, E, k, H, F, 4, sizes)
    prob = gu.problem(cfg)
    P = L["P"]
    # activations: oracle-quantised random h (so both sides see the same codes)
    rng = np.random.default_rng(9)
    h = (rng.standard_normal((P, F)) * rng.uniform(0.1, 3, (P, 1))).astype(np.float32)
    qa, sa = O.quant_1x128(h)
    wq, ws = zip(*[O.quant_weight_128x128(gu.f64(wd[e]).astype(np.float32)) for e in range(E)])
    wq, ws = np.stack(wq), np.stack(ws)
    refy = np.zeros((P, H))
    for e in range(E):
        a, b = ref["group_offsets"][e], ref["group_offsets"][e + 1]
        if b > a:
            refy[a:b] = O.fp8_block_scaled_matmul(qa[a:b], sa[a:b], wq[e], ws[e])
    for f32 in (False, True):
        y = torch.full((P, H), float("nan"), dtype=torch.float32 if f32 else torch.bfloat16,
                       device="cuda")
        call = lambda: M.moe_grouped_gemm(prob, 0, H, F, torch.from_numpy(qa).cuda(),
                                          torch.from_numpy(sa).cuda(), torch.from_numpy(wq).cuda(),
                                          torch.from_numpy(ws).cuda(), tables,
                                          (M.MOE_EPI_STORE_F32 if f32 else M.MOE_EPI_STORE) | tiling,
                                          y, None, None, status)
        if _pair_unsupported(tiling, H, fp8=True):
            _expect_unsupported(call)
            continue
        call()
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        if f32:
            gu.assert_within_tol(gu.f64(y), refy, "fp8 down f32", rtol=1e-4, atol=1e-4)
        else:
            gu.assert_within_tol(gu.f64(y), refy, "fp8 down")


@pytest.mark.parametrize("tiling", TILINGS)
@pytest.mark.parametrize("M_rows,N,K", [(1, 128, 64), (300, 512, 448), (4096 + 17, 256, 256)])
def test_dense_gemm_store(M_rows, N, K, tiling):
    gu = _gu()
    import moe_routed_expert_top_b200 as M
    g = torch.Generator(device="cuda")
    g.manual_seed(M_rows)
    A = torch.randn(M_rows, K, generator=g, device="cuda").to(torch.bfloat16)
    B = (torch.randn(N, K, generator=g, device="cuda") * 0.05).to(torch.bfloat16)
    C = torch.empty(M_rows, N, dtype=torch.bfloat16, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    call = lambda: M.moe_grouped_gemm(None, M_rows, N, K, A, None, B, None, None,
                                      M.MOE_EPI_STORE | tiling, C, None, None, status)
    if _pair_unsupported(tiling, N):
        _expect_unsupported(call)
        return
    call()
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    gu.assert_within_tol(gu.f64(C), gu.f64(A) @ gu.f64(B).T, "dense")


@pytest.mark.parametrize("Mr,F", [(0, 128), (1, 6144), (127, 6144), (128, 6144), (129, 6144),
                                  (37, 200)])
def test_swiglu_quant_from_h_bit_exact(Mr, F):
    import moe_routed_expert_top_b200 as M
    rng = np.random.default_rng(Mr + F)
    h = (rng.standard_normal((Mr, F)) * rng.uniform(1e-3, 30, (Mr, 1))).astype(np.float32)
    if Mr > 3:
        h[1, :128] = 0.0
        h[2, 5] = -1e-30
        h[3, :] *= 1e-4
    q = torch.zeros(Mr, F, dtype=torch.uint8, device="cuda")
    s = torch.zeros(Mr, -(-F // 128), dtype=torch.float32, device="cuda")
    M.moe_swiglu_quant(Mr, F, None, torch.from_numpy(h).cuda() if Mr else None, 1, q, s)
    torch.cuda.synchronize()
    rq, rs = O.quant_1x128(h)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), rs.view(np.uint32))
    assert np.array_equal(q.cpu().numpy(), rq)


def test_e4m3_encoder_sweep_through_quant():
    """Rows whose amax is exactly 448 have scale 1, so the kernel's codes are
    the E4M3 encoding of h itself: sweep dense values in [-448, 448]."""
    import moe_routed_expert_top_b200 as M
    rng = np.random.default_rng(0)
    n = 1 << 22
    mags = np.exp(rng.uniform(np.log(2.0 ** -12), np.log(448.0), n))
    vals = (mags * rng.choice([-1.0, 1.0], n)).astype(np.float32)
    v = O.e4m3_decode_table()
    finite = v[np.isfinite(v)]
    mids = ((np.sort(finite)[1:] + np.sort(finite)[:-1]) / 2).astype(np.float32)
    vals = np.concatenate([vals, mids, finite.astype(np.float32), -mids,
                           np.array([-0.0, 0.0, 2.0 ** -11, -(2.0 ** -11)], np.float32)])
    vals = np.clip(vals, -448, 448)
    cols = 128
    rows = -(-vals.size // (cols - 1))
    h = np.zeros((rows, cols), np.float32)
    flat = np.zeros(rows * (cols - 1), np.float32)
    flat[:vals.size] = vals
    h[:, 1:] = flat.reshape(rows, cols - 1)
    h[:, 0] = 448.0
    q = torch.zeros(rows, cols, dtype=torch.uint8, device="cuda")
    s = torch.zeros(rows, 1, dtype=torch.float32, device="cuda")
    M.moe_swiglu_quant(rows, cols, None, torch.from_numpy(h).cuda(), 1, q, s)
    torch.cuda.synchronize()
    assert np.all(s.cpu().numpy() == 1.0)
    assert np.array_equal(q.cpu().numpy(), O.e4m3_encode(h))


@pytest.mark.parametrize("out_fp8", [0, 1])
def test_swiglu_quant_from_gate_up(out_fp8):
    gu = _gu()
    import moe_routed_expert_top_b200 as M
    Mr, F = 257, 384
    g = torch.Generator(device="cuda")
    g.manual_seed(3)
    gate_up = (torch.randn(Mr, 2 * F, generator=g, device="cuda") * 2).to(torch.bfloat16)
    h_ref = O.swiglu(gu.f64(gate_up), F)
    if out_fp8:
        q = torch.zeros(Mr, F, dtype=torch.uint8, device="cuda")
        s = torch.zeros(Mr, F // 128, dtype=torch.float32, device="cuda")
        M.moe_swiglu_quant(Mr, F, gate_up, None, 1, q, s)
        torch.cuda.synchronize()
        deq = O.e4m3_value(q.cpu().numpy()) * np.repeat(s.cpu().numpy().astype(np.float64), 128, 1)
        amax = np.abs(h_ref).reshape(Mr, F // 128, 128).max(2)
        assert np.allclose(s.cpu().numpy(), amax / 448, rtol=1e-5)
        # E4M3 keeps 3 mantissa bits: half-ulp relative error 2**-4 (plus subnormals)
        err = np.abs(deq - h_ref)
        assert np.all(err <= np.abs(h_ref) * (2.0 ** -4 + 1e-5) + np.repeat(amax / 448, 128, 1) * 2.0 ** -9)
    else:
        out = torch.empty(Mr, F, dtype=torch.bfloat16, device="cuda")
        M.moe_swiglu_quant(Mr, F, gate_up, None, 0, out, None)
        torch.cuda.synchronize()
        gu.assert_within_tol(gu.f64(out), O.bf16_round(h_ref), "swiglu bf16", rtol=1e-2, atol=1e-3)


def test_weight_quant_bit_exact():
    gu = _gu()
    import moe_routed_expert_top_b200 as M
    E, N, K = 3, 384, 256
    g = torch.Generator(device="cuda")
    g.manual_seed(8)
    w = (torch.randn(E, N, K, generator=g, device="cuda") * 0.02).to(torch.bfloat16)
    w[1, 128:256, 128:] = 0
    q = torch.zeros(E, N, K, dtype=torch.uint8, device="cuda")
    s = torch.zeros(E, N // 128, K // 128, dtype=torch.float32, device="cuda")
    M.moe_quantize_weight_128x128(E, N, K, w, q, s)
    torch.cuda.synchronize()
    for e in range(E):
        rq, rs = O.quant_weight_128x128(gu.f64(w[e]).astype(np.float32))
        assert np.array_equal(q[e].cpu().numpy(), rq)
        assert np.array_equal(s[e].cpu().numpy().view(np.uint32), rs.view(np.uint32))


def test_swiglu_fp8_epilogue_full_size_bits():
    """The fused SwiGLU + 1x128 FP8 epilogue on the DeepSeek-V3 decode workload
    (T 512, E 256, k 8, H 7168, F 2048, skewed routing): every code and scale
    equals the oracle's quantiser applied to the kernel's own fp32 h."""
    gu = _gu()
    import moe_routed_expert_top_b200 as M
    from moe_inputs import make_hidden, make_logits, make_weights
    cfg = get_config("dsv3_decode_fp8")
    ids, _ = O.route_topk(make_logits(cfg), cfg.top_k, gu.score_code(cfg), cfg.renormalize)
    hidden = make_hidden(cfg, "cuda")
    weights = make_weights(cfg, "cuda")
    wgu = weights.pop("w_gate_up")
    del weights
    L, tables, status, x_perm = gu.gpu_tables(cfg, ids, hidden=hidden)
    prob = gu.problem(cfg)
    P, F = L["P"], cfg.F
    q = torch.zeros(P, F, dtype=torch.uint8, device="cuda")
    sc = torch.zeros(P, F // 128, dtype=torch.float32, device="cuda")
    dh = torch.zeros(P, F, dtype=torch.float32, device="cuda")
    M.moe_grouped_gemm(prob, 0, 2 * F, cfg.H, x_perm, None, wgu, None, tables,
                       M.MOE_EPI_SWIGLU_FP8, q, sc, dh, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    q_ref, s_ref = O.quant_1x128(dh.cpu().numpy())
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(sc.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert (s_ref > 0).all()


def _f16e_decode(c16: torch.Tensor, exps: torch.Tensor) -> np.ndarray:
    """y = C16 * 2^e per row and 128-column block (exact in float64)."""
    c = c16.float().cpu().numpy().astype(np.float64)
    e = exps.cpu().numpy().astype(np.int64)
    return c * np.repeat(np.ldexp(1.0, e), 128, axis=1)


def _check_f16e(dec, ref, what):
    """Every value within the fp32 store's tolerance of the oracle's (the
    tensor core's fp32 sums: 1e-4 + 1e-4*|ref|) plus fp16's rounding (11
    significant bits: 2^-11 relative, and the subnormal step of its block)."""
    rows, n = ref.shape
    bmax = np.abs(ref).reshape(rows, n // 128, 128).max(2)
    step = np.repeat(bmax, 128, axis=1) * 2.0 ** -38
    err = np.abs(dec - ref)
    bound = 1e-4 + np.abs(ref) * (1e-4 + 2.0 ** -11) + step
    assert np.all(err <= bound), (what, float((err / bound).max()))


@pytest.mark.parametrize("tiling", TILINGS)
@pytest.mark.parametrize("T,E,k,H,F,sizes", [(200, 8, 2, 256, 384, None),
                                            (260, 8, 3, 512, 256, [0, 1, 127, 128, 129, 0, 255, 140]),
                                            (546, 8, 4, 256, 256, [257, 288, 289, 517, 544, 256, 0, 33])])
def test_grouped_gemm_store_f16e(T, E, k, H, F, sizes, tiling):
    """MOE_EPI_STORE_F16E (the forward's down-GEMM output): fp16 values and one
    int8 exponent per row and 128 columns, decoded against the oracle's
    float64 product; the token-row tiling refuses it."""
    gu = _gu()
    import moe_routed_expert_top_b200 as M
    cfg, ids, hidden, L, tables, status, x_perm, ref, wgu, wd = _setup(T, E, k, H, F, 6, sizes)
    prob = gu.problem(cfg)
    P, N = L["P"], 2 * F
    c16 = torch.full((P, N), float("nan"), dtype=torch.float16, device="cuda")
    ex = torch.zeros(P, N // 128, dtype=torch.int8, device="cuda")
    call = lambda: M.moe_grouped_gemm(prob, 0, N, H, x_perm, None, wgu, None, tables,
                                      M.MOE_EPI_STORE_F16E | tiling, c16, ex, None, status)
    if tiling == 0x10 or _pair_unsupported(tiling, N):
        _expect_unsupported(call)
        return
    call()
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    refC = _oracle_rows_gemm(hidden, wgu, ref, E, k)
    dec = _f16e_decode(c16, ex)
    _check_f16e(dec, refC, "f16e store")
    # and, value for value, the same tiling's fp32 store rounded once to fp16
    # under the block exponent (the encoding is exact apart from that rounding)
    c32 = torch.empty(P, N, dtype=torch.float32, device="cuda")
    M.moe_grouped_gemm(prob, 0, N, H, x_perm, None, wgu, None, tables,
                       M.MOE_EPI_STORE_F32 | tiling, c32, None, None, status)
    torch.cuda.synchronize()
    y32 = c32.cpu().numpy().astype(np.float64)
    scale = np.repeat(np.ldexp(1.0, ex.cpu().numpy().astype(np.int64)), 128, axis=1)
    assert np.array_equal((y32 / scale).astype(np.float16).astype(np.float64) * scale, dec)
    # the exponent rule: each block's largest magnitude in [2^14, 2^15] * 2^e
    e = ex.cpu().numpy().astype(np.int64)
    cmax = np.abs(c16.float().cpu().numpy()).reshape(P, N // 128, 128).max(2)
    nz = cmax > 0
    assert np.all((cmax[nz] >= 2.0 ** 14) & (cmax[nz] <= 2.0 ** 15))
    assert np.all(e[~nz] == 0)


def test_grouped_gemm_fp8_store_f16e():
    """The FP8 block-scaled down GEMM (weight-row tiling) stores f16e too."""
    gu = _gu()
    import moe_routed_expert_top_b200 as M
    T, E, k, H, F = 200, 8, 2, 256, 384
    cfg, ids, hidden, L, tables, status, x_perm, ref, wgu, wd = _setup(T, E, k, H, F, 4)
    prob = gu.problem(cfg)
    P = L["P"]
    rng = np.random.default_rng(9)
    h = (rng.standard_normal((P, F)) * rng.uniform(0.1, 3, (P, 1))).astype(np.float32)
    qa, sa = O.quant_1x128(h)
    wq, ws = zip(*[O.quant_weight_128x128(gu.f64(wd[e]).astype(np.float32)) for e in range(E)])
    wq, ws = np.stack(wq), np.stack(ws)
    refy = np.zeros((P, H))
    for e in range(E):
        a, b = ref["group_offsets"][e], ref["group_offsets"][e + 1]
        if b > a:
            refy[a:b] = O.fp8_block_scaled_matmul(qa[a:b], sa[a:b], wq[e], ws[e])
    c16 = torch.full((P, H), float("nan"), dtype=torch.float16, device="cuda")
    ex = torch.zeros(P, H // 128, dtype=torch.int8, device="cuda")
    M.moe_grouped_gemm(prob, 0, H, F, torch.from_numpy(qa).cuda(), torch.from_numpy(sa).cuda(),
                       torch.from_numpy(wq).cuda(), torch.from_numpy(ws).cuda(), tables,
                       M.MOE_EPI_STORE_F16E | 0x20, c16, ex, None, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    # the fp32 accumulation of the scaled K-blocks (as the fp32 store) before the fp16 rounding
    gu.assert_within_tol(_f16e_decode(c16, ex), refy, "fp8 f16e", rtol=1e-3, atol=1e-4)
