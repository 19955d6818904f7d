"""Pins for the oracle's expert MLP, unpermute and whole forward (CPU only).

The pages print no output values for the experts forward, so these pins are:
the reduction of E=1, top_k=1, weight 1 to a textbook dense SwiGLU MLP written
as scalar loops; brute-force scalar loops on tiny MoE shapes; agreement of the
table-driven pipeline (tables -> permute -> per-block GEMMs -> unpermute) with
the per-token definition; linearity in routed_scaling_factor (TileOPs PR #1580
§Test Plan checks it at 2.827); FP8 block-scaled down GEMM exactness on
constructed inputs; and bf16 rounding against torch's float32 -> bfloat16 cast.
"""
import math

import numpy as np
import pytest
import torch

from oracle import moe_oracle as O


def _bf16(a):
    return torch.from_numpy(np.asarray(a, np.float32)).to(torch.bfloat16)


def _silu(v):
    return v / (1.0 + math.exp(-v))


def _textbook_mlp_token(x, wgu, wd, F):
    """Scalar-loop SwiGLU MLP for one token: gate = rows [0,F), up = rows [F,2F)."""
    H = len(x)
    h = []
    for f in range(F):
        g = 0.0
        u = 0.0
        for i in range(H):
            g += float(x[i]) * float(wgu[f][i])
            u += float(x[i]) * float(wgu[F + f][i])
        h.append(float(O.bf16_round(_silu(g) * u)))
    y = []
    for n in range(H):
        acc = 0.0
        for f in range(F):
            acc += h[f] * float(wd[n][f])
        y.append(acc)
    return y


def test_bf16_round_matches_torch_from_float32():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000) * 10.0 ** rng.integers(-30, 30, 100000),
                        [0.0, -0.0, 1.0, 3.0e38, -3.0e38, 1e-40, -1e-41]]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).float().numpy().astype(np.float64)
    got = O.bf16_round(x.astype(np.float64))
    assert np.array_equal(got, ref)


def test_bf16_round_single_rounding_from_float64():
    # 1 + 2**-8 + 2**-30: above the midpoint between bf16 neighbours 1 and 1+2**-7;
    # a float32 detour would land exactly on the midpoint and round to even (1.0)
    x = 1.0 + 2.0 ** -8 + 2.0 ** -30
    assert O.bf16_round(x) == 1.0 + 2.0 ** -7
    assert O.bf16_round(1.0 + 2.0 ** -8) == 1.0                    # tie -> even
    assert O.bf16_round(1.0 + 3 * 2.0 ** -8) == 1.0 + 2 * 2.0 ** -7  # tie -> even


def test_silu_identities():
    xs = np.linspace(-20, 20, 2001)
    s = O.silu(xs)
    assert O.silu(0.0) == 0.0
    assert np.allclose(O.silu(-xs), s - xs, atol=1e-12)
    assert np.allclose(s, xs / (1 + np.exp(-xs)))
    assert abs(O.silu(40.0) - 40.0) < 1e-12


def test_dense_reduction_to_textbook_swiglu_mlp():
    rng = np.random.default_rng(1)
    T, H, F = 5, 16, 8
    x = _bf16(rng.standard_normal((T, H)))
    wgu = _bf16(rng.standard_normal((1, 2 * F, H)) * 0.3)
    wd = _bf16(rng.standard_normal((1, H, F)) * 0.3)
    ids = np.zeros((T, 1), np.int32)
    w = np.ones((T, 1), np.float32)
    out = O.experts_forward(x, ids, w, wgu, wd, 1.0, round_output=False)
    xs, g, d = x.float().numpy(), wgu[0].float().numpy(), wd[0].float().numpy()
    for t in range(T):
        ref = _textbook_mlp_token(xs[t], g, d, F)
        assert np.allclose(out[t], ref, rtol=1e-12, atol=1e-12)


def _shard_token_loops(x, wgu, wd, F_s, tp, r):
    """Scalar loops over rank r's FFN columns f in [r*F_s/tp, (r+1)*F_s/tp):
    gate row f, up row F_s + f, down column f of the complete weights."""
    Fp = F_s // tp
    H = len(x)
    y = [0.0] * H
    for f in range(r * Fp, (r + 1) * Fp):
        g = sum(float(x[i]) * float(wgu[f][i]) for i in range(H))
        u = sum(float(x[i]) * float(wgu[F_s + f][i]) for i in range(H))
        h = float(O.bf16_round(_silu(g) * u))
        for n in range(H):
            y[n] += h * float(wd[n][f])
    return y


@pytest.mark.parametrize("tp", [1, 2, 4])
def test_shared_partial_brute_force_and_sum_of_shards(tp):
    """Each rank's partial follows the pages' column/row-parallel split of the
    complete weights (checked by scalar loops over the rank's columns), and the
    partials of all ranks add up to the unsharded shared expert."""
    rng = np.random.default_rng(40 + tp)
    T, H, F_s = 3, 8, 8
    x = _bf16(rng.standard_normal((T, H)))
    wgu = _bf16(rng.standard_normal((2 * F_s, H)) * 0.3)
    wd = _bf16(rng.standard_normal((H, F_s)) * 0.3)
    xs, g, d = x.float().numpy(), wgu.float().numpy(), wd.float().numpy()
    total = np.zeros((T, H))
    for r in range(tp):
        part = O.shared_expert_partial(x, wgu, wd, tp, r)
        for t in range(T):
            assert np.allclose(part[t], _shard_token_loops(xs[t], g, d, F_s, tp, r),
                               rtol=1e-12, atol=1e-12)
        total += part
    full = O.dense_swiglu_mlp(x, wgu, wd)
    assert np.allclose(total, full, rtol=1e-12, atol=1e-12)
    for t in range(T):
        assert np.allclose(full[t], _textbook_mlp_token(xs[t], g, d, F_s), rtol=1e-12, atol=1e-12)
    with pytest.raises(ValueError):
        O.shared_expert_partial(x, wgu, wd, 3, 0)      # F_s % tp != 0
    with pytest.raises(ValueError):
        O.shared_expert_partial(x, wgu, wd, tp, tp)    # rank out of range


def test_brute_force_tiny_moe():
    rng = np.random.default_rng(2)
    T, E, k, H, F = 4, 3, 2, 8, 4
    x = _bf16(rng.standard_normal((T, H)))
    wgu = _bf16(rng.standard_normal((E, 2 * F, H)) * 0.3)
    wd = _bf16(rng.standard_normal((E, H, F)) * 0.3)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    ids, w = O.route_topk(logits, k, O.SOFTMAX, True)
    s = 1.7
    out = O.experts_forward(x, ids, w, wgu, wd, s, round_output=False)
    xs = x.float().numpy()
    for t in range(T):
        ref = [0.0] * H
        for j in range(k):
            e = int(ids[t, j])
            y = _textbook_mlp_token(xs[t], wgu[e].float().numpy(), wd[e].float().numpy(), F)
            for n in range(H):
                ref[n] += float(w[t, j]) * y[n]
        ref = [s * v for v in ref]
        assert np.allclose(out[t], ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("fp8", [False, True])
def test_table_pipeline_equals_per_token_definition(fp8):
    rng = np.random.default_rng(3)
    T, E, k, H, F = 37, 6, 3, 128, 256
    x = _bf16(rng.standard_normal((T, H)))
    wgu = _bf16(rng.standard_normal((E, 2 * F, H)) * 0.05)
    wd = _bf16(rng.standard_normal((E, H, F)) * 0.05)
    logits = rng.standard_normal((T, E)).astype(np.float32)
    ids, w = O.route_topk(logits, k, O.SIGMOID, True)
    s = 2.5
    ref = O.experts_forward(x, ids, w, wgu, wd, s, fp8=fp8, round_output=False)
    # pipeline: tables -> permute -> per M-block expert MLP -> unpermute
    bt = 16
    t = O.dispatch_tables(ids, E, bt)
    xp = O.permute(x.float().numpy().astype(np.float64), t["pair_of_row"], k)
    y = np.zeros((T * k, H))
    for bx in range(t["M_blk"]):
        g, m0, rows = O.block_rows(t, bx, bt)
        if rows:
            y[m0:m0 + rows] = O.expert_mlp(xp[m0:m0 + rows], wgu[g], wd[g], fp8=fp8)
    out = O.unpermute(y, t["row_of_pair"], w, s, round_output=False)
    assert np.allclose(out, ref, rtol=1e-12, atol=1e-12)
    # the sampled-token form gives the same rows
    sample = np.array([0, 5, 36])
    sub = O.experts_forward(x, ids, w, wgu, wd, s, tokens=sample, fp8=fp8, round_output=False)
    assert np.allclose(sub, ref[sample], rtol=0, atol=0)


def test_linearity_in_routed_scaling_factor():
    rng = np.random.default_rng(4)
    T, E, k, H, F = 20, 4, 2, 64, 64
    x = _bf16(rng.standard_normal((T, H)))
    wgu = _bf16(rng.standard_normal((E, 2 * F, H)) * 0.05)
    wd = _bf16(rng.standard_normal((E, H, F)) * 0.05)
    ids, w = O.route_topk(rng.standard_normal((T, E)).astype(np.float32), k)
    base = O.experts_forward(x, ids, w, wgu, wd, 1.0, round_output=False)
    for s in (2.5, 2.827):
        scaled = O.experts_forward(x, ids, w, wgu, wd, s, round_output=False)
        assert np.allclose(scaled, s * base, rtol=1e-14, atol=0)
        rounded = O.experts_forward(x, ids, w, wgu, wd, s)
        # after the bf16 cast the error is at most half a bf16 ulp of the value
        assert np.all(np.abs(rounded - s * base) <= np.abs(s * base) * 2.0 ** -8 + 1e-30)


def test_unpermute_properties():
    rng = np.random.default_rng(5)
    T, k, H = 6, 3, 16
    y = rng.standard_normal((T * k, H))
    rop = rng.permutation(T * k).astype(np.int32)
    zero = O.unpermute(y, rop, np.zeros((T, k), np.float32), 2.0)
    assert np.all(zero == 0)
    onehot = np.zeros((T, k), np.float32)
    onehot[:, 1] = 1.0
    out = O.unpermute(y, rop, onehot, 1.0, round_output=False)
    assert np.array_equal(out, y[rop.reshape(T, k)[:, 1]])
    add = rng.standard_normal((T, H))
    out2 = O.unpermute(y, rop, onehot, 1.0, addend=add, round_output=False)
    assert np.allclose(out2, out + add)


def test_fp8_block_scaled_matmul_exact_on_constructed_inputs():
    rng = np.random.default_rng(6)
    M, N, K = 3, 256, 384
    v = O.e4m3_decode_table()
    small_int_codes = np.array([c for c in range(256) if np.isfinite(v[c]) and v[c] == np.round(v[c])
                                and abs(v[c]) <= 8], dtype=np.uint8)
    qa = rng.choice(small_int_codes, (M, K))
    qw = rng.choice(small_int_codes, (N, K))
    sa = 2.0 ** rng.integers(-3, 3, (M, K // 128)).astype(np.float32)
    sw = 2.0 ** rng.integers(-3, 3, (N // 128, K // 128)).astype(np.float32)
    got = O.fp8_block_scaled_matmul(qa, sa, qw, sw)
    ref = np.zeros((M, N))
    for r in range(M):
        for n in range(N):
            acc = 0.0
            for f in range(K):
                acc += float(sa[r, f // 128]) * float(sw[n // 128, f // 128]) * v[qa[r, f]] * v[qw[n, f]]
            ref[r, n] = acc
    assert np.array_equal(got, ref)
    ones = O.fp8_block_scaled_matmul(qa, np.ones_like(sa), qw, np.ones_like(sw))
    assert np.array_equal(ones, v[qa] @ v[qw].T)


def test_fp8_expert_close_to_bf16_expert():
    rng = np.random.default_rng(7)
    H, F = 256, 256
    x = _bf16(rng.standard_normal((9, H)))
    wgu = _bf16(rng.standard_normal((2 * F, H)) * 0.02)
    wd = _bf16(rng.standard_normal((H, F)) * 0.02)
    yb = O.expert_mlp(x, wgu, wd)
    yq = O.expert_mlp(x, wgu, wd, fp8=True)
    rel = np.linalg.norm(yq - yb) / np.linalg.norm(yb)
    assert rel < 0.08, rel
