"""CPU oracle for the routed mixture-of-experts expert forward.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
module. The product path (``moe_routed_expert_top_b200``) never imports it and
shares no code, constants or helpers with it.

It is a plain, slow, obviously correct restatement of what the path computes,
written from these pages:

* TileLang tutorial "Example 07: MoE dispatch contract and quantised GEMM",
  §1 ``moe_dispatch_contract.py`` (the four dispatch tables, the m_start row
  recovery formula and its three self-checks, the 9-token worked example) and
  §2 ``skeletons.py`` (routed grouped GEMM gate/up -> SiLU -> down -> weighted
  write-back).
* TileOPs PR #1580 "Grouped-GEMM TMA OOB zero-fill + unpermute out=",
  §Grouped-GEMM kernel (C[e] = A[e] @ B[e]^T over each expert's rows) and
  §Unpermute (weighted gather-reduce with routed_scaling_factor folded in
  before the cast/store).
* TileOPs PR #778 "SharedFusedMoE with native shared expert kernel and TP
  support", §Design (gate+up GEMM -> SiLU-mul -> down GEMM; gate rows first,
  then up rows, in the merged gate_up weight) and §Benchmark (sigmoid routing).
* XTuner PR #2089 "Fuse MoE activation FP8 quantization kernels", §Changes
  (SiLU(gate)*up fused with W2-input 1x128 per-tile FP8 quantisation) and the
  review thread (fp32 tile arithmetic, FP8 max constant, bitwise tests).

Precision: every sum and product the pages leave open runs in float64. Where a
floating-point value decides an integer (the FP8 code, the top-k order) the
oracle takes that decision in float32, the precision the kernels use. Two bf16
roundings belong to the method itself and are done here as exact
round-to-nearest-even from float64: h, because the down GEMM multiplies bf16
(or E4M3) operands, and the final bf16 output. The down GEMM's result y and the
shared expert's output are sums, kept in float64 up to the final cast.

Parity status per function (what pins it is in ``tests/test_oracle_*.py``):
every function below is pinned except ``experts_forward`` end-to-end values,
for which the pages print no numbers: they are pinned by the dense-MLP
reduction (E=1, k=1, weight 1), brute-force loops on tiny shapes and linearity
in routed_scaling_factor.
"""
from __future__ import annotations

import math

import numpy as np

F32 = np.float32

# ---------------------------------------------------------------------------
# bf16 helpers (round-to-nearest-even, exact from float64)
# ---------------------------------------------------------------------------


def bf16_round(x) -> np.ndarray:
    """Round float64 (or float32) values to the nearest bfloat16 value, ties to
    even, in ONE rounding step; returns float64 holding bf16-exact values.

    bfloat16 keeps 8 significant bits and float32's exponent range (normal
    down to 2**-126, subnormal spacing 2**-133)."""
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros_like(x)
    nz = (x != 0) & np.isfinite(x)
    m, e = np.frexp(x[nz])          # x = m * 2**e, 0.5 <= |m| < 1
    e = np.maximum(e, -125)         # below 2**-126 the grid is fixed at 2**-133
    q = np.rint(np.ldexp(x[nz], 8 - e))  # exact scaling, then ties-to-even
    out[nz] = np.ldexp(q, e - 8)
    out[~nz] = x[~nz]
    big = np.abs(out) > float(np.ldexp(255.0, 120))  # above the largest finite bf16
    out[big] = np.copysign(np.inf, out[big])
    return out


def bf16_bits(x) -> np.ndarray:
    """uint16 bit patterns of bf16-exact float64 values (after ``bf16_round``)."""
    f = np.asarray(x, dtype=np.float64).astype(np.float32)
    return (f.view(np.uint32) >> 16).astype(np.uint16)


def bf16_from_bits(b) -> np.ndarray:
    b = np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


# ---------------------------------------------------------------------------
# moe_exp: exp in float32 by Cody-Waite range reduction and a Taylor polynomial
# ---------------------------------------------------------------------------
# Method (Cody & Waite, "Software Manual for the Elementary Functions", 1980):
# n = rint(x*log2(e)); r = (x - n*ln2_hi) - n*ln2_lo with ln2_hi = 355/512
# (9 significant bits, so n*ln2_hi is exact); e**r by its degree-7 Taylor
# polynomial in Horner form; result = p * 2**n applied in two exact power-of-two
# steps so the final multiply is the only rounding. Every step is one float32
# operation rounded to nearest even; nothing is fused. The pages state no exp
# algorithm: routing weights are defined with this one so that a GPU kernel
# following the same steps reproduces them bit for bit.

_LOG2E = F32(float.fromhex("0x1.715476p+0"))
_LN2_HI = F32(0.693359375)
_LN2_LO = F32(float.fromhex("-0x1.bd0106p-13"))
_TAYLOR = [F32(1.0 / math.factorial(i)) for i in range(8)]
_EXP_XMAX = F32(89.0)
_EXP_XMIN = F32(-104.0)


def moe_exp(x) -> np.ndarray:
    """float32 exp(x) by the Cody-Waite/Taylor steps above (vectorised)."""
    x = np.asarray(x, dtype=np.float32)
    x = np.minimum(np.maximum(x, _EXP_XMIN), _EXP_XMAX)
    old = np.seterr(over="ignore", under="ignore")
    n = np.rint(x * _LOG2E).astype(np.float32)        # float32 mul, then ties-to-even
    r = (x - n * _LN2_HI).astype(np.float32)          # n*ln2_hi exact
    r = (r - (n * _LN2_LO).astype(np.float32)).astype(np.float32)
    p = _TAYLOR[7]
    for c in _TAYLOR[6::-1]:
        p = ((p * r).astype(np.float32) + c).astype(np.float32)
    ni = n.astype(np.int64)
    half = ni // 2
    rest = ni - half
    s1 = np.ldexp(np.float32(1.0), rest.astype(np.int32)).astype(np.float32)
    s2 = np.ldexp(np.float32(1.0), half.astype(np.int32)).astype(np.float32)
    out = ((p * s1).astype(np.float32) * s2).astype(np.float32)
    np.seterr(**old)
    return out


# ---------------------------------------------------------------------------
# a1: top-k routing
# ---------------------------------------------------------------------------

SOFTMAX, SIGMOID = 0, 1


def topk_ids(logits: np.ndarray, k: int) -> np.ndarray:
    """Per token, the k experts with the largest router logit, largest first;
    equal logits go to the lower expert index. Softmax and sigmoid are
    increasing, so these are also the k largest scores (TileOPs PR #778
    §Benchmark routes Kimi-K2/DeepSeek by sigmoid scores; the tutorial's MoE
    skeleton in "Example 07" §2 consumes the resulting topk ids)."""
    logits = np.asarray(logits, dtype=np.float32)
    order = np.argsort(-logits, axis=1, kind="stable")   # stable: lower index first on ties
    return order[:, :k].astype(np.int32)


def route_topk(logits: np.ndarray, k: int, score_fn: int = SOFTMAX,
               renormalize: bool = True):
    """Top-k ids and their weights, fp32, with the float32 steps fixed here
    (the pages fix none):

    softmax, renormalised: e_j = moe_exp(l_j - l_top1), w_j = e_j / sum_{i<k} e_i
      (the full softmax denominator cancels in the renormalisation);
    softmax, not renormalised: e_j = moe_exp(l_j - max_e l_e),
      w_j = e_j / sum over all E experts in index order;
    sigmoid: s_j = 1 / (1 + moe_exp(-l_j)); renormalised w_j = s_j / sum_{i<k} s_i,
      otherwise w_j = s_j.
    Sums run in slot (or index) order, one float32 rounding per operation."""
    logits = np.asarray(logits, dtype=np.float32)
    T, E = logits.shape
    ids = topk_ids(logits, k)
    sel = np.take_along_axis(logits, ids, axis=1)        # [T, k] fp32
    if score_fn == SOFTMAX:
        if renormalize:
            e = moe_exp((sel - sel[:, :1]).astype(np.float32))
            den = np.zeros(T, dtype=np.float32)
            for j in range(k):
                den = (den + e[:, j]).astype(np.float32)
        else:
            mx = sel[:, :1]
            e = moe_exp((sel - mx).astype(np.float32))
            eall = moe_exp((logits - mx).astype(np.float32))
            den = np.zeros(T, dtype=np.float32)
            for j in range(E):
                den = (den + eall[:, j]).astype(np.float32)
        w = (e / den[:, None]).astype(np.float32)
    elif score_fn == SIGMOID:
        s = (F32(1.0) / (F32(1.0) + moe_exp((-sel).astype(np.float32))).astype(np.float32))
        s = s.astype(np.float32)
        if renormalize:
            den = np.zeros(T, dtype=np.float32)
            for j in range(k):
                den = (den + s[:, j]).astype(np.float32)
            w = (s / den[:, None]).astype(np.float32)
        else:
            w = s
    else:
        raise ValueError(score_fn)
    return ids, w


# ---------------------------------------------------------------------------
# a2: dispatch tables and the expert-sorted permutation
# ---------------------------------------------------------------------------


def ceil_div(a, b):
    return -(-a // b)


def dispatch_tables(topk_ids_: np.ndarray, E: int, padding_M: int,
                    block_token: int | None = None) -> dict:
    """The four host-side tables of the TileLang tutorial "Example 07" §1, plus
    the permutation that sorts (token, expert) pairs by expert.

    pairs: flat index p = t*k + j with expert e(p) = topk_ids[t, j].
    group_sizes[e]          = #{p : e(p) = e}
    group_offsets[e]        = sum_{e' < e} group_sizes[e']   (E+1 entries; last = P)
    group_padded_offsets[e] = sum_{e' < e} ceil(size/padding_M)*padding_M  (E+1 entries)
    M_blk                   = ceil(P / block_token) + E
    group_idx_for_bx[bx]    = largest g with group_padded_offsets[g] <= bx*block_token
    row_of_pair[p]          = group_offsets[e(p)] + #{p' < p : e(p') = e(p)}  (stable)
    pair_of_row             = inverse of row_of_pair
    Readings where the tutorial is silent: within one expert pairs keep their
    flat order (stable); an empty expert gets an empty padded interval; the
    tie-break "largest g" sends a block to the non-empty expert when empty
    experts share its offset."""
    ids = np.asarray(topk_ids_, dtype=np.int64).reshape(-1)
    P = ids.size
    bt = padding_M if block_token is None else block_token
    if np.any((ids < 0) | (ids >= E)):
        raise ValueError("expert id out of range")
    sizes = np.zeros(E, dtype=np.int64)
    for e in ids:
        sizes[e] += 1
    offsets = np.zeros(E + 1, dtype=np.int64)
    padded = np.zeros(E + 1, dtype=np.int64)
    for e in range(E):
        offsets[e + 1] = offsets[e] + sizes[e]
        padded[e + 1] = padded[e] + ceil_div(int(sizes[e]), padding_M) * padding_M
    M_blk = ceil_div(P, bt) + E
    idx_for_bx = np.zeros(M_blk, dtype=np.int64)
    for bx in range(M_blk):
        g = 0
        for cand in range(E):
            if padded[cand] <= bx * bt:
                g = cand
        idx_for_bx[bx] = g
    row_of_pair = np.zeros(P, dtype=np.int64)
    seen = np.zeros(E, dtype=np.int64)
    for p in range(P):
        e = ids[p]
        row_of_pair[p] = offsets[e] + seen[e]
        seen[e] += 1
    pair_of_row = np.zeros(P, dtype=np.int64)
    pair_of_row[row_of_pair] = np.arange(P)
    return {
        "group_sizes": sizes.astype(np.int32),
        "group_offsets": offsets.astype(np.int32),
        "group_padded_offsets": padded.astype(np.int32),
        "group_idx_for_bx": idx_for_bx.astype(np.int32),
        "row_of_pair": row_of_pair.astype(np.int32),
        "pair_of_row": pair_of_row.astype(np.int32),
        "M_blk": int(M_blk),
        "group_sum": int(P),
        "waste": int(M_blk * bt - P),
    }


def block_rows(tables: dict, bx: int, block_token: int):
    """Rows handled by M-block ``bx``, by the tutorial's recovery formula
    m_start = m_start_padded - group_padded_offsets[g] + group_offsets[g], with
    m_start_padded = bx*block_token, and actual_rows = the rows of expert g left
    from there, clamped to [0, block_token] ("Example 07" §1, self-check 3)."""
    g = int(tables["group_idx_for_bx"][bx])
    gpo = int(tables["group_padded_offsets"][g])
    go = int(tables["group_offsets"][g])
    size = int(tables["group_sizes"][g])
    m_start_padded = bx * block_token
    m_start = m_start_padded - gpo + go
    actual_rows = min(max(size - (m_start_padded - gpo), 0), block_token)
    return g, m_start, actual_rows


# ---------------------------------------------------------------------------
# a3: permute gather
# ---------------------------------------------------------------------------


def permute(hidden: np.ndarray, pair_of_row: np.ndarray, k: int) -> np.ndarray:
    """x_perm[r] = hidden[pair_of_row[r] // k]: each expert's rows contiguous."""
    return np.asarray(hidden)[np.asarray(pair_of_row) // k]


# ---------------------------------------------------------------------------
# a5: SwiGLU and FP8 E4M3 1x128 quantisation
# ---------------------------------------------------------------------------


def silu(x):
    """SiLU(x) = x * sigmoid(x) = x / (1 + e**-x), float64."""
    x = np.asarray(x, dtype=np.float64)
    return x / (1.0 + np.exp(-x))


def swiglu(gate_up: np.ndarray, F: int) -> np.ndarray:
    """h = SiLU(gate) * up with gate = columns [0, F), up = columns [F, 2F)
    (TileOPs PR #778 §Design merged gate_up layout; XTuner PR #2089 §Changes
    ``SiLU(gate) * up``). float64."""
    g = np.asarray(gate_up, dtype=np.float64)
    return silu(g[..., :F]) * g[..., F:2 * F]


E4M3_MAX = 448.0


def e4m3_decode_table() -> np.ndarray:
    """Value of each of the 256 OCP FP8 E4M3 ("E4M3FN") codes: sign bit 7,
    exponent bits 6..3 with bias 7, mantissa bits 2..0; exponent 0 is
    subnormal (m/8 * 2**-6); S.1111.111 is NaN; no infinities."""
    vals = np.zeros(256, dtype=np.float64)
    for c in range(256):
        s = -1.0 if c & 0x80 else 1.0
        e = (c >> 3) & 0xF
        m = c & 0x7
        if e == 0xF and m == 0x7:
            vals[c] = np.nan
        elif e == 0:
            vals[c] = s * (m / 8.0) * 2.0 ** -6
        else:
            vals[c] = s * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return vals


def e4m3_encode(x) -> np.ndarray:
    """float32 -> E4M3 code, round to nearest even, saturating to +-448 for
    |x| >= 448 (``satfinite``), sign of zero kept. NaN is out of scope."""
    x = np.asarray(x, dtype=np.float32).astype(np.float64)   # exact widening
    sign = np.signbit(x).astype(np.uint8) << 7
    a = np.abs(x)
    code = np.zeros(a.shape, dtype=np.int64)
    sat = a >= E4M3_MAX
    sub = a < 2.0 ** -6
    nrm = ~sat & ~sub
    # subnormal grid: multiples of 2**-9; m == 8 lands exactly on code 0x08 = 2**-6
    code[sub] = np.rint(a[sub] * 2.0 ** 9).astype(np.int64)
    if np.any(nrm):
        m, e = np.frexp(a[nrm])            # a = m * 2**e, m in [0.5, 1)
        e = e - 1                           # a = (2m) * 2**e, 2m in [1, 2)
        q = np.rint((2.0 * m - 1.0) * 8.0).astype(np.int64)  # exact, ties to even
        carry = q == 8
        q[carry] = 0
        e[carry] += 1
        c = ((e + 7) << 3) | q
        c = np.minimum(c, 0x7E)
        code[nrm] = c
    code[sat] = 0x7E
    return (code.astype(np.uint8) | sign).astype(np.uint8)


def quant_1x128(h32: np.ndarray):
    """Per-row, per-128-column-tile FP8 quantisation of float32 activations
    (XTuner PR #2089 §Changes, ``per_tile_quant``; fp32 tile arithmetic as in
    its review thread):

      amax = max |h| over the tile's valid columns (float32, exact)
      s    = amax / 448                 (float32 IEEE division)
      q    = e4m3_encode(h / s)         (float32 IEEE division per element)
      amax == 0  ->  s = 0 and every code 0x00.
    Returns codes uint8 [M, F] and scales float32 [M, ceil(F/128)]."""
    h = np.asarray(h32, dtype=np.float32)
    M, F = h.shape
    nt = ceil_div(F, 128)
    q = np.zeros((M, F), dtype=np.uint8)
    s = np.zeros((M, nt), dtype=np.float32)
    for c in range(nt):
        blk = h[:, c * 128:(c + 1) * 128]
        amax = np.max(np.abs(blk), axis=1).astype(np.float32) if blk.shape[1] else np.zeros(M, np.float32)
        sc = (amax / F32(E4M3_MAX)).astype(np.float32)
        nz = amax > 0
        tile = np.zeros(blk.shape, dtype=np.uint8)
        if np.any(nz):
            tile[nz] = e4m3_encode((blk[nz] / sc[nz, None]).astype(np.float32))
        q[:, c * 128:(c + 1) * 128] = tile
        s[:, c] = np.where(nz, sc, F32(0.0))
    return q, s


def quant_weight_128x128(w: np.ndarray):
    """128x128 block FP8 quantisation of a weight matrix w [N, K] (same rule
    as ``quant_1x128`` over each 128x128 block): codes uint8 [N, K] and
    float32 scales [ceil(N/128), ceil(K/128)]. N and K are padded with zeros
    to whole blocks for the block maxima; padding never changes a maximum."""
    w = np.asarray(w, dtype=np.float32)
    N, K = w.shape
    nb, kb = ceil_div(N, 128), ceil_div(K, 128)
    wp = np.zeros((nb * 128, kb * 128), dtype=np.float32)
    wp[:N, :K] = w
    blocks = wp.reshape(nb, 128, kb, 128)
    amax = np.abs(blocks).max(axis=(1, 3)).astype(np.float32)        # [nb, kb]
    s = (amax / F32(E4M3_MAX)).astype(np.float32)
    safe = np.where(amax > 0, s, F32(1.0)).astype(np.float32)
    scaled = (blocks / safe[:, None, :, None]).astype(np.float32)
    q = e4m3_encode(scaled)
    q[np.broadcast_to((amax == 0)[:, None, :, None], q.shape)] = 0
    q = q.reshape(nb * 128, kb * 128)[:N, :K]
    s = np.where(amax > 0, s, F32(0.0)).astype(np.float32)
    return np.ascontiguousarray(q), s


_E4M3_VALUES = e4m3_decode_table()


def e4m3_value(codes) -> np.ndarray:
    return _E4M3_VALUES[np.asarray(codes, dtype=np.uint8)]


# ---------------------------------------------------------------------------
# Training-side FP8 layouts and the SwiGLU backward (XTuner PR #2089,
# §Changes: per_tile_quant_with_trans_per_block / _per_tile,
# swiglu_per_tile_quant_with_trans_per_block, swiglu_backward)
# ---------------------------------------------------------------------------


def padded_columns(tables: dict) -> np.ndarray:
    """Column of every row on the expert-padded token axis ("expand_128x"):
    row r of expert g (rows go[g] .. go[g]+size[g]-1) goes to column
    gpo[g] + (r - go[g]), i.e. each expert's rows start a fresh 128-row block
    of the TileLang tutorial "Example 07" §1 layout (padding_M = 128)."""
    sizes = np.asarray(tables["group_sizes"])
    go = np.asarray(tables["group_offsets"])
    gpo = np.asarray(tables["group_padded_offsets"])
    cols = np.zeros(int(sizes.sum()), dtype=np.int64)
    for g in range(len(sizes)):
        n = int(sizes[g])
        cols[go[g]:go[g] + n] = gpo[g] + np.arange(n)
    return cols


def quant_transposed(x32: np.ndarray, cols: np.ndarray, Mp: int, per_block: bool):
    """The transposed, expert-padded FP8 copy of activations x [M, K] (the
    operand of a weight-gradient GEMM, which contracts over tokens):
    xT[k, cols[r]] = x[r, k], zero in the padding columns, xT [K, Mp]; then
      per_block: one scale per 128x128 block of xT,
      per tile : one scale per 1x128 tile of an xT row (128 padded tokens),
    each with the rule of ``quant_1x128`` (s = amax/448, q = e4m3(x / s),
    an all-zero block or tile has s = 0 and codes 0).
    Returns qT uint8 [K, Mp] and sT float32 [K/128, Mp/128] or [K, Mp/128]."""
    x = np.asarray(x32, dtype=np.float32)
    M, K = x.shape
    if K % 128 or Mp % 128:
        raise ValueError("K and Mp must be multiples of 128")
    xT = np.zeros((K, Mp), dtype=np.float32)
    xT[:, cols] = x.T
    if not per_block:
        return quant_1x128(xT)
    blocks = np.abs(xT).reshape(K // 128, 128, Mp // 128, 128)
    amax = blocks.max(axis=(1, 3)).astype(np.float32)                  # [K/128, Mp/128]
    s = (amax / F32(E4M3_MAX)).astype(np.float32)
    s_full = np.repeat(np.repeat(s, 128, axis=0), 128, axis=1)
    q = np.zeros((K, Mp), dtype=np.uint8)
    nz = s_full > 0
    q[nz] = e4m3_encode((xT[nz] / s_full[nz]).astype(np.float32))
    return q, np.where(amax > 0, s, F32(0.0)).astype(np.float32)


def quant_dual(x32: np.ndarray, cols: np.ndarray, Mp: int, per_block: bool):
    """Both layouts of one activation: the forward 1x128 row quantisation
    (``quant_1x128``) and the transposed, expert-padded copy
    (``quant_transposed``). Returns (q, s, qT, sT)."""
    q, s = quant_1x128(x32)
    qT, sT = quant_transposed(x32, cols, Mp, per_block)
    return q, s, qT, sT


def swiglu_backward(gate_up, grad_h) -> np.ndarray:
    """Gradient of h = SiLU(gate) * up with respect to [gate, up] given dL/dh,
    float64: with s = 1 / (1 + e^-g),
      dL/dgate = dL/dh * up * s * (1 + g * (1 - s))   (d SiLU/dg)
      dL/dup   = dL/dh * g * s                        (SiLU(g))
    Returns grad_gate_up [M, 2F] (gate columns first, as in gate_up)."""
    G = as_f64(gate_up)
    dh = as_f64(grad_h)
    F = dh.shape[1]
    g, u = G[:, :F], G[:, F:]
    s = 1.0 / (1.0 + np.exp(-g))
    return np.concatenate([dh * u * s * (1.0 + g * (1.0 - s)), dh * g * s], axis=1)


# ---------------------------------------------------------------------------
# a4 + a5 + a6: one expert's SwiGLU MLP on its rows
# ---------------------------------------------------------------------------


def as_f64(t) -> np.ndarray:
    """float64 copy of a bf16/fp32 array-like (torch tensors accepted)."""
    if hasattr(t, "detach"):
        import torch
        return t.detach().to("cpu", torch.float64).numpy()
    return np.asarray(t, dtype=np.float64)


def gate_up_rows(x: np.ndarray, w_gate_up_e: np.ndarray) -> np.ndarray:
    """G = x @ w_gate_up[e]^T over the expert's rows, float64 (TileOPs PR #1580
    §Grouped-GEMM kernel: C[e] = A[e] @ B[e]^T)."""
    return as_f64(x) @ as_f64(w_gate_up_e).T


def expert_mlp(x: np.ndarray, w_gate_up_e, w_down_e, fp8: bool = False,
               w_down_q_e=None, w_down_s_e=None, return_parts: bool = False):
    """One expert's gate+up GEMM -> SiLU(gate)*up -> down GEMM on rows x [n, H].

    bf16 path: h is rounded to bf16 (the down GEMM's operand type) and
      y = h_bf16 @ w_down[e]^T in float64.
    FP8 path: h is taken to float32, quantised per 1x128 tile (``quant_1x128``),
      and y[r, n] = sum over 128-wide K-blocks kb, in kb order, of
      (sa[r, kb] * sw[n//128, kb]) * sum_{f in kb} dec(q_a[r, f]) * dec(q_w[n, f]),
      with w_down quantised per 128x128 block (``quant_weight_128x128``).
    Returns y float64 [n, H] (and the intermediates when ``return_parts``)."""
    G = gate_up_rows(x, w_gate_up_e)
    F = G.shape[1] // 2
    h = swiglu(G, F)
    parts = {"G": G, "h": h}
    if not fp8:
        hb = bf16_round(h)
        y = hb @ as_f64(w_down_e).T
        parts["h_bf16"] = hb
    else:
        if w_down_q_e is None:
            w_down_q_e, w_down_s_e = quant_weight_128x128(as_f64(w_down_e).astype(np.float32))
        h32 = h.astype(np.float32)
        qa, sa = quant_1x128(h32)
        y = fp8_block_scaled_matmul(qa, sa, w_down_q_e, w_down_s_e)
        parts.update(h32=h32, q=qa, sa=sa)
    return (y, parts) if return_parts else y


def fp8_block_scaled_matmul(qa, sa, qw, sw) -> np.ndarray:
    """y[r, n] = sum over 128-wide K-blocks kb, in kb order, of
    (sa[r, kb] * sw[n // 128, kb]) * sum_{f in kb} dec(qa[r, f]) * dec(qw[n, f]),
    float64: E4M3 activations with one scale per 1x128 tile times E4M3
    weights with one scale per 128x128 block."""
    A = e4m3_value(qa)
    B = e4m3_value(qw)
    K = A.shape[1]
    Hn = B.shape[0]
    sa = np.asarray(sa, np.float64)
    sw = np.asarray(sw, np.float64)
    y = np.zeros((A.shape[0], Hn), dtype=np.float64)
    for kb in range(ceil_div(K, 128)):
        inner = A[:, kb * 128:(kb + 1) * 128] @ B[:, kb * 128:(kb + 1) * 128].T
        swn = np.repeat(sw[:, kb], 128)[:Hn]
        y += (sa[:, kb][:, None] * swn[None, :]) * inner
    return y


def dense_swiglu_mlp(x, w_gate_up, w_down):
    """The shared expert: a dense SwiGLU MLP on all tokens (TileOPs PR #778
    §Design, SharedExpertMLPKernel), bf16 h, float64 sums."""
    return expert_mlp(x, w_gate_up, w_down)


def shared_expert_partial(x, w_gate_up, w_down, tp_size: int = 1, tp_rank: int = 0):
    """Tensor-parallel rank ``tp_rank``'s partial output of the shared expert
    (TileOPs PR #778, TP split convention and Partial output contract). The
    complete weights are w_gate_up [2*F_s, H] (gate rows [0, F_s), up rows
    [F_s, 2*F_s)) and w_down [H, F_s]; with F_p = F_s / tp_size the rank owns
    gate rows [r*F_p, (r+1)*F_p), the up rows F_s above them (column
    parallel) and w_down columns [r*F_p, (r+1)*F_p) (row parallel). The
    partials of all ranks sum to the whole shared expert's output (float64)."""
    two_fs = w_gate_up.shape[0]
    F_s = two_fs // 2
    if tp_size < 1 or not 0 <= tp_rank < tp_size or F_s % tp_size:
        raise ValueError("need 0 <= tp_rank < tp_size and F_s % tp_size == 0")
    Fp = F_s // tp_size
    lo, hi = tp_rank * Fp, (tp_rank + 1) * Fp
    gate = as_f64(w_gate_up[lo:hi])
    up = as_f64(w_gate_up[F_s + lo:F_s + hi])
    down = as_f64(w_down[:, lo:hi])
    return dense_swiglu_mlp(x, np.concatenate([gate, up]), down)


# ---------------------------------------------------------------------------
# a7: weighted unpermute with routed_scaling_factor folded in
# ---------------------------------------------------------------------------


def unpermute(y: np.ndarray, row_of_pair: np.ndarray, topk_weights: np.ndarray,
              scale: float, addend=None, round_output: bool = True) -> np.ndarray:
    """out[t] = bf16( scale * sum_j w[t,j] * y[row_of_pair[t*k + j]] + addend[t] )
    (TileOPs PR #1580 §Unpermute: scale folded in before the cast/store, output
    written directly). Sum over j in slot order, float64. Returns bf16-exact
    float64 [T, H] (the float64 value before the cast if not ``round_output``)."""
    w = np.asarray(topk_weights, dtype=np.float64)
    T, k = w.shape
    y = as_f64(y)
    rows = np.asarray(row_of_pair).reshape(T, k)
    acc = np.zeros((T, y.shape[1]), dtype=np.float64)
    for j in range(k):
        acc += w[:, j:j + 1] * y[rows[:, j]]
    acc = float(scale) * acc
    if addend is not None:
        acc = acc + as_f64(addend)
    return bf16_round(acc) if round_output else acc


def weighted_rows(y: np.ndarray, pair_of_row: np.ndarray, topk_weights: np.ndarray,
                  scale: float, round_output: bool = True):
    """The down projection's rows with the routing weight and scale applied,
    moved to flat pair order (the routing weight x scale folded into the
    down-GEMM epilogue: TileOPs PR #1580 §Unpermute's scale folding done one
    step earlier, as pypto-lib PR #809's per-row scale x routing weight):
        y_w[p] = bf16( scale * w[p] * y[r] )   for every row r with p = pair_of_row[r] >= 0
    The bf16 rounding is the one the pages put on the down GEMM's output (y is
    bf16 [P, H] in their layout); ``round_output=False`` keeps the float64
    product. Returns (y_w float64 [P, H], written bool [P]); rows of pairs with
    no permuted row stay 0 / unwritten."""
    w = np.asarray(topk_weights, dtype=np.float64).reshape(-1)
    y = as_f64(y)
    por = np.asarray(pair_of_row).reshape(-1)
    P = w.shape[0]
    out = np.zeros((P, y.shape[1]), dtype=np.float64)
    written = np.zeros(P, dtype=bool)
    for r in range(por.shape[0]):
        p = int(por[r])
        if p < 0:
            continue
        v = float(scale) * w[p] * y[r]
        out[p] = bf16_round(v) if round_output else v
        written[p] = True
    return out, written


def combine(y_w: np.ndarray, row_of_pair: np.ndarray, k: int, addend=None,
            round_output: bool = True) -> np.ndarray:
    """out[t] = bf16( sum_{j<k, row_of_pair[t*k+j] >= 0} y_w[t*k+j] + addend[t] )
    (TileOPs PR #1580 §Unpermute's gather-reduce once the weights are applied:
    the deterministic combine). Sum over j in slot order, float64."""
    y_w = as_f64(y_w)
    rop = np.asarray(row_of_pair).reshape(-1)
    P, H = y_w.shape
    T = P // k
    acc = np.zeros((T, H), dtype=np.float64)
    for j in range(k):
        has = rop[j::k] >= 0
        acc[has] += y_w[j::k][has]
    if addend is not None:
        acc = acc + as_f64(addend)
    return bf16_round(acc) if round_output else acc


# ---------------------------------------------------------------------------
# whole experts forward, by its plain definition per token
# ---------------------------------------------------------------------------


def experts_forward(hidden, topk_ids_, topk_weights, w_gate_up, w_down, scale: float,
                    tokens=None, fp8: bool = False, w_down_q=None, w_down_s=None,
                    ws_gate_up=None, ws_down=None, weight_loader=None,
                    round_output: bool = True):
    """out[t] = bf16( scale * sum_j w[t,j] * MLP_{e(t,j)}(hidden[t]) + shared(hidden[t]) )

    Computed straight from the definition, per (token, expert) pair, with no
    permutation: pairs are grouped by expert only so each expert's weights are
    widened to float64 once. ``tokens`` restricts the computation to a sample of
    token indices (the result has one row per sampled token).
    ``weight_loader(name, e)`` may supply one expert's weights at a time (used
    when the weights live on a GPU)."""
    ids = np.asarray(topk_ids_)
    w = np.asarray(topk_weights, dtype=np.float64)
    T, k = ids.shape
    toks = np.arange(T) if tokens is None else np.asarray(tokens)
    X = as_f64(hidden[toks]) if tokens is not None else as_f64(hidden)
    H = X.shape[1]
    acc = np.zeros((len(toks), H), dtype=np.float64)

    def load(name, e):
        if weight_loader is not None:
            return weight_loader(name, e)
        src = {"w_gate_up": w_gate_up, "w_down": w_down,
               "w_down_q": w_down_q, "w_down_s": w_down_s}[name]
        return None if src is None else src[e]

    sub_ids = ids[toks]
    Y = np.zeros((len(toks), k, H), dtype=np.float64)   # MLP output of every pair
    for e in np.unique(sub_ids):
        ti, ji = np.nonzero(sub_ids == e)
        Y[ti, ji] = expert_mlp(X[ti], load("w_gate_up", e), load("w_down", e), fp8=fp8,
                               w_down_q_e=load("w_down_q", e) if fp8 else None,
                               w_down_s_e=load("w_down_s", e) if fp8 else None)
    for j in range(k):                                   # slot order
        acc += w[toks, j][:, None] * Y[:, j]
    acc = float(scale) * acc
    if ws_gate_up is not None:
        acc = acc + dense_swiglu_mlp(X, ws_gate_up, ws_down)
    return bf16_round(acc) if round_output else acc
