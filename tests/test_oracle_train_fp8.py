"""Pins of the oracle's training-side FP8 layouts and SwiGLU backward
(XTuner PR #2089, Changes): the expert-padded token axis against the TileLang
tutorial "Example 07" §1 block layout, the transposed copies against a plain
transpose (every real element once, padding exactly zero), the per-block and
per-tile scale rules by their invariants, and the backward against central
finite differences of the forward SwiGLU definition."""
import numpy as np
import pytest

from oracle import moe_oracle as O


def _routing(M, E, seed, empty=()):
    rng = np.random.default_rng(seed)
    ids = rng.integers(0, E, size=(M, 1)).astype(np.int32)
    for e in empty:
        ids[ids == e] = (e + 1) % E
    return ids


def _layout(ids, E):
    tab = O.dispatch_tables(ids, E, 128)
    cols = O.padded_columns(tab)
    Mp = 128 * int(tab["M_blk"])
    return tab, cols, Mp


def test_padded_columns_follow_the_block_layout():
    ids = _routing(700, 9, 1, empty=(3,))
    tab, cols, Mp = _layout(ids, 9)
    # a bijection of the rows onto distinct columns, each inside its expert's blocks
    assert len(np.unique(cols)) == 700 and cols.max() < Mp
    for bx, g in enumerate(tab["group_idx_for_bx"]):
        _, m_start, rows = O.block_rows(tab, bx, 128)
        for i in range(rows):
            assert cols[m_start + i] == bx * 128 + i      # the tutorial's m_start recovery
    # expert boundaries start fresh 128-column blocks
    for g in range(9):
        if tab["group_sizes"][g]:
            assert cols[tab["group_offsets"][g]] % 128 == 0


def _deq_check(x_blocks, q, s):
    v = O.e4m3_decode_table()
    amax = np.abs(x_blocks).max()
    if amax == 0:
        assert s == 0 and np.all(q == 0)
        return
    assert s == np.float32(np.float32(amax) / np.float32(448.0))
    assert np.any((q & 0x7F) == 0x7E)
    deq = v[q] * float(s)
    assert np.all(np.abs(deq - x_blocks) <= np.abs(x_blocks) * (2.0 ** -4 + 2.0 ** -22)
                  + 2.0 ** -10 * float(s) * (1 + 2.0 ** -20))


@pytest.mark.parametrize("per_block", [True, False])
def test_transposed_copy_and_scales(per_block):
    rng = np.random.default_rng(2)
    E, K = 6, 256
    ids = _routing(500, E, 3, empty=(2,))
    tab, cols, Mp = _layout(ids, E)
    x = (rng.standard_normal((500, K)) * rng.uniform(0.01, 5, (500, 1))).astype(np.float32)
    x[:, 128:] *= 1e-3                                  # a second K-block of small values
    qT, sT = O.quant_transposed(x, cols, Mp, per_block)
    assert qT.shape == (K, Mp)
    assert sT.shape == ((K // 128, Mp // 128) if per_block else (K, Mp // 128))
    # padding columns are exactly zero codes
    pad = np.setdiff1d(np.arange(Mp), cols)
    assert np.all(qT[:, pad] == 0)
    xT = np.zeros((K, Mp), np.float32)
    xT[:, cols] = x.T
    for kb in range(K // 128):
        for mb in range(Mp // 128):
            blk = xT[kb * 128:(kb + 1) * 128, mb * 128:(mb + 1) * 128]
            qb = qT[kb * 128:(kb + 1) * 128, mb * 128:(mb + 1) * 128]
            if per_block:
                _deq_check(blk, qb, sT[kb, mb])
            else:
                for k in range(0, 128, 37):
                    _deq_check(blk[k], qb[k], sT[kb * 128 + k, mb])


def test_transposed_is_exact_on_representable_values():
    """Power-of-two magnitudes that are E4M3 values times the block scale come
    back exactly: the transpose places every element, the rule keeps it."""
    rng = np.random.default_rng(4)
    E, M, K = 3, 300, 128
    ids = _routing(M, E, 5)
    tab, cols, Mp = _layout(ids, E)
    x = (2.0 ** rng.integers(-4, 5, size=(M, K)) * rng.choice([-1, 1], size=(M, K))).astype(
        np.float32)
    x[0, 0] = 448.0 * 2.0 ** -3                          # fixes every block's amax to 56
    x[:, :] = np.clip(x, -56, 56)
    for per_block in (True, False):
        qT, sT = O.quant_transposed(x, cols, Mp, per_block)
        v = O.e4m3_decode_table()
        s_full = (np.repeat(np.repeat(sT, 128, 0), 128, 1) if per_block
                  else np.repeat(sT, 128, 1))
        deq = v[qT] * s_full
        xT = np.zeros((K, Mp))
        xT[:, cols] = x.T
        nz = s_full > 0
        # an amax of 2^k gives s = 2^k/448; codes of 2^j/s are exact in E4M3
        rel = np.abs(deq[nz] - xT[nz]) <= np.abs(xT[nz]) * 2.0 ** -20
        assert np.mean(rel) > 0.999


def test_dual_is_row_and_transposed():
    rng = np.random.default_rng(6)
    ids = _routing(260, 4, 7)
    tab, cols, Mp = _layout(ids, 4)
    x = rng.standard_normal((260, 256)).astype(np.float32)
    q, s, qT, sT = O.quant_dual(x, cols, Mp, True)
    q1, s1 = O.quant_1x128(x)
    assert np.array_equal(q, q1) and np.array_equal(s, s1)
    # dense (one group) layout: columns are the rows themselves, padded to 128
    qd, sd = O.quant_transposed(x, np.arange(260), 384, False)
    q2, s2 = O.quant_1x128(np.pad(x.T, ((0, 0), (0, 124))))
    assert np.array_equal(qd, q2) and np.array_equal(sd, s2)


def test_swiglu_backward_matches_finite_differences():
    rng = np.random.default_rng(8)
    M, F = 7, 5
    gu = rng.standard_normal((M, 2 * F)) * 3
    dh = rng.standard_normal((M, F))
    grad = O.swiglu_backward(gu, dh)
    eps = 1e-6

    def loss(z):
        return float(np.sum(dh * O.swiglu(z, F)))

    for r in range(M):
        for c in range(2 * F):
            zp, zm = gu.copy(), gu.copy()
            zp[r, c] += eps
            zm[r, c] -= eps
            fd = (loss(zp) - loss(zm)) / (2 * eps)
            assert abs(fd - grad[r, c]) <= 1e-7 * (1 + abs(fd))
    # closed forms at g = 0: dSiLU/dg = 1/2, SiLU = 0
    z = np.zeros((1, 2))
    z[0, 1] = 3.0
    g0 = O.swiglu_backward(z, np.ones((1, 1)))
    assert g0[0, 0] == 1.5 and g0[0, 1] == 0.0
