"""Pins for the oracle's weighted rows and combine (CPU only).

The down projection's rows with the routing weight and scale applied, in flat
pair order, then summed per token in slot order (TileOPs PR #1580
"Grouped-GEMM TMA OOB zero-fill + unpermute out=", §Unpermute, with the
weight fold moved into the down projection). Pinned by a hand-computed
example, by agreement with the separately pinned ``unpermute`` whenever every
weighted term is exactly representable in bf16, and by special cases.
"""
from __future__ import annotations

import numpy as np

from oracle import moe_oracle as O


def _tables(ids, E):
    t = O.dispatch_tables(np.asarray(ids, dtype=np.int32), E, 128)
    return t["row_of_pair"], t["pair_of_row"]


def test_hand_computed_example():
    # T=2 tokens, k=2, E=3 experts, H=2 columns
    ids = [[2, 0], [0, 1]]
    rop, por = _tables(ids, 3)
    # pairs p = t*k+j: p0 -> e2, p1 -> e0, p2 -> e0, p3 -> e1
    # rows in expert order: e0 holds p1, p2 (rows 0, 1); e1 holds p3 (row 2); e2 holds p0 (row 3)
    assert list(rop) == [3, 0, 1, 2]
    assert list(por) == [1, 2, 3, 0]
    y = np.array([[1.0, 2.0],     # row 0 = pair 1
                  [4.0, -8.0],    # row 1 = pair 2
                  [0.5, 0.25],    # row 2 = pair 3
                  [3.0, 6.0]])    # row 3 = pair 0
    w = np.array([[0.5, 0.25], [0.75, 0.125]])
    y_w, written = O.weighted_rows(y, por, w, 2.0)
    assert written.all()
    # y_w[p] = 2 * w[p] * y[row_of_pair[p]]
    assert np.array_equal(y_w, [[3.0, 6.0],      # p0: 2*0.5*[3, 6]
                                [0.5, 1.0],      # p1: 2*0.25*[1, 2]
                                [6.0, -12.0],    # p2: 2*0.75*[4, -8]
                                [0.125, 0.0625]])  # p3: 2*0.125*[0.5, 0.25]
    out = O.combine(y_w, rop, 2, addend=np.array([[1.0, 1.0], [0.0, -1.0]]))
    assert np.array_equal(out, [[4.5, 8.0], [6.125, -12.9375]])


def test_matches_unpermute_when_every_term_is_bf16_exact():
    rng = np.random.default_rng(11)
    T, k, E, H = 7, 3, 5, 12
    ids = np.stack([rng.choice(E, k, replace=False) for _ in range(T)])
    rop, por = _tables(ids, E)
    # small integers times powers of two: scale * w * y is exact in bf16 and
    # every partial sum is exact in float64, so both orders agree exactly
    y = rng.integers(-8, 9, (T * k, H)).astype(np.float64)
    w = (2.0 ** rng.integers(-3, 1, (T, k))).astype(np.float32)
    add = rng.integers(-4, 5, (T, H)).astype(np.float64)
    y_w, written = O.weighted_rows(y, por, w, 0.5)
    assert written.all()
    got = O.combine(y_w, rop, k, addend=add, round_output=False)
    ref = O.unpermute(y, rop, w, 0.5, addend=add, round_output=False)
    assert np.array_equal(got, ref)


def test_single_slot_unit_weight_is_the_rounded_row():
    rng = np.random.default_rng(12)
    T, H = 9, 8
    ids = rng.integers(0, 4, (T, 1))
    rop, por = _tables(ids, 4)
    y = rng.standard_normal((T, H))
    y_w, _ = O.weighted_rows(y, por, np.ones((T, 1), np.float32), 1.0)
    assert np.array_equal(y_w, O.bf16_round(y[rop]))
    assert np.array_equal(O.combine(y_w, rop, 1), O.bf16_round(y[rop]))


def test_rounding_happens_per_term_then_once_more():
    # two terms that each round in bf16, then their sum rounds again
    rop = np.array([0, 1])
    por = np.array([0, 1])
    y = np.array([[1.0 + 2.0 ** -9], [1.0 + 3 * 2.0 ** -9]])
    y_w, _ = O.weighted_rows(y, por, np.array([[1.0, 1.0]], np.float32), 1.0)
    # 1 + 2^-9 -> 1 (tie to even); 1 + 3*2^-9 -> 1 + 2^-7 (nearest)
    assert list(y_w[:, 0]) == [1.0, 1.0 + 2.0 ** -7]
    assert O.combine(y_w, rop, 2)[0, 0] == 2.0   # 2 + 2^-7 is a tie: even -> 2


def test_pairs_without_a_row_are_skipped():
    rng = np.random.default_rng(13)
    T, k, H = 4, 2, 4
    rop = np.array([2, -1, 0, 1, -1, -1, 3, 4])
    por = np.array([2, 3, 0, 6, 7])            # rows 0..4 -> pairs
    y = rng.standard_normal((5, H))
    w = rng.random((T, k)).astype(np.float32)
    y_w, written = O.weighted_rows(y, por, w, 1.0)
    assert list(written) == [True, False, True, True, False, False, True, True]
    assert np.all(y_w[~written] == 0)
    out = O.combine(y_w, rop, k, round_output=False)
    assert np.array_equal(out[2], np.zeros(H))          # both of token 2's pairs missing
    assert np.array_equal(out[0], y_w[0])               # token 0: only slot 0
    assert np.array_equal(out[3], y_w[6] + y_w[7])


def test_mistakes_are_caught():
    # indexing y_w by row instead of pair, or y by pair instead of row, changes
    # the hand example's result
    ids = [[2, 0], [0, 1]]
    rop, por = _tables(ids, 3)
    y = np.array([[1.0, 2.0], [4.0, -8.0], [0.5, 0.25], [3.0, 6.0]])
    w = np.array([[0.5, 0.25], [0.75, 0.125]])
    y_w, _ = O.weighted_rows(y, por, w, 2.0)
    wrong = np.stack([O.bf16_round(2.0 * w.reshape(-1)[p] * y[p]) for p in range(4)])
    assert not np.array_equal(wrong, y_w)
