"""Pins for the oracle's dispatch tables and permutation (CPU only).

Pinned by the worked example printed in the TileLang tutorial "Example 07: MoE
dispatch contract and quantised GEMM" §1 (tests/golden/dispatch_example_tutorial07.json),
by the tutorial's three self-checks (exact-once coverage, padded intervals
cover compact ones, the m_start recovery formula) run on seeded random
routings including the tutorial's second command-line configuration, and by an
independent brute-force recount.
"""
import json
import os

import numpy as np
import pytest

from oracle import moe_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "dispatch_example_tutorial07.json")


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


def test_worked_example_tables():
    g = _golden()
    ids = np.array(g["topk_ids"], dtype=np.int32)
    assert ids.shape == (g["tokens"], g["top_k"])
    t = O.dispatch_tables(ids, g["experts"], g["padding_M"], g["block_token"])
    assert t["group_sizes"].tolist() == g["group_sizes"]
    assert t["group_offsets"][:-1].tolist() == g["group_offsets"]
    assert t["group_offsets"][-1] == g["group_sum"]
    assert t["group_padded_offsets"][:-1].tolist() == g["group_padded_offsets"]
    lens = np.diff(t["group_padded_offsets"]).tolist()
    assert lens == g["padded_interval_lengths"]
    assert t["group_sum"] == g["group_sum"]
    assert t["M_blk"] == g["M_blk"]
    assert t["waste"] == g["waste"]
    assert t["group_idx_for_bx"].tolist() == g["group_idx_for_bx"]


def _random_ids(T, E, k, rng, skew=False):
    ids = np.zeros((T, k), dtype=np.int32)
    p = None
    if skew:
        p = 1.0 / np.arange(1, E + 1) ** 1.5
        p /= p.sum()
    for t in range(T):
        ids[t] = rng.choice(E, size=k, replace=False, p=p)
    return ids


def _check_contract(ids, E, padding_M, bt):
    """The tutorial's three self-checks plus a brute-force recount."""
    T, k = ids.shape
    P = T * k
    t = O.dispatch_tables(ids, E, padding_M, bt)
    flat = ids.reshape(-1)
    # brute-force recount of every table
    for e in range(E):
        assert t["group_sizes"][e] == sum(1 for x in flat if x == e)
        assert t["group_offsets"][e] == sum(1 for x in flat if x < e)
        assert t["group_padded_offsets"][e] == sum(
            -(-sum(1 for x in flat if x == ee) // padding_M) * padding_M for ee in range(e))
    assert int(t["group_sizes"].sum()) == P
    assert t["M_blk"] == -(-P // bt) + E
    # permutation: bijection, sorted by expert, stable within an expert
    rop, por = t["row_of_pair"], t["pair_of_row"]
    assert sorted(rop.tolist()) == list(range(P))
    assert np.all(por[rop] == np.arange(P))
    experts_by_row = flat[por]
    assert np.all(np.diff(experts_by_row) >= 0)
    for e in range(E):
        rows = np.nonzero(experts_by_row == e)[0]
        assert np.all(np.diff(por[rows]) > 0)          # stable: flat order kept
    # self-check 2: each padded interval covers its compact interval
    go, gpo, gs = t["group_offsets"], t["group_padded_offsets"], t["group_sizes"]
    for e in range(E):
        assert gpo[e + 1] - gpo[e] >= gs[e]
        assert (gpo[e + 1] - gpo[e]) % padding_M == 0
    # self-checks 1 and 3: walk every M-block with the recovery formula;
    # every (token, expert) pair is reached exactly once and no row leaves its group
    covered = np.zeros(P, dtype=np.int64)
    for bx in range(t["M_blk"]):
        g, m_start, rows = O.block_rows(t, bx, bt)
        assert 0 <= rows <= bt
        if rows:
            assert go[g] <= m_start and m_start + rows <= go[g] + gs[g]
            for r in range(m_start, m_start + rows):
                assert experts_by_row[r] == g
                covered[por[r]] += 1
    assert np.all(covered == 1)
    return t


def test_worked_example_contract():
    g = _golden()
    _check_contract(np.array(g["topk_ids"], dtype=np.int32), g["experts"],
                    g["padding_M"], g["block_token"])


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_second_cli_configuration_contract(seed):
    c = _golden()["second_cli_configuration"]
    rng = np.random.default_rng(100 + seed)
    ids = _random_ids(c["tokens"], c["experts"], c["top_k"], rng)
    _check_contract(ids, c["experts"], c["padding_M"], c["block_token"])


@pytest.mark.parametrize("T,E,k,pad,skew", [(33, 16, 4, 16, True), (64, 32, 8, 128, True),
                                            (17, 5, 5, 8, False), (1, 8, 2, 128, False)])
def test_random_routing_contract(T, E, k, pad, skew):
    rng = np.random.default_rng(T * 1000 + E)
    ids = _random_ids(T, E, k, rng, skew=skew)
    _check_contract(ids, E, pad, pad)


def test_empty_experts_get_empty_intervals_and_blocks_skip_them():
    # experts 1, 2 and 4 receive nothing; blocks must go to non-empty experts
    ids = np.array([[0, 3], [3, 5], [0, 5], [5, 3]], dtype=np.int32)
    t = _check_contract(ids, 6, 4, 4)
    assert t["group_sizes"].tolist() == [2, 0, 0, 3, 0, 3]
    assert t["group_padded_offsets"].tolist() == [0, 4, 4, 4, 8, 8, 12]
    # the block starting at row 4 belongs to expert 3 (largest g with offset <= 4)
    assert t["group_idx_for_bx"][1] == 3
    assert t["group_idx_for_bx"][2] == 5


def test_permute_gathers_token_rows():
    rng = np.random.default_rng(5)
    ids = _random_ids(7, 6, 3, rng)
    hidden = rng.standard_normal((7, 4))
    t = O.dispatch_tables(ids, 6, 4)
    xp = O.permute(hidden, t["pair_of_row"], 3)
    for p in range(21):
        assert np.array_equal(xp[t["row_of_pair"][p]], hidden[p // 3])


def test_out_of_range_id_rejected():
    with pytest.raises(ValueError):
        O.dispatch_tables(np.array([[0, 4]], dtype=np.int32), 4, 128)
