"""GPU parity of a7, the weighted unpermute (moe_unpermute), against the
oracle: fp32 y rows gathered by row_of_pair, weighted in slot order, scaled by
routed_scaling_factor, plus the optional addend, one bf16 cast."""
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


@pytest.mark.parametrize("T,E,k,H,scale,addend", [(9, 4, 2, 128, 1.0, False),
                                                   (300, 16, 8, 2048, 2.5, True),
                                                   (77, 7, 3, 7168, 2.827, False)])
def test_unpermute(T, E, k, H, scale, addend):
    from tests import gpu_util as gu
    import moe_routed_expert_top_b200 as M
    cfg = get_config("tiny", T=T, E=E, top_k=k, H=H, F=64)
    rng = np.random.default_rng(T)
    ids = gu.random_ids(T, E, k, rng)
    _, w = O.route_topk(rng.standard_normal((T, E)).astype(np.float32), k, O.SIGMOID, True)
    L, tables, status, _ = gu.gpu_tables(cfg, ids)
    ref_t = O.dispatch_tables(ids, E, 128)
    y = (rng.standard_normal((T * k, H)) * 1.5).astype(np.float32)
    add = (rng.standard_normal((T, H))).astype(np.float32) if addend else None
    out = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
    M.moe_unpermute(gu.problem(cfg), torch.from_numpy(y).cuda(), tables, torch.from_numpy(w).cuda(),
                    scale, torch.from_numpy(add).cuda() if addend else None, out)
    torch.cuda.synchronize()
    ref = O.unpermute(y, ref_t["row_of_pair"], w, scale, addend=add)
    gu.assert_within_tol(gu.f64(out), ref, "unpermute")
    # one bf16 cast of an fp32 sum: within one bf16 ulp of the exact value
    exact = O.unpermute(y, ref_t["row_of_pair"], w, scale, addend=add, round_output=False)
    assert np.all(np.abs(gu.f64(out) - exact) <= np.abs(exact) * 2.0 ** -7 + 1e-6)


def _f16e_encode(y):
    """fp16 codes and int8 exponents of rows y [P, H] (per 128 columns, the
    block maximum in [2^14, 2^15)), written from the format's definition."""
    P, H = y.shape
    b = np.abs(y).reshape(P, H // 128, 128).max(2)
    e = np.where(b > 0, np.floor(np.log2(np.where(b > 0, b, 1.0))) - 14, 0).astype(np.int64)
    e = np.maximum(e, -100)
    c = (y / np.repeat(np.ldexp(1.0, e), 128, axis=1)).astype(np.float16)
    return c, e.astype(np.int8)


@pytest.mark.parametrize("T,E,k,H,scale,addend", [(9, 4, 2, 128, 1.0, False),
                                                   (300, 16, 8, 2048, 2.5, True),
                                                   (77, 7, 3, 7168, 2.827, False)])
def test_unpermute_f16e(T, E, k, H, scale, addend):
    """moe_unpermute_f16e against the oracle's unpermute of the exactly decoded
    rows (wide-range rows: some blocks far above fp16's range, some far below)."""
    from tests import gpu_util as gu
    import moe_routed_expert_top_b200 as M
    cfg = get_config("tiny", T=T, E=E, top_k=k, H=H, F=64)
    rng = np.random.default_rng(T + 1)
    ids = gu.random_ids(T, E, k, rng)
    _, w = O.route_topk(rng.standard_normal((T, E)).astype(np.float32), k, O.SIGMOID, True)
    L, tables, status, _ = gu.gpu_tables(cfg, ids)
    ref_t = O.dispatch_tables(ids, E, 128)
    y = rng.standard_normal((T * k, H)) * 1.5
    y *= np.repeat(2.0 ** rng.integers(-40, 40, (T * k, H // 128)), 128, axis=1)
    c16, ex = _f16e_encode(y)
    dec = c16.astype(np.float64) * np.repeat(np.ldexp(1.0, ex.astype(np.int64)), 128, axis=1)
    add = (rng.standard_normal((T, H))).astype(np.float32) if addend else None
    out = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
    M.moe_unpermute_f16e(gu.problem(cfg), torch.from_numpy(c16).cuda(), torch.from_numpy(ex).cuda(),
                         tables, torch.from_numpy(w).cuda(), scale,
                         torch.from_numpy(add).cuda() if addend else None, out)
    torch.cuda.synchronize()
    exact = O.unpermute(dec, ref_t["row_of_pair"], w, scale, addend=add, round_output=False)
    # one bf16 cast of an fp32 sum of the decoded rows: the cast (2^-8 relative,
    # with margin) plus fp32 rounding of the k-term sum (bounded by the sum of
    # the terms' magnitudes)
    mag = O.unpermute(np.abs(dec), ref_t["row_of_pair"], np.abs(w), abs(scale),
                      addend=np.abs(add) if addend else None, round_output=False)
    bound = np.abs(exact) * 2.0 ** -8 + mag * (k + 2) * 2.0 ** -23 + 1e-38
    assert np.all(np.abs(gu.f64(out) - exact) <= bound)
