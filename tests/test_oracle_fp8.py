"""Pins for the oracle's E4M3 encoder and FP8 quantisation (CPU only).

The encoder is pinned by the OCP FP8 E4M3 ("E4M3FN") format definition (code
values, round trip of every finite code, ties-to-even at every midpoint,
saturation) and by torch's own float32 -> float8_e4m3fn conversion on dense
samples. 1x128 activation and 128x128 weight quantisation are pinned by their
invariants: every tile with a non-zero maximum has a +-448 code, the
dequantisation error bound, the zero-tile rule, and the row-count edge cases
[0, 1, 127, 128, 129] at width 6144 from XTuner PR #2089's parametrised tests.
"""
import numpy as np
import pytest
import torch

from oracle import moe_oracle as O


def test_decode_table_known_codes():
    v = O.e4m3_decode_table()
    assert v[0x00] == 0.0 and np.signbit(v[0x80])
    assert v[0x01] == 2.0 ** -9            # smallest subnormal
    assert v[0x07] == 7 * 2.0 ** -9        # largest subnormal
    assert v[0x08] == 2.0 ** -6            # smallest normal
    assert v[0x38] == 1.0
    assert v[0x7E] == 448.0 and v[0xFE] == -448.0
    assert np.isnan(v[0x7F]) and np.isnan(v[0xFF])
    finite = v[np.isfinite(v)]
    assert len(finite) == 254


def test_round_trip_every_finite_code():
    v = O.e4m3_decode_table()
    codes = np.array([c for c in range(256) if np.isfinite(v[c])], dtype=np.uint8)
    got = O.e4m3_encode(v[codes].astype(np.float32))
    assert np.array_equal(got, codes)


def test_midpoints_round_to_even_and_nearest():
    v = O.e4m3_decode_table()
    pos = [c for c in range(0x7F)]           # 0x00 .. 0x7E, increasing values
    for a, b in zip(pos[:-1], pos[1:]):
        mid = (v[a] + v[b]) / 2
        m32 = np.float32(mid)
        assert float(m32) == mid            # midpoints are exact in float32
        even = a if (a & 1) == 0 else b
        assert O.e4m3_encode(m32) == even, (hex(a), hex(b))
        lo = np.nextafter(m32, np.float32(-1))
        hi = np.nextafter(m32, np.float32(1000))
        assert O.e4m3_encode(lo) == a
        assert O.e4m3_encode(hi) == b
        assert O.e4m3_encode(-hi) == (b | 0x80)


def test_saturation_and_signed_zero():
    xs = np.array([448.0, 449.0, 463.99, 464.0, 480.0, 1e30, np.inf], dtype=np.float32)
    assert np.all(O.e4m3_encode(xs) == 0x7E)
    assert np.all(O.e4m3_encode(-xs) == 0xFE)
    assert O.e4m3_encode(np.float32(-0.0)) == 0x80
    assert O.e4m3_encode(np.float32(2.0 ** -11)) == 0x00     # rounds to +0
    assert O.e4m3_encode(np.float32(-(2.0 ** -11))) == 0x80  # rounds to -0


def test_matches_torch_float8_cast_on_dense_samples():
    rng = np.random.default_rng(0)
    mags = np.exp(rng.uniform(np.log(2.0 ** -12), np.log(447.9), 400000))
    x = (mags * rng.choice([-1.0, 1.0], mags.size)).astype(np.float32)
    x = np.concatenate([x, np.linspace(-447.9, 447.9, 200001).astype(np.float32)])
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = O.e4m3_encode(x)
    assert np.array_equal(got, ref)


def _check_quant(h, q, s, tile_cols=128):
    M, F = h.shape
    v = O.e4m3_decode_table()
    for r in range(M):
        for c in range(-(-F // tile_cols)):
            blk = h[r, c * tile_cols:(c + 1) * tile_cols].astype(np.float64)
            qb = q[r, c * tile_cols:(c + 1) * tile_cols]
            amax = np.abs(blk).max() if blk.size else 0.0
            if amax == 0:
                assert s[r, c] == 0 and np.all(qb == 0)
                continue
            assert s[r, c] == np.float32(np.float32(amax) / np.float32(448.0))
            assert np.any((qb & 0x7F) == 0x7E)
            deq = v[qb] * float(s[r, c])
            normal = np.abs(blk) >= 2.0 ** -6 * float(s[r, c])
            err = np.abs(deq - blk)
            # half an E4M3 ulp (2**-4 relative) plus the float32 division's rounding
            assert np.all(err[normal] <= np.abs(blk[normal]) * (2.0 ** -4 + 2.0 ** -22))
            assert np.all(err[~normal] <= 2.0 ** -10 * float(s[r, c]) * (1 + 2.0 ** -20))


@pytest.mark.parametrize("M", [0, 1, 127, 128, 129])
def test_quant_1x128_row_edge_cases(M):
    rng = np.random.default_rng(M)
    h = (rng.standard_normal((M, 6144)) * rng.uniform(0.01, 10, (M, 1))).astype(np.float32)
    q, s = O.quant_1x128(h)
    assert q.shape == (M, 6144) and q.dtype == np.uint8
    assert s.shape == (M, 48) and s.dtype == np.float32
    if M:
        _check_quant(h[:8], q[:8], s[:8])


def test_quant_1x128_partial_tile_zero_tile_and_subnormals():
    rng = np.random.default_rng(3)
    h = rng.standard_normal((5, 200)).astype(np.float32)
    h[1, :128] = 0.0                       # an all-zero tile
    h[2, 128:] = 0.0                       # an all-zero partial tile
    h[3, :127] *= 1e-6                     # one large value, the rest subnormal in E4M3
    h[4, 7] = -h[4].__abs__().max() * 3    # negative amax
    q, s = O.quant_1x128(h)
    assert s.shape == (5, 2)
    assert s[1, 0] == 0 and np.all(q[1, :128] == 0)
    assert s[2, 1] == 0 and np.all(q[2, 128:] == 0)
    assert q[4, 7] == 0xFE
    _check_quant(h, q, s)


def test_quant_weight_128x128_blocks():
    rng = np.random.default_rng(4)
    w = (rng.standard_normal((256, 384)) * 0.02).astype(np.float32)
    w[128:, 256:] = 0.0
    q, s = O.quant_weight_128x128(w)
    assert s.shape == (2, 3)
    assert s[1, 2] == 0 and np.all(q[128:, 256:] == 0)
    v = O.e4m3_decode_table()
    for i in range(2):
        for j in range(3):
            blk = w[i * 128:(i + 1) * 128, j * 128:(j + 1) * 128]
            if not np.any(blk):
                continue
            qb = q[i * 128:(i + 1) * 128, j * 128:(j + 1) * 128]
            assert s[i, j] == np.float32(np.float32(np.abs(blk).max()) / np.float32(448))
            assert np.any((qb & 0x7F) == 0x7E)
            # same rule as a 1x128 row tile applied to the whole block
            q1 = O.e4m3_encode((blk / s[i, j]).astype(np.float32))
            assert np.array_equal(q1, qb)
            assert np.all(np.abs(v[qb] * s[i, j] - blk) <= np.abs(blk) * 2.0 ** -4 + 2.0 ** -10 * s[i, j] * 1.001)
