"""Pins of the oracle's 4-bit latent cache row (CPU only).

GLM on CUDA names an opt-in 4-bit latent cache (--kv-dtype fp4) and gives no format; the reading is
E2M1 codes (sign, two exponent bits with bias 1, one mantissa bit) with one E4M3 scale for every 16
values and one fp32 scale per row: s_row = amax / 2688, e_k = the E4M3 value nearest
bmax_k / (6 s_row), code = the E2M1 value nearest x / (value(e_k) s_row), ties to the even code,
saturating at +-6, the sign kept; 304 bytes (256 code pairs, 32 block scales, s_row, 12 zeros).
The decoder is checked against the format's value list, the encoder against a brute-force search
and the interval table of the rounding, the row against hand-derived bytes and invariants.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from synth import f32_to_bf16_bits
from tests.conftest import GOLDEN

E2M1 = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def _row(nonzero):
    x = np.zeros(512, dtype=np.float32)
    for k, v in nonzero.items():
        x[int(k)] = v
    return f32_to_bf16_bits(x)


def test_decode_is_the_value_list():
    for c in range(8):
        assert oracle.e2m1_value(c) == E2M1[c]
        assert oracle.e2m1_value(c | 8) == -E2M1[c] and math.copysign(1.0, oracle.e2m1_value(c | 8)) == -1.0


def _nearest(x):
    """Brute force over the magnitudes: nearest, the even code on a tie, the sign kept."""
    sign = 8 if math.copysign(1.0, x) < 0 else 0
    best = None
    for c in range(8):
        d = abs(abs(x) - E2M1[c])
        if best is None or d < best[0] or (d == best[0] and c % 2 == 0):
            best = (d, c)
    return sign | best[1]


def test_encode_interval_table():
    # rounding to nearest, ties to the even code: the closed and open ends of each interval
    table = [(0.0, 0), (0.25, 0), (np.nextafter(0.25, 1), 1), (0.5, 1), (np.nextafter(0.75, 0), 1), (0.75, 2),
             (1.25, 2), (np.nextafter(1.25, 2), 3), (np.nextafter(1.75, 0), 3), (1.75, 4), (2.5, 4),
             (np.nextafter(2.5, 3), 5), (np.nextafter(3.5, 0), 5), (3.5, 6), (5.0, 6), (np.nextafter(5.0, 6), 7),
             (6.0, 7), (1e30, 7)]
    for x, c in table:
        assert oracle.e2m1_encode(x) == c, x
        assert oracle.e2m1_encode(-x) == c | 8, -x


def test_encode_is_the_nearest_value():
    rng = np.random.default_rng(4)
    xs = list(rng.uniform(-8, 8, 500)) + list(np.exp2(rng.uniform(-6, 3, 300)) * rng.choice([-1, 1], 300))
    for x in xs:
        assert oracle.e2m1_encode(x) == _nearest(float(x)), x


def test_golden_row():
    g = json.load(open(os.path.join(GOLDEN, "store_fp4_row.json")))
    cache = np.full((2, 304), 0xA5, np.uint8)
    oracle.store_fp4(_row(g["nonzero"])[None], np.array([1], np.int64), cache)
    want = np.zeros(256, np.uint8)
    for k, v in g["code_bytes"].items():
        want[int(k)] = v
    sc = np.zeros(32, np.uint8)
    for k, v in g["block_scales"].items():
        sc[int(k)] = v
    r = cache[1]
    assert np.array_equal(r[:256], want)
    assert np.array_equal(r[256:288], sc)
    assert list(r[288:292]) == g["row_scale_bytes_le"]
    assert not r[292:].any()
    assert (cache[0] == 0xA5).all()
    deq = oracle.dequant_rows_fp4(cache, [1])[0]
    for k, v in g["dequant"].items():
        assert deq[int(k)] == v, k


def _blocks(cache, slots):
    r = cache[slots]
    codes = np.stack([r[:, :256] & 15, r[:, :256] >> 4], axis=2).reshape(len(slots), 512)
    return codes, r[:, 256:288], r[:, 288:292].copy().view(np.float32)[:, 0].astype(np.float64)


def test_row_invariants():
    rng = np.random.default_rng(11)
    n = 30
    x32 = (rng.standard_normal((n, 512)) * rng.uniform(0.01, 30, (n, 1))).astype(np.float32)
    x32[:, 96:112] *= 1e-3                                           # a block far below the row's range
    x32[2, 208:224] = 0.0                                            # an all-zero block
    lat = f32_to_bf16_bits(x32)
    cache = np.zeros((n + 8, 304), np.uint8)
    slots = np.arange(n, dtype=np.int64) + 4
    oracle.store_fp4(lat, slots, cache)
    x = (lat.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    codes, esc, s_row = _blocks(cache, slots)
    amax = np.abs(x).max(axis=1)
    assert np.array_equal(s_row, (amax / 2688.0).astype(np.float32).astype(np.float64))
    u = (6.0 * s_row).astype(np.float32).astype(np.float64)
    deq = oracle.dequant_rows_fp4(cache, slots)
    for i in range(n):
        for k in range(32):
            xb = x[i, 16 * k:16 * k + 16]
            t = float(np.float32(np.abs(xb).max() / u[i]))
            assert esc[i, k] == oracle.e4m3_encode(t)                # the pinned E4M3 rounding
            d = float(np.float32(oracle.e4m3_value(esc[i, k]) * s_row[i]))
            for j in range(16):
                c = int(codes[i, 16 * k + j])
                want = _nearest(float(np.float32(xb[j] / d))) if d > 0 else 0
                assert c == want, (i, k, j)
                assert deq[i, 16 * k + j] == E2M1[c & 7] * (-1 if c & 8 else 1) * oracle.e4m3_value(esc[i, k]) * s_row[i]
        assert esc[i].max() <= 0x7E
    # the row's largest value maps to +-6 x 448 x s_row
    arg = np.abs(x).argmax(axis=1)
    assert ((codes[np.arange(n), arg] & 7) == 7).all() and (esc[np.arange(n), arg // 16] == 0x7E).all()
    assert esc[2, 13] == 0 and not codes[2, 208:224].any()
    assert not cache[:4].any() and not cache[n + 4:].any() and not cache[slots, 292:].any()


def test_exactly_representable_row_round_trips():
    # s_row = 1 (amax 2688); each block's values are E2M1 magnitudes times its own scale
    rng = np.random.default_rng(5)
    x = np.zeros(512, np.float64)
    scales = [448.0, 1.0, 2.0 ** -9, 16.0, 0.5, 240.0, 3.5] + [1.0] * 25
    for k in range(32):
        v = rng.choice(E2M1, 16) * rng.choice([-1, 1], 16) * scales[k]
        v[0] = 6.0 * scales[k]                                        # the block's largest value
        x[16 * k:16 * k + 16] = v
    lat = f32_to_bf16_bits(x.astype(np.float32))
    assert np.array_equal((lat.astype(np.uint32) << 16).view(np.float32).astype(np.float64), x)
    cache = np.zeros((1, 304), np.uint8)
    oracle.store_fp4(lat[None], np.zeros(1, np.int64), cache)
    assert np.array_equal(oracle.dequant_rows_fp4(cache, [0])[0], x)


def test_zero_row_padding_and_bounds():
    cache = np.full((3, 304), 7, np.uint8)
    oracle.store_fp4(np.zeros((2, 512), np.uint16), np.array([1, -1], np.int64), cache)
    floor = np.float32(np.float64(np.float32(1e-4)) / 2688.0)
    assert cache[1, 288:292].copy().view(np.float32)[0] == floor
    assert not cache[1, :288].any() and not cache[1, 292:].any()
    assert (cache[0] == 7).all() and (cache[2] == 7).all()
    with pytest.raises(ValueError):
        oracle.store_fp4(np.zeros((1, 512), np.uint16), np.array([3], np.int64), cache)
