"""Pins of the oracle's FP8 latent cache row (CPU only).

GLM on CUDA names an opt-in FP8 latent cache and gives no format; the readings are E4M3 codes
(the OCP E4M3FN form: exponent bias 7, subnormals, no infinities, largest finite 448) with one fp32
scale per row in the INT8 row's 528-byte layout: scale = amax / 448 (amax floored as for INT8),
code = the E4M3 value nearest x / scale with ties to the even code, saturating at +-448.
The encoder is checked against a brute-force search over the decoded table, which shares none of
its arithmetic; the decoder against the format's definition at fixed points; the row against
hand-derived bytes and invariants.
"""
import json
import math
import os

import numpy as np

import oracle
from synth import f32_to_bf16_bits
from tests.conftest import GOLDEN

FINITE = [c for c in range(256) if (c & 0x7F) != 0x7F]


def _row(nonzero):
    x = np.zeros(512, dtype=np.float32)
    for k, v in nonzero.items():
        x[int(k)] = v
    return f32_to_bf16_bits(x)


def test_decode_fixed_points_and_order():
    v = oracle.e4m3_value
    assert v(0x00) == 0.0 and v(0x01) == 2.0 ** -9 and v(0x07) == 7 * 2.0 ** -9
    assert v(0x08) == 2.0 ** -6                                     # the smallest normal
    assert v(0x38) == 1.0 and v(0x40) == 2.0 and v(0x7E) == 448.0
    assert math.isnan(v(0x7F)) and math.isnan(v(0xFF))
    pos = [v(c) for c in range(0x7F)]
    assert all(a < b for a, b in zip(pos, pos[1:]))                  # strictly increasing
    assert len(pos) == 127
    for c in range(0x7F):
        assert v(c | 0x80) == -pos[c] and math.copysign(1.0, v(c | 0x80)) == -1.0


def _nearest(x):
    """Brute force: the finite code of x's sign whose value is nearest x, ties to the even code;
    beyond the largest value, the largest value."""
    sign = 0x80 if math.copysign(1.0, x) < 0 else 0
    best = None
    for c in range(0x7F):
        d = abs(abs(x) - oracle.e4m3_value(c))
        if best is None or d < best[0] or (d == best[0] and c % 2 == 0):
            best = (d, c)
    return sign | best[1]


def test_encode_is_the_nearest_value_ties_to_even():
    rng = np.random.default_rng(9)
    xs = list(rng.uniform(-460, 460, 300)) + list(np.exp2(rng.uniform(-12, 9, 300)) * rng.choice([-1, 1], 300))
    vals = [oracle.e4m3_value(c) for c in range(0x7F)]
    for a, b in zip(vals, vals[1:]):                                # every midpoint and its neighbours
        m = (a + b) / 2
        xs += [m, -m, np.nextafter(m, 0.0), np.nextafter(m, 1e9)]
    for x in xs:
        assert oracle.e4m3_encode(x) == _nearest(float(x)), x


def test_encode_saturates_and_keeps_the_sign():
    assert oracle.e4m3_encode(448.0) == 0x7E and oracle.e4m3_encode(1e9) == 0x7E
    assert oracle.e4m3_encode(-500.0) == 0xFE
    assert oracle.e4m3_encode(-0.0) == 0x80 and oracle.e4m3_encode(0.0) == 0x00
    assert oracle.e4m3_encode(-1e-9) == 0x80                        # rounds to -0


def test_golden_rows():
    g = json.load(open(os.path.join(GOLDEN, "store_fp8_rows.json")))
    for case in g["cases"]:
        cache = np.full((1, 528), 0xA5, np.uint8)
        oracle.store_fp8(_row(case["nonzero"])[None], np.zeros(1, np.int64), cache)
        want = np.zeros(512, np.uint8)
        for k, v in case["codes"].items():
            want[int(k)] = v
        assert np.array_equal(cache[0, :512], want), case["name"]
        assert list(cache[0, 512:516]) == case["scale_bytes_le"], case["name"]
        assert not cache[0, 516:].any()


def test_row_invariants():
    rng = np.random.default_rng(10)
    lat = f32_to_bf16_bits((rng.standard_normal((40, 512)) * rng.uniform(0.01, 30, (40, 1))).astype(np.float32))
    cache = np.zeros((50, 528), np.uint8)
    slots = np.arange(40, dtype=np.int64) + 5
    oracle.store_fp8(lat, slots, cache)
    x = (lat.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    deq = oracle.dequant_rows_fp8(cache, slots)
    scales = cache[slots, 512:516].copy().view(np.float32)[:, 0].astype(np.float64)
    amax = np.abs(x).max(axis=1)
    assert np.array_equal(scales, (amax / 448.0).astype(np.float32).astype(np.float64))
    arg = np.abs(x).argmax(axis=1)
    assert ((cache[slots, arg] & 0x7F) == 0x7E).all()               # the largest maps to 448
    # within half a step of the E4M3 grid: 2^-4 relative for normals, 2^-10 absolute (x scale) below
    err = np.abs(x - deq)
    bound = np.maximum(np.abs(x) * 2.0 ** -4, 2.0 ** -10 * scales[:, None]) * (1 + 1e-6)
    assert (err <= bound).all()
    assert not cache[:5].any() and not cache[45:].any()              # other rows untouched
    assert not cache[slots, 516:].any()


def test_zero_row_and_padding_slot():
    cache = np.full((3, 528), 7, np.uint8)
    oracle.store_fp8(np.zeros((2, 512), np.uint16), np.array([1, -1], np.int64), cache)
    floor = np.float32(np.float64(np.float32(1e-4)) / 448.0)
    assert cache[1, 512:516].copy().view(np.float32)[0] == floor
    assert not cache[1, :512].any() and not cache[1, 516:].any()
    assert (cache[0] == 7).all() and (cache[2] == 7).all()           # a negative slot writes nothing
