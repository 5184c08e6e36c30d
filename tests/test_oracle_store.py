"""Pins of the oracle's store_int8 and the NoPE geometry check (CPU only).

store_int8 follows "GLM-5.3 Kernels" README, 'Included' table (titan_kv.store_int8): 512 int8
values, one fp32 scale, 12 zero bytes per 528-byte row, scattered by slot, negative slot = padding.
"""
import json
import os

import numpy as np
import pytest

import oracle
from synth import f32_to_bf16_bits, bf16_bits_to_f32
from tests.conftest import GOLDEN

ROW = 528


def _row_from_sparse(nonzero):
    x = np.zeros(512, dtype=np.float32)
    for k, v in nonzero.items():
        x[int(k)] = v
    b = f32_to_bf16_bits(x)
    assert np.array_equal(bf16_bits_to_f32(b), x), "golden values must be exact in bf16"
    return b


def test_golden_rows_bytes():
    g = json.load(open(os.path.join(GOLDEN, "store_int8_rows.json")))
    for case in g["cases"]:
        lat = _row_from_sparse(case["nonzero"])[None]
        cache = np.full((3, ROW), 0x5A, dtype=np.int8)
        oracle.store_int8(lat, np.array([1], dtype=np.int64), cache)
        row = cache[1].view(np.uint8)
        codes = np.zeros(512, dtype=np.int8)
        for k, v in case["codes"].items():
            codes[int(k)] = v
        assert np.array_equal(cache[1, :512], codes), case["name"]
        assert list(row[512:516]) == case["scale_bytes_le"], case["name"]
        assert not row[516:].any(), case["name"]
        # rows 0 and 2 untouched
        assert (cache[0] == 0x5A).all() and (cache[2] == 0x5A).all()


def _quantise(lat, n_rows=None):
    n = lat.shape[0]
    cache = np.full((n if n_rows is None else n_rows, ROW), 0x5A, dtype=np.int8)
    oracle.store_int8(lat, np.arange(n, dtype=np.int64), cache)
    return cache


def _scales(cache):
    return cache[:, 512:516].copy().view(np.float32)[:, 0]


def test_random_rows_invariants():
    rng = np.random.default_rng(7)
    x = rng.standard_normal((64, 512)).astype(np.float32) * rng.uniform(0.01, 30, (64, 1)).astype(np.float32)
    lat = f32_to_bf16_bits(x)
    xv = bf16_bits_to_f32(lat).astype(np.float64)
    cache = _quantise(lat)
    codes = cache[:, :512].astype(np.float64)
    scale = _scales(cache).astype(np.float64)
    amax = np.abs(xv).max(1)
    # the scale is amax / 127 rounded to fp32
    assert np.array_equal(scale.astype(np.float32), (amax / 127.0).astype(np.float32))
    # the element of largest magnitude maps to +-127
    j = np.abs(xv).argmax(1)
    assert np.array_equal(np.abs(codes[np.arange(64), j]), np.full(64, 127.0))
    assert np.array_equal(np.sign(codes[np.arange(64), j]), np.sign(xv[np.arange(64), j]))
    # reconstruction error within half a step (plus the fp32 rounding of the quotient)
    err = np.abs(xv - codes * scale[:, None])
    # (half an ulp of a quotient below 128 is 2**-18, i.e. < 4e-6 of a step)
    assert (err <= scale[:, None] * (0.5 + 4e-6)).all()
    # codes never reach -128; trailing 12 bytes are zero
    assert codes.min() >= -127 and codes.max() <= 127
    assert not cache[:, 516:].any()


def test_zero_and_tiny_rows_use_the_floor():
    lat = np.zeros((2, 512), dtype=np.uint16)
    lat[1, 3] = f32_to_bf16_bits(np.array([1e-6], dtype=np.float32))[0]
    cache = _quantise(lat)
    floor_scale = np.float32(np.float32(1e-4) / np.float32(127.0))
    assert _scales(cache)[0] == floor_scale and _scales(cache)[1] == floor_scale
    assert not cache[0, :512].any()
    # 1e-6 / (1e-4/127) = 1.27 -> 1
    assert cache[1, 3] == 1 and np.count_nonzero(cache[1, :512]) == 1


def test_negative_slots_write_nothing_and_order_is_by_slot():
    rng = np.random.default_rng(3)
    lat = f32_to_bf16_bits(rng.standard_normal((5, 512)).astype(np.float32))
    slots = np.array([4, -1, 0, -7, 2], dtype=np.int64)
    cache = np.full((6, ROW), 0x5A, dtype=np.int8)
    oracle.store_int8(lat, slots, cache)
    ref = _quantise(lat)
    assert np.array_equal(cache[4], ref[0])
    assert np.array_equal(cache[0], ref[2])
    assert np.array_equal(cache[2], ref[4])
    for r in (1, 3, 5):
        assert (cache[r] == 0x5A).all()


def test_slot_past_cache_is_an_error():
    lat = np.zeros((1, 512), dtype=np.uint16)
    cache = np.zeros((2, ROW), dtype=np.int8)
    with pytest.raises(ValueError):
        oracle.store_int8(lat, np.array([2], dtype=np.int64), cache)


def test_sign_symmetry():
    # quantising -x gives exactly the negated codes and the same scale (round half to even is odd)
    rng = np.random.default_rng(11)
    x = rng.standard_normal((16, 512)).astype(np.float32)
    a = _quantise(f32_to_bf16_bits(x))
    b = _quantise(f32_to_bf16_bits(-x))
    assert np.array_equal(a[:, :512], -b[:, :512])
    assert np.array_equal(a[:, 512:], b[:, 512:])


def test_dequant_row_is_code_times_scale():
    lat = _row_from_sparse({"0": 254.0, "1": 5.0, "2": -7.0})[None]
    cache = _quantise(lat)
    d = oracle.dequant_rows(cache, [0])[0]
    assert d[0] == 254.0 and d[1] == 4.0 and d[2] == -8.0 and not d[3:].any()


def test_nope_dims_check():
    # "Module glm5next_dsa_ref" NoPE trap: qk_rope_head_dim = 0, the k_rot slice is zero-width;
    # the latent consumed is exactly kv_lora_rank = 512 wide.
    assert oracle.check_dims(512, 0, 64, 32, 128, 4)
    assert not oracle.check_dims(512, 64, 64, 32, 128, 4)
    assert not oracle.check_dims(576, 0, 64, 32, 128, 4)
    assert not oracle.check_dims(512, 0, 0, 32, 128, 4)
