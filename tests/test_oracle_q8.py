"""Pins of the oracle's INT8 indexer state (CPU only).

GLM-5.3-Flash (pypto-lib) page, 'What is quantized': the indexer state cache is FP32 today; the
sibling port quantizes it to INT8 with one FP32 scale per row. Each 128-value pooled key becomes
128 int8 codes and one fp32 scale with the row recipe of the same section (amax floored at
INT8_AMAX_EPS, rescaled to 127); the index scores then use code * scale in place of the key.
"""
import json
import os

import numpy as np

import oracle
from synth import f32_to_bf16_bits
from tests.conftest import GOLDEN


def _row(nonzero, d=128):
    x = np.zeros(d, dtype=np.float32)
    for k, v in nonzero.items():
        x[int(k)] = v
    return x


def test_golden_rows():
    g = json.load(open(os.path.join(GOLDEN, "pool_q8_rows.json")))
    for case in g["cases"]:
        codes, scales = oracle.pool_q8(_row(case["nonzero"])[None])
        want = np.zeros(128, dtype=np.int8)
        for k, v in case["codes"].items():
            want[int(k)] = v
        assert np.array_equal(codes[0], want), case["name"]
        assert scales[0] == np.float32(case["scale"]), case["name"]


def test_floor_rows():
    # an all-zero row and a tiny row take the amax floor: scale = fl32(fl32(1e-4) / 127)
    floor = np.float32(np.float64(np.float32(1e-4)) / 127.0)
    codes, scales = oracle.pool_q8(np.stack([_row({}), _row({"0": 1e-6, "1": -1e-6})]))
    assert (scales == floor).all()
    assert not codes[0].any()
    assert codes[1, 0] == 1 and codes[1, 1] == -1 and not codes[1, 2:].any()   # 1e-6 / scale = 1.27


def test_invariants_on_random_rows():
    rng = np.random.default_rng(5)
    x = (rng.standard_normal((300, 128)) * rng.uniform(0.01, 50, (300, 1))).astype(np.float32)
    codes, scales = oracle.pool_q8(x)
    amax = np.abs(x).max(axis=1)
    assert np.array_equal(scales, (amax.astype(np.float64) / 127.0).astype(np.float32))
    arg = np.abs(x).argmax(axis=1)
    assert (np.abs(codes[np.arange(300), arg]) == 127).all()               # the largest maps to 127
    err = np.abs(x.astype(np.float64) - codes * scales[:, None].astype(np.float64))
    assert (err <= scales[:, None] * (0.5 + 4e-6)).all()                     # within half a step
    assert (np.abs(codes.astype(np.int32)) <= 127).all()
    neg_codes, neg_scales = oracle.pool_q8(-x)
    assert np.array_equal(neg_codes, -codes) and np.array_equal(neg_scales, scales)


def test_scores_q8_are_scores_of_the_dequantised_keys():
    # the q8 score equals index_scores (pinned on its own) applied to code * scale in fp64
    rng = np.random.default_rng(6)
    H, D, P = 32, 128, 40
    q = f32_to_bf16_bits(rng.standard_normal((H, D)).astype(np.float32))
    w = rng.uniform(0, 1, H).astype(np.float32)
    pooled = rng.standard_normal((P, D)).astype(np.float32)
    codes, scales = oracle.pool_q8(pooled)
    deq = codes.astype(np.float64) * scales[:, None].astype(np.float64)
    assert np.array_equal(oracle.index_scores_q8(q, w, codes, scales, P), oracle.index_scores(q, w, deq, P))
    s_q8 = oracle.index_scores_q8(q, w, codes, scales, 30)
    assert s_q8.shape == (30,)


def test_scores_q8_within_the_quantisation_bound():
    # |s_q8 - s| <= sum_h |w_h| sum_d |q_hd| * scale_p / 2 (relu is 1-Lipschitz)
    rng = np.random.default_rng(7)
    H, D, P = 32, 128, 200
    q = f32_to_bf16_bits(rng.standard_normal((H, D)).astype(np.float32))
    qf = q.astype(np.uint32) << 16
    qf = qf.view(np.float32).astype(np.float64)
    w = rng.uniform(0, 1, H).astype(np.float32)
    pooled = rng.standard_normal((P, D)).astype(np.float32)
    codes, scales = oracle.pool_q8(pooled)
    s = oracle.index_scores(q, w, pooled, P)
    s_q8 = oracle.index_scores_q8(q, w, codes, scales, P)
    bound = (w.astype(np.float64) * np.abs(qf).sum(axis=1)).sum() * scales.astype(np.float64) * (0.5 + 1e-5)
    assert (np.abs(s_q8 - s) <= bound).all()
    assert np.abs(s_q8 - s).max() > 0          # the quantisation is not a no-op
