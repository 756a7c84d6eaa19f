"""Pins of the W4 (symmetric int4, 128-block, fp16 scale) oracle.

Each test checks the oracle against something other than itself: values
worked by hand from the format's reading, the rounding error bound of
round-to-nearest, the statistics of uniform rounding error, the relative
error the DeepSeek-V4-Pro-671B-GALE-1bit-v4 card prints, and brute-force
loops.  A plausible slip (truncation instead of rounding, scale amax / 8,
the wrong nibble order, a transposed product) fails at least one of them.
"""
import json
import os

import numpy as np
import pytest

import gale_synth as gs
from oracle import w4_oracle as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pages_numbers.json")


def _rng_matrix(rows, cols, tag):
    return gs.normal(gs.stream_key(70, tag), rows * cols).astype(np.float32).reshape(rows, cols)


def test_w4_layout_sizes():
    L = W.w4_layout(4096, 4096)
    assert L["q_bytes"] == 4096 * 4096 // 2
    assert L["s_off"] == L["q_bytes"]                     # already 256-aligned
    assert L["s_bytes"] == 4096 * 32 * 2
    assert L["total"] == L["q_bytes"] + L["s_bytes"]
    # 4 bits per weight plus one fp16 per 128 weights: 4.125 bits/weight
    assert 8 * L["total"] / (4096 * 4096) == pytest.approx(4.125)
    L2 = W.w4_layout(3, 128)
    assert (L2["q_bytes"], L2["s_off"], L2["s_bytes"], L2["total"]) == (192, 256, 6, 512)


def test_w4_quantize_by_hand():
    # block 0: amax 7 -> s = 1 exactly; codes are rint(w) with ties to even
    w = np.zeros((1, 256), dtype=np.float32)
    w[0, :8] = [7.0, -7.0, 2.5, 3.5, -0.5, 0.49, -2.51, 6.4]
    # block 1: amax 0.7 -> s = fp16(0.1); w = 0.35 is 3.5 s (about) -> nearest
    w[0, 128] = 0.7
    w[0, 129] = -0.35
    q, s = W.w4_quantize(w)
    assert s[0, 0] == np.float16(1.0)
    assert list(q[0, :8]) == [7, -7, 2, 4, 0, 0, -3, 6]
    assert (q[0, 8:128] == 0).all()
    s1 = np.float16(np.float32(0.7) / np.float32(7.0))
    assert s[0, 1] == s1
    assert q[0, 128] == 7
    assert q[0, 129] == int(np.rint(np.float32(-0.35) / np.float32(s1)))
    assert q[0, 129] in (-3, -4)


def test_w4_zero_block_and_clamp():
    w = np.zeros((2, 128), dtype=np.float32)
    q, s = W.w4_quantize(w)
    assert (q == 0).all() and (s == 0).all()
    # the amax element always maps to +-7 (the fp16 scale is within 2^-11 of amax / 7)
    w = _rng_matrix(64, 512, 1) * np.float32(37.0)
    q, s = W.w4_quantize(w)
    assert q.min() >= -7 and q.max() <= 7
    for r in range(64):
        for b in range(4):
            blk = w[r, 128 * b:128 * (b + 1)]
            i = int(np.argmax(np.abs(blk)))
            assert abs(int(q[r, 128 * b + i])) == 7


def test_w4_round_to_nearest_bound():
    # |w - s q| <= s / 2 (+ fp32 rounding of w / s) for every weight: round to nearest
    w = _rng_matrix(32, 1024, 2)
    q, s = W.w4_quantize(w)
    sd = np.repeat(s.astype(np.float64), 128, axis=1)
    err = np.abs(w.astype(np.float64) - sd * q)
    assert (err <= sd * (0.5 + 1e-6) + 1e-30).all()
    # and truncation would break it: some weights are more than s/2 from trunc(w/s) s
    tq = np.trunc(w / np.repeat(s.astype(np.float32), 128, axis=1))
    assert (np.abs(w - sd * tq) > sd * 0.5 * 1.01).any()


def test_w4_error_statistics_match_uniform_rounding_and_the_card():
    # For rounding to nearest the error is uniform in [-s/2, s/2]: its mean square is s^2 / 12.
    w = _rng_matrix(256, 4096, 3)
    q, s = W.w4_quantize(w)
    err2 = (w.astype(np.float64) - W.w4_dequant(q, s)) ** 2
    want = np.repeat(s.astype(np.float64) ** 2 / 12.0, 128, axis=1)
    assert err2.mean() == pytest.approx(want.mean(), rel=0.03)
    # relative Frobenius error of N(0,1) weights: about 0.12, as the card's 0.119 on real weights
    rel = np.sqrt(err2.sum() / (w.astype(np.float64) ** 2).sum())
    card = json.load(open(GOLDEN))["w4_nonexpert"]["relative_error_real_weights"]
    assert abs(rel - card) < 0.015, rel


def test_w4_pack_nibble_order_by_hand():
    q = np.zeros((1, 128), dtype=np.int8)
    q[0, :4] = [1, -1, 7, -7]
    s = np.full((1, 1), 0.5, dtype=np.float16)
    buf = W.w4_pack(q, s)
    # byte 0 = low nibble q[0] = 0x1, high nibble q[1] = -1 = 0xF; byte 1 = 7 | (-7 & 0xF) << 4 = 0x97
    assert buf[0] == 0xF1 and buf[1] == 0x97 and (buf[2:64] == 0).all()
    assert buf[256:258].view(np.float16)[0] == np.float16(0.5)


def test_w4_pack_unpack_round_trip():
    w = _rng_matrix(48, 384, 4)
    q, s = W.w4_quantize(w)
    q2, s2 = W.w4_unpack(W.w4_pack(q, s), 48, 384)
    assert np.array_equal(q, q2) and np.array_equal(s.view(np.uint16), s2.view(np.uint16))


def test_w4_gemv_brute_force():
    rows, cols, B = 5, 256, 3
    w = _rng_matrix(rows, cols, 5)
    q, s = W.w4_quantize(w)
    x = gs.bf16_bits_to_f32(gs.f32_to_bf16_bits(gs.normal(gs.stream_key(71, 0), B * cols).astype(np.float32))).reshape(B, cols)
    y = W.w4_gemv(q, s, x)
    for t in range(B):
        for r in range(rows):
            acc = 0.0
            for c in range(cols):
                acc += float(s[r, c // 128]) * int(q[r, c]) * float(x[t, c])
            assert y[t, r] == pytest.approx(acc, rel=1e-12, abs=1e-12)


def test_w4_unit_scales_reduce_to_integer_matmul():
    rng = np.random.default_rng(9)
    q = rng.integers(-7, 8, size=(7, 256)).astype(np.int8)
    s = np.ones((7, 2), dtype=np.float16)
    x = rng.integers(-3, 4, size=(2, 256)).astype(np.float64)
    y = W.w4_gemv(q, s, x)
    assert np.array_equal(y, (x.astype(np.int64) @ q.astype(np.int64).T).astype(np.float64))
