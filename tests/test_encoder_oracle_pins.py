"""Pins of the GALE 1-bit encoder oracle (dense -> rotated -> sign + LS block
scale + top-1 % outliers with a per-row int4 scale).

Checked against: the dense Hadamard transform of the main oracle (and its
closed forms), an exactly representable matrix that must come back unchanged,
hand-worked rows (signs, outlier choice and order, ties), the least-squares
property of the block scale, the rounding bound of the outlier codes, and the
closed-form error of sign rounding with an LS scale on Gaussian weights,
sqrt(1 - 2/pi).
"""
import math

import numpy as np
import pytest

import gale_synth as gs
from oracle import encoder_oracle as E
from oracle import gale_oracle as O


def _gauss(rows, cols, tag):
    return gs.normal(gs.stream_key(74, tag), rows * cols).astype(np.float32).reshape(rows, cols)


def test_staged_fwht_matches_dense_hadamard():
    x = _gauss(3, 2048, 1).astype(np.float64)
    a = E.fwht_staged(x)
    b = O.fwht_blocked(x)
    assert np.max(np.abs(a - b)) < 1e-12 * np.max(np.abs(b))
    assert np.max(np.abs(E.fwht_staged(a) - x)) < 1e-12 * np.max(np.abs(x))   # involution


def _representable(rows, cols, rng):
    """W_rot whose every block has one magnitude 7 * 2^-e (e in 4..9) and random
    signs: every step of the encoder is exact on it."""
    nb = cols // 128
    e = rng.integers(4, 10, size=(rows, nb))
    mag = np.repeat(7.0 * 2.0 ** -e, 128, axis=1)
    return np.where(rng.random((rows, cols)) < 0.5, -mag, mag)


def test_representable_matrix_round_trips_exactly():
    rng = np.random.default_rng(3)
    wr = _representable(6, 2048, rng)
    w = E.fwht_staged(wr)                   # dyadic sums: exact in fp32 and fp64
    assert np.array_equal(w.astype(np.float32).astype(np.float64), w)
    c = E.encode(w.astype(np.float32))
    assert np.array_equal(O.dequant(c), wr)
    # and through the packed bytes
    assert np.array_equal(O.dequant_packed(O.pack(c), 6, 2048), wr)


def test_signs_outliers_and_ties_by_hand():
    cols = 1024                              # k = 10
    wr = np.full((2, cols), 0.25)
    wr[0, 1::2] = -0.25                      # odd columns negative
    big = {900: 3.0, 5: -2.5, 77: 2.0, 640: -1.5, 12: 1.25, 300: 1.0, 301: -1.0, 1000: 0.75, 3: 0.5, 8: -0.5}
    for cc, v in big.items():
        wr[0, cc] = v
    wr[0, 9] = 0.5                           # ties with columns 3 and 8 at |0.5|: the lower columns win
    wr[1] = 0.0                              # zero row: signs 0, every scale 0, first ten columns chosen
    c = E.encode(E.fwht_staged(wr).astype(np.float32))
    assert list(c["idx"][0]) == [3, 5, 8, 12, 77, 300, 301, 640, 900, 1000]
    assert list(c["idx"][1]) == list(range(10))
    assert np.array_equal(c["signs"][0], (wr[0] < 0).astype(np.uint8))
    assert (c["signs"][1] == 0).all() and (c["s_blk"][1] == 0).all() and c["s_row"][1] == 0
    sr = np.float16(3.0 / 7.0)
    assert c["s_row"][0] == sr
    want = [np.clip(np.rint(wr[0, j] / np.float64(sr)), -7, 7) for j in c["idx"][0]]
    assert list(c["q"][0]) == want
    assert c["q"][0][list(c["idx"][0]).index(900)] == 7
    # blocks hold 0.25 magnitudes apart from the outliers, but block 0 also keeps
    # column 9 (0.5, the tie it lost): its scale is the mean over its 127 kept weights
    assert c["s_blk"][0][0] == np.float16((126 * 0.25 + 0.5) / 127)
    assert (c["s_blk"][0][1:] == np.float16(0.25)).all()


def test_block_scale_is_the_least_squares_scale():
    w = _gauss(8, 4096, 4)
    c = E.encode(w)
    wr = E.fwht_staged(w.astype(np.float64))
    out = np.zeros_like(wr, dtype=bool)
    np.put_along_axis(out, c["idx"].astype(np.int64), True, axis=1)
    for r in range(8):
        for b in range(32):
            sl = slice(128 * b, 128 * b + 128)
            keep = ~out[r, sl]
            a = np.abs(wr[r, sl][keep])
            err = lambda s: float(np.sum((a - s) ** 2))   # |w - s sign(w)|^2 = (|w| - s)^2
            s = float(c["s_blk"][r, b])
            up = float(np.nextafter(np.float16(s), np.float16(np.inf)))
            dn = float(np.nextafter(np.float16(s), np.float16(-np.inf)))
            assert err(s) <= err(up) and err(s) <= err(dn)
            assert abs(s - a.mean()) <= abs(up - s) / 2 + 1e-12


def test_outlier_codes_round_to_nearest():
    w = _gauss(16, 2048, 5)
    c = E.encode(w)
    wr = E.fwht_staged(w.astype(np.float64))
    for r in range(16):
        sr = float(c["s_row"][r])
        v = wr[r, c["idx"][r].astype(np.int64)]
        err = np.abs(v - c["q"][r] * sr)
        assert (err <= sr / 2 * (1 + 1e-9) + 1e-300).all() or (np.abs(c["q"][r]) == 7).any()
        assert np.abs(c["q"][r]).max() == 7                      # the row's largest maps to +-7


def test_sign_rounding_error_closed_form():
    # LS-scaled sign rounding of iid Gaussian weights: relative error sqrt(1 - 2/pi)
    w = _gauss(64, 4096, 6)
    wr = E.fwht_staged(w.astype(np.float64))
    c0 = E.encode(w, frac=0.0)
    rel0 = np.linalg.norm(O.dequant(c0) - wr) / np.linalg.norm(wr)
    assert rel0 == pytest.approx(math.sqrt(1 - 2 / math.pi), rel=0.01)
    c1 = E.encode(w)                          # 1 % outliers lower it
    rel1 = np.linalg.norm(O.dequant(c1) - wr) / np.linalg.norm(wr)
    assert rel1 < rel0 - 0.01
