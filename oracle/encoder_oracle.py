"""Plain CPU oracle of a GALE 1-bit encoder (dense matrix -> packed record).

TEST INFRASTRUCTURE ONLY.  Only the test-suite, the package's smoke check and
the CPU-baseline leg of the benchmark may import this module.  The product
path never calls it and shares no code with it.

What the pages fix (DeepSeek-V4-Pro-671B-GALE-1bit-v4 card, weights table and
the paragraph under it; DeepSeek-V4-Flash card, "What is in the pack"):
one sign bit per weight under a blocked FWHT-1024 rotation of the input
dimension, one fp16 scale per 128-weight block, 1 % of each row's weights as
int4 outliers with one fp16 scale per row that replace the signed weight; the
v3 pack rounded each weight to its sign (the v4 sign choice needs real
activations and is not this function).

The steps, in the pages' order: rotate, then sign, block scale and outliers.
Readings of what the pages leave open (each taken below):

* Rotation: W_rot = W H with H the normalised blocked Hadamard matrix (the
  inference path multiplies the rotated activation H x, and H H = I), i.e. a
  blocked FWHT-1024 of every row, here in fp64 with the butterfly stages taken
  for h = 1, 2, 4, ..., 512 (a + b to the lower, a - b to the upper element)
  and the 1/32 applied at the end.  Both sides decide signs, outliers and
  codes from these fp64 values computed in this order.
* Sign: bit 1 (weight -1) where W_rot < 0, bit 0 elsewhere (0 included),
  for every column, outlier columns too (the format stores and ignores them).
* Outliers: the k = round(cols / 100) columns of largest |W_rot| in the row,
  the lower column first on equal magnitudes, stored in ascending order.
* Outlier values: symmetric int4, s_row = fp16(max |W_rot| of the row / 7)
  (fp64 division, round to nearest even), q = clamp(rint(W_rot / s_row),
  -7, 7) in fp64; q = 0 when s_row is 0.
* Block scale: the least-squares scale of sign(w) for the block's weights
  that are not outliers, which is their mean |W_rot|: the sum taken in fp64
  in column order, divided by their count, rounded to fp16; 0 when a block
  holds outliers only.
"""
from __future__ import annotations

import numpy as np

from . import gale_oracle as O


def fwht_staged(x: np.ndarray, block: int = O.FWHT_N) -> np.ndarray:
    """Normalised blocked FWHT along the last axis in fp64, stages h = 1..block/2."""
    v = np.array(x, dtype=np.float64, copy=True)
    n = v.shape[-1]
    if n % block:
        raise ValueError("length must be a multiple of the block")
    lead = v.shape[:-1]
    v = v.reshape(*lead, n // block, block)
    h = 1
    while h < block:
        w = v.reshape(*lead, n // block, block // (2 * h), 2, h)
        a = w[..., 0, :].copy()
        b = w[..., 1, :].copy()
        w[..., 0, :] = a + b
        w[..., 1, :] = a - b
        v = w.reshape(*lead, n // block, block)
        h *= 2
    return (v * (1.0 / 32.0 if block == 1024 else 1.0 / np.sqrt(block))).reshape(*lead, n)


def encode(w: np.ndarray, frac: float = 0.01) -> dict:
    """Canonical unpacked matrix (signs, s_blk, s_row, idx, q) of a dense
    [rows, cols] matrix, ready for ``gale_oracle.pack``."""
    w = np.asarray(w, dtype=np.float32)
    rows, cols = w.shape
    k = O.outliers_per_row(cols, frac)
    wr = fwht_staged(w.astype(np.float64))
    a = np.abs(wr)
    signs = (wr < 0).astype(np.uint8)
    col = np.arange(cols)
    idx = np.zeros((rows, k), dtype=np.int64)
    q = np.zeros((rows, k), dtype=np.int8)
    s_row = np.zeros(rows, dtype=np.float16)
    out_mask = np.zeros((rows, cols), dtype=bool)
    for r in range(rows):
        order = np.lexsort((col, -a[r]))        # |w| descending, then column ascending
        pick = np.sort(order[:k])
        idx[r] = pick
        out_mask[r, pick] = True
        amax = a[r, order[0]] if k else 0.0
        sr = np.float16(amax / 7.0)
        s_row[r] = sr
        if k and float(sr) > 0.0:
            q[r] = np.clip(np.rint(wr[r, pick] / np.float64(sr)), -7, 7).astype(np.int8)
    nb = cols // O.BLOCK
    am = np.where(out_mask, 0.0, a).reshape(rows, nb, O.BLOCK)
    sums = np.cumsum(am, axis=2)[:, :, -1]      # sequential, in column order
    cnt = O.BLOCK - out_mask.reshape(rows, nb, O.BLOCK).sum(axis=2)
    mean = np.where(cnt > 0, sums / np.maximum(cnt, 1), 0.0)
    s_blk = mean.astype(np.float16)
    return {"rows": rows, "cols": cols, "signs": signs, "s_blk": s_blk, "s_row": s_row,
            "idx": idx.astype(np.uint16), "q": q}
