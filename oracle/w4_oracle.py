"""Plain CPU oracle for the 4-bit non-expert weight format (W4, g128).

TEST INFRASTRUCTURE ONLY.  Only the test-suite, the package's smoke check and
the CPU-baseline leg of the benchmark may import this module.  The product
path never calls it and shares no code with it.

What the pages fix:

* DeepSeek-V4-Pro-671B-GALE-1bit-v4 card, paragraph under the weights table:
  the 4-bit non-expert weights are symmetric int4 per 128-block with fp16
  scales (0.119 relative error on that model's weights; a Hadamard rotation
  was measured there and not kept, so this format is not rotated).
* DeepSeek-V4-Flash card, "What is in the pack", non-expert row: attention,
  shared experts and the head are kept 4-bit in VRAM (quantized at load).

Readings of what the pages leave open (each used below):

* "symmetric int4": codes q in [-7, 7] (the -8 code is never produced) and a
  scale s = amax / 7 per (row, 128-column block) of the [rows, cols] matrix;
  the block is the 128 consecutive weights of a row, as for the GALE block
  scales.
* Precision of the decisions (a quantised code is decided in floating point,
  so both sides decide in the same precision): amax and amax / 7 in fp32,
  the scale rounded to fp16 (round to nearest even), q = rint(w / s) with
  the fp32 value of that fp16 scale (IEEE fp32 division, ties to even),
  clamped to [-7, 7].  A block whose amax is 0 has s = 0 and q = 0.
* Storage: q as 4-bit two's complement, two per byte, the low nibble holding
  the even column, rows contiguous ([rows][cols / 2] bytes); then the fp16
  scales [rows][cols / 128]; each section starts on a 256-byte boundary.
* The product: y[t, r] = sum_c s[r, c // 128] q[r, c] x[t, c] with bf16
  activations x, evaluated here in fp64.
"""
from __future__ import annotations

import numpy as np

W4_BLOCK = 128
W4_QMAX = 7
W4_ALIGN = 256


def _align(n: int, a: int = W4_ALIGN) -> int:
    return (n + a - 1) // a * a


def w4_layout(rows: int, cols: int) -> dict:
    """Byte offsets and sizes of the two sections of one packed matrix."""
    if cols % W4_BLOCK:
        raise ValueError("cols must be a multiple of 128")
    q_bytes = rows * cols // 2
    s_off = _align(q_bytes)
    s_bytes = rows * (cols // W4_BLOCK) * 2
    return {"rows": rows, "cols": cols, "q_off": 0, "q_bytes": q_bytes, "s_off": s_off,
            "s_bytes": s_bytes, "total": _align(s_off + s_bytes)}


def w4_quantize(w: np.ndarray):
    """(q int8 [rows, cols], s float16 [rows, cols // 128]) of an fp32 matrix."""
    w = np.asarray(w, dtype=np.float32)
    rows, cols = w.shape
    nb = cols // W4_BLOCK
    q = np.zeros((rows, cols), dtype=np.int8)
    s = np.zeros((rows, nb), dtype=np.float16)
    for r in range(rows):
        for b in range(nb):
            blk = w[r, b * W4_BLOCK:(b + 1) * W4_BLOCK]
            amax = np.float32(np.max(np.abs(blk)))
            sh = np.float16(np.float32(amax) / np.float32(W4_QMAX))
            s[r, b] = sh
            sf = np.float32(sh)
            if sf > 0:
                qq = np.rint(blk / sf)
                q[r, b * W4_BLOCK:(b + 1) * W4_BLOCK] = np.clip(qq, -W4_QMAX, W4_QMAX).astype(np.int8)
    return q, s


def w4_pack(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    """Bytes of one packed matrix (uint8 array of w4_layout(...)['total'])."""
    rows, cols = q.shape
    L = w4_layout(rows, cols)
    out = np.zeros(L["total"], dtype=np.uint8)
    nib = (q.astype(np.int16) & 0xF).astype(np.uint8)
    out[:L["q_bytes"]] = (nib[:, 0::2] | (nib[:, 1::2] << 4)).reshape(-1)
    out[L["s_off"]:L["s_off"] + L["s_bytes"]] = np.ascontiguousarray(s, dtype=np.float16).view(np.uint8).reshape(-1)
    return out


def w4_unpack(buf: np.ndarray, rows: int, cols: int):
    """(q, s) back from the bytes of one packed matrix."""
    L = w4_layout(rows, cols)
    b = np.asarray(buf, dtype=np.uint8)
    pb = b[:L["q_bytes"]].reshape(rows, cols // 2)
    q = np.zeros((rows, cols), dtype=np.int8)
    for half, shift in ((0, 0), (1, 4)):
        n = ((pb >> shift) & 0xF).astype(np.int16)
        q[:, half::2] = np.where(n >= 8, n - 16, n).astype(np.int8)
    s = b[L["s_off"]:L["s_off"] + L["s_bytes"]].view(np.float16).reshape(rows, cols // W4_BLOCK).copy()
    return q, s


def w4_dequant(q: np.ndarray, s: np.ndarray) -> np.ndarray:
    """Dense fp64 weights s[r, c // 128] * q[r, c]."""
    return q.astype(np.float64) * np.repeat(s.astype(np.float64), W4_BLOCK, axis=1)


def w4_gemv(q: np.ndarray, s: np.ndarray, x: np.ndarray) -> np.ndarray:
    """y [B, rows] = x [B, cols] @ dequant(q, s).T in fp64 (a library matmul)."""
    return np.asarray(x, dtype=np.float64) @ w4_dequant(q, s).T
