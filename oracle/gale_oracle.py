"""Plain fp64 CPU oracle for the GALE 1-bit routed-expert forward.

TEST INFRASTRUCTURE ONLY.  Only the test-suite, the package's smoke check and
the CPU-baseline leg of the benchmark may import this module.  The product
path (the CUDA library and its Python binding) never calls it and shares no
code with it.

Everything here is written from the definition of the format and of the
expert function, in fp64, with no blocking, fusion or reordering:

* Format (DeepSeek-V4-Flash -- GALE 1-bit experts, "What is in the pack",
  routed-experts row; repeated on the DeepSeek-V4-Pro-671B-GALE-1bit-v4 card,
  weights table): one sign bit per weight in the domain rotated by a blocked
  FWHT-1024 along the input dimension, one fp16 scale per 128-weight block
  along the row, 1 % outliers per row as int4 values with a per-row fp16
  scale.  The outlier value replaces the signed weight at its column.
* Shapes (same table): routed experts w1/w3 [2048, 4096] and w2 [4096, 2048].
* Expert: SwiGLU, ``w2 @ (silu(w1 x) * (w3 x))``; at inference the rotation
  is applied to the activation instead of the weight, ``W x = W_rot (H x)``.
* Layer: ``y[t] = sum_k g[t,k] * expert_{ids[t,k]}(x[t])``.

Readings of points the pages leave open (sign polarity, bit order, section
order, nibble order, Hadamard ordering, outlier count per row, chain norm
placement) are stated next to the code that takes them.

Parity pins: every function here is pinned by ``tests/test_oracle_pins.py``.
The only quantity with no pin is the real-weight quality figure
(expert_out_rel of 0.357 in the "Accuracy" section), which needs trained
weights and calibration data: parity unpinned for that number, and this
oracle does not try to reproduce it.
"""
from __future__ import annotations

import math

import numpy as np
import scipy.linalg

SECTION_ALIGN = 256          # every section starts on a 256-byte boundary
BLOCK = 128                  # weights per fp16 block scale
FWHT_N = 1024                # rotation block length


# ----------------------------------------------------------------------------
# layout (sizes and offsets of the five sections of one packed matrix)
# ----------------------------------------------------------------------------

def _align(n: int, a: int = SECTION_ALIGN) -> int:
    return (n + a - 1) // a * a


def outliers_per_row(cols: int, frac: float = 0.01) -> int:
    """k = the nearest integer to frac * cols (41 for 4096 columns, 20 for 2048).

    Reading: the pages give only "1 % outliers"; the nearest integer is the
    count that reproduces the printed 1.329 bits/weight and 46.0 GB.
    """
    return int(math.floor(frac * cols + 0.5))


def layout(rows: int, cols: int, frac: float = 0.01) -> dict:
    """Byte layout of one packed matrix: signs, s_blk, s_row, idx, q.

    signs : rows*cols/8 bytes, uint32 words, row-major, column c of row r is
            bit (c % 32) of word r*(cols/32) + c/32; a set bit means -1.
    s_blk : fp16 [rows, cols/128] row-major.
    s_row : fp16 [rows].
    idx   : uint16 [rows, k] row-major, strictly ascending within a row.
    q     : int4 two's complement, value j of row r is nibble n = r*k + j,
            stored in byte n // 2, low nibble first.
    """
    k = outliers_per_row(cols, frac)
    sizes = [rows * cols // 8, rows * (cols // BLOCK) * 2, rows * 2, rows * k * 2,
             (rows * k + 1) // 2]
    offs, o = [], 0
    for s in sizes:
        offs.append(o)
        o = _align(o + s)
    return {"rows": rows, "cols": cols, "k": k, "sizes": sizes, "offsets": offs,
            "total": o}


def expert_bytes(d_model: int, d_ff: int, frac: float = 0.01) -> int:
    """Bytes of one expert record w1 || w3 || w2."""
    return (2 * layout(d_ff, d_model, frac)["total"]
            + layout(d_model, d_ff, frac)["total"])


# ----------------------------------------------------------------------------
# pack / unpack
# ----------------------------------------------------------------------------

def pack(c: dict, frac: float = 0.01) -> np.ndarray:
    """Canonical unpacked matrix -> packed bytes (uint8 array)."""
    rows, cols = c["rows"], c["cols"]
    L = layout(rows, cols, frac)
    k = L["k"]
    idx = np.asarray(c["idx"], dtype=np.int64).reshape(rows, k)
    q = np.asarray(c["q"], dtype=np.int64).reshape(rows, k)
    if k:
        if (np.diff(idx, axis=1) <= 0).any() or idx.min() < 0 or idx.max() >= cols:
            raise ValueError("outlier columns must be strictly ascending and in range")
        if q.min() < -8 or q.max() > 7:
            raise ValueError("int4 outlier value out of range")
    out = np.zeros(L["total"], dtype=np.uint8)
    o = L["offsets"]
    # signs: little-endian bit order inside each byte == LSB-first uint32 words
    sg = np.packbits(np.asarray(c["signs"], dtype=np.uint8).reshape(rows, cols),
                     axis=1, bitorder="little")
    out[o[0]:o[0] + L["sizes"][0]] = sg.reshape(-1)
    out[o[1]:o[1] + L["sizes"][1]] = np.asarray(c["s_blk"], dtype="<f2").reshape(-1).view(np.uint8)
    out[o[2]:o[2] + L["sizes"][2]] = np.asarray(c["s_row"], dtype="<f2").reshape(-1).view(np.uint8)
    out[o[3]:o[3] + L["sizes"][3]] = idx.astype("<u2").reshape(-1).view(np.uint8)
    nib = (q.reshape(-1) & 0xF).astype(np.uint8)
    if nib.size % 2:
        nib = np.concatenate([nib, np.zeros(1, np.uint8)])
    out[o[4]:o[4] + L["sizes"][4]] = nib[0::2] | (nib[1::2] << 4)
    return out


def unpack(buf: np.ndarray, rows: int, cols: int, frac: float = 0.01) -> dict:
    """Packed bytes -> canonical unpacked matrix (inverse of ``pack``)."""
    L = layout(rows, cols, frac)
    k, o, s = L["k"], L["offsets"], L["sizes"]
    b = np.asarray(buf, dtype=np.uint8)
    signs = np.unpackbits(b[o[0]:o[0] + s[0]].reshape(rows, cols // 8), axis=1,
                          bitorder="little")
    s_blk = b[o[1]:o[1] + s[1]].view("<f2").reshape(rows, cols // BLOCK)
    s_row = b[o[2]:o[2] + s[2]].view("<f2").copy()
    idx = b[o[3]:o[3] + s[3]].view("<u2").reshape(rows, k)
    qb = b[o[4]:o[4] + s[4]]
    nib = np.empty(2 * qb.size, dtype=np.int64)
    nib[0::2] = qb & 0xF
    nib[1::2] = qb >> 4
    nib = nib[:rows * k]
    q = np.where(nib >= 8, nib - 16, nib).astype(np.int8).reshape(rows, k)
    return {"rows": rows, "cols": cols, "signs": signs, "s_blk": s_blk.astype(np.float16),
            "s_row": s_row.astype(np.float16), "idx": idx.astype(np.uint16), "q": q}


def dequant(c: dict) -> np.ndarray:
    """Dense fp64 weights Q(W_rot): sign times block scale, outliers replaced.

    Wd[r, c] = (signs[r, c] ? -1 : +1) * s_blk[r, c // 128]
    Wd[r, idx[r, j]] = q[r, j] * s_row[r]        (the outlier replaces the weight)
    """
    rows, cols = c["rows"], c["cols"]
    sgn = 1.0 - 2.0 * np.asarray(c["signs"], dtype=np.float64).reshape(rows, cols)
    sb = np.repeat(np.asarray(c["s_blk"], dtype=np.float64).reshape(rows, -1), BLOCK, axis=1)
    W = sgn * sb
    idx = np.asarray(c["idx"], dtype=np.int64).reshape(rows, -1)
    if idx.shape[1]:
        val = (np.asarray(c["q"], dtype=np.float64).reshape(rows, -1)
               * np.asarray(c["s_row"], dtype=np.float64)[:, None])
        np.put_along_axis(W, idx, val, axis=1)
    return W


def dequant_packed(buf: np.ndarray, rows: int, cols: int, frac: float = 0.01) -> np.ndarray:
    return dequant(unpack(buf, rows, cols, frac))


# ----------------------------------------------------------------------------
# rotation
# ----------------------------------------------------------------------------

def hadamard(n: int) -> np.ndarray:
    """Sylvester Hadamard matrix in natural order, H_2n = [[H, H], [H, -H]].

    Reading: a "butterfly" Walsh-Hadamard transform (the pages' FWHT kernel)
    produces natural (Sylvester) order; it is symmetric and, normalised by
    1/sqrt(n), its own inverse, so the direction of the rotation is moot.
    """
    return scipy.linalg.hadamard(n).astype(np.float64)


def fwht_blocked(x: np.ndarray, block: int = FWHT_N) -> np.ndarray:
    """Blocked, normalised FWHT along the last axis: every run of ``block``
    consecutive elements [block*b, block*b + block) is multiplied by
    H_block / sqrt(block) (1/32 for block 1024)."""
    x = np.asarray(x, dtype=np.float64)
    n = x.shape[-1]
    if n % block:
        raise ValueError("length must be a multiple of the block")
    H = hadamard(block) / math.sqrt(block)
    xb = x.reshape(*x.shape[:-1], n // block, block)
    return (xb @ H.T).reshape(x.shape)


# ----------------------------------------------------------------------------
# expert, layer, chain
# ----------------------------------------------------------------------------

def silu(z: np.ndarray) -> np.ndarray:
    return z / (1.0 + np.exp(-z))


def gemv(Wd: np.ndarray, x_rot: np.ndarray) -> np.ndarray:
    """y[t] = Q(W_rot) x_rot[t] for x_rot of shape [..., cols]."""
    return np.asarray(x_rot, dtype=np.float64) @ Wd.T


def swiglu_hidden(W1d: np.ndarray, W3d: np.ndarray, x_rot: np.ndarray) -> np.ndarray:
    """h = silu(Q(W1) x_rot) * (Q(W3) x_rot)."""
    return silu(gemv(W1d, x_rot)) * gemv(W3d, x_rot)


def expert_forward(dense: list, x: np.ndarray) -> np.ndarray:
    """One SwiGLU expert on un-rotated inputs x [..., d_model].

    dense = [Q(W1_rot), Q(W3_rot), Q(W2_rot)] as fp64 arrays; the rotation of
    each matrix's input dimension is applied to the activation feeding it.
    """
    W1d, W3d, W2d = dense
    h = swiglu_hidden(W1d, W3d, fwht_blocked(x))
    return gemv(W2d, fwht_blocked(h))


def moe_layer(dense_of, x: np.ndarray, ids: np.ndarray, gates: np.ndarray) -> np.ndarray:
    """y[t] = sum_k gates[t,k] * expert_{ids[t,k]}(x[t]) (fp64).

    ``dense_of(e)`` returns the three dense matrices of expert e.
    """
    x = np.asarray(x, dtype=np.float64)
    ids = np.asarray(ids)
    gates = np.asarray(gates, dtype=np.float64)
    y = np.zeros_like(x)
    for e in np.unique(ids):
        tok, slot = np.nonzero(ids == e)
        o = expert_forward(dense_of(int(e)), x[tok])
        y[tok] += gates[tok, slot][:, None] * o
    return y


def rmsnorm(v: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    """RMSNorm with unit weight along the last axis."""
    v = np.asarray(v, dtype=np.float64)
    return v / np.sqrt(np.mean(v * v, axis=-1, keepdims=True) + eps)


def chain_step(dense_of, x_bf16_values: np.ndarray, ids, gates, eps: float = 1e-6):
    """One post-norm layer of the expert-only chain:
    x_{l+1} = RMSNorm(x_l + MoE_l(x_l)), returned in fp64 before the bf16
    rounding that the caller applies to the next layer's input.

    Reading: the chained workload says only "through the expert output plus a
    residual add and RMSNorm"; post-norm with unit weight is the plain reading.
    """
    x = np.asarray(x_bf16_values, dtype=np.float64)
    return rmsnorm(x + moe_layer(dense_of, x, ids, gates), eps)


# ----------------------------------------------------------------------------
# router and routing permute
# ----------------------------------------------------------------------------

def route_topk(logits: np.ndarray, k: int):
    """Top-k routing of every token: the k experts of largest fp32 logit, in
    descending order (a lower expert index first on equal logits), and their
    gates, the softmax over the k selected logits taken in fp64 and rounded
    to fp32.

    Reading: the cards give "top-6 of 256 experts" per token; the benchmark
    configuration normalises the gates over the selected six.  Written as a
    plain sort of (-logit, index) and exp / sum.
    """
    lg = np.asarray(logits, dtype=np.float32)
    B, E = lg.shape
    ids = np.zeros((B, k), dtype=np.int32)
    gates = np.zeros((B, k), dtype=np.float32)
    for t in range(B):
        order = sorted(range(E), key=lambda e: (-float(lg[t, e]), e))[:k]
        sel = [float(lg[t, e]) for e in order]
        m = max(sel)
        ex = [math.exp(v - m) for v in sel]
        tot = sum(ex)
        ids[t] = order
        gates[t] = [v / tot for v in ex]
    return ids, gates



def route_permute(ids: np.ndarray, n_experts: int):
    """Group the (token, slot) pairs by expert, stable in (token, slot) order.

    Returns counts[E], offsets[E+1] and perm[B*K], where perm lists the pair
    indices t*K + k sorted by (expert, t, k).  Written as a plain sort.
    """
    ids = np.asarray(ids, dtype=np.int64)
    B, K = ids.shape
    pairs = sorted(range(B * K), key=lambda p: (ids[p // K, p % K], p))
    counts = np.zeros(n_experts, dtype=np.int64)
    for p in range(B * K):
        counts[ids[p // K, p % K]] += 1
    offsets = np.concatenate([[0], np.cumsum(counts)])
    return counts.astype(np.int32), offsets.astype(np.int32), np.asarray(pairs, dtype=np.int32)
