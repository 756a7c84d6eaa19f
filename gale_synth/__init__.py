"""Seeded synthetic inputs for the GALE 1-bit expert path.

This module is shared by the CUDA-side tests/benchmark and by the CPU oracle.
It holds random-number generation only: no packing, no dequantisation, no
Hadamard transform and no expert arithmetic.  Everything it returns is a
*canonical, unpacked* description of an expert matrix (one sign per weight,
scales, outlier positions and values) or an activation/routing input.

Generator definition (counter based, so any element can be drawn on its own):

* ``mix64`` is the SplitMix64 output function of Steele, Lea and Flood,
  "Fast splittable pseudorandom number generators" (OOPSLA 2014).
* A *stream key* is derived from a tuple of integer fields by
  ``k <- mix64((k ^ f) + GOLDEN)`` for each field ``f``, starting from the seed.
* Element ``i`` of a stream is ``mix64(key + (i + 1) * GOLDEN) mod 2**64``, i.e. the
  ``i``-th output of a SplitMix64 generator whose state starts at ``key``.
* A uniform double in (0, 1) is ``((u >> 11) + 0.5) * 2**-53``.
* A standard normal is Box-Muller's cosine branch on elements ``2i`` and ``2i+1``.
* A bounded integer in ``[0, n)`` is ``((u >> 32) * n) >> 32``.

Shapes and distributions follow the synthetic workloads of the GALE 1-bit
expert pack (DeepSeek-V4-Flash -- GALE 1-bit experts, "What is in the pack"):
signs i.i.d. Bernoulli(0.5); block scales fp16 lognormal(-4, 0.3) per 128
weights; 1 % of columns per row as outliers (uniform, distinct) with int4
values uniform in [-8, 7] and a per-row fp16 scale lognormal(-3, 0.3).
"""
from __future__ import annotations

import numpy as np

SEED = 0x6A1E
GOLDEN = 0x9E3779B97F4A7C15
_M64 = (1 << 64) - 1

# stream-kind tags (first field after the seed)
KIND_MATRIX = 1
KIND_ACT = 2
KIND_LOGITS = 3
KIND_BIAS = 4
KIND_X_F32 = 5

# matrix ids inside an expert record and section ids inside a matrix
W1, W3, W2 = 0, 1, 2
SEC_SIGNS, SEC_SBLK, SEC_SROW, SEC_IDX, SEC_Q = 0, 1, 2, 3, 4

BLK_MU, BLK_SIGMA = -4.0, 0.3
ROW_MU, ROW_SIGMA = -3.0, 0.3


def _mix64_int(z: int) -> int:
    z &= _M64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _M64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _M64
    return z ^ (z >> 31)


def mix64(z: np.ndarray) -> np.ndarray:
    """SplitMix64 output function on a uint64 array (wrapping arithmetic)."""
    z = np.asarray(z, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
    return z ^ (z >> np.uint64(31))


def stream_key(*fields: int, seed: int = SEED) -> int:
    k = seed & _M64
    for f in fields:
        k = _mix64_int(((k ^ (int(f) & _M64)) + GOLDEN) & _M64)
    return k


def u64(key: int, idx) -> np.ndarray:
    """Elements ``idx`` (uint64 array) of the stream ``key``."""
    idx = np.asarray(idx, dtype=np.uint64)
    with np.errstate(over="ignore"):
        state = np.uint64(key) + (idx + np.uint64(1)) * np.uint64(GOLDEN)
    return mix64(state)


def uniform(key: int, idx) -> np.ndarray:
    u = u64(key, idx)
    return ((u >> np.uint64(11)).astype(np.float64) + 0.5) * (2.0 ** -53)


def normal(key: int, n: int, start: int = 0) -> np.ndarray:
    """``n`` standard normals: element i uses stream elements 2i and 2i+1."""
    i = np.arange(start, start + n, dtype=np.uint64)
    u1 = uniform(key, 2 * i)
    u2 = uniform(key, 2 * i + np.uint64(1))
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)


def bounded(u: np.ndarray, n) -> np.ndarray:
    """Map uint64 draws to integers in [0, n) by a 32x32 multiply-high."""
    hi = (u >> np.uint64(32)).astype(np.uint64)
    return ((hi * np.asarray(n, dtype=np.uint64)) >> np.uint64(32)).astype(np.int64)


def outlier_count(cols: int, frac: float = 0.01) -> int:
    """Outliers per row: the nearest integer to ``frac * cols``."""
    return int(np.floor(frac * cols + 0.5))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (round to nearest, ties to even); returns uint16 bits."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rnd = ((b >> np.uint64(16)) & np.uint64(1)) + np.uint64(0x7FFF)
    return ((b + rnd) >> np.uint64(16)).astype(np.uint16)


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    return (np.asarray(h, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# ----------------------------------------------------------------------------
# expert matrices
# ----------------------------------------------------------------------------

def matrix_canonical(rows: int, cols: int, layer: int = 0, expert: int = 0,
                     matrix: int = W1, frac: float = 0.01, seed: int = SEED) -> dict:
    """One expert matrix in canonical unpacked form.

    Returns ``signs`` uint8 [rows, cols] (1 means the weight is negative),
    ``s_blk`` fp16 [rows, cols/128], ``s_row`` fp16 [rows],
    ``idx`` uint16 [rows, k] (strictly ascending per row) and
    ``q`` int8 [rows, k] in [-8, 7].
    """
    assert cols % 128 == 0 and cols % 64 == 0
    base = (KIND_MATRIX, layer, expert, matrix)
    # signs: bit (c % 64) of draw r*(cols/64) + c/64
    kw = stream_key(*base, SEC_SIGNS, seed=seed)
    words = u64(kw, np.arange(rows * (cols // 64), dtype=np.uint64))
    signs = np.unpackbits(words.astype("<u8").view(np.uint8), bitorder="little")
    signs = signs.reshape(rows, cols)
    # block scales: fp16(exp(mu + sigma z))
    nb = cols // 128
    z = normal(stream_key(*base, SEC_SBLK, seed=seed), rows * nb)
    s_blk = np.exp(BLK_MU + BLK_SIGMA * z).astype(np.float16).reshape(rows, nb)
    z = normal(stream_key(*base, SEC_SROW, seed=seed), rows)
    s_row = np.exp(ROW_MU + ROW_SIGMA * z).astype(np.float16)
    # outlier columns: Floyd's sampling of k distinct columns per row
    k = outlier_count(cols, frac)
    ki = stream_key(*base, SEC_IDX, seed=seed)
    sel = np.zeros((rows, k), dtype=np.int64)
    r_ids = np.arange(rows, dtype=np.uint64)
    for step in range(k):
        j = cols - k + step
        t = bounded(u64(ki, r_ids * np.uint64(k) + np.uint64(step)), j + 1)
        if step:
            dup = (sel[:, :step] == t[:, None]).any(axis=1)
            t = np.where(dup, j, t)
        sel[:, step] = t
    idx = np.sort(sel, axis=1).astype(np.uint16)
    # int4 values: top 4 bits of a draw, shifted to [-8, 7]
    kq = stream_key(*base, SEC_Q, seed=seed)
    n = np.arange(rows * k, dtype=np.uint64)
    q = ((u64(kq, n) >> np.uint64(60)).astype(np.int64) - 8).astype(np.int8).reshape(rows, k)
    return {"rows": rows, "cols": cols, "signs": signs, "s_blk": s_blk,
            "s_row": s_row, "idx": idx, "q": q}


def expert_canonical(d_model: int, d_ff: int, layer: int = 0, expert: int = 0,
                     frac: float = 0.01, seed: int = SEED) -> list:
    """[w1, w3, w2] of one SwiGLU expert: w1, w3 are [d_ff, d_model], w2 is [d_model, d_ff]."""
    return [matrix_canonical(d_ff, d_model, layer, expert, W1, frac, seed),
            matrix_canonical(d_ff, d_model, layer, expert, W3, frac, seed),
            matrix_canonical(d_model, d_ff, layer, expert, W2, frac, seed)]


# ----------------------------------------------------------------------------
# activations and routing
# ----------------------------------------------------------------------------

def x_f32(n: int, tag: int = 0, seed: int = SEED) -> np.ndarray:
    """fp32 N(0, 1) vector (the single-expert workload's input)."""
    return normal(stream_key(KIND_X_F32, tag, seed=seed), n).astype(np.float32)


def hidden_bf16(tokens: int, d_model: int, tag: int = 0, seed: int = SEED):
    """bf16 N(0,1) hidden states [tokens, d_model]: (uint16 bits, fp32 values)."""
    z = normal(stream_key(KIND_ACT, tag, seed=seed), tokens * d_model)
    bits = f32_to_bf16_bits(z.astype(np.float32)).reshape(tokens, d_model)
    return bits, bf16_bits_to_f32(bits)


def router_logits(tokens: int, n_experts: int, tag: int = 0, bias_sigma: float = 0.0,
                  seed: int = SEED) -> np.ndarray:
    """fp32 router logits N(0,1) [tokens, n_experts], plus an optional per-expert
    popularity bias N(0, bias_sigma) shared by all tokens (skewed routing)."""
    z = normal(stream_key(KIND_LOGITS, tag, seed=seed), tokens * n_experts)
    lg = z.reshape(tokens, n_experts)
    if bias_sigma > 0.0:
        lg = lg + bias_sigma * normal(stream_key(KIND_BIAS, tag, seed=seed), n_experts)[None, :]
    return lg.astype(np.float32)


def route_topk(logits: np.ndarray, k: int):
    """Top-k experts per token (descending logit, lower index first on ties) and
    their gates, softmax-normalised over the selected k (fp64, rounded to fp32)."""
    lg = np.asarray(logits, dtype=np.float32)
    order = np.argsort(-lg.astype(np.float64), axis=1, kind="stable")[:, :k]
    sel = np.take_along_axis(lg, order, axis=1).astype(np.float64)
    e = np.exp(sel - sel.max(axis=1, keepdims=True))
    gates = (e / e.sum(axis=1, keepdims=True)).astype(np.float32)
    return order.astype(np.int32), gates


# ----------------------------------------------------------------------------
# the same matrix generator on a torch device (for large resident workloads)
# ----------------------------------------------------------------------------

def _t_mix64(z):
    """SplitMix64 output function on an int64 torch tensor holding uint64 bit
    patterns (wrapping multiply; logical right shifts by masking)."""
    import torch
    m30 = (1 << 34) - 1
    m27 = (1 << 37) - 1
    m31 = (1 << 33) - 1
    c1 = 0xBF58476D1CE4E5B9 - (1 << 64)
    c2 = 0x94D049BB133111EB - (1 << 64)
    z = (z ^ ((z >> 30) & m30)) * c1
    z = (z ^ ((z >> 27) & m27)) * c2
    return z ^ ((z >> 31) & m31)


def _t_u64(keys, idx):
    """Elements idx (int64 tensor, broadcast against keys) of the streams keys."""
    g = GOLDEN - (1 << 64)
    return _t_mix64(keys + (idx + 1) * g)


def _t_uniform(keys, idx):
    import torch
    u = _t_u64(keys, idx)
    hi = (u >> 11) & ((1 << 53) - 1)
    return (hi.to(torch.float64) + 0.5) * (2.0 ** -53)


def _t_normal(keys, n):
    import torch
    i = torch.arange(n, dtype=torch.int64, device=keys.device)
    u1 = _t_uniform(keys, 2 * i)
    u2 = _t_uniform(keys, 2 * i + 1)
    return torch.sqrt(-2.0 * torch.log(u1)) * torch.cos(2.0 * torch.pi * u2)


def normal_torch(key: int, n: int, device="cuda", start: int = 0):
    """Elements start .. start + n of the N(0, 1) stream `key` as an fp64
    tensor on a torch device (Box-Muller of the same SplitMix64 draws as
    ``normal``; the device's fp64 log and cos may round a last bit apart)."""
    import torch
    k = torch.tensor([key - (1 << 64) if key >= (1 << 63) else key], dtype=torch.int64, device=device)
    i = torch.arange(start, start + n, dtype=torch.int64, device=device)
    u1 = _t_uniform(k, 2 * i)
    u2 = _t_uniform(k, 2 * i + 1)
    return torch.sqrt(-2.0 * torch.log(u1)) * torch.cos(2.0 * torch.pi * u2)


def _t_keys(fields_list, device):
    import torch
    ks = [stream_key(*f) for f in fields_list]
    return torch.tensor([k - (1 << 64) if k >= (1 << 63) else k for k in ks], dtype=torch.int64, device=device)


def matrices_canonical_torch(rows: int, cols: int, layer: int, experts, matrix: int, device="cuda",
                             frac: float = 0.01) -> dict:
    """``matrix_canonical`` for several experts at once on a torch device.

    Integer draws (signs, outlier columns, outlier values) are bit-identical to
    the numpy version; the scales go through the device's fp64 log, cos and
    exp, which may round a rare value to a neighbouring fp16.  Tensors carry a
    leading expert dimension.
    """
    import torch
    E = len(experts)
    base = [(KIND_MATRIX, layer, e, matrix) for e in experts]
    col = lambda t: t.view(E, 1)
    # signs: bit (c % 64) of draw r*(cols/64) + c/64
    kw = col(_t_keys([b + (SEC_SIGNS,) for b in base], device))
    nw = rows * (cols // 64)
    words = _t_u64(kw, torch.arange(nw, dtype=torch.int64, device=device).view(1, nw))
    bits = torch.arange(64, dtype=torch.int64, device=device)
    signs = ((words.view(E, nw, 1) >> bits) & 1).to(torch.uint8).view(E, rows, cols)
    nb = cols // 128
    z = _t_normal(col(_t_keys([b + (SEC_SBLK,) for b in base], device)), rows * nb)
    s_blk = torch.exp(BLK_MU + BLK_SIGMA * z).to(torch.float16).view(E, rows, nb)
    z = _t_normal(col(_t_keys([b + (SEC_SROW,) for b in base], device)), rows)
    s_row = torch.exp(ROW_MU + ROW_SIGMA * z).to(torch.float16).view(E, rows)
    k = outlier_count(cols, frac)
    ki = col(_t_keys([b + (SEC_IDX,) for b in base], device)).view(E, 1, 1)
    r_ids = torch.arange(rows, dtype=torch.int64, device=device).view(1, rows, 1)
    sel = torch.zeros((E, rows, k), dtype=torch.int64, device=device)
    for step in range(k):
        j = cols - k + step
        u = _t_u64(ki, r_ids * k + step).view(E, rows)
        t = (((u >> 32) & 0xFFFFFFFF) * (j + 1)) >> 32
        if step:
            dup = (sel[:, :, :step] == t.unsqueeze(-1)).any(dim=-1)
            t = torch.where(dup, torch.full_like(t, j), t)
        sel[:, :, step] = t
    idx = torch.sort(sel, dim=-1).values.to(torch.int32).to(torch.int16)
    kq = col(_t_keys([b + (SEC_Q,) for b in base], device))
    n = torch.arange(rows * k, dtype=torch.int64, device=device).view(1, rows * k)
    q = (((_t_u64(kq, n) >> 60) & 0xF) - 8).to(torch.int8).view(E, rows, k)
    return {"rows": rows, "cols": cols, "signs": signs, "s_blk": s_blk, "s_row": s_row, "idx": idx, "q": q}
