"""GPU parity: every entry point of libgale against the fp64 oracle.

Bit-exact for packing, dense dequantisation and the routing permute; within
a relative L2 error of 2e-3 (bf16 activations, fp32 accumulation) for the
expert GEMV, the SwiGLU expert and the MoE layer; FWHT within fp32 rounding.
"""
import ctypes

import numpy as np
import pytest

import gale_synth as gs
from oracle import gale_oracle as O

from .helpers import REL_L2_TOL, Layer, assert_tokens, bf16_round, edge_hidden, gpu_pack, rel_l2, to_dev

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
G = pytest.importorskip("bit_expert_gemv_b200")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    G.lib()


def _empty_u8(n):
    return torch.zeros(n, dtype=torch.uint8, device="cuda")


# ----------------------------------------------------------------------------
# pack / unpack
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("rows,cols", [(1, 1024), (37, 2048), (100, 3072), (2048, 4096), (4096, 2048)])
def test_pack_bit_exact(rows, cols):
    c = gs.matrix_canonical(rows, cols, expert=rows + cols)
    want = O.pack(c)
    dst = _empty_u8(G.gale_pack_layout(rows, cols)["total"])
    status = gpu_pack(c, dst)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert np.array_equal(dst.cpu().numpy(), want)


def test_pack_rejects_unsorted_idx():
    c = gs.matrix_canonical(8, 1024, expert=1)
    c["idx"] = c["idx"].copy()
    c["idx"][3, 4] = c["idx"][3, 3]
    dst = _empty_u8(G.gale_pack_layout(8, 1024)["total"])
    status = gpu_pack(c, dst)
    torch.cuda.synchronize()
    assert int(status.item()) == G.GALE_ERR_ARG


@pytest.mark.parametrize("rows,cols", [(3, 1024), (129, 2048), (2048, 4096)])
def test_unpack_bit_exact(rows, cols):
    c = gs.matrix_canonical(rows, cols, expert=5)
    dst = _empty_u8(G.gale_pack_layout(rows, cols)["total"])
    gpu_pack(c, dst)
    dense = torch.empty(rows, cols, dtype=torch.float32, device="cuda")
    G.gale_unpack(dst, rows, cols, dense)
    torch.cuda.synchronize()
    want = O.dequant(c)
    assert np.array_equal(dense.cpu().numpy().astype(np.float64), want)


# ----------------------------------------------------------------------------
# FWHT
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("rows,cols", [(1, 1024), (3, 4096), (37, 2048), (0, 1024)])
def test_fwht_f32(rows, cols):
    x = np.stack([gs.x_f32(cols, tag=100 + r) for r in range(rows)]) if rows else np.zeros((0, cols), np.float32)
    xd = to_dev(x.astype(np.float32))
    y = torch.empty_like(xd)
    G.gale_fwht1024(xd, y)
    torch.cuda.synchronize()
    if rows:
        want = O.fwht_blocked(x.astype(np.float64))
        assert np.max(np.abs(y.cpu().numpy() - want)) < 2e-5 * max(1.0, np.max(np.abs(want)))


def test_fwht_bf16_in_place_involution():
    bits, vals = gs.hidden_bf16(5, 4096, tag=9)
    xd = to_dev(bits, torch.bfloat16)
    y = torch.empty(5, 4096, dtype=torch.float32, device="cuda")
    G.gale_fwht1024(xd, y)
    want = O.fwht_blocked(vals.astype(np.float64))
    z = y.clone()
    G.gale_fwht1024(z, z)      # in place, back to x
    torch.cuda.synchronize()
    assert np.max(np.abs(y.cpu().numpy() - want)) < 2e-5 * np.max(np.abs(want))
    assert np.max(np.abs(z.cpu().numpy() - vals)) < 1e-5


# ----------------------------------------------------------------------------
# expert GEMV
# ----------------------------------------------------------------------------

def _packed_dev(c):
    dst = _empty_u8(G.gale_pack_layout(c["rows"], c["cols"])["total"])
    gpu_pack(c, dst)
    return dst


@pytest.mark.parametrize("rows,cols,ntok", [(2048, 4096, 1), (4096, 2048, 1), (4096, 2048, 2), (100, 1024, 1),
                                             (37, 2048, 2), (300, 4096, 2), (17, 3072, 1), (1, 1024, 1),
                                             (100, 1024, 3), (37, 2048, 8), (300, 4096, 5), (64, 3072, 64),
                                             (17, 1024, 9)])
def test_gemv_plain(rows, cols, ntok):
    c = gs.matrix_canonical(rows, cols, expert=rows, matrix=gs.W2)
    W = _packed_dev(c)
    x = np.stack([gs.x_f32(cols, tag=t) for t in range(ntok)])
    y = torch.empty(ntok, rows, dtype=torch.float32, device="cuda")
    G.gale_expert_gemv(W, rows, cols, to_dev(x), y)
    torch.cuda.synchronize()
    want = O.gemv(O.dequant(c), x.astype(np.float64))
    assert_tokens(y.cpu().numpy(), want, what=f"{rows}x{cols} ntok {ntok}")


@pytest.mark.parametrize("rows,cols,ntok", [(2048, 4096, 1), (2048, 4096, 2), (2048, 4096, 8), (200, 2048, 2),
                                             (33, 1024, 1), (48, 1024, 33)])
def test_gemv_swiglu(rows, cols, ntok):
    c1 = gs.matrix_canonical(rows, cols, expert=7, matrix=gs.W1)
    c3 = gs.matrix_canonical(rows, cols, expert=7, matrix=gs.W3)
    W1, W3 = _packed_dev(c1), _packed_dev(c3)
    x = np.stack([gs.x_f32(cols, tag=50 + t) for t in range(ntok)])
    y = torch.empty(ntok, rows, dtype=torch.float32, device="cuda")
    G.gale_expert_gemv(W1, rows, cols, to_dev(x), y, W3=W3, mode=G.GALE_MODE_SWIGLU)
    torch.cuda.synchronize()
    want = O.swiglu_hidden(O.dequant(c1), O.dequant(c3), x.astype(np.float64))
    assert_tokens(y.cpu().numpy(), want, what=f"{rows}x{cols} ntok {ntok}")


@pytest.mark.parametrize("rows,cols", [(64, 2048), (50, 4096)])
def test_gemv_unit_scale_integer_exact(rows, cols):
    """All-unit-scale pack and integer x: the product is an exact integer sum,
    so the GPU must match the oracle bit for bit (both the int8 tensor-core
    path, whose fixed-point digits hold small integers exactly, and the
    CUDA-core path)."""
    c = gs.matrix_canonical(rows, cols, expert=11)
    c["s_blk"] = np.ones_like(c["s_blk"])
    c["s_row"] = np.ones_like(c["s_row"])
    W = _packed_dev(c)
    for ntok in (1, 2, 4):
        x = np.random.default_rng(3 + ntok).integers(-8, 9, size=(ntok, cols)).astype(np.float32)
        y = torch.empty(ntok, rows, dtype=torch.float32, device="cuda")
        G.gale_expert_gemv(W, rows, cols, to_dev(x), y)
        torch.cuda.synchronize()
        want = O.gemv(O.dequant(c), x.astype(np.float64))
        assert np.array_equal(y.cpu().numpy().astype(np.float64), want), ntok


# ----------------------------------------------------------------------------
# routing permute
# ----------------------------------------------------------------------------

def _route(ids, E, counts, offsets, perm, status, grid):
    """gale_route_permute, or its many-CTA form with a scratch buffer."""
    if grid:
        B, K = ids.shape
        scratch = torch.empty(G.gale_route_permute_scratch_bytes(B, K, E), dtype=torch.uint8, device="cuda")
        G.gale_route_permute_grid(to_dev(ids), E, counts, offsets, perm, status, scratch)
    else:
        G.gale_route_permute(to_dev(ids), E, counts, offsets, perm, status)
    torch.cuda.synchronize()


@pytest.mark.parametrize("grid", [False, True])
@pytest.mark.parametrize("B,K,E,skew", [(1, 6, 256, 0.0), (8, 6, 256, 0.0), (64, 6, 256, 0.5),
                                         (4096, 6, 256, 0.5), (3, 2, 4, 0.0), (200, 16, 1024, 0.0),
                                         (20000, 6, 256, 0.5)])
def test_route_permute_bit_exact(B, K, E, skew, grid):
    ids, _ = gs.route_topk(gs.router_logits(B, E, tag=B, bias_sigma=skew), K)
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.empty(B * K, dtype=torch.int32, device="cuda")
    status = torch.ones(1, dtype=torch.int32, device="cuda")
    _route(ids, E, counts, offsets, perm, status, grid)
    wc, wo, wp = O.route_permute(ids, E)
    assert int(status.item()) == 0
    assert np.array_equal(counts.cpu().numpy(), wc)
    assert np.array_equal(offsets.cpu().numpy(), wo)
    assert np.array_equal(perm.cpu().numpy(), wp)


def test_route_permute_flags_bad_ids():
    ids = np.array([[0, 1, 2], [3, 3, 4], [5, 300, 6]], np.int32)
    E = 256
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.full((9,), -7, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    G.gale_route_permute(to_dev(ids), E, counts, offsets, perm, status)
    torch.cuda.synchronize()
    assert int(status.item()) == G.GALE_ERR_ARG
    assert int(counts.sum().item()) == 7      # the repeated 3 and the id 300 are dropped


@pytest.mark.parametrize("grid", [False, True])
def test_route_permute_drops_repeats_at_walk_boundaries(grid):
    """Repeated ids planted where a token's pairs straddle the boundaries of
    the kernel's walk: B = 4001, K = 6 gives 32 warp ranges of 751 pairs,
    walked 32 pairs a step and eight steps per batch of loads.  Token 125
    straddles warp ranges 0 / 1 (pair 751), token 5 a step boundary (pair 32),
    token 167 the batch boundary of range 1 (pair 751 + 256 = 1007), token 42
    the batch boundary of range 0 (pair 256), which is also the boundary of
    the many-CTA form's first 256-pair range.  The later pair of each repeat
    is dropped; the rest is the stable sort by (expert, pair), checked
    against a plain sort of the valid pairs."""
    B, K, E = 4001, 6, 256
    ids, _ = gs.route_topk(gs.router_logits(B, E, tag=4001, bias_sigma=0.5), K)
    ids = ids.copy()
    ids[125, 1] = ids[125, 0]   # pairs 750 | 751
    ids[5, 3] = ids[5, 0]       # pairs 30 | 33
    ids[167, 5] = ids[167, 1]   # pairs 1003 | 1007
    ids[42, 5] = ids[42, 0]     # pairs 252 | 257
    flat = ids.reshape(-1)
    valid = [p for p in range(B * K) if flat[p] not in flat[p - p % K:p]]
    assert len(valid) == B * K - 4
    want_counts = np.bincount(flat[valid], minlength=E).astype(np.int32)
    want_perm = np.array(sorted(valid, key=lambda p: (flat[p], p)), np.int32)
    counts = torch.empty(E, dtype=torch.int32, device="cuda")
    offsets = torch.empty(E + 1, dtype=torch.int32, device="cuda")
    perm = torch.full((B * K,), -7, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    _route(ids, E, counts, offsets, perm, status, grid)
    assert int(status.item()) == G.GALE_ERR_ARG
    assert np.array_equal(counts.cpu().numpy(), want_counts)
    assert np.array_equal(offsets.cpu().numpy(), np.concatenate([[0], np.cumsum(want_counts)]).astype(np.int32))
    assert np.array_equal(perm.cpu().numpy()[:len(valid)], want_perm)


# ----------------------------------------------------------------------------
# MoE layer
# ----------------------------------------------------------------------------

@pytest.fixture(scope="module")
def small_layer():
    return Layer(16, 2048, 1024, layer=1)


def _moe(layer, bits, ids, gates, out_dtype=None, flags=0, eps=1e-6):
    B, K = ids.shape
    ws = torch.empty(G.gale_moe_workspace_size(layer.desc, B, K), dtype=torch.uint8, device="cuda")
    out = torch.empty(B, layer.d_model, dtype=out_dtype or torch.float32, device="cuda")
    G.gale_moe_forward(layer.desc, to_dev(bits, torch.bfloat16), to_dev(ids), to_dev(gates), out, ws,
                       flags=flags, eps=eps)
    torch.cuda.synchronize()
    return out, int(ws[:4].view(torch.int32).item())


@pytest.mark.parametrize("B,K", [(1, 6), (5, 6), (33, 4), (2, 1), (70, 6), (1, 16), (2, 16), (3, 10)])
def test_moe_small(small_layer, B, K):
    """Decode and prefill paths on a 16-expert layer: batch 1-2 (x rotated
    while the routing runs), one-warp routing up to 32 pairs, block routing
    above, and combines over K = 10 and 16 experts (more than one batch of
    eight expert loads)."""
    L = small_layer
    bits, xv = gs.hidden_bf16(B, L.d_model, tag=B)
    ids, gates = gs.route_topk(gs.router_logits(B, L.E, tag=B), K)
    out, st = _moe(L, bits, ids, gates)
    assert st == 0
    want = O.moe_layer(L.dense, xv, ids, gates)
    assert_tokens(out.cpu().numpy(), want, what=f"B={B} K={K}")


def test_moe_fused_rmsnorm(small_layer):
    L = small_layer
    B = 3
    bits, xv = gs.hidden_bf16(B, L.d_model, tag=77)
    ids, gates = gs.route_topk(gs.router_logits(B, L.E, tag=77), 6)
    out, st = _moe(L, bits, ids, gates, out_dtype=torch.bfloat16, flags=G.GALE_FLAG_RESIDUAL_RMSNORM)
    assert st == 0
    # the output is bf16: compare with the oracle rounded to bf16, per token
    want = bf16_round(O.chain_step(L.dense, xv, ids, gates))
    assert_tokens(out.float().cpu().numpy(), want, what="fused norm")


@pytest.mark.parametrize("B,K", [(1, 6), (2, 16)])
def test_moe_fused_rmsnorm_small_batch(small_layer, B, K):
    """Residual + RMSNorm through the decode kernel at batch 1-2 (the last
    64-row block of a token normalises the row)."""
    L = small_layer
    bits, xv = gs.hidden_bf16(B, L.d_model, tag=88 + B)
    ids, gates = gs.route_topk(gs.router_logits(B, L.E, tag=88 + B), K)
    out, st = _moe(L, bits, ids, gates, out_dtype=torch.bfloat16, flags=G.GALE_FLAG_RESIDUAL_RMSNORM)
    assert st == 0
    want = bf16_round(O.chain_step(L.dense, xv, ids, gates))
    assert_tokens(out.float().cpu().numpy(), want, what=f"fused norm B={B} K={K}")


@pytest.mark.parametrize("kind", ["spikes", "zero", "scaled"])
@pytest.mark.parametrize("B", [1, 2, 5, 40, 200])
def test_moe_edge_inputs(small_layer, kind, B):
    """Hard activations through every path (one or two tokens: the small-batch
    kernel; 5 and 40: the streaming kernel; 200: the tensor-core tiles): three
    features per token at 300x the rms, an all-zero token (its output must be
    exactly zero), and hidden states scaled by 1000 (h reaches ~10^6, past the
    fp16 range unless the paths scale it).  Per-token parity."""
    L = small_layer
    bits, xv = edge_hidden(B, L.d_model, kind, tag=3000 + B)
    ids, gates = gs.route_topk(gs.router_logits(B, L.E, tag=3000 + B), 6)
    out, st = _moe(L, bits, ids, gates)
    assert st == 0
    assert_tokens(out.cpu().numpy(), O.moe_layer(L.dense, xv, ids, gates), what=f"{kind} B={B}")
    outn, st = _moe(L, bits, ids, gates, out_dtype=torch.bfloat16, flags=G.GALE_FLAG_RESIDUAL_RMSNORM)
    assert st == 0
    want = bf16_round(O.chain_step(L.dense, xv, ids, gates))
    assert_tokens(outn.float().cpu().numpy(), want, what=f"{kind} B={B} fused norm")


def test_moe_empty_batch(small_layer):
    """B = 0: nothing to do, status 0."""
    L = small_layer
    bits = np.zeros((0, L.d_model), np.uint16)
    ids = np.zeros((0, 6), np.int32)
    gates = np.zeros((0, 6), np.float32)
    out, st = _moe(L, bits, ids, gates)
    assert st == 0 and out.shape == (0, L.d_model)


@pytest.mark.parametrize("B,K,fused", [(1, 6, False), (2, 16, True), (200, 6, False)])
def test_moe_forward_host_matches_device(small_layer, B, K, fused):
    """Host-buffer entry point: one packed input copy, the result written into
    pinned host memory (or copied back when over 1 MiB, B = 200); bit-identical
    to the device-buffer call."""
    L = small_layer
    bits, _ = gs.hidden_bf16(B, L.d_model, tag=300 + B)
    ids, gates = gs.route_topk(gs.router_logits(B, L.E, tag=300 + B), K)
    flags = G.GALE_FLAG_RESIDUAL_RMSNORM if fused else 0
    dt = torch.bfloat16 if fused else torch.float32
    want, st = _moe(L, bits, ids, gates, out_dtype=dt, flags=flags)
    assert st == 0
    x_h = torch.from_numpy(np.ascontiguousarray(bits)).view(torch.bfloat16)
    ids_h, gates_h = torch.from_numpy(ids), torch.from_numpy(gates)
    staging = torch.empty(G.gale_moe_host_staging_bytes(B, K, L.d_model), dtype=torch.uint8).pin_memory()
    ws = torch.empty(G.gale_moe_host_workspace_size(L.desc, B, K), dtype=torch.uint8, device="cuda")
    out_h = torch.empty(B, L.d_model, dtype=dt).pin_memory()
    G.gale_moe_forward_host(L.desc, x_h, ids_h, gates_h, out_h, ws, staging, flags=flags)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0
    assert torch.equal(out_h, want.cpu())


def test_moe_forward_host_rejects_pageable_output(small_layer):
    L = small_layer
    bits, _ = gs.hidden_bf16(1, L.d_model, tag=5)
    ids, gates = gs.route_topk(gs.router_logits(1, L.E, tag=5), 6)
    staging = torch.empty(G.gale_moe_host_staging_bytes(1, 6, L.d_model), dtype=torch.uint8).pin_memory()
    ws = torch.empty(G.gale_moe_host_workspace_size(L.desc, 1, 6), dtype=torch.uint8, device="cuda")
    out_pageable = torch.empty(1, L.d_model, dtype=torch.float32)
    with pytest.raises(G.GaleError):
        G.gale_moe_forward_host(L.desc, torch.from_numpy(np.ascontiguousarray(bits)).view(torch.bfloat16),
                                torch.from_numpy(ids), torch.from_numpy(gates), out_pageable, ws, staging)


def test_moe_general_path_wide_ff():
    """d_ff = 16384: more outliers per w2 row (164) than the tile path stages
    and wider than the decode kernel takes, so the layer runs on the general
    kernels (routing permute, FWHT, grouped GEMVs, combine)."""
    L = Layer(2, 1024, 16384, layer=2)
    for B, K in [(1, 2), (3, 1)]:
        bits, xv = gs.hidden_bf16(B, L.d_model, tag=500 + B)
        ids, gates = gs.route_topk(gs.router_logits(B, L.E, tag=500 + B), K)
        out, st = _moe(L, bits, ids, gates)
        assert st == 0
        assert_tokens(out.cpu().numpy(), O.moe_layer(L.dense, xv, ids, gates), what=f"B={B} K={K}")


def test_moe_bad_ids_status(small_layer):
    L = small_layer
    bits, _ = gs.hidden_bf16(2, L.d_model, tag=5)
    ids = np.array([[0, 1, 2, 3, 4, 99], [1, 1, 2, 3, 4, 5]], np.int32)
    gates = np.full((2, 6), 1.0 / 6, np.float32)
    _, st = _moe(L, bits, ids, gates)
    assert st == G.GALE_ERR_ARG


@pytest.fixture(scope="module")
def full_layer():
    """256 experts of w1/w3 [2048 x 4096], w2 [4096 x 2048] (about 1.07 GB packed)."""
    return Layer(256, 4096, 2048, layer=0)


@pytest.mark.parametrize("B,skew", [(1, 0.0), (8, 0.0), (64, 0.5)])
def test_moe_full_size(full_layer, B, skew):
    L = full_layer
    bits, xv = gs.hidden_bf16(B, L.d_model, tag=1000 + B)
    ids, gates = gs.route_topk(gs.router_logits(B, L.E, tag=1000 + B, bias_sigma=skew), 6)
    out, st = _moe(L, bits, ids, gates)
    assert st == 0
    assert_tokens(out.cpu().numpy(), O.moe_layer(L.dense, xv, ids, gates), what=f"B={B}")


# ----------------------------------------------------------------------------
# MoE layer, tensor-core (prefill) path: batches past the decode limit
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("B,K,skew", [(70, 6, 0.0), (200, 6, 0.0), (1000, 6, 0.0), (500, 1, 0.0),
                                      (300, 4, 2.0)])
def test_moe_prefill_small(small_layer, B, K, skew):
    """Several 128-row tiles (w2: several pairs of them) and K-steps per
    matrix; experts with more than 128 tokens split into chunks of 128 with a
    ragged last chunk (B = 1000: ~375 tokens per expert, and the skewed
    routing)."""
    L = small_layer
    bits, xv = gs.hidden_bf16(B, L.d_model, tag=2000 + B)
    ids, gates = gs.route_topk(gs.router_logits(B, L.E, tag=2000 + B, bias_sigma=skew), K)
    out, st = _moe(L, bits, ids, gates)
    assert st == 0
    got = out.cpu().numpy()
    toks = np.arange(B) if B <= 300 else np.arange(0, B, 7)
    assert_tokens(got[toks], O.moe_layer(L.dense, xv[toks], ids[toks], gates[toks]), what=f"B={B} K={K}")
    # every token, not only the sampled ones, is finite and nonzero
    assert np.isfinite(got).all() and (np.abs(got).sum(axis=1) > 0).all()


def test_moe_prefill_fused_rmsnorm(small_layer):
    L = small_layer
    B = 150
    bits, xv = gs.hidden_bf16(B, L.d_model, tag=78)
    ids, gates = gs.route_topk(gs.router_logits(B, L.E, tag=78), 6)
    out, st = _moe(L, bits, ids, gates, out_dtype=torch.bfloat16, flags=G.GALE_FLAG_RESIDUAL_RMSNORM)
    assert st == 0
    want = bf16_round(O.chain_step(L.dense, xv, ids, gates))
    assert_tokens(out.float().cpu().numpy(), want, what="prefill fused norm")


def test_moe_prefill_bad_ids(small_layer):
    """An invalid expert id drops its pair and raises the status; the other
    tokens are still computed."""
    L = small_layer
    B = 100
    bits, xv = gs.hidden_bf16(B, L.d_model, tag=6)
    ids, gates = gs.route_topk(gs.router_logits(B, L.E, tag=6), 6)
    ids = ids.copy()
    ids[37, 2] = 4000
    out, st = _moe(L, bits, ids, gates)
    assert st == G.GALE_ERR_ARG
    toks = np.array([0, 36, 38, 99])
    assert_tokens(out.cpu().numpy()[toks], O.moe_layer(L.dense, xv[toks], ids[toks], gates[toks]))


@pytest.mark.parametrize("skew", [0.0, 1.0])
def test_moe_prefill_full_size(full_layer, skew):
    """4096 tokens, top-6 of 256 experts, per-token parity on every token
    routed to the three hottest experts (under the skewed routing hundreds
    each: several 128-token chunks and the persistent kernel's tail items)
    and on every 16th token."""
    L = full_layer
    B = 4096
    bits, xv = gs.hidden_bf16(B, L.d_model, tag=4096)
    ids, gates = gs.route_topk(gs.router_logits(B, L.E, tag=4096, bias_sigma=skew), 6)
    out, st = _moe(L, bits, ids, gates)
    assert st == 0
    got = out.cpu().numpy()
    assert np.isfinite(got).all()
    counts = np.bincount(ids.reshape(-1), minlength=L.E)
    hot = np.argsort(-counts, kind="stable")[:3]
    if skew > 0:
        assert counts[hot].min() > 128   # the skewed routing splits them into several chunks
    toks = np.union1d(np.nonzero(np.isin(ids, hot).any(axis=1))[0], np.arange(0, B, 16))
    assert_tokens(got[toks], O.moe_layer(L.dense, xv[toks], ids[toks], gates[toks]), what=f"skew {skew}")


def test_selftest():
    scratch = torch.empty(G.gale_selftest_scratch_bytes(), dtype=torch.uint8, device="cuda")
    assert G.gale_selftest(scratch) == G.GALE_OK


# ----------------------------------------------------------------------------
# router
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("B,E,K,skew", [(1, 256, 6, 0.0), (8, 256, 6, 0.0), (64, 256, 6, 0.5), (4096, 256, 6, 0.5),
                                         (5, 16, 16, 0.0), (33, 1000, 8, 0.0), (7, 1024, 1, 0.0)])
def test_route_topk_matches_oracle(B, E, K, skew):
    """Ids bit-exact, gates within 1e-6, against the oracle's router."""
    lg = gs.router_logits(B, E, tag=6000 + B, bias_sigma=skew)
    ids = torch.empty(B, K, dtype=torch.int32, device="cuda")
    gates = torch.empty(B, K, dtype=torch.float32, device="cuda")
    G.gale_route_topk(to_dev(lg), ids, gates)
    torch.cuda.synchronize()
    wi, wg = O.route_topk(lg, K)
    assert np.array_equal(ids.cpu().numpy(), wi)
    assert np.max(np.abs(gates.cpu().numpy().astype(np.float64) - wg)) < 1e-6


def test_route_topk_ties_and_nan():
    """Equal logits go to the lower expert index; NaN ranks last."""
    lg = np.array([[0.5, 2.0, 2.0, np.nan, 2.0, -1.0, 0.5, 0.5]] * 3, np.float32)
    lg[1, 1] = np.nan
    lg[2] = 1.0
    ids = torch.empty(3, 4, dtype=torch.int32, device="cuda")
    gates = torch.empty(3, 4, dtype=torch.float32, device="cuda")
    G.gale_route_topk(to_dev(lg), ids, gates)
    torch.cuda.synchronize()
    assert ids.cpu().numpy().tolist() == [[1, 2, 4, 0], [2, 4, 0, 6], [0, 1, 2, 3]]
    wi, wg = O.route_topk(np.nan_to_num(lg, nan=-np.inf), 4)
    assert np.array_equal(ids.cpu().numpy(), wi)
    assert np.max(np.abs(gates.cpu().numpy().astype(np.float64) - wg)) < 1e-6


@pytest.mark.parametrize("shape,e,B", [("small", 3, 1), ("small", 15, 2), ("small", 0, 5), ("full", 7, 1),
                                       ("full", 200, 3)])
def test_expert_forward(small_layer, full_layer, shape, e, B):
    """One expert's SwiGLU forward on fp32 tokens in one launch
    (gale_expert_forward) against the oracle's expert_forward, per token."""
    L = small_layer if shape == "small" else full_layer
    x = np.stack([gs.x_f32(L.d_model, tag=1000 + 10 * B + t) for t in range(B)])
    ws = torch.empty(G.gale_expert_forward_workspace_size(L.desc, B), dtype=torch.uint8, device="cuda")
    out = torch.full((B, L.d_model), float("nan"), device="cuda")
    G.gale_expert_forward(L.desc, e, to_dev(x), out, ws)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0
    assert_tokens(out.cpu().numpy(), O.expert_forward(L.dense(e), x.astype(np.float64)), what=f"expert {e} B={B}")


def test_expert_forward_rejects_bad_expert(small_layer):
    L = small_layer
    x = torch.zeros(1, L.d_model, device="cuda")
    out = torch.zeros(1, L.d_model, device="cuda")
    ws = torch.empty(G.gale_expert_forward_workspace_size(L.desc, 1), dtype=torch.uint8, device="cuda")
    rc = G.lib().gale_expert_forward(ctypes.byref(L.desc), L.E, x.data_ptr(), 1, out.data_ptr(), ws.data_ptr(),
                                     ws.numel(), None)
    assert rc == G.GALE_ERR_ARG
