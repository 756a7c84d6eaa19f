"""gale_moe_forward_noalloc: the MoE layer for callers that cannot allocate
device memory (a plugin inside a runtime that owns the device memory pool, or
a process with a device footprint fixed at start-up).  Its scratch is a fixed
array inside the library; the test checks two calls in a row against the
workspace entry point, through the C ABI, within the layer tolerance.

Kept in a file of its own that collects last, so that a run stopping at the
first failure has already run every other test.
"""
import numpy as np
import pytest

import gale_synth as gs

from .helpers import REL_L2_TOL, Layer, rel_l2, to_dev

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
G = pytest.importorskip("bit_expert_gemv_b200")


@pytest.fixture(scope="module")
def layer():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return Layer(16, 2048, 1024, layer=3)


def _with_workspace(L, xd, idd, gd):
    B, K = idd.shape
    ws = torch.empty(G.gale_moe_workspace_size(L.desc, B, K), dtype=torch.uint8, device="cuda")
    out = torch.empty(B, L.d_model, dtype=torch.float32, device="cuda")
    G.gale_moe_forward(L.desc, xd, idd, gd, out, ws)
    return out


def test_noalloc_matches_workspace_entry_point_twice(layer):
    L = layer
    for call, (B, K, tag) in enumerate([(4, 6, 901), (9, 4, 902)]):
        bits, _ = gs.hidden_bf16(B, L.d_model, tag=tag)
        ids, gates = gs.route_topk(gs.router_logits(B, L.E, tag=tag), K)
        xd, idd, gd = to_dev(bits, torch.bfloat16), to_dev(ids), to_dev(gates)
        want = _with_workspace(L, xd, idd, gd)
        got = torch.full((B, L.d_model), float("nan"), dtype=torch.float32, device="cuda")
        status = torch.full((1,), 12345, dtype=torch.int32, device="cuda")
        G.gale_moe_forward_noalloc(L.desc, xd, idd, gd, got, status=status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0, call
        assert rel_l2(got.cpu().numpy(), want.cpu().numpy()) < REL_L2_TOL, call


def test_noalloc_rejects_oversized_call(layer):
    L = layer
    B, K = 4096, 6
    assert G.gale_moe_workspace_size(L.desc, B, K) > G.GALE_NOALLOC_SCRATCH_BYTES
    ids = torch.zeros(B, K, dtype=torch.int32, device="cuda")
    x = torch.zeros(B, L.d_model, dtype=torch.bfloat16, device="cuda")
    g = torch.zeros(B, K, dtype=torch.float32, device="cuda")
    out = torch.empty(B, L.d_model, dtype=torch.float32, device="cuda")
    with pytest.raises(G.GaleError) as e:
        G.gale_moe_forward_noalloc(L.desc, x, ids, g, out)
    assert e.value.code == G.GALE_ERR_WORKSPACE


@pytest.fixture(scope="module")
def full_shape_layer():
    """Eight experts of the full shapes (w1/w3 [2048 x 4096], w2 [4096 x 2048])."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return Layer(8, 4096, 2048, layer=4)


def test_noalloc_full_shape_fused_norm_bf16(full_shape_layer):
    """Batch 1, top-6, residual + RMSNorm into bf16 at the full expert shapes
    (the combine stages v = x + y in the scratch array): the same result as
    the workspace entry point, on two calls in a row."""
    L = full_shape_layer
    for tag in (911, 912):
        bits, _ = gs.hidden_bf16(1, L.d_model, tag=tag)
        ids, gates = gs.route_topk(gs.router_logits(1, L.E, tag=tag), 6)
        xd, idd, gd = to_dev(bits, torch.bfloat16), to_dev(ids), to_dev(gates)
        ws = torch.empty(G.gale_moe_workspace_size(L.desc, 1, 6), dtype=torch.uint8, device="cuda")
        want = torch.empty(1, L.d_model, dtype=torch.bfloat16, device="cuda")
        G.gale_moe_forward(L.desc, xd, idd, gd, want, ws, flags=G.GALE_FLAG_RESIDUAL_RMSNORM)
        got = torch.full((1, L.d_model), float("nan"), dtype=torch.bfloat16, device="cuda")
        status = torch.full((1,), 12345, dtype=torch.int32, device="cuda")
        G.gale_moe_forward_noalloc(L.desc, xd, idd, gd, got, status=status, flags=G.GALE_FLAG_RESIDUAL_RMSNORM)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert rel_l2(got.float().cpu().numpy(), want.float().cpu().numpy()) < REL_L2_TOL


def test_noalloc_reports_bad_ids_in_status(full_shape_layer):
    """An expert id out of range drops its pair and reaches the caller's
    status word as GALE_ERR_ARG; a clean call afterwards reports 0."""
    L = full_shape_layer
    bits, _ = gs.hidden_bf16(1, L.d_model, tag=913)
    ids, gates = gs.route_topk(gs.router_logits(1, L.E, tag=913), 6)
    bad = ids.copy()
    bad[0, 3] = L.E + 5
    xd, gd = to_dev(bits, torch.bfloat16), to_dev(gates)
    out = torch.empty(1, L.d_model, dtype=torch.float32, device="cuda")
    status = torch.full((1,), 12345, dtype=torch.int32, device="cuda")
    G.gale_moe_forward_noalloc(L.desc, xd, to_dev(bad), gd, out, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == G.GALE_ERR_ARG
    G.gale_moe_forward_noalloc(L.desc, xd, to_dev(ids), gd, out, status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
