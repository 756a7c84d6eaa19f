"""The failure path of the streaming decode kernel, without faulting or
hanging the GPU: every device-side wait of the kernel is bounded, and a wait
that runs out reports GALE_ERR_TIMEOUT in the status word while every CTA
drains its copies and returns.  The test shortens the bound to 1 ms and has
one CTA withhold its h-readiness counts (a flag that nothing else sets), so
that the phase-2 waits of the CTAs needing those h blocks run out; a normal
call on the same workspace afterwards must be correct."""
import numpy as np
import pytest

import gale_synth as gs
from oracle import gale_oracle as O

from .helpers import Layer, assert_tokens, to_dev

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
G = pytest.importorskip("bit_expert_gemv_b200")


@pytest.fixture(scope="module")
def layer():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    return Layer(16, 2048, 1024, layer=5)


def test_stream_wait_runs_out_then_recovers(layer):
    L = layer
    B, K = 5, 6   # 30 pairs: the streaming decode kernel
    bits, xv = gs.hidden_bf16(B, L.d_model, tag=55)
    ids, gates = gs.route_topk(gs.router_logits(B, L.E, tag=55), K)
    xd, idd, gd = to_dev(bits, torch.bfloat16), to_dev(ids), to_dev(gates)
    ws = torch.empty(G.gale_moe_workspace_size(L.desc, B, K), dtype=torch.uint8, device="cuda")
    out = torch.empty(B, L.d_model, dtype=torch.float32, device="cuda")
    try:
        G.gale_debug_set_failure(1_000_000, 0)
        G.gale_moe_forward(L.desc, xd, idd, gd, out, ws)
        torch.cuda.synchronize()
        assert int(ws[:4].view(torch.int32).item()) == G.GALE_ERR_TIMEOUT
    finally:
        G.gale_debug_set_failure(0, -1)
    out.fill_(float("nan"))
    G.gale_moe_forward(L.desc, xd, idd, gd, out, ws)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0
    assert_tokens(out.cpu().numpy(), O.moe_layer(L.dense, xv, ids, gates), what="after the timeout")


def test_chain_wait_runs_out_then_recovers():
    """The same failure in a three-layer stack (gale_moe_chain): the phase-2
    waits of layer 0 run out, the CTAs that finished their part wait (bounded)
    for the layer's outputs, every CTA leaves the layer loop, and the call
    reports GALE_ERR_TIMEOUT; a normal call on the same workspace afterwards
    matches the layers run one call at a time."""
    from .test_gpu_chain import _stack
    n_layers, E, d, dff, B, K = 3, 16, 2048, 1024, 5, 6
    buf, stride, _ = _stack(n_layers, E, d, dff)
    first = G.make_layer(buf, stride, E, d, dff)
    bits, _ = gs.hidden_bf16(B, d, tag=56)
    ids = np.zeros((n_layers, B, K), dtype=np.int32)
    gates = np.zeros((n_layers, B, K), dtype=np.float32)
    for l in range(n_layers):
        ids[l], gates[l] = gs.route_topk(gs.router_logits(B, E, tag=560 + l), K)
    x0, idd, gd = to_dev(bits, torch.bfloat16), to_dev(ids), to_dev(gates)
    ws = torch.empty(G.gale_moe_chain_workspace_size(first, n_layers, B, K), dtype=torch.uint8, device="cuda")
    out = torch.empty(B, d, dtype=torch.bfloat16, device="cuda")
    try:
        G.gale_debug_set_failure(1_000_000, 0)
        G.gale_moe_chain(first, n_layers, E * stride, x0, idd, gd, out, ws)
        torch.cuda.synchronize()
        assert int(ws[:4].view(torch.int32).item()) == G.GALE_ERR_TIMEOUT
    finally:
        G.gale_debug_set_failure(0, -1)
    G.gale_moe_chain(first, n_layers, E * stride, x0, idd, gd, out, ws)
    x = x0
    for l in range(n_layers):
        Ll = G.make_layer(buf[l * E * stride:], stride, E, d, dff)
        wsl = torch.empty(G.gale_moe_workspace_size(Ll, B, K), dtype=torch.uint8, device="cuda")
        xn = torch.empty(B, d, dtype=torch.bfloat16, device="cuda")
        G.gale_moe_forward(Ll, x, idd[l], gd[l], xn, wsl, flags=G.GALE_FLAG_RESIDUAL_RMSNORM, eps=1e-6)
        x = xn
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0
    assert torch.equal(out.view(torch.int16), x.view(torch.int16))
