"""Chained decode: three layers of x_{l+1} = bf16(RMSNorm(x_l + MoE_l(x_l)))
(residual + RMSNorm fused into gale_moe_forward) against the oracle chain
with the same bf16 rounding of every layer's input."""
import numpy as np
import pytest

import gale_synth as gs
from oracle import gale_oracle as O
from tests.helpers import Layer, rel_l2, to_dev

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


def test_three_layer_chain():
    import bit_expert_gemv_b200 as G
    E, d, dff, K = 8, 4096, 2048, 6
    layers = [Layer(E, d, dff, layer=l) for l in range(3)]
    bits, xv = gs.hidden_bf16(1, d, tag=4242)
    x_dev = to_dev(bits, torch.bfloat16)
    x_ref = xv.astype(np.float64)
    for l, L in enumerate(layers):
        ids, gates = gs.route_topk(gs.router_logits(1, E, tag=100 + l), K)
        ws = torch.empty(G.gale_moe_workspace_size(L.desc, 1, K), dtype=torch.uint8, device="cuda")
        out = torch.empty(1, d, dtype=torch.bfloat16, device="cuda")
        G.gale_moe_forward(L.desc, x_dev, to_dev(ids), to_dev(gates), out, ws,
                           flags=G.GALE_FLAG_RESIDUAL_RMSNORM, eps=1e-6)
        torch.cuda.synchronize()
        assert int(ws[:4].view(torch.int32).item()) == 0
        y = O.chain_step(L.dense, x_ref, ids, gates)
        # the oracle's next input is its own output rounded to bf16, as on the device
        x_ref = gs.bf16_bits_to_f32(gs.f32_to_bf16_bits(y.astype(np.float32))).astype(np.float64)
        x_dev = out
        got = out.float().cpu().numpy()
        assert rel_l2(got, x_ref) < 4e-3, f"layer {l}"


def _stack(n_layers, E, d, dff):
    """n_layers layers of E experts packed back to back in one buffer (layer l's
    expert e is record l * E + e) and the oracle's dense views."""
    import bit_expert_gemv_b200 as G
    from tests.helpers import gpu_pack
    stride = G.gale_expert_bytes(d, dff)
    l1 = G.gale_pack_layout(dff, d)["total"]
    buf = torch.empty(n_layers * E * stride, dtype=torch.uint8, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    dense = []
    for l in range(n_layers):
        dl = {}
        for e in range(E):
            cs = gs.expert_canonical(d, dff, layer=l, expert=e)
            for m, c in enumerate(cs):
                gpu_pack(c, buf[(l * E + e) * stride + m * l1:], status)
            dl[e] = [O.dequant_packed(O.pack(c), c["rows"], c["cols"]) for c in cs]
        dense.append(dl)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return buf, stride, dense


@pytest.mark.parametrize("n_layers,E,d,dff,B,K", [(4, 8, 4096, 2048, 1, 6), (5, 16, 2048, 1024, 3, 4),
                                                  (3, 12, 4096, 2048, 8, 6), (2, 16, 2048, 1024, 2, 16),
                                                  (3, 32, 2048, 1024, 32, 6)])
def test_chain_kernel(n_layers, E, d, dff, B, K):
    """gale_moe_chain (one persistent launch for the whole stack):
    - from three tokens on, bit-identical to the same layers run one call at a
      time through gale_moe_forward with the fused norm (the same kernel);
    - against the oracle chain with the same bf16 rounding between layers, at
      2e-3 per layer: where the two sides' values straddle a bf16 rounding
      boundary their outputs differ by one ulp, and the next layer carries
      the difference on, so the one-layer tolerance grows with depth."""
    import bit_expert_gemv_b200 as G
    from tests.helpers import assert_tokens
    buf, stride, dense = _stack(n_layers, E, d, dff)
    first = G.make_layer(buf, stride, E, d, dff)
    bits, xv = gs.hidden_bf16(B, d, tag=777 + B)
    ids = np.zeros((n_layers, B, K), dtype=np.int32)
    gates = np.zeros((n_layers, B, K), dtype=np.float32)
    x_ref = xv.astype(np.float64)
    for l in range(n_layers):
        ids[l], gates[l] = gs.route_topk(gs.router_logits(B, E, tag=300 + 10 * l + B), K)
        y = O.chain_step(lambda e, l=l: dense[l][e], x_ref, ids[l], gates[l])
        x_ref = gs.bf16_bits_to_f32(gs.f32_to_bf16_bits(y.astype(np.float32))).astype(np.float64)
    x0 = to_dev(bits, torch.bfloat16)
    ws = torch.empty(G.gale_moe_chain_workspace_size(first, n_layers, B, K), dtype=torch.uint8, device="cuda")
    out = torch.empty(B, d, dtype=torch.bfloat16, device="cuda")
    G.gale_moe_chain(first, n_layers, E * stride, x0, to_dev(ids), to_dev(gates), out, ws)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0
    assert_tokens(out.float().cpu().numpy(), x_ref, tol=2e-3 * n_layers, what=f"{n_layers}-layer chain B={B}")
    if B >= 3:
        x = x0
        for l in range(n_layers):
            Ll = G.make_layer(buf[l * E * stride:], stride, E, d, dff)
            wsl = torch.empty(G.gale_moe_workspace_size(Ll, B, K), dtype=torch.uint8, device="cuda")
            xn = torch.empty(B, d, dtype=torch.bfloat16, device="cuda")
            G.gale_moe_forward(Ll, x, to_dev(ids[l]), to_dev(gates[l]), xn, wsl, flags=G.GALE_FLAG_RESIDUAL_RMSNORM,
                               eps=1e-6)
            x = xn
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), x.view(torch.int16))


def test_chain_kernel_one_layer_equals_forward():
    """A one-layer stack is bit-identical to gale_moe_forward with the fused norm
    (both on the streaming kernel at three tokens)."""
    import bit_expert_gemv_b200 as G
    E, d, dff, B, K = 16, 2048, 1024, 3, 6
    buf, stride, _ = _stack(1, E, d, dff)
    first = G.make_layer(buf, stride, E, d, dff)
    bits, _ = gs.hidden_bf16(B, d, tag=31)
    ids, gates = gs.route_topk(gs.router_logits(B, E, tag=31), K)
    x = to_dev(bits, torch.bfloat16)
    out1 = torch.empty(B, d, dtype=torch.bfloat16, device="cuda")
    ws1 = torch.empty(G.gale_moe_chain_workspace_size(first, 1, B, K), dtype=torch.uint8, device="cuda")
    G.gale_moe_chain(first, 1, E * stride, x, to_dev(ids[None]), to_dev(gates[None]), out1, ws1)
    out2 = torch.empty(B, d, dtype=torch.bfloat16, device="cuda")
    ws2 = torch.empty(G.gale_moe_workspace_size(first, B, K), dtype=torch.uint8, device="cuda")
    G.gale_moe_forward(first, x, to_dev(ids), to_dev(gates), out2, ws2, flags=G.GALE_FLAG_RESIDUAL_RMSNORM, eps=1e-6)
    torch.cuda.synchronize()
    assert int(ws1[:4].view(torch.int32).item()) == 0 and int(ws2[:4].view(torch.int32).item()) == 0
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))
