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
