"""GPU encoder (gale_encode) against the encoder oracle: the packed record bit
for bit, at several shapes, on hand-made rows (ties, a zero row, an exactly
representable matrix), at the widest supported row, and end to end: experts
encoded on the device drive gale_moe_forward to the oracle's layer output.
"""
import numpy as np
import pytest

import gale_synth as gs
from oracle import encoder_oracle as E
from oracle import gale_oracle as O

from .helpers import assert_tokens, to_dev

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
G = pytest.importorskip("bit_expert_gemv_b200")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    G.lib()


def _gauss(rows, cols, tag, scale=0.02):
    return (gs.normal(gs.stream_key(75, tag), rows * cols) * scale).astype(np.float32).reshape(rows, cols)


def _encode_gpu(w):
    rows, cols = w.shape
    L = G.gale_pack_layout(rows, cols)
    dst = torch.full((L["total"],), 0xAB, dtype=torch.uint8, device="cuda")
    G.gale_encode(to_dev(w), dst)
    torch.cuda.synchronize()
    return dst.cpu().numpy()


def _assert_same(got, want, rows, cols):
    if not np.array_equal(got, want):
        L = O.layout(rows, cols)
        names = ["signs", "s_blk", "s_row", "idx", "q"]
        first = int(np.argmax(got != want))
        sec = max(i for i in range(5) if L["offsets"][i] <= first)
        raise AssertionError(f"first differing byte {first} in section {names[sec]}")


@pytest.mark.parametrize("rows,cols", [(1, 1024), (37, 2048), (64, 4096), (5, 16384)])
def test_encode_bit_exact(rows, cols):
    w = _gauss(rows, cols, rows + cols)
    _assert_same(_encode_gpu(w), O.pack(E.encode(w)), rows, cols)


def test_encode_ties_zero_row_and_representable():
    rng = np.random.default_rng(11)
    cols = 2048
    e = rng.integers(4, 10, size=(4, cols // 128))
    mag = np.repeat(7.0 * 2.0 ** -e, 128, axis=1)
    wr = np.where(rng.random((4, cols)) < 0.5, -mag, mag)       # equal magnitudes per block: ties everywhere
    wr[2] = 0.0                                                  # a zero row
    w = E.fwht_staged(wr).astype(np.float32)
    got = _encode_gpu(w)
    _assert_same(got, O.pack(E.encode(w)), 4, cols)
    assert np.array_equal(O.dequant_packed(got, 4, cols), wr)   # and it decodes to the rotated matrix exactly


def test_encode_errors():
    L = G.lib()
    w = torch.zeros((2, 1024), dtype=torch.float32, device="cuda")
    dst = torch.zeros(G.gale_pack_layout(2, 1024)["total"] + 64, dtype=torch.uint8, device="cuda")
    assert L.gale_encode(w.data_ptr(), 2, 1000, dst.data_ptr(), None) == G.GALE_ERR_ARG
    assert L.gale_encode(w.data_ptr(), 0, 1024, dst.data_ptr(), None) == G.GALE_ERR_ARG
    assert L.gale_encode(w.data_ptr(), 2, 1024, dst.data_ptr() + 8, None) == G.GALE_ERR_ALIGN
    assert L.gale_encode(w.data_ptr(), 1, 17408, dst.data_ptr(), None) == G.GALE_ERR_UNSUPPORTED


def test_encoded_experts_drive_the_layer():
    E_, dm, dff, B, K = 4, 2048, 1024, 3, 2
    stride = G.gale_expert_bytes(dm, dff)
    l1 = G.gale_pack_layout(dff, dm)["total"]
    buf = torch.zeros(E_ * stride, dtype=torch.uint8, device="cuda")
    dense = []
    for e in range(E_):
        mats = [_gauss(dff, dm, 100 + 3 * e), _gauss(dff, dm, 101 + 3 * e), _gauss(dm, dff, 102 + 3 * e)]
        offs = [0, l1, 2 * l1]
        for m, off in zip(mats, offs):
            G.gale_encode(to_dev(m), buf[e * stride + off:])
        dense.append([O.dequant(E.encode(m)) for m in mats])
    layer = G.make_layer(buf, stride, E_, dm, dff)
    bits, xv = gs.hidden_bf16(B, dm, tag=5)
    ids, gates = gs.route_topk(gs.router_logits(B, E_, tag=5), K)
    out = torch.empty(B, dm, device="cuda")
    ws = torch.empty(G.gale_moe_workspace_size(layer, B, K), dtype=torch.uint8, device="cuda")
    G.gale_moe_forward(layer, torch.from_numpy(bits).view(torch.bfloat16).cuda(), torch.from_numpy(ids).cuda(),
                       torch.from_numpy(gates).cuda(), out, ws)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0
    assert_tokens(out.cpu().numpy(), O.moe_layer(lambda e: dense[e], xv, ids, gates), what="encoded layer")
