"""GPU parity of the 4-bit non-expert weights (W4, g128) against the oracle.

The quantizer is compared byte for byte with the oracle's pack (a code is a
float decision taken in fp32 on both sides); the GEMV per token against the
oracle's fp64 product of the oracle's own pack, at several tiles and ragged
token counts, at the benchmark's full shape (sampled rows), and on hard
activations (spikes, a zero token, values x1000).
"""
import numpy as np
import pytest

import gale_synth as gs
from oracle import w4_oracle as W

from .helpers import REL_L2_TOL, assert_tokens, edge_hidden, to_dev

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
G = pytest.importorskip("bit_expert_gemv_b200")


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    G.lib()


def _weights(rows, cols, tag, scale=1.0):
    return (gs.normal(gs.stream_key(72, tag), rows * cols).astype(np.float32) * np.float32(scale)).reshape(rows, cols)


def _gpu_quantize(w):
    rows, cols = w.shape
    L = G.gale_w4_layout(rows, cols)
    packed = torch.zeros(L.total, dtype=torch.uint8, device="cuda")
    G.gale_w4_quantize(to_dev(w), packed)
    torch.cuda.synchronize()
    return packed.cpu().numpy(), L


def _gemv(buf_np, rows, cols, xbits):
    B = xbits.shape[0]
    packed = to_dev(buf_np)
    x = to_dev(xbits.astype(np.uint16), torch.int16)
    y = torch.full((B, rows), float("nan"), device="cuda")
    ws = torch.zeros(G.gale_w4_workspace_size(rows, cols, B), dtype=torch.uint8, device="cuda")
    G.gale_w4_gemv(packed, rows, cols, x, y, ws)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0
    return y.cpu().numpy()


@pytest.mark.parametrize("rows,cols,scale", [(1, 128, 1.0), (37, 384, 1.0), (64, 4096, 0.02), (300, 1024, 250.0)])
def test_w4_quantize_bit_exact(rows, cols, scale):
    w = _weights(rows, cols, rows + cols, scale)
    if rows > 2:
        w[1, :128] = 0.0                                   # a zero block
        w[2, :8] = [7.0, -7.0, 2.5, 3.5, -0.5, 0.5, 1.5, -6.5]   # ties at s = 1
        w[2, 8:128] = 0.0
    got, L = _gpu_quantize(w)
    want = W.w4_pack(*W.w4_quantize(w))
    n = L.q_bytes
    assert np.array_equal(got[:n], want[:n]), f"codes differ at byte {int(np.argmax(got[:n] != want[:n]))}"
    s0 = L.s_offset
    assert np.array_equal(got[s0:s0 + L.s_bytes], want[s0:s0 + L.s_bytes])


@pytest.mark.parametrize("rows,cols,B", [(16, 1024, 1), (64, 2048, 2), (128, 4096, 3), (512, 4096, 8),
                                         (48, 3072, 5), (2048, 4096, 1), (96, 8192, 4), (32, 1024, 7),
                                         (4752, 1024, 2), (32, 7168, 6), (16, 8192, 8), (48, 16384, 3),
                                         (16, 34816, 1)])
def test_w4_gemv_parity(rows, cols, B):
    """Shapes: one tile (one CTA), more tiles than SMs with a ragged last
    round (4752 rows = 297 tiles), rows of several units with a narrower last
    unit (7168, 16384), and the widest rows the shared memory holds at 8 and
    at 1 token."""
    w = _weights(rows, cols, 1000 + rows + B)
    q, s = W.w4_quantize(w)
    xbits, xv = gs.hidden_bf16(B, cols, tag=rows + cols + B)
    got = _gemv(W.w4_pack(q, s), rows, cols, xbits)
    assert_tokens(got, W.w4_gemv(q, s, xv), what=f"w4 {rows}x{cols} B={B}")


@pytest.mark.parametrize("B", [1, 8])
def test_w4_gemv_full_shape_sampled_rows(B):
    # the benchmark's shape: [65536 x 4096], weights drawn and quantized on the device
    rows, cols = 65536, 4096
    w = torch.empty(rows, cols, dtype=torch.float32, device="cuda")
    for r0 in range(0, rows, 4096):
        w[r0:r0 + 4096] = (gs.normal_torch(gs.stream_key(73, 0), 4096 * cols, start=r0 * cols) * 0.02).view(4096, cols)
    L = G.gale_w4_layout(rows, cols)
    packed = torch.zeros(L.total, dtype=torch.uint8, device="cuda")
    G.gale_w4_quantize(w, packed)
    xbits, xv = gs.hidden_bf16(B, cols, tag=17)
    x = to_dev(xbits.astype(np.uint16), torch.int16)
    y = torch.full((B, rows), float("nan"), device="cuda")
    ws = torch.zeros(G.gale_w4_workspace_size(rows, cols, B), dtype=torch.uint8, device="cuda")
    G.gale_w4_gemv(packed, rows, cols, x, y, ws)
    torch.cuda.synchronize()
    assert int(ws[:4].view(torch.int32).item()) == 0
    sel = np.r_[0:16, 30000:30016, rows - 16:rows]
    q, s = W.w4_quantize(w[torch.from_numpy(sel).cuda()].cpu().numpy())
    assert_tokens(y.cpu().numpy()[:, sel], W.w4_gemv(q, s, xv), what=f"w4 {rows}x{cols} B={B} sampled rows")


@pytest.mark.parametrize("kind", ["spikes", "zero", "scaled"])
def test_w4_gemv_hard_inputs(kind):
    rows, cols, B = 256, 4096, 5
    w = _weights(rows, cols, 11)
    q, s = W.w4_quantize(w)
    xbits, xv = edge_hidden(B, cols, kind, tag=23)
    got = _gemv(W.w4_pack(q, s), rows, cols, xbits)
    assert_tokens(got, W.w4_gemv(q, s, xv), what=f"w4 {kind}")


def test_w4_unit_scales_small_integers():
    # s = 1 and small integer activations: the int32 MMA sums are exact and
    # only the fp32 combination of the digit sums rounds (relative 1e-7)
    rows, cols, B = 64, 2048, 2
    rng = np.random.default_rng(5)
    q = rng.integers(-7, 8, size=(rows, cols)).astype(np.int8)
    s = np.ones((rows, cols // 128), dtype=np.float16)
    xv = rng.integers(-4, 5, size=(B, cols)).astype(np.float32)
    got = _gemv(W.w4_pack(q, s), rows, cols, gs.f32_to_bf16_bits(xv))
    assert_tokens(got, W.w4_gemv(q, s, xv), tol=1e-6, what="w4 unit scales")


def test_w4_argument_errors():
    rows, cols = 32, 1024
    q, s = W.w4_quantize(_weights(rows, cols, 3))
    packed = to_dev(W.w4_pack(q, s))
    x = torch.zeros((1, cols), dtype=torch.int16, device="cuda")
    y = torch.zeros((1, rows), device="cuda")
    ws = torch.empty(G.gale_w4_workspace_size(rows, cols, 1), dtype=torch.uint8, device="cuda")
    L = G.lib()
    args = lambda r, c, B, wsb: L.gale_w4_gemv(packed.data_ptr(), r, c, x.data_ptr(), B, y.data_ptr(),
                                                ws.data_ptr(), wsb, None)
    assert args(rows, 1536, 1, ws.numel()) == G.GALE_ERR_ARG      # cols % 1024
    assert args(24, cols, 1, ws.numel()) == G.GALE_ERR_ARG        # rows % 16
    assert args(rows, cols, 9, ws.numel()) == G.GALE_ERR_ARG      # B > 8
    assert args(rows, cols, 1, 16) == G.GALE_ERR_WORKSPACE
    assert L.gale_w4_gemv(packed.data_ptr() + 16, rows, cols, x.data_ptr(), 1, y.data_ptr(), ws.data_ptr(),
                          ws.numel(), None) == G.GALE_ERR_ALIGN
    assert G.gale_w4_workspace_size(rows, 1000, 1) == 0
    # beyond the shared-memory limit: 8 tokens of 9216 columns
    c2 = 9216
    x8 = torch.zeros((8, c2), dtype=torch.int16, device="cuda")
    y8 = torch.zeros((8, 16), device="cuda")
    assert G.gale_w4_workspace_size(16, c2, 8) == 0
    ws8 = torch.zeros(256, dtype=torch.uint8, device="cuda")
    p8 = torch.zeros(G.gale_w4_layout(16, c2).total, dtype=torch.uint8, device="cuda")
    assert L.gale_w4_gemv(p8.data_ptr(), 16, c2, x8.data_ptr(), 8, y8.data_ptr(), ws8.data_ptr(), ws8.numel(),
                          None) == G.GALE_ERR_UNSUPPORTED
