"""CPU-side checks of the C ABI: the library loads, exports every symbol that
include/gale.h declares, and its host-side layout and argument validation
agree with the oracle's layout.  No compute call is made (no GPU here)."""
import ctypes
import os
import re

import pytest

import bit_expert_gemv_b200 as G
from oracle import gale_oracle as O

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "gale.h")


def declared_symbols():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gale_[a-z0-9_]+)\s*\(", text)))


def test_library_exports_every_declared_symbol():
    lib = G.lib()
    names = declared_symbols()
    assert names, "no declarations parsed"
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(G.EXPORTS) == names


@pytest.mark.parametrize("rows,cols", [(2048, 4096), (4096, 2048), (1, 1024), (37, 2048), (100, 3072),
                                        (5, 8192)])
def test_layout_matches_oracle(rows, cols):
    L = G.gale_pack_layout(rows, cols)
    Lo = O.layout(rows, cols)
    assert L["k"] == Lo["k"]
    assert L["offsets"] == Lo["offsets"]
    assert L["sizes"] == Lo["sizes"]
    assert L["total"] == Lo["total"]


def test_expert_bytes():
    assert G.gale_expert_bytes(4096, 2048) == O.expert_bytes(4096, 2048) == 4179968
    assert G.gale_expert_bytes(4096, 1000) == 0


def test_host_argument_validation():
    lib = G.lib()
    out = G.gale_layout()
    assert lib.gale_pack_layout(0, 1024, ctypes.byref(out)) == G.GALE_ERR_ARG
    assert lib.gale_pack_layout(4, 1000, ctypes.byref(out)) == G.GALE_ERR_ARG
    assert lib.gale_pack_layout(4, 1024, None) == G.GALE_ERR_ARG
    # rejected before any CUDA call
    assert lib.gale_fwht1024(None, 0, None, 0, 4, 1000, None) == G.GALE_ERR_ARG
    assert lib.gale_fwht1024(None, 0, None, 0, 0, 1024, None) == G.GALE_OK
    assert lib.gale_fwht1024(8, 7, 8, 0, 1, 1024, None) == G.GALE_ERR_ARG
    assert lib.gale_fwht1024(6, 0, 8, 0, 1, 1024, None) == G.GALE_ERR_ALIGN
    assert lib.gale_expert_gemv(None, None, None, 1, None, 0, None) == G.GALE_ERR_ARG
    assert lib.gale_route_permute(None, 1, 0, 256, None, None, None, None, None) == G.GALE_ERR_ARG
    # the many-CTA permute: scratch of one int per (256-pair range, expert), checked before any CUDA call
    assert G.gale_route_permute_scratch_bytes(4096, 6, 256) == 96 * 256 * 4
    assert G.gale_route_permute_scratch_bytes(1, 6, 256) == 256 * 4
    assert G.gale_route_permute_scratch_bytes(0, 6, 256) == 0
    assert G.gale_route_permute_scratch_bytes(4, 17, 256) == 0
    assert lib.gale_route_permute_grid(None, 1, 0, 256, None, None, None, None, None, 0, None) == G.GALE_ERR_ARG
    assert lib.gale_route_permute_grid(16, 4, 6, 256, 16, 16, 16, 16, 16, 1023, None) == G.GALE_ERR_WORKSPACE
    assert lib.gale_route_permute_grid(16, 4, 6, 256, 16, 16, 16, 16, 18, 1024, None) == G.GALE_ERR_ALIGN
    assert lib.gale_selftest(None, None) == G.GALE_ERR_ARG
    assert G.status_string(G.GALE_ERR_TIMEOUT).startswith("GALE_ERR_TIMEOUT")


def test_workspace_size_and_layer_validation():
    lib = G.lib()
    good = G.gale_layer(0x100000, 4179968, 256, 4096, 2048, 0)
    n1 = G.gale_moe_workspace_size(good, 1, 6)
    n64 = G.gale_moe_workspace_size(good, 64, 6)
    assert 0 < n1 < n64
    bad_stride = G.gale_layer(0x100000, 4179968 - 256, 256, 4096, 2048, 0)
    assert G.gale_moe_workspace_size(bad_stride, 1, 6) == 0
    bad = G.gale_layer(0x100000, 4179968, 256, 4096, 2048, 0)
    rc = lib.gale_moe_forward(ctypes.byref(bad), None, None, None, 1, 6, None, 0, 0, ctypes.c_float(1e-6),
                              None, 0, None)
    assert rc == G.GALE_ERR_WORKSPACE
    rc = lib.gale_moe_forward(ctypes.byref(bad), None, None, None, 1, 6, None, 5, 0, ctypes.c_float(1e-6),
                              None, 0, None)
    assert rc == G.GALE_ERR_ARG


def test_w4_supported_sizes():
    """The 4-bit GEMV's documented limits, from the host-only workspace query:
    the widest row (a multiple of 1024) whose activation digits and two ring
    stages fit the shared memory, per token count, and 0 one step beyond."""
    limits = {1: 34816, 2: 34816, 3: 16384, 4: 16384, 5: 11264, 6: 11264, 7: 8192, 8: 8192}
    for B, cols in limits.items():
        assert G.gale_w4_workspace_size(16, cols, B) == 256, (B, cols)
        assert G.gale_w4_workspace_size(16, cols + 1024, B) == 0, (B, cols)
    assert G.gale_w4_workspace_size(16, 4096, 9) == 0
    assert G.gale_w4_workspace_size(24, 4096, 1) == 0
    assert G.gale_w4_workspace_size(16, 1536, 1) == 0
