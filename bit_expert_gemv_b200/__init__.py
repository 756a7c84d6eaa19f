"""Python binding of libgale, the sm_100a GALE 1-bit routed-expert library.

Argument marshalling only: every function forwards torch tensors (device
memory owned by the caller) as raw pointers to the C ABI declared in
``include/gale.h``, under the same names.  There is no CPU fallback: if the
library is missing, loading it raises.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libgale.so")

GALE_OK = 0
GALE_ERR_ARG = -1
GALE_ERR_ALIGN = -2
GALE_ERR_WORKSPACE = -3
GALE_ERR_CUDA = -4
GALE_ERR_TIMEOUT = -5
GALE_ERR_UNSUPPORTED = -6
GALE_ERR_SELFTEST = -7

GALE_F32, GALE_BF16, GALE_F16 = 0, 1, 2
GALE_MODE_PLAIN, GALE_MODE_SWIGLU = 0, 1
GALE_FLAG_RESIDUAL_RMSNORM = 1

# every symbol include/gale.h declares
EXPORTS = (
    "gale_status_string", "gale_pack_layout", "gale_expert_bytes", "gale_pack", "gale_unpack",
    "gale_fwht1024", "gale_expert_gemv", "gale_route_permute", "gale_route_permute_scratch_bytes",
    "gale_route_permute_grid", "gale_moe_workspace_size",
    "gale_moe_forward", "gale_moe_forward_noalloc", "gale_selftest_scratch_bytes", "gale_selftest",
    "gale_moe_host_staging_bytes", "gale_moe_host_workspace_size", "gale_moe_forward_host",
    "gale_debug_set_failure", "gale_route_topk",
    "gale_w4_layout", "gale_w4_quantize", "gale_w4_workspace_size", "gale_w4_gemv", "gale_encode",
    "gale_moe_chain", "gale_moe_chain_workspace_size", "gale_expert_forward", "gale_expert_forward_workspace_size",
)

GALE_NOALLOC_SCRATCH_BYTES = 4 << 20


class GaleError(RuntimeError):
    def __init__(self, code: int, where: str = ""):
        self.code = code
        super().__init__(f"{where}: {status_string(code)}" if where else status_string(code))


class gale_layout(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_int32), ("cols", ctypes.c_int32), ("k", ctypes.c_int32),
                ("reserved", ctypes.c_int32), ("offset", ctypes.c_int64 * 5),
                ("size", ctypes.c_int64 * 5), ("total", ctypes.c_int64)]


class gale_matrix(ctypes.Structure):
    _fields_ = [("packed", ctypes.c_void_p), ("rows", ctypes.c_int32), ("cols", ctypes.c_int32)]


class gale_w4_layout_t(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_int64), ("cols", ctypes.c_int64), ("q_offset", ctypes.c_int64),
                ("q_bytes", ctypes.c_int64), ("s_offset", ctypes.c_int64), ("s_bytes", ctypes.c_int64),
                ("total", ctypes.c_int64)]


class gale_layer(ctypes.Structure):
    _fields_ = [("base", ctypes.c_void_p), ("expert_stride", ctypes.c_int64),
                ("n_experts", ctypes.c_int32), ("d_model", ctypes.c_int32),
                ("d_ff", ctypes.c_int32), ("reserved", ctypes.c_int32)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libgale.so (built in-tree by ``bit_expert_gemv_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: run `python -m bit_expert_gemv_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
        sig = {
            "gale_status_string": (ctypes.c_char_p, [i32]),
            "gale_pack_layout": (i32, [i32, i32, ctypes.POINTER(gale_layout)]),
            "gale_expert_bytes": (i64, [i32, i32]),
            "gale_pack": (i32, [vp, vp, vp, vp, vp, i32, i32, vp, vp, vp]),
            "gale_unpack": (i32, [vp, i32, i32, vp, vp]),
            "gale_fwht1024": (i32, [vp, i32, vp, i32, i64, i32, vp]),
            "gale_expert_gemv": (i32, [ctypes.POINTER(gale_matrix), ctypes.POINTER(gale_matrix), vp, i32,
                                       vp, i32, vp]),
            "gale_route_permute": (i32, [vp, i32, i32, i32, vp, vp, vp, vp, vp]),
            "gale_route_permute_scratch_bytes": (sz, [i32, i32, i32]),
            "gale_route_permute_grid": (i32, [vp, i32, i32, i32, vp, vp, vp, vp, vp, sz, vp]),
            "gale_moe_workspace_size": (sz, [ctypes.POINTER(gale_layer), i32, i32]),
            "gale_moe_forward": (i32, [ctypes.POINTER(gale_layer), vp, vp, vp, i32, i32, vp, i32, i32,
                                       ctypes.c_float, vp, sz, vp]),
            "gale_moe_forward_noalloc": (i32, [ctypes.POINTER(gale_layer), vp, vp, vp, i32, i32, vp, i32, i32,
                                               ctypes.c_float, vp, vp]),
            "gale_moe_host_staging_bytes": (sz, [i32, i32, i32]),
            "gale_moe_host_workspace_size": (sz, [ctypes.POINTER(gale_layer), i32, i32]),
            "gale_moe_forward_host": (i32, [ctypes.POINTER(gale_layer), vp, vp, vp, i32, i32, vp, i32, i32,
                                            ctypes.c_float, vp, sz, vp, sz, vp]),
            "gale_debug_set_failure": (i32, [ctypes.c_uint64, i32]),
            "gale_route_topk": (i32, [vp, i32, i32, i32, vp, vp, vp]),
            "gale_encode": (i32, [vp, i32, i32, vp, vp]),
            "gale_moe_chain_workspace_size": (sz, [ctypes.POINTER(gale_layer), i32, i32, i32]),
            "gale_expert_forward_workspace_size": (sz, [ctypes.POINTER(gale_layer), i32]),
            "gale_expert_forward": (i32, [ctypes.POINTER(gale_layer), i32, vp, i32, vp, vp, sz, vp]),
            "gale_moe_chain": (i32, [ctypes.POINTER(gale_layer), i32, i64, vp, vp, vp, i32, i32, vp, ctypes.c_float,
                                     vp, sz, vp]),
            "gale_w4_layout": (i32, [i64, i64, ctypes.POINTER(gale_w4_layout_t)]),
            "gale_w4_quantize": (i32, [vp, i64, i64, vp, vp]),
            "gale_w4_workspace_size": (sz, [i64, i64, i32]),
            "gale_w4_gemv": (i32, [vp, i64, i64, vp, i32, vp, vp, sz, vp]),
            "gale_selftest_scratch_bytes": (sz, []),
            "gale_selftest": (i32, [vp, vp]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def status_string(code: int) -> str:
    return lib().gale_status_string(int(code)).decode()


def _check(rc: int, where: str):
    if rc != GALE_OK:
        raise GaleError(rc, where)


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    import torch
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _dtype_code(t) -> int:
    import torch
    return {torch.float32: GALE_F32, torch.bfloat16: GALE_BF16, torch.float16: GALE_F16}[t.dtype]


# ----------------------------------------------------------------------------
# entry points (same names as the C ABI)
# ----------------------------------------------------------------------------

def gale_pack_layout(rows: int, cols: int) -> dict:
    out = gale_layout()
    _check(lib().gale_pack_layout(rows, cols, ctypes.byref(out)), "gale_pack_layout")
    return {"rows": out.rows, "cols": out.cols, "k": out.k, "offsets": list(out.offset),
            "sizes": list(out.size), "total": out.total}


def gale_expert_bytes(d_model: int, d_ff: int) -> int:
    return int(lib().gale_expert_bytes(d_model, d_ff))


def gale_pack(signs, s_blk, s_row, idx, q, rows: int, cols: int, dst, status, stream=None):
    _check(lib().gale_pack(_ptr(signs), _ptr(s_blk), _ptr(s_row), _ptr(idx), _ptr(q), rows, cols,
                           _ptr(dst), _ptr(status), _stream(stream)), "gale_pack")


def gale_unpack(packed, rows: int, cols: int, dense, stream=None):
    _check(lib().gale_unpack(_ptr(packed), rows, cols, _ptr(dense), _stream(stream)), "gale_unpack")


def gale_fwht1024(x, y, stream=None):
    cols = x.shape[-1]
    rows = x.numel() // cols if cols else 0
    _check(lib().gale_fwht1024(_ptr(x), _dtype_code(x), _ptr(y), _dtype_code(y), rows, cols,
                               _stream(stream)), "gale_fwht1024")


def gale_expert_gemv(W, rows: int, cols: int, x_rot, y, W3=None, mode: int = GALE_MODE_PLAIN,
                     stream=None):
    a = gale_matrix(_ptr(W), rows, cols)
    b = gale_matrix(_ptr(W3), rows, cols) if W3 is not None else None
    ntok = x_rot.numel() // cols
    _check(lib().gale_expert_gemv(ctypes.byref(a), ctypes.byref(b) if b is not None else None,
                                  _ptr(x_rot), ntok, _ptr(y), mode, _stream(stream)), "gale_expert_gemv")


def gale_route_permute(ids, n_experts: int, counts, offsets, perm, status, stream=None):
    B, K = ids.shape
    _check(lib().gale_route_permute(_ptr(ids), B, K, n_experts, _ptr(counts), _ptr(offsets), _ptr(perm),
                                    _ptr(status), _stream(stream)), "gale_route_permute")


def gale_route_permute_scratch_bytes(B: int, K: int, n_experts: int) -> int:
    return int(lib().gale_route_permute_scratch_bytes(B, K, n_experts))


def gale_route_permute_grid(ids, n_experts: int, counts, offsets, perm, status, scratch, stream=None):
    """The many-CTA routing permute (same results as gale_route_permute);
    `scratch` is a device byte tensor of gale_route_permute_scratch_bytes()."""
    B, K = ids.shape
    _check(lib().gale_route_permute_grid(_ptr(ids), B, K, n_experts, _ptr(counts), _ptr(offsets), _ptr(perm),
                                         _ptr(status), _ptr(scratch), scratch.numel() * scratch.element_size(),
                                         _stream(stream)), "gale_route_permute_grid")


def gale_route_topk(logits, ids, gates, stream=None):
    """Top-K experts of every token (K = ids.shape[1]) and their softmax gates."""
    B, E = logits.shape
    _check(lib().gale_route_topk(_ptr(logits), B, E, ids.shape[1], _ptr(ids), _ptr(gates), _stream(stream)),
           "gale_route_topk")


def gale_expert_forward_workspace_size(layer: gale_layer, B: int) -> int:
    return int(lib().gale_expert_forward_workspace_size(ctypes.byref(layer), B))


def gale_expert_forward(layer: gale_layer, expert: int, x, out, ws, stream=None):
    """out [B, d_model] fp32 = the SwiGLU forward of one expert on fp32 x [B, d_model] (one launch)."""
    B = x.shape[0]
    _check(lib().gale_expert_forward(ctypes.byref(layer), expert, _ptr(x), B, _ptr(out), _ptr(ws),
                                     ws.numel() * ws.element_size(), _stream(stream)), "gale_expert_forward")


def gale_moe_chain_workspace_size(first: gale_layer, n_layers: int, B: int, K: int) -> int:
    return int(lib().gale_moe_chain_workspace_size(ctypes.byref(first), n_layers, B, K))


def gale_moe_chain(first: gale_layer, n_layers: int, layer_stride: int, x0, ids, gates, out, ws, eps: float = 1e-6,
                   stream=None):
    """x_L of a stack of n_layers layers: x_{l+1} = bf16(RMSNorm(x_l + MoE_l(x_l))); ids/gates [n_layers, B, K]."""
    B, K = ids.shape[1], ids.shape[2]
    _check(lib().gale_moe_chain(ctypes.byref(first), n_layers, layer_stride, _ptr(x0), _ptr(ids), _ptr(gates), B, K,
                                _ptr(out), eps, _ptr(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "gale_moe_chain")


def gale_encode(w, dst, stream=None):
    """Encode a device fp32 [rows, cols] matrix into one packed GALE record (dst: device bytes)."""
    rows, cols = w.shape
    _check(lib().gale_encode(_ptr(w), rows, cols, _ptr(dst), _stream(stream)), "gale_encode")


def gale_w4_layout(rows: int, cols: int) -> gale_w4_layout_t:
    out = gale_w4_layout_t()
    _check(lib().gale_w4_layout(rows, cols, ctypes.byref(out)), "gale_w4_layout")
    return out


def gale_w4_quantize(w, packed, stream=None):
    """Quantize a device fp32 [rows, cols] matrix into the W4 g128 layout (packed: device bytes)."""
    rows, cols = w.shape
    _check(lib().gale_w4_quantize(_ptr(w), rows, cols, _ptr(packed), _stream(stream)), "gale_w4_quantize")


def gale_w4_workspace_size(rows: int, cols: int, B: int) -> int:
    return int(lib().gale_w4_workspace_size(rows, cols, B))


def gale_w4_gemv(packed, rows: int, cols: int, x, y, ws, stream=None):
    """y [B, rows] fp32 = x [B, cols] (bf16 bits) times the W4 matrix transposed."""
    B = x.shape[0]
    _check(lib().gale_w4_gemv(_ptr(packed), rows, cols, _ptr(x), B, _ptr(y), _ptr(ws), ws.numel() * ws.element_size(),
                              _stream(stream)), "gale_w4_gemv")


def make_layer(base, expert_stride: int, n_experts: int, d_model: int, d_ff: int) -> gale_layer:
    return gale_layer(_ptr(base), expert_stride, n_experts, d_model, d_ff, 0)


def gale_moe_workspace_size(layer: gale_layer, B: int, K: int) -> int:
    return int(lib().gale_moe_workspace_size(ctypes.byref(layer), B, K))


def gale_moe_forward(layer: gale_layer, x, ids, gates, out, ws, flags: int = 0, eps: float = 1e-6,
                     stream=None):
    B, K = ids.shape
    _check(lib().gale_moe_forward(ctypes.byref(layer), _ptr(x), _ptr(ids), _ptr(gates), B, K, _ptr(out),
                                  _dtype_code(out), flags, eps, _ptr(ws), ws.numel() * ws.element_size(),
                                  _stream(stream)), "gale_moe_forward")


def gale_moe_forward_noalloc(layer: gale_layer, x, ids, gates, out, status=None, flags: int = 0,
                             eps: float = 1e-6, stream=None):
    """gale_moe_forward with the library's fixed scratch array instead of a
    caller workspace (for callers that cannot allocate device memory)."""
    B, K = ids.shape
    _check(lib().gale_moe_forward_noalloc(ctypes.byref(layer), _ptr(x), _ptr(ids), _ptr(gates), B, K,
                                          _ptr(out), _dtype_code(out), flags, eps, _ptr(status),
                                          _stream(stream)), "gale_moe_forward_noalloc")


def gale_moe_host_staging_bytes(B: int, K: int, d_model: int) -> int:
    return int(lib().gale_moe_host_staging_bytes(B, K, d_model))


def gale_moe_host_workspace_size(layer: gale_layer, B: int, K: int) -> int:
    return int(lib().gale_moe_host_workspace_size(ctypes.byref(layer), B, K))


def gale_moe_forward_host(layer: gale_layer, x, ids, gates, out, ws, staging, flags: int = 0,
                          eps: float = 1e-6, stream=None):
    """gale_moe_forward with x, ids, gates in host memory and out in pinned
    host memory; `staging` is a pinned host byte tensor of at least
    gale_moe_host_staging_bytes() bytes, `ws` a device workspace of at least
    gale_moe_host_workspace_size() bytes.  Asynchronous: synchronise the
    stream before reading `out` or refilling `staging`."""
    B, K = ids.shape
    _check(lib().gale_moe_forward_host(ctypes.byref(layer), _ptr(x), _ptr(ids), _ptr(gates), B, K, _ptr(out),
                                       _dtype_code(out), flags, eps, _ptr(ws), ws.numel() * ws.element_size(),
                                       _ptr(staging), staging.numel() * staging.element_size(), _stream(stream)),
           "gale_moe_forward_host")


def gale_debug_set_failure(wait_limit_ns: int, withhold_cta: int):
    """Failure-path testing: bound of the streaming decode kernel's device
    waits (0 = default 2 s) and a CTA whose h tiles are never counted (-1 = none)."""
    _check(lib().gale_debug_set_failure(int(wait_limit_ns), int(withhold_cta)), "gale_debug_set_failure")


def gale_selftest_scratch_bytes() -> int:
    return int(lib().gale_selftest_scratch_bytes())


def gale_selftest(scratch, stream=None) -> int:
    return int(lib().gale_selftest(_ptr(scratch), _stream(stream)))
