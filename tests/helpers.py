"""Shared helpers of the test-suite: build packed layers on the GPU from the
seeded canonical matrices (through the library's own packer), and the
oracle's dense view of the same experts (through the oracle's own packer and
unpacker).  The two sides share only the seeded canonical inputs."""
from __future__ import annotations

import numpy as np

import gale_synth as gs
from oracle import gale_oracle as O

REL_L2_TOL = 2e-3   # expert-output tolerance (bf16 activations, fp32 accumulation)


def rel_l2(a, b) -> float:
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def rel_l2_rows(a, b) -> np.ndarray:
    """Relative L2 error of every row (token) of a against b."""
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return np.linalg.norm(a - b, axis=-1) / np.maximum(np.linalg.norm(b, axis=-1), 1e-300)


def assert_tokens(got, want, tol=REL_L2_TOL, what=""):
    """Per-token parity: every row within `tol` relative L2; rows the oracle
    gives as exact zeros must be exact zeros."""
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    assert got.shape == want.shape, what
    assert np.isfinite(got).all(), what
    zero = np.all(want == 0.0, axis=-1)
    assert np.all(got[zero] == 0.0), f"{what}: rows {np.nonzero(zero)[0][:8]} should be exactly zero"
    if (~zero).any():
        e = rel_l2_rows(got[~zero], want[~zero])
        worst = int(np.argmax(e))
        assert e.max() < tol, f"{what}: token {np.nonzero(~zero)[0][worst]} rel-L2 {e.max():.3g} >= {tol}"


def bf16_round(v) -> np.ndarray:
    """fp64 values rounded to bf16 (round to nearest even), back as fp64."""
    return gs.bf16_bits_to_f32(gs.f32_to_bf16_bits(np.asarray(v, dtype=np.float32))).astype(np.float64)


def edge_hidden(B: int, d: int, kind: str, tag: int):
    """bf16 hidden states with a hard case planted: "spikes" puts three
    features of every token at 300x the rms, "zero" makes the middle token all
    zeros, "scaled" multiplies every value by 1000.  Returns (bits, values)."""
    _, v = gs.hidden_bf16(B, d, tag=tag)
    v = v.astype(np.float32).copy()
    if kind == "spikes":
        rng = np.random.default_rng(tag)
        for t in range(B):
            cols = rng.choice(d, size=3, replace=False)
            v[t, cols] = 300.0 * np.sign(v[t, cols] + 0.5)
    elif kind == "zero":
        v[B // 2] = 0.0
    elif kind == "scaled":
        v *= 1000.0
    else:
        raise ValueError(kind)
    bits = gs.f32_to_bf16_bits(v)
    return bits, gs.bf16_bits_to_f32(bits)


def to_dev(a, dtype=None):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.cuda()


def gpu_pack(c: dict, dst, status=None):
    """Pack one canonical matrix into the device buffer ``dst`` (uint8 view)."""
    import torch
    import bit_expert_gemv_b200 as G
    if status is None:
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
    k = c["idx"].shape[1]
    G.gale_pack(to_dev(c["signs"]), to_dev(c["s_blk"].view(np.uint16)), to_dev(c["s_row"].view(np.uint16)),
                to_dev(c["idx"]) if k else None, to_dev(c["q"]) if k else None,
                c["rows"], c["cols"], dst, status)
    return status


class Layer:
    """A packed MoE layer resident on the GPU plus lazy oracle access."""

    DENSE_CACHE = 48

    def __init__(self, n_experts: int, d_model: int, d_ff: int, layer: int = 0):
        import torch
        import bit_expert_gemv_b200 as G
        self.E, self.d_model, self.d_ff, self.layer_id = n_experts, d_model, d_ff, layer
        self.stride = G.gale_expert_bytes(d_model, d_ff)
        self.buf = torch.empty(n_experts * self.stride, dtype=torch.uint8, device="cuda")
        l1 = G.gale_pack_layout(d_ff, d_model)["total"]
        self.mat_off = [0, l1, 2 * l1]
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        for e in range(n_experts):
            cs = gs.expert_canonical(d_model, d_ff, layer=layer, expert=e)
            for m, c in enumerate(cs):
                off = e * self.stride + self.mat_off[m]
                gpu_pack(c, self.buf[off:], status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        self.desc = G.make_layer(self.buf, self.stride, n_experts, d_model, d_ff)
        self._dense = {}

    def dense(self, e: int):
        if e not in self._dense:
            if len(self._dense) >= self.DENSE_CACHE:   # fp64 experts are large: keep the newest few
                self._dense.pop(next(iter(self._dense)))
            cs = gs.expert_canonical(self.d_model, self.d_ff, layer=self.layer_id, expert=e)
            self._dense[e] = [O.dequant_packed(O.pack(c), c["rows"], c["cols"]) for c in cs]
        return self._dense[e]
