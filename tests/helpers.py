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
