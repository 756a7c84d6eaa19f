"""The torch port of the seeded matrix generator (used to build large resident
workloads on the device) draws the same canonical matrices as the numpy
generator: integer draws bit-identical, scales equal up to a rare last-place
rounding of the device's transcendental functions."""
import numpy as np
import pytest

import gale_synth as gs


def _compare(t, experts, rows, cols, layer, matrix, min_scale_equal):
    for i, e in enumerate(experts):
        c = gs.matrix_canonical(rows, cols, layer, e, matrix)
        assert np.array_equal(t["signs"][i].cpu().numpy(), c["signs"])
        assert np.array_equal(t["idx"][i].cpu().numpy().view(np.uint16), c["idx"])
        assert np.array_equal(t["q"][i].cpu().numpy(), c["q"])
        assert (t["s_blk"][i].cpu().numpy() == c["s_blk"]).mean() >= min_scale_equal
        assert (t["s_row"][i].cpu().numpy() == c["s_row"]).mean() >= min_scale_equal


@pytest.mark.parametrize("rows,cols,layer,experts,matrix", [(64, 1024, 3, [0, 5], gs.W1), (32, 2048, 1, [7], gs.W2)])
def test_torch_generator_matches_numpy_cpu(rows, cols, layer, experts, matrix):
    t = gs.matrices_canonical_torch(rows, cols, layer, experts, matrix, device="cpu")
    _compare(t, experts, rows, cols, layer, matrix, 1.0)


@pytest.mark.gpu
def test_torch_generator_matches_numpy_gpu():
    t = gs.matrices_canonical_torch(256, 4096, 11, [1, 200], gs.W3, device="cuda")
    _compare(t, [1, 200], 256, 4096, 11, gs.W3, 0.999)
