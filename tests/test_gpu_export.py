"""GPU test of the export of the block scales into the 128-row x 4-column tiled
layout of block-scaled FP4 GEMM operands, bit-exact against the oracle's
definition (pinned in tests/test_oracle_pins.py), on ragged shapes and on the
scales of a solved layer.

Method: "Replay the Curvature", Abstract, infrastructure sentence (layers are
exported before their full-precision weights are retired).
"""
import numpy as np
import pytest
import torch

import oracle as O
from nvfp4_post_weight_b200 import binding as B
from nvfp4_post_weight_b200 import synth
from nvfp4_post_weight_b200.layer import LayerSolver

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def export(scales_np):
    rows, nb = scales_np.shape
    sc = torch.from_numpy(np.ascontiguousarray(scales_np)).to(DEV)
    out = torch.full((B.nvfp4_export_scales_size(rows, nb * 16),), 0xAB, dtype=torch.uint8,
                     device=DEV)
    B.nvfp4_export_scales(sc, out)
    torch.cuda.synchronize()
    return out.cpu().numpy()


@pytest.mark.parametrize("rows,nb", [(1, 1), (7, 3), (128, 4), (200, 6), (4097, 257)])
def test_export_scales_bitexact(rows, nb):
    rng = np.random.default_rng(rows + nb)
    sc = rng.integers(0, 127, size=(rows, nb)).astype(np.uint8)
    np.testing.assert_array_equal(export(sc), O.scales_to_tiled(sc))


def test_export_scales_of_a_solved_layer():
    W, X = synth.small_outlier()
    s = LayerSolver(*W.shape, DEV, out_dtype=torch.float32)
    s.step(W.to(DEV), X.to(DEV))
    torch.cuda.synchronize()
    sc = s.scales.cpu().numpy()
    np.testing.assert_array_equal(export(sc), O.scales_to_tiled(sc))
