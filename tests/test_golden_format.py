"""The oracle against the format facts the pages state (tests/golden/nvfp4_format.txt).

"Replay the Curvature" (arXiv 2609.36654v1), Abstract, NVFP4 sentence: every
16 E2M1 weights share one E4M3 block scale.  The value sets are built here from
the format names alone (one sign bit, E exponent bits with bias 2^(E-1) - 1,
M mantissa bits, subnormals at the zero exponent; for E4M3 the "fn" variant
whose all-ones pattern is NaN, the reading the oracle states), and a solved
layer is checked to be made of 16-weight blocks that share one scale.
"""
from pathlib import Path

import numpy as np
import pytest

import oracle as O

GOLDEN = Path(__file__).parent / "golden" / "nvfp4_format.txt"


def fixture():
    out = {}
    for line in GOLDEN.read_text().splitlines():
        line = line.strip()
        if line and not line.startswith("#"):
            k, v = line.split()
            out[k] = v
    return out


def field_widths(name):
    assert name[0] == "E" and "M" in name
    e, m = name[1:].split("M")
    return int(e), int(m)


def magnitudes(e_bits, m_bits, drop_all_ones=False):
    """Every finite non-negative value of a sign/exponent/mantissa format."""
    bias = 2 ** (e_bits - 1) - 1
    vals = set()
    for e in range(2 ** e_bits):
        for m in range(2 ** m_bits):
            if drop_all_ones and e == 2 ** e_bits - 1 and m == 2 ** m_bits - 1:
                continue   # NaN in the fn variant
            if e == 0:
                v = (m / 2 ** m_bits) * 2.0 ** (1 - bias)
            else:
                v = (1 + m / 2 ** m_bits) * 2.0 ** (e - bias)
            vals.add(v)
    return np.array(sorted(vals))


def test_fixture_block_size_is_the_oracles():
    assert int(fixture()["block_size"]) == O.BLOCK == 16


def test_e2m1_values_follow_from_the_format_name():
    e, m = field_widths(fixture()["element_format"])
    assert (e, m) == (2, 1)
    assert np.array_equal(magnitudes(e, m), O.E2M1_MAGNITUDE)
    assert O.E2M1_MAX == magnitudes(e, m)[-1]


def test_e4m3_values_follow_from_the_format_name():
    e, m = field_widths(fixture()["scale_format"])
    assert (e, m) == (4, 3)
    vals = magnitudes(e, m, drop_all_ones=True)
    assert np.array_equal(vals, O.E4M3_TABLE)     # codes 0 .. 126, 0 .. 448
    assert O.E4M3_MAX == vals[-1] == 448.0


@pytest.mark.parametrize("d_out,d_in", [(6, 64), (3, 160)])
def test_solved_layer_is_blocks_of_16_sharing_one_scale(d_out, d_in):
    rng = np.random.default_rng(d_out * 1000 + d_in)
    W = rng.standard_normal((d_out, d_in)) * np.exp(rng.standard_normal((d_out, 1)))
    X = rng.standard_normal((4 * d_in, d_in))
    res = O.solve_layer(W, X)
    blk = int(fixture()["block_size"])
    assert res["codes"].shape == (d_out, d_in)
    assert res["scales"].shape == (d_out, d_in // blk)
    e2m1 = magnitudes(*field_widths(fixture()["element_format"]))
    e4m3 = magnitudes(*field_widths(fixture()["scale_format"]), drop_all_ones=True)
    scale = e4m3[res["scales"]] * float(np.float32(res["s_g"]))   # one value per block
    q = res["q"].reshape(d_out, d_in // blk, blk)
    live = scale > 0
    ratio = np.abs(q[live]) / scale[live][:, None]
    # every weight of a block is an E2M1 value times the block's one scale
    assert np.all(np.isin(ratio, e2m1))
    assert np.all(q[~live] == 0.0)
