"""GPU parity of the independent-block scale rules that Schur Replay is compared
with: the amax scale and the per-block squared-error search without replay
("Replay the Curvature", Abstract: evaluating a block independently can
misestimate its final reconstruction error once GPTQ updates the columns that
follow).  Both run the same GPTQ sweep as Schur Replay; only the scale decision
differs, so the same parity bar applies: bit-exact on small layers, the near-tie
rule of tests/parity.py on the 4096 x 4096 layer (every row), layer error
within 1e-4.  The last test is the comparison itself on the GPU: Schur
Replay's layer error is below both rules' on that layer.
"""
import numpy as np
import pytest
import torch

import oracle as O
from nvfp4_post_weight_b200 import binding as B
from nvfp4_post_weight_b200 import synth
from nvfp4_post_weight_b200.layer import LayerSolver
from parity import classify, report, unpack_codes

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
RULES = ["amax", "block_mse"]


def gpu_quantize(W, U32, rule):
    d_out, d_in = W.shape
    Wd = W.to(DEV)
    Ud = torch.as_tensor(U32, dtype=torch.float32).to(DEV)
    codes = torch.empty((d_out, d_in // 2), dtype=torch.uint8, device=DEV)
    scales = torch.empty((d_out, d_in // 16), dtype=torch.uint8, device=DEV)
    sg = torch.empty(1, dtype=torch.float32, device=DEV)
    err = torch.empty(1, dtype=torch.float64, device=DEV)
    ws = B.workspace(B.nvfp4_quantize_workspace_size(d_out, d_in), DEV)
    B.nvfp4_gptq_schur_replay_quantize(Wd, Ud, codes, scales, sg, err, None, ws,
                                       B.solve_params(rule))
    torch.cuda.synchronize()
    assert B.nvfp4_workspace_status(ws) == 0
    return (unpack_codes(codes.cpu().numpy()), scales.cpu().numpy().astype(np.int64),
            float(sg.item()), float(err.item()))


@pytest.mark.parametrize("rule", RULES)
@pytest.mark.parametrize("d_out,d_in", [(1, 16), (33, 144), (5, 272), (64, 256)])
def test_rule_given_oracle_factor_bitexact(rule, d_out, d_in):
    rng = np.random.default_rng(d_out * 1000 + d_in + 7)
    W64 = rng.normal(0, 0.02, size=(d_out, d_in))
    W64[:, rng.integers(0, d_in)] *= 20
    W64 = W64.astype(np.float32).astype(np.float64)      # both sides see the same fp32 W
    X = rng.standard_normal((2 * d_in, d_in)) * rng.lognormal(0, 1, size=d_in)
    Hd, _, _ = O.damp(X.T @ X)
    U32 = O.inverse_cholesky_upper(Hd).astype(np.float32)
    sg = O.global_scale(W64)
    ref = O.schur_replay_gptq(W64, U32.astype(np.float64), sg, rule=rule)
    codes, scales, sg_gpu, err = gpu_quantize(torch.from_numpy(W64.astype(np.float32)), U32, rule)
    assert np.float32(sg_gpu) == sg
    assert np.array_equal(scales, ref["scales"])
    assert np.array_equal(codes, ref["codes"])
    # past the first 128 columns W~ carries the 3xTF32 trailing update
    # (~2^-22 relative per product, fp32 sums), so the sum of delta^2 agrees
    # to ~1e-7 while the discrete outputs stay identical
    assert abs(err - ref["err_sum"]) <= 1e-6 * ref["err_sum"]


@pytest.mark.parametrize("rule", RULES)
def test_rule_small_outlier_solve_bitexact(rule):
    W, X = synth.small_outlier()
    ref = O.solve_layer(W.double().numpy(), X.double().numpy(), rule=rule)
    s = LayerSolver(*W.shape, DEV, out_dtype=torch.float32, scale_rule=rule)
    s.step(W.to(DEV), X.to(DEV))
    torch.cuda.synchronize()
    assert s.status() == (0, 0)
    assert np.array_equal(s.scales.cpu().numpy().astype(np.int64), ref["scales"])
    assert np.array_equal(unpack_codes(s.codes.cpu().numpy()), ref["codes"])
    L = ref["layer_error"]
    assert abs(s.layer_err.item() - L) <= 1e-4 * L


@pytest.fixture(scope="module")
def attn_layer():
    W, X = synth.attn_massive()
    H = O.hessian(X.double().numpy())
    Hd, _, _ = O.damp(H)
    U = O.inverse_cholesky_upper(Hd)
    return dict(W=W, X=X, H=H, U=U, W64=W.double().numpy())


def solve_gpu(layer, rule):
    W, X = layer["W"], layer["X"]
    s = LayerSolver(*W.shape, DEV, out_dtype=torch.bfloat16, scale_rule=rule)
    s.step(W.to(DEV), X.to(DEV))
    torch.cuda.synchronize()
    assert s.status() == (0, 0)
    return s


@pytest.mark.parametrize("rule", RULES)
def test_rule_attn_4096_all_rows(attn_layer, rule):
    s = solve_gpu(attn_layer, rule)
    W64, U, H = attn_layer["W64"], attn_layer["U"], attn_layer["H"]
    sg = O.global_scale(W64)
    assert np.float32(s.s_g.item()) == sg
    ref = O.schur_replay_gptq(W64, U, sg, return_diag=True, rule=rule)
    codes = unpack_codes(s.codes.cpu().numpy())
    scales = s.scales.cpu().numpy().astype(np.int64)
    c = classify(ref, U, sg, codes, scales)
    report(f"attn_massive_4096x4096 rule {rule}", c)
    assert c["frac"] <= 1e-3, c
    assert not c["bad_first"], c
    Q = O.dequant(codes, scales, sg).astype(np.float64)
    L_gpu = O.layer_error(W64, Q, H)
    L_ref = O.layer_error(W64, ref["q"], H)
    assert abs(L_gpu - L_ref) <= 1e-4 * L_ref
    assert abs(s.layer_err.item() - L_ref) <= 1e-4 * L_ref


def test_schur_replay_lowers_layer_error_on_the_gpu(attn_layer):
    """The comparison the method is about, on the 4096 x 4096 layer: the GPU's
    own layer errors tr((W-Q) H (W-Q)^T) under the three rules."""
    L = {r: solve_gpu(attn_layer, r).layer_err.item() for r in ["schur_replay"] + RULES}
    assert L["schur_replay"] < L["block_mse"] and L["schur_replay"] < L["amax"], L
