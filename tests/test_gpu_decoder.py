"""GPU tests on the 70B-shaped dense decoder layer (hidden 8192, kv 1024,
intermediate 28672, 16384 calibration tokens per Hessian, lognormal(0, 1.5)
channel scales), solved as the layer is: one Hessian and one factor U shared by
q, k and v, and one by gate and up, each tensor with its own global scale.

* Attention (q/k/v + o) and gate/up: the GPU Hessian against the oracle's fp64
  one (1e-4 Frobenius); then the GPU factor from the oracle's fp32-rounded
  Hessian and the GPU quantize of every tensor with the shared U, compared
  with the oracle on a seeded sample of rows per tensor (rows are independent
  given U) under the near-tie rule of parity.py, and the sampled rows' layer
  error within 1e-4.
* down (d_in = 28672, where the oracle's fp64 Hessian and inverse take many
  minutes): properties that hold at any size -- sampled Hessian entries
  against exact dot products of the bf16 tokens, U upper with a positive
  diagonal, codes and scales of every block well formed, and the library's
  layer error (<H, E^T E> on the 3xTF32 Gram tiles) against tr(E H E^T)
  evaluated in fp64.

Method: "Replay the Curvature", Abstract (GPTQ with Schur Replay on every
linear of a layer; shared second-order state for inputs that are shared).
"""
import numpy as np
import pytest
import torch

import oracle as O
from nvfp4_post_weight_b200 import binding as B
from nvfp4_post_weight_b200 import synth
from parity import classify, report, unpack_codes

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
ROWS = 256   # sampled rows per tensor


def rel_frob(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def gpu_hessian(X):
    d = X.shape[1]
    H = torch.empty((d, d), dtype=torch.float32, device=DEV)
    B.nvfp4_hessian_accumulate(H, X.to(DEV))
    torch.cuda.synchronize()
    assert B.nvfp4_hessian_status() == 0
    return H


def gpu_prepare(H32):
    d = H32.shape[0]
    U = torch.empty_like(H32)
    ws = B.workspace(B.nvfp4_prepare_workspace_size(d), DEV)
    B.nvfp4_gptq_prepare(H32, 0.01, U, None, None, ws)
    torch.cuda.synchronize()
    assert B.nvfp4_workspace_status(ws) == 0
    return U


def gpu_quantize(W, U):
    d_out, d_in = W.shape
    codes = torch.empty((d_out, d_in // 2), dtype=torch.uint8, device=DEV)
    scales = torch.empty((d_out, d_in // 16), dtype=torch.uint8, device=DEV)
    sg = torch.empty(1, dtype=torch.float32, device=DEV)
    err = torch.empty(1, dtype=torch.float64, device=DEV)
    ws = B.workspace(B.nvfp4_quantize_workspace_size(d_out, d_in), DEV)
    B.nvfp4_gptq_schur_replay_quantize(W.to(DEV), U, codes, scales, sg, err, None, ws)
    torch.cuda.synchronize()
    assert B.nvfp4_workspace_status(ws) == 0
    return codes, scales, sg, err


def check_group(layer, x_name, w_names, seed):
    """One shared Hessian: GPU H vs oracle, then every tensor of the group
    quantized with the one GPU factor of the oracle's fp32 H, sampled rows vs
    the oracle."""
    X = layer[x_name]()
    Xn = X.double().numpy()
    H = O.hessian(Xn)
    del Xn
    Hg = gpu_hessian(X)
    assert rel_frob(Hg.cpu().numpy().astype(np.float64), H) < 1e-4
    del Hg, X
    H32 = H.astype(np.float32)
    U = gpu_prepare(torch.from_numpy(H32).to(DEV))
    Hd, _, _ = O.damp(H32.astype(np.float64))
    Uo = O.inverse_cholesky_upper(Hd)
    rng = np.random.default_rng(seed)
    for name in w_names:
        W = layer[name]()
        codes, scales, sg_gpu, _ = gpu_quantize(W, U)
        W64 = W.double().numpy()
        sg = O.global_scale(W64)
        assert np.float32(sg_gpu.item()) == sg, name
        rows = np.sort(rng.choice(W64.shape[0], ROWS, replace=False))
        c_g = unpack_codes(codes[rows].cpu().numpy())
        s_g = scales[rows].cpu().numpy().astype(np.int64)
        ref = O.schur_replay_gptq(W64[rows], Uo, sg, return_diag=True)
        c = classify(ref, Uo, sg, c_g, s_g, rows)
        report(f"dense_decoder_70b {name}", c)
        assert c["frac"] <= 1e-3, (name, c)
        assert not c["bad_first"], (name, c)
        Q = O.dequant(c_g, s_g, sg).astype(np.float64)
        L_gpu = O.layer_error(W64[rows], Q, H)
        L_ref = O.layer_error(W64[rows], ref["q"], H)
        assert abs(L_gpu - L_ref) <= 1e-4 * L_ref, name


@pytest.fixture(scope="module")
def layer():
    return synth.dense_decoder_layer()


def test_attention_qkv_shared_factor_and_o(layer):
    check_group(layer, "X_attn", ["q", "k", "v"], seed=31)
    check_group(layer, "X_o", ["o"], seed=32)


def test_mlp_gate_up_shared_factor(layer):
    check_group(layer, "X_mlp", ["gate", "up"], seed=33)


def test_down_28672_properties(layer):
    X = layer["X_down"]()
    n_tok, d = X.shape
    H = gpu_hessian(X)
    # sampled entries against exact dot products of the bf16 tokens
    rng = np.random.default_rng(34)
    ii = rng.integers(0, d, 256)
    jj = rng.integers(0, d, 256)
    Xc = X.float()
    xi = Xc[:, ii].double().numpy()
    xj = Xc[:, jj].double().numpy()
    exact = np.einsum("ti,ti->i", xi, xj)
    absum = np.einsum("ti,ti->i", np.abs(xi), np.abs(xj))
    Hs = H[torch.from_numpy(ii).to(DEV), torch.from_numpy(jj).to(DEV)].double().cpu().numpy()
    assert np.all(np.abs(Hs - exact) <= 1e-5 * absum)
    del Xc, X
    U = gpu_prepare(H)
    assert torch.isfinite(U).all().item()
    assert torch.count_nonzero(torch.tril(U, -1)).item() == 0
    assert (torch.diagonal(U) > 0).all().item()
    W = layer["down"]()
    d_out = W.shape[0]
    codes, scales, sg, err = gpu_quantize(W, U)
    del U
    # every block well formed: an all-zero block has scale 0 and codes 0,
    # any other block a positive E4M3 scale code
    sc = scales.to(torch.int32)
    assert int(sc.max().item()) <= 126 and int(sc.min().item()) >= 0
    nz = (sc > 0)
    cd = codes.view(d_out, d // 16, 8)
    assert torch.count_nonzero(cd[~nz]).item() == 0
    assert nz.float().mean().item() > 0.99
    # the layer error through the library against tr(E H E^T) in fp64
    Q = torch.empty((d_out, d), dtype=torch.float32, device=DEV)
    B.nvfp4_dequant(codes, scales, sg, Q)
    Lg = torch.empty(1, dtype=torch.float64, device=DEV)
    wse = B.workspace(B.nvfp4_layer_error_workspace_size(d_out, d), DEV)
    B.nvfp4_layer_error(W.to(DEV), codes, scales, sg, H, Lg, wse)
    torch.cuda.synchronize()
    del wse
    E = W.to(DEV).double() - Q.double()
    del Q
    H64 = H.double()
    L = 0.0
    for r0 in range(0, d_out, 1024):
        Er = E[r0:r0 + 1024]
        L += float((Er @ H64 * Er).sum().item())
    assert abs(Lg.item() - L) <= 1e-6 * L
    assert err.item() > 0
