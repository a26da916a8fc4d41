"""The fp64-accurate Hessian (nvfp4_hessian_accumulate_f64) and the prepare
that reads it (nvfp4_gptq_prepare_f64), against the oracle.

* Exactness: tokens that are small integers give an integer H, which the fp64
  path must reproduce exactly (a ragged token count exercises the padding).
* Accuracy: a lognormal-scaled layer and one with more tokens than one pass
  takes (several passes added in fp64) against the oracle's fp64 Hessian,
  within 1e-12 relative Frobenius.
* Rank-deficient layers end to end: fewer calibration tokens than channels
  give a damped Hessian of condition number 1e4-1e5, where the fp32 storage of
  H alone moves decisions beyond near ties.  With the fp64 Hessian the whole
  chain -- tokens -> H -> U -> codes -- matches the oracle's fp64 solve under
  the near-tie rule of parity.py: the MLP down-projection layer (8192 tokens
  for 14336 channels) and MoE experts with 97 and 266 tokens for 4096 and 1536
  channels.

Method: "Replay the Curvature", Abstract (second-order state from the
calibration activations; GPTQ with Schur Replay).
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


def hessian_f64(X):
    n_tok, d = X.shape
    H = torch.empty((d, d), dtype=torch.float64, device=DEV)
    ws = B.workspace(B.nvfp4_hessian_f64_workspace_size(n_tok, d), DEV)
    B.nvfp4_hessian_accumulate_f64(H, X.to(DEV), ws)
    torch.cuda.synchronize()
    assert B.nvfp4_workspace_status(ws) == 0
    return H


def rel_frob(a, b):
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def test_integer_tokens_give_an_exact_hessian():
    rng = np.random.default_rng(41)
    Xi = rng.integers(-255, 256, size=(300, 256))
    X = torch.from_numpy(Xi.astype(np.float32)).to(torch.bfloat16)   # exact in bf16
    H = hessian_f64(X).cpu().numpy()
    ref = (Xi.T @ Xi).astype(np.float64)
    assert np.array_equal(H, ref)


@pytest.mark.parametrize("n_tok,d", [(1000, 512), (20000, 256)])
def test_fp64_hessian_against_the_oracle(n_tok, d):
    ss = np.random.SeedSequence(42 + d)
    X = synth.lognormal_acts_fast(n_tok, d, 1.5, ss)
    H = hessian_f64(X).cpu().numpy()
    ref = O.hessian(X.double().numpy())
    assert rel_frob(H, ref) < 1e-12
    assert np.array_equal(H, H.T)


def solve_f64(X, Ws):
    """fp64 Hessian -> prepare_f64 -> quantize every W (device results)."""
    d = X.shape[1]
    H = hessian_f64(X)
    U = torch.empty((d, d), dtype=torch.float32, device=DEV)
    wsp = B.workspace(B.nvfp4_prepare_workspace_size(d), DEV)
    B.nvfp4_gptq_prepare_f64(H, 0.01, U, None, None, wsp)
    out = []
    for W in Ws:
        d_out = W.shape[0]
        c = torch.empty((d_out, d // 2), dtype=torch.uint8, device=DEV)
        s = torch.empty((d_out, d // 16), dtype=torch.uint8, device=DEV)
        g = torch.empty(1, dtype=torch.float32, device=DEV)
        wq = B.workspace(B.nvfp4_quantize_workspace_size(d_out, d), DEV)
        B.nvfp4_gptq_schur_replay_quantize(W.to(DEV), U, c, s, g, None, None, wq)
        torch.cuda.synchronize()
        assert B.nvfp4_workspace_status(wq) == 0
        out.append((unpack_codes(c.cpu().numpy()), s.cpu().numpy().astype(np.int64),
                    float(g.item())))
    assert B.nvfp4_workspace_status(wsp) == 0
    return out


def check(label, X, Ws, n_rows, seed):
    Hn = O.hessian(X.double().numpy())
    Hd, _, _ = O.damp(Hn)
    U = O.inverse_cholesky_upper(Hd)
    del Hd
    rng = np.random.default_rng(seed)
    for (name, W), (codes, scales, sg_gpu) in zip(Ws, solve_f64(X, [w for _, w in Ws])):
        W64 = W.double().numpy()
        sg = O.global_scale(W64)
        assert np.float32(sg_gpu) == sg
        rows = np.sort(rng.choice(W64.shape[0], min(n_rows, W64.shape[0]), replace=False))
        ref = O.schur_replay_gptq(W64[rows], U, sg, return_diag=True)
        c = classify(ref, U, sg, codes[rows], scales[rows], rows)
        report(f"{label} {name} end to end with the fp64 Hessian: {len(rows)} rows", c)
        assert c["frac"] <= 1e-3, (name, c)
        assert not c["bad_first"], (name, c)
        Q = O.dequant(codes[rows], scales[rows], sg).astype(np.float64)
        L_gpu = O.layer_error(W64[rows], Q, Hn)
        L_ref = O.layer_error(W64[rows], ref["q"], Hn)
        assert abs(L_gpu - L_ref) <= 1e-4 * L_ref, name


def test_mlp_down_14336_end_to_end_with_fp64_hessian():
    W, X = synth.mlp_down_silu()
    check("mlp_down_silu_4096x14336", X, [("W", W)], 512, 102)


@pytest.mark.parametrize("e", [127, 50])
def test_low_token_experts_end_to_end_with_fp64_hessian(e):
    counts, make = synth.moe_layer()
    ex = make(e)
    n = int(counts[e])
    check(f"moe_128_experts expert {e} ({n} tokens) input", ex["X_in"],
          [("gate", ex["gate"]), ("up", ex["up"])], 256, 3000 + e)
    check(f"moe_128_experts expert {e} ({n} tokens) intermediate", ex["X_mid"],
          [("down", ex["down"])], 256, 4000 + e)
