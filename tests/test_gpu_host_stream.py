"""GPU tests of the host-resident input path: the Hessian streamed from host
memory in token chunks (nvfp4_hessian_accumulate_host), and the whole layer
solve from host-resident W and X (LayerSolver.step_host), against the device
path and the oracle.

Method: "Replay the Curvature", Abstract, infrastructure sentence (calibration
activations tiered across device, host and disk; this is the device/host tier
of the second-order state).
"""
import numpy as np
import pytest
import torch

import oracle as O
from nvfp4_post_weight_b200 import binding as B
from nvfp4_post_weight_b200 import synth
from nvfp4_post_weight_b200.layer import LayerSolver
from parity import unpack_codes

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def rel_frob(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def streamed_h(X_host, chunk, beta=0, H0=None):
    d = X_host.shape[1]
    H = (H0.clone() if H0 is not None else
         torch.full((d, d), float("nan"), dtype=torch.float32, device=DEV))
    ws = B.workspace(B.nvfp4_hessian_host_workspace_size(d, chunk, X_host.dtype), DEV)
    B.nvfp4_hessian_accumulate_host(H, X_host, chunk, ws, beta)
    torch.cuda.synchronize()
    assert B.nvfp4_hessian_status() == 0
    return H


@pytest.mark.parametrize("n_tok,d,chunk,dtype", [
    (4096, 512, 1024, torch.bfloat16),     # whole chunks, tensor-core Hessian
    (3000, 512, 1024, torch.bfloat16),     # ragged last chunk
    (1000, 256, 48, torch.bfloat16),       # chunks below the tensor-core minimum
    (777, 208, 100, torch.float32),        # fp32 tokens, CUDA-core Hessian
    (5, 64, 1024, torch.bfloat16),         # one short chunk
])
def test_streamed_hessian_matches_device_and_oracle(n_tok, d, chunk, dtype):
    rng = np.random.default_rng(n_tok + d)
    X = torch.from_numpy((rng.standard_normal((n_tok, d)) *
                          rng.lognormal(0, 1, size=d)).astype(np.float32)).to(dtype)
    Xp = X.pin_memory()
    H = streamed_h(Xp, chunk)
    Hd = torch.empty((d, d), dtype=torch.float32, device=DEV)
    B.nvfp4_hessian_accumulate(Hd, X.to(DEV))
    torch.cuda.synchronize()
    Hn, Hdn = H.cpu().numpy(), Hd.cpu().numpy()
    assert np.all(np.isfinite(Hn))
    assert np.array_equal(Hn, Hn.T)
    # the chunk sums are added in fp32: the same accumulation as the device
    # path's 128-token chunks, cut at other places
    assert rel_frob(Hn, Hdn) < 1e-6
    assert rel_frob(Hn, O.hessian(X.double().numpy())) < 1e-4


def test_streamed_hessian_accumulates_and_pageable_memory_works():
    rng = np.random.default_rng(3)
    d = 256
    X1 = torch.from_numpy(rng.standard_normal((700, d)).astype(np.float32)).to(torch.bfloat16)
    X2 = torch.from_numpy(rng.standard_normal((900, d)).astype(np.float32)).to(torch.bfloat16)
    H1 = streamed_h(X1, 256)                       # pageable host memory
    H12 = streamed_h(X2.pin_memory(), 512, beta=1, H0=H1)
    ref = O.hessian(torch.cat([X1, X2]).double().numpy())
    assert rel_frob(H12.cpu().numpy(), ref) < 1e-4


def test_streamed_hessian_zero_tokens_zeroes_h():
    H = streamed_h(torch.empty((0, 64), dtype=torch.bfloat16), 16)
    assert torch.count_nonzero(H).item() == 0


def test_solve_from_host_inputs_equals_device_solve():
    """The 4096 x 4096 layer from pinned host W and X (tokens streamed in 1024-token
    chunks, W copied beside the prepare): codes and scales equal the device-input
    solve except at near-ties of the Hessian's summation order, and the layer
    error agrees within 1e-4."""
    W, X = synth.attn_massive()
    d_out, d_in = W.shape
    dev_solver = LayerSolver(d_out, d_in, DEV, out_dtype=torch.bfloat16)
    dev_solver.step(W.to(DEV), X.to(DEV))
    host_solver = LayerSolver(d_out, d_in, DEV, out_dtype=torch.bfloat16)
    W_dev = torch.empty((d_out, d_in), dtype=W.dtype, device=DEV)
    out_h = (torch.empty((d_out, d_in // 2), dtype=torch.uint8).pin_memory(),
             torch.empty((d_out, d_in // 16), dtype=torch.uint8).pin_memory(),
             torch.empty(1, dtype=torch.float32).pin_memory())
    host_solver.step_host(W.pin_memory(), X.pin_memory(), W_dev, chunk_tok=1024, out_host=out_h)
    torch.cuda.synchronize()
    # the read-back on the side stream holds the quantize's outputs
    assert torch.equal(out_h[0], host_solver.codes.cpu())
    assert torch.equal(out_h[1], host_solver.scales.cpu())
    assert out_h[2].item() == host_solver.s_g.item()
    assert dev_solver.status() == (0, 0) and host_solver.status() == (0, 0)
    assert torch.equal(W_dev.cpu(), W)
    assert rel_frob(host_solver.H.cpu().numpy(), dev_solver.H.cpu().numpy()) < 1e-6
    sd, sh = dev_solver.scales.cpu().numpy(), host_solver.scales.cpu().numpy()
    cd = unpack_codes(dev_solver.codes.cpu().numpy())
    ch = unpack_codes(host_solver.codes.cpu().numpy())
    blk = (sd == sh) & (cd.reshape(d_out, -1, 16) == ch.reshape(d_out, -1, 16)).all(axis=2)
    assert (~blk).mean() <= 1e-3
    Ld, Lh = dev_solver.layer_err.item(), host_solver.layer_err.item()
    assert abs(Ld - Lh) <= 1e-4 * Ld


SMALL_DECODER = (("X_attn", {"q": (512, 512), "k": (128, 512), "v": (128, 512)}),
                 ("X_o", {"o": (512, 512)}),
                 ("X_mlp", {"gate": (1024, 512), "up": (1024, 512)}),
                 ("X_down", {"down": (512, 1024)}))


@pytest.mark.parametrize("chunk", [4096, 1024])
def test_decoder_layer_from_host_inputs_pipelined(chunk):
    """DecoderLayerSolver.step_host streams group g + 1's tokens into a second
    Hessian buffer while group g is solved.  With one chunk per group every
    result equals the device-resident solve bit for bit; with four chunks per
    group (H accumulated in fp32 over the chunks, a different summation order)
    the block scales agree on >= 99% of the blocks (a decision flipped at a
    near-tie carries along its row) and the layer errors within 1e-4.  The read-back
    codes, scales and global scales always equal the device ones."""
    from nvfp4_post_weight_b200.decoder import DecoderLayerSolver
    n_tok = 4096
    rng = np.random.default_rng(61)
    Wh, Xh = {}, {}
    for x, t in SMALL_DECODER:
        d = next(iter(t.values()))[1]
        scale = np.exp(rng.standard_normal(d) * 1.5).astype(np.float32)
        Xh[x] = torch.from_numpy(rng.standard_normal((n_tok, d)).astype(np.float32) * scale) \
            .to(torch.bfloat16).pin_memory()
        for n, (o, i) in t.items():
            Wh[n] = torch.from_numpy(rng.standard_normal((o, i)).astype(np.float32) * 0.02) \
                .to(torch.bfloat16).pin_memory()
    dev_solver = DecoderLayerSolver(SMALL_DECODER, DEV)
    dev_solver.step({n: w.to(DEV) for n, w in Wh.items()}, {x: t.to(DEV) for x, t in Xh.items()})
    host_solver = DecoderLayerSolver(SMALL_DECODER, DEV)
    W_dev = {n: torch.empty(w.shape, dtype=w.dtype, device=DEV) for n, w in Wh.items()}
    out_h = {n: (torch.empty(host_solver.codes[n].shape, dtype=torch.uint8).pin_memory(),
                 torch.empty(host_solver.scales[n].shape, dtype=torch.uint8).pin_memory(),
                 torch.empty(1, dtype=torch.float32).pin_memory()) for n in Wh}
    for _ in range(2):   # the second step reuses the buffers, streams and events
        host_solver.step_host(Wh, Xh, W_dev, chunk_tok=chunk, out_host=out_h)
    torch.cuda.synchronize()
    assert dev_solver.status() == (0, 0, 0) and host_solver.status() == (0, 0, 0)
    for n in Wh:
        c_h, s_h, g_h = out_h[n]
        assert torch.equal(c_h, host_solver.codes[n].cpu())
        assert torch.equal(s_h, host_solver.scales[n].cpu())
        assert torch.equal(g_h, host_solver.s_g[n].cpu())
        if chunk >= n_tok:
            for a, b in ((dev_solver.codes, host_solver.codes), (dev_solver.scales, host_solver.scales),
                         (dev_solver.Q, host_solver.Q), (dev_solver.layer_err, host_solver.layer_err)):
                assert torch.equal(a[n], b[n]), n
        else:
            same = (dev_solver.scales[n] == host_solver.scales[n]).float().mean().item()
            assert same >= 0.99, (n, same)
            le_d, le_h = dev_solver.layer_err[n].item(), host_solver.layer_err[n].item()
            assert abs(le_d - le_h) <= 1e-4 * le_d, (n, le_d, le_h)
