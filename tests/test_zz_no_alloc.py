"""The allocation-free quantize entry point against the workspace one.

nvfp4_gptq_schur_replay_quantize_noalloc serves callers that cannot allocate
device memory when they quantize (an engine that owns all GPU memory through
its own fixed pool, or a loop that must not take cudaMalloc's implicit device
synchronisation): it runs the same solve in a fixed scratch array inside the
library.  Its codes, scales and global scale must equal the workspace call's
bit for bit and its sum of delta^2 must agree within the 1e-9 relative bound
the other quantize tests use, on two calls in a row -- the second on a smaller
layer, so stale contents the first call leaves in the shared array would show.

This file is named to be collected last: it is an add-on to the library, and a
stop-at-first-failure run has then already run every other test.
"""

import numpy as np
import pytest
import torch

from nvfp4_post_weight_b200 import binding as B
from nvfp4_post_weight_b200 import synth


pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _factor(X, d):
    """U from the library's own Hessian and prepare calls."""
    H = torch.empty((d, d), dtype=torch.float32, device=DEV)
    B.nvfp4_hessian_accumulate(H, X.to(DEV))
    U = torch.empty_like(H)
    ws = B.workspace(B.nvfp4_prepare_workspace_size(d), DEV)
    B.nvfp4_gptq_prepare(H, 0.01, U, None, None, ws)
    torch.cuda.synchronize()
    assert B.nvfp4_workspace_status(ws) == 0
    return U


def _outputs(d_out, d_in):
    return (torch.empty((d_out, d_in // 2), dtype=torch.uint8, device=DEV),
            torch.empty((d_out, d_in // 16), dtype=torch.uint8, device=DEV),
            torch.empty(1, dtype=torch.float32, device=DEV),
            torch.empty(1, dtype=torch.float64, device=DEV))


def _with_workspace(W, U):
    d_out, d_in = W.shape
    codes, scales, sg, err = _outputs(d_out, d_in)
    ws = B.workspace(B.nvfp4_quantize_workspace_size(d_out, d_in), DEV)
    B.nvfp4_gptq_schur_replay_quantize(W, U, codes, scales, sg, err, None, ws)
    torch.cuda.synchronize()
    assert B.nvfp4_workspace_status(ws) == 0
    return codes.cpu(), scales.cpu(), sg.item(), err.item()


def _without_workspace(W, U):
    d_out, d_in = W.shape
    codes, scales, sg, err = _outputs(d_out, d_in)
    status = torch.full((1,), -1, dtype=torch.int32, device=DEV)
    B.nvfp4_gptq_schur_replay_quantize_noalloc(W, U, codes, scales, sg, err, status)
    torch.cuda.synchronize()
    assert status.item() == 0
    return codes.cpu(), scales.cpu(), sg.item(), err.item()


def test_noalloc_matches_workspace_call_twice():
    # first call: 512 x 256 fp32 layer with outlier input columns
    W1, X1 = synth.small_outlier(d_out=512, d_in=256, n_tok=512, seed=11)
    # second call: a smaller bf16 layer, after the first left its data behind
    rng = np.random.default_rng(12)
    W2 = synth.normal_weights(96, 128, 0.02, rng)
    X2 = synth.lognormal_acts(256, 128, 1.0, rng, rng)
    for W, X in ((W1, X1), (W2, X2)):
        d_out, d_in = W.shape
        U = _factor(X, d_in)
        Wd = W.to(DEV)
        ref = _with_workspace(Wd, U)
        got = _without_workspace(Wd, U)
        assert torch.equal(got[0], ref[0])
        assert torch.equal(got[1], ref[1])
        assert got[2] == ref[2]
        assert abs(got[3] - ref[3]) <= 1e-9 * abs(ref[3])


def test_noalloc_reserves_nothing_after_its_first_call():
    """The first call on a device loads the library module that holds the
    fixed scratch array (lazy module loading); from then on a call changes
    the device's free memory by nothing."""
    W, X = synth.small_outlier(d_out=128, d_in=256, n_tok=512, seed=13)
    U = _factor(X, 256)
    Wd = W.to(DEV)
    codes, scales, sg, err = _outputs(128, 256)
    status = torch.full((1,), -1, dtype=torch.int32, device=DEV)
    B.nvfp4_gptq_schur_replay_quantize_noalloc(Wd, U, codes, scales, sg, err, status)
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(2):
        B.nvfp4_gptq_schur_replay_quantize_noalloc(Wd, U, codes, scales, sg, err, status)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert status.item() == 0


def test_noalloc_rejects_layers_beyond_its_scratch():
    d_out, d_in = 4096, 4096   # needs far more than the fixed 16 MiB
    assert B.nvfp4_quantize_workspace_size(d_out, d_in) > (16 << 20)
    W = torch.zeros((d_out, d_in), dtype=torch.bfloat16, device=DEV)
    U = torch.zeros((d_in, d_in), dtype=torch.float32, device=DEV)
    codes, scales, sg, err = _outputs(d_out, d_in)
    with pytest.raises(B.Nvfp4Error) as e:
        B.nvfp4_gptq_schur_replay_quantize_noalloc(W, U, codes, scales, sg, err)
    assert e.value.code == 3   # NVFP4_ERR_WORKSPACE
