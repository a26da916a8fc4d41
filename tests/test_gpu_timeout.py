"""Failure detection on the GPU without a fault: the bounded waits.

Every pipeline wait inside the library's tensor-core kernels gives up after a
limit that the host sets (nvfp4_set_wait_limit_ns; 4 s by default).  With the
limit at 1 ns a wait gives up as soon as one non-blocking probe finds that what
it waits for has not happened yet -- the first copy of every kernel takes
longer than that -- so each tensor-core kernel of a call runs into the timeout
path: it records NVFP4_ERR_TIMEOUT in the call's status word, waits (with the
fixed 4 s bound) for the copies and MMAs it has already issued, frees its
tensor memory and returns.  The tests check that the status reaches the host
and that the context stays usable: with the default limit back, the same calls
succeed and give the results of a run that never timed out.

Nothing here faults, traps or spins without a bound.
"""
import numpy as np
import pytest
import torch

from nvfp4_post_weight_b200 import binding as B
from nvfp4_post_weight_b200 import synth

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
TIMEOUT = 6   # NVFP4_ERR_TIMEOUT


class tiny_wait_limit:
    """Pipeline-wait limit of 1 ns inside the block, the default after it
    (also when the block raises)."""

    def __enter__(self):
        torch.cuda.synchronize()
        B.nvfp4_set_wait_limit_ns(1)

    def __exit__(self, *a):
        torch.cuda.synchronize()
        B.nvfp4_set_wait_limit_ns(0)


def test_gemm_timeout_is_reported_and_the_context_survives():
    g = torch.Generator(device=DEV).manual_seed(5)
    P = torch.randn((1024, 512), device=DEV, generator=g)
    Q = torch.randn((768, 512), device=DEV, generator=g)
    C = torch.zeros((1024, 768), device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    with tiny_wait_limit():
        B.nvfp4_gemm_nt_f32(P, Q, C, status=status)
    assert status.item() == TIMEOUT
    status.zero_()
    B.nvfp4_gemm_nt_f32(P, Q, C, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    ref = P.double() @ Q.double().T
    assert torch.allclose(C.double(), ref, rtol=1e-5, atol=1e-4)


def test_hessian_timeout_is_reported_then_cleared():
    W, X = synth.small_outlier(d_out=16, d_in=512, n_tok=1024, seed=21)
    Xb = X.to(torch.bfloat16).to(DEV)
    H = torch.empty((512, 512), device=DEV)
    assert B.nvfp4_hessian_status() == 0
    with tiny_wait_limit():
        B.nvfp4_hessian_accumulate(H, Xb)
    assert B.nvfp4_hessian_status() == TIMEOUT
    assert B.nvfp4_hessian_status() == 0          # read and cleared
    B.nvfp4_hessian_accumulate(H, Xb)
    assert B.nvfp4_hessian_status() == 0
    ref = Xb.double().T @ Xb.double()
    assert (torch.linalg.norm(H.double() - ref) / torch.linalg.norm(ref)).item() < 1e-6


def test_layer_solve_timeout_then_same_results():
    """A whole prepare + quantize with every wait timing out reports the
    timeout in both workspaces; afterwards the same calls give exactly the
    results of the undisturbed solve."""
    W, X = synth.attn_massive(d_out=512, d_in=2048, n_tok=1024, seed=22)
    d_out, d_in = W.shape
    Wd = W.to(DEV)
    H = torch.empty((d_in, d_in), device=DEV)
    B.nvfp4_hessian_accumulate(H, X.to(DEV))
    wsp = B.workspace(B.nvfp4_prepare_workspace_size(d_in), DEV)
    wsq = B.workspace(B.nvfp4_quantize_workspace_size(d_out, d_in), DEV)

    def solve():
        U = torch.empty_like(H)
        B.nvfp4_gptq_prepare(H, 0.01, U, None, None, wsp)
        codes = torch.empty((d_out, d_in // 2), dtype=torch.uint8, device=DEV)
        scales = torch.empty((d_out, d_in // 16), dtype=torch.uint8, device=DEV)
        sg = torch.empty(1, device=DEV)
        B.nvfp4_gptq_schur_replay_quantize(Wd, U, codes, scales, sg, None, None, wsq)
        return U, codes, scales

    ref = solve()
    assert B.nvfp4_workspace_status(wsp) == 0 and B.nvfp4_workspace_status(wsq) == 0
    with tiny_wait_limit():
        solve()
    assert B.nvfp4_workspace_status(wsp) == TIMEOUT
    assert B.nvfp4_workspace_status(wsq) == TIMEOUT
    again = solve()
    assert B.nvfp4_workspace_status(wsp) == 0 and B.nvfp4_workspace_status(wsq) == 0
    for a, b in zip(ref, again):
        assert torch.equal(a, b)
    assert np.isfinite(ref[0].cpu().numpy()).all()
