"""The debug build (libnvfp4pw_debug.so, compiled with NVFP4_DEBUG: the
tensor-core kernels check every tile their decomposition hands out against
the output before touching it and record NVFP4_ERR_BOUNDS otherwise) runs the
whole solve with no check failing and gives exactly the release build's
results: on a layer with ragged rows, on one wide enough for the int8-slice
engine and the super-batch 3xTF32 update, and on a batched group of three
problems of different sizes.  This stands in for a memory checker, which is
not available here."""
import numpy as np
import pytest
import torch

from nvfp4_post_weight_b200 import binding as B
from nvfp4_post_weight_b200 import synth
from nvfp4_post_weight_b200.layer import LayerSolver

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def solve(W, X):
    s = LayerSolver(W.shape[0], W.shape[1], DEV)
    s.step(W.to(DEV), X.to(DEV))
    torch.cuda.synchronize()
    st = s.status()
    return st, [t.clone() for t in (s.H, s.U, s.codes, s.scales, s.s_g, s.Q, s.layer_err)]


def with_library(monkeypatch, L, fn, *args):
    monkeypatch.setattr(B, "_lib", L)
    try:
        return fn(*args)
    finally:
        monkeypatch.undo()


@pytest.mark.parametrize("d_out,d_in,n_tok", [(33, 272, 300), (1000, 2080, 2500)])
def test_debug_build_solves_like_the_release_build(monkeypatch, d_out, d_in, n_tok):
    assert B.lib().nvfp4_debug_build() == 0
    D = B.debug_lib()
    assert D.nvfp4_debug_build() == 1
    W, X = synth.attn_massive(d_out=d_out, d_in=d_in, n_tok=n_tok, seed=31)
    st_r, out_r = solve(W, X)
    st_d, out_d = with_library(monkeypatch, D, solve, W, X)
    assert st_r == (0, 0) and st_d == (0, 0), (st_r, st_d)
    assert D.nvfp4_hessian_status(None) == 0
    for a, b in zip(out_r, out_d):
        assert torch.equal(a, b)


def test_debug_build_batched_group(monkeypatch):
    """Three problems of different sizes through the batched calls (grouped
    launches, ragged token counts)."""
    shapes = [(64, 512, 700), (48, 512, 97), (40, 1040, 1500)]
    data = [synth.attn_massive(d_out=o, d_in=i, n_tok=n, seed=40 + k)
            for k, (o, i, n) in enumerate(shapes)]

    def run():
        Hs = [torch.empty((W.shape[1],) * 2, device=DEV) for W, _ in data]
        B.nvfp4_hessian_accumulate_batched(Hs, [X.to(DEV) for _, X in data])
        Us = [torch.empty_like(h) for h in Hs]
        ds = [h.shape[0] for h in Hs]
        wsp = B.workspace(B.nvfp4_prepare_batched_workspace_size(ds), DEV)
        B.nvfp4_gptq_prepare_batched(Hs, 0.01, Us, ws=wsp)
        torch.cuda.synchronize()
        assert B.nvfp4_batched_workspace_status(wsp, len(Hs))[0] == 0
        assert B.nvfp4_hessian_status() == 0
        return [h.clone() for h in Hs] + [u.clone() for u in Us]

    ref = run()
    got = with_library(monkeypatch, B.debug_lib(), run)
    for a, b in zip(ref, got):
        assert torch.equal(a, b)
