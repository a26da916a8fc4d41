"""GPU tests of the row-shard entry points (nvfp4_weight_amax,
nvfp4_gptq_schur_replay_quantize_rows): the 4096 x 4096 layer quantized as
three row shards with the layer's amax must give the whole-layer call's codes,
scales and global scale bit for bit (rows are independent given U), and the
shards' sums of delta^2 and layer errors must add up to the whole layer's.
The shards run one after another on this GPU: the collectives of a real
multi-GPU run are scalar reductions of the host (MAX of the amax, SUM of the
errors), done here by hand.  A one-rank NCCL group runs ShardedLayerSolver's
own path end to end.

Method: "Replay the Curvature", Abstract, infrastructure sentence (independent
output rows distributed across tensor-parallel ranks).
"""
import os

import numpy as np
import pytest
import torch

from nvfp4_post_weight_b200 import binding as B
from nvfp4_post_weight_b200 import synth
from nvfp4_post_weight_b200.layer import LayerSolver
from nvfp4_post_weight_b200.sharded import ShardedLayerSolver, row_range

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module")
def whole():
    W, X = synth.attn_massive()
    s = LayerSolver(*W.shape, DEV, out_dtype=torch.bfloat16)
    s.step(W.to(DEV), X.to(DEV))
    torch.cuda.synchronize()
    assert s.status() == (0, 0)
    return W, X, s


def test_weight_amax(whole):
    W, _, s = whole
    a = torch.empty(1, dtype=torch.float32, device=DEV)
    B.nvfp4_weight_amax(W.to(DEV), a)
    torch.cuda.synchronize()
    assert a.item() == W.float().abs().max().item()
    B.nvfp4_weight_amax(torch.empty((0, 16), dtype=torch.bfloat16, device=DEV), a)
    torch.cuda.synchronize()
    assert a.item() == 0.0


def test_row_shards_equal_whole_layer(whole):
    W, _, s = whole
    d_out, d_in = W.shape
    Wd = W.to(DEV)
    world = 3
    amaxes = []
    for r in range(world):
        r0, r1 = row_range(d_out, r, world)
        a = torch.empty(1, dtype=torch.float32, device=DEV)
        B.nvfp4_weight_amax(Wd[r0:r1], a, s.dead)
        amaxes.append(a)
    amax = torch.stack(amaxes).max().reshape(1)            # the MAX all-reduce
    codes, scales, err_sum, lerr_sum = [], [], 0.0, 0.0
    for r in range(world):
        r0, r1 = row_range(d_out, r, world)
        sh = LayerSolver(r1 - r0, d_in, DEV, out_dtype=torch.bfloat16)
        sh.U, sh.dead, sh.H = s.U, s.dead, s.H             # the shared factor
        B.nvfp4_gptq_schur_replay_quantize_rows(Wd[r0:r1], s.U, amax, sh.codes, sh.scales,
                                                sh.s_g, sh.err, s.dead, sh.ws_quant)
        sh.layer_error(Wd[r0:r1])
        torch.cuda.synchronize()
        assert B.nvfp4_workspace_status(sh.ws_quant) == 0
        assert sh.s_g.item() == s.s_g.item()
        codes.append(sh.codes.cpu())
        scales.append(sh.scales.cpu())
        err_sum += sh.err.item()
        lerr_sum += sh.layer_err.item()
    assert torch.equal(torch.cat(codes), s.codes.cpu())
    assert torch.equal(torch.cat(scales), s.scales.cpu())
    assert err_sum == pytest.approx(s.err.item(), rel=1e-12)
    assert lerr_sum == pytest.approx(s.layer_err.item(), rel=1e-6)


def test_sharded_solver_one_rank_nccl(whole):
    import torch.distributed as tdist
    W, X, s = whole
    os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
    os.environ.setdefault("MASTER_PORT", str(29800 + os.getpid() % 1000))
    tdist.init_process_group("nccl", rank=0, world_size=1)
    try:
        sh = ShardedLayerSolver(*W.shape, device=DEV)
        sh.step(W.to(DEV), X.to(DEV), tokens_split=True)
        codes, scales = sh.gather()
        torch.cuda.synchronize()
        assert sh.backend.status() == (0, 0)
        assert torch.equal(codes.cpu(), s.codes.cpu()) and torch.equal(scales.cpu(), s.scales.cpu())
        assert sh.layer_err.item() == pytest.approx(s.layer_err.item(), rel=1e-12)
    finally:
        tdist.destroy_process_group()
