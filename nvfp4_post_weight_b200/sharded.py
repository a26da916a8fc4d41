"""Row-sharded solve of one layer over the ranks of a torch.distributed group.

"Replay the Curvature", Abstract, infrastructure sentence: independent output
rows are distributed across tensor-parallel ranks.  Given the factor U the
rows of the GPTQ solve are independent, so rank r quantizes the contiguous
rows [r0, r1) of W and the ranks exchange only:

  * the Hessian, when the calibration tokens are split over the ranks
    (all-reduce SUM of each rank's X_r^T X_r; with every rank holding all
    tokens there is no exchange);
  * the layer's max |W| (all-reduce MAX of a scalar): the global scale is the
    layer's, not the shard's;
  * the layer error and sum of delta^2 (all-reduce SUM of two scalars);
  * optionally the codes and scales (all-gather), for a rank that needs the
    whole layer.

Every rank prepares U from the same reduced H itself (the prepare is
deterministic, so all ranks hold the same U) instead of receiving it: no
64 MB broadcast, and the prepare is not the part that shards.

The per-rank compute goes through a backend object; the default one is the
CUDA library (LayerSolver and the row-shard entry points of the C ABI).
"""
from __future__ import annotations

import torch
import torch.distributed as tdist

from . import binding as B
from .layer import LayerSolver


def row_range(d_out: int, rank: int, world: int):
    """Contiguous, balanced row range [r0, r1) of `rank` among `world` ranks."""
    base, extra = divmod(int(d_out), int(world))
    r0 = rank * base + min(rank, extra)
    return r0, r0 + base + (1 if rank < extra else 0)


class CudaBackend:
    """The per-rank compute on this rank's GPU through the C ABI."""

    def __init__(self, rows: int, d_in: int, device, out_dtype=torch.bfloat16):
        self.s = LayerSolver(rows, d_in, device, out_dtype=out_dtype)
        self.device = self.s.device
        self.amax = torch.empty(1, dtype=torch.float32, device=self.device)

    def hessian(self, X):
        self.s.hessian(X)
        return self.s.H

    def prepare(self, H):
        self.s.prepare()

    def weight_amax(self, W):
        B.nvfp4_weight_amax(W, self.amax, self.s.dead)
        return self.amax

    def quantize_rows(self, W, amax):
        s = self.s
        B.nvfp4_gptq_schur_replay_quantize_rows(W, s.U, amax, s.codes, s.scales, s.s_g, s.err,
                                                s.dead, s.ws_quant, s.params)
        s.dequant()
        s.layer_error(W)
        return s.codes, s.scales, s.s_g, s.err, s.layer_err

    def status(self):
        return self.s.status()


class ShardedLayerSolver:
    """One layer (d_out x d_in) solved with its rows split over the group."""

    def __init__(self, d_out: int, d_in: int, group=None, device=None, backend=None,
                 out_dtype=torch.bfloat16):
        self.group = group
        self.rank = tdist.get_rank(group)
        self.world = tdist.get_world_size(group)
        self.d_out, self.d_in = int(d_out), int(d_in)
        self.r0, self.r1 = row_range(d_out, self.rank, self.world)
        self.backend = backend if backend is not None else CudaBackend(
            self.r1 - self.r0, d_in, device, out_dtype)

    def step(self, W_rows, X, tokens_split: bool = True):
        """W_rows: this rank's rows [r0, r1) of W; X: this rank's tokens (its
        share of the calibration set when tokens_split, else all of them).
        Returns (codes, scales, s_g, sum delta^2, layer error) with the last two
        summed over the group."""
        H = self.backend.hessian(X)
        if tokens_split and self.world > 1:
            tdist.all_reduce(H, op=tdist.ReduceOp.SUM, group=self.group)
        self.backend.prepare(H)
        amax = self.backend.weight_amax(W_rows)
        if self.world > 1:
            tdist.all_reduce(amax, op=tdist.ReduceOp.MAX, group=self.group)
        codes, scales, sg, err, lerr = self.backend.quantize_rows(W_rows, amax)
        tot = torch.cat([err.reshape(1).double(), lerr.reshape(1).double()])
        if self.world > 1:
            tdist.all_reduce(tot, op=tdist.ReduceOp.SUM, group=self.group)
        self.codes, self.scales, self.s_g = codes, scales, sg
        self.err, self.layer_err = tot[0], tot[1]
        return codes, scales, sg, tot[0], tot[1]

    def gather(self):
        """The whole layer's codes and scales on every rank (all-gather of the
        row shards, padded to the largest shard)."""
        rows = self.r1 - self.r0
        pad = -(-self.d_out // self.world)
        out = []
        for t in (self.codes, self.scales):
            buf = torch.zeros((pad,) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device)
            buf[:rows] = t
            parts = [torch.empty_like(buf) for _ in range(self.world)]
            tdist.all_gather(parts, buf, group=self.group)
            out.append(torch.cat([p[:row_range(self.d_out, r, self.world)[1] -
                                   row_range(self.d_out, r, self.world)[0]]
                                  for r, p in enumerate(parts)]))
        return out[0], out[1]
