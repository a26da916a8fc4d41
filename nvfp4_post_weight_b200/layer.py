"""Per-layer solve through the C ABI: the calls a user strings together.

LayerSolver owns the device buffers of one layer shape so that repeated solves
(benchmark steps, several weights sharing one Hessian) allocate nothing.
"""
from __future__ import annotations

import torch

from . import binding as B


class LayerSolver:
    """Hessian -> prepare -> Schur Replay quantize -> dequant -> layer error for
    one (d_out, d_in) layer on one CUDA device.  scale_rule picks the block-scale
    rule (binding.SCALE_RULES; Schur Replay by default, the independent-block
    rules for comparison)."""

    def __init__(self, d_out: int, d_in: int, device="cuda", damp: float = 0.01,
                 out_dtype=torch.bfloat16, scale_rule="schur_replay"):
        self.d_out, self.d_in, self.damp = int(d_out), int(d_in), float(damp)
        self.params = B.solve_params(scale_rule)
        dev = torch.device(device)
        self.device = dev
        d = self.d_in
        self.H = torch.empty((d, d), dtype=torch.float32, device=dev)
        self.U = torch.empty((d, d), dtype=torch.float32, device=dev)
        self.dead = torch.empty(d, dtype=torch.uint8, device=dev)
        self.lam = torch.empty(1, dtype=torch.float32, device=dev)
        self.codes = torch.empty((d_out, d // 2), dtype=torch.uint8, device=dev)
        self.scales = torch.empty((d_out, d // 16), dtype=torch.uint8, device=dev)
        self.s_g = torch.empty(1, dtype=torch.float32, device=dev)
        self.err = torch.empty(1, dtype=torch.float64, device=dev)
        self.layer_err = torch.empty(1, dtype=torch.float64, device=dev)
        self.Q = torch.empty((d_out, d), dtype=out_dtype, device=dev)
        self.ws_prep = B.workspace(B.nvfp4_prepare_workspace_size(d), dev)
        self.ws_quant = B.workspace(B.nvfp4_quantize_workspace_size(d_out, d), dev)
        self.ws_err = B.workspace(B.nvfp4_layer_error_workspace_size(d_out, d), dev)

    def hessian(self, X, beta=0, stream=None):
        B.nvfp4_hessian_accumulate(self.H, X, beta, stream)

    def prepare(self, stream=None):
        B.nvfp4_gptq_prepare(self.H, self.damp, self.U, self.dead, self.lam, self.ws_prep, stream)

    def quantize(self, W, stream=None):
        B.nvfp4_gptq_schur_replay_quantize(W, self.U, self.codes, self.scales, self.s_g,
                                           self.err, self.dead, self.ws_quant, self.params,
                                           stream)

    def dequant(self, stream=None):
        B.nvfp4_dequant(self.codes, self.scales, self.s_g, self.Q, stream)

    def layer_error(self, W, stream=None):
        B.nvfp4_layer_error(W, self.codes, self.scales, self.s_g, self.H, self.layer_err,
                            self.ws_err, stream)

    def step(self, W, X, stream=None, with_error=True):
        """One whole solve of the layer from its weights and calibration
        activations (both already on the device)."""
        self.hessian(X, 0, stream)
        self.prepare(stream)
        self.quantize(W, stream)
        self.dequant(stream)
        if with_error:
            self.layer_error(W, stream)

    def status(self, stream=None):
        """Device status words of the prepare and quantize workspaces."""
        return (B.nvfp4_workspace_status(self.ws_prep, stream),
                B.nvfp4_workspace_status(self.ws_quant, stream))
