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

    def hessian_host(self, X_host, chunk_tok=1024, beta=0, stream=None):
        """H from host-resident tokens, streamed through the device in chunks
        (the copy of the next chunk overlaps the Hessian of the current one)."""
        key = (int(chunk_tok), X_host.dtype)
        if getattr(self, "_ws_host_key", None) != key:
            self.ws_host = B.workspace(
                B.nvfp4_hessian_host_workspace_size(self.d_in, chunk_tok, X_host.dtype),
                self.device)
            self._ws_host_key = key
        B.nvfp4_hessian_accumulate_host(self.H, X_host, chunk_tok, self.ws_host, beta, stream)

    def step_host(self, W_host, X_host, W_dev, chunk_tok=1024, stream=None, with_error=True,
                  out_host=None):
        """One whole solve from host-resident inputs: the tokens stream into the
        Hessian chunk by chunk; W is copied into W_dev on a side stream once the
        last token chunk is on the device (so the two copies do not share the
        host link while the Hessian waits), beside the prepare; quantize waits
        for it.  With out_host = (codes_h, scales_h, s_g_h) (pinned host
        tensors) the codes, scales and global scale are read back on the side
        stream as soon as quantize has written them, beside dequant and the
        layer error; the caller's stream waits for that read-back at the end."""
        st = stream if stream is not None else torch.cuda.current_stream(self.device)
        if not hasattr(self, "_side"):
            self._side = torch.cuda.Stream(self.device)
            self._x_done = torch.cuda.Event()
            self._w_ready = torch.cuda.Event()
            self._q_done = torch.cuda.Event()
            self._d2h_done = torch.cuda.Event()
        self.hessian_host(X_host, chunk_tok, 0, st)
        self._x_done.record(st)           # all tokens are on the device (and W_dev is free)
        self._side.wait_event(self._x_done)
        with torch.cuda.stream(self._side):
            W_dev.copy_(W_host, non_blocking=True)
            self._w_ready.record(self._side)
        self.prepare(st)
        st.wait_event(self._w_ready)
        self.quantize(W_dev, st)
        if out_host is not None:
            self._q_done.record(st)
            self._side.wait_event(self._q_done)
            with torch.cuda.stream(self._side):
                codes_h, scales_h, sg_h = out_host
                codes_h.copy_(self.codes, non_blocking=True)
                scales_h.copy_(self.scales, non_blocking=True)
                sg_h.copy_(self.s_g, non_blocking=True)
                self._d2h_done.record(self._side)
        self.dequant(st)
        if with_error:
            self.layer_error(W_dev, st)
        if out_host is not None:
            st.wait_event(self._d2h_done)

    def status(self, stream=None):
        """Device status words of the prepare and quantize workspaces."""
        return (B.nvfp4_workspace_status(self.ws_prep, stream),
                B.nvfp4_workspace_status(self.ws_quant, stream))
