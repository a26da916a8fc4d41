"""Whole-layer solves through the C ABI: a dense decoder layer whose linears
are solved in sequence with shared Hessians, and a mixture-of-experts layer
whose experts are solved together through the batched calls.

"Replay the Curvature", Abstract: every linear layer is quantized with GPTQ
and Schur Replay from its own second-order state H = X^T X; linears that read
the same input (q/k/v, gate/up) share one H and therefore one factor U, and
each tensor keeps its own global scale.  The experts of an MoE layer are
independent linear layers, each with its own H.

Both solvers own every device buffer they need, so repeated solves allocate
nothing; the big scratch buffers (prepare, quantize and layer-error
workspaces) are shared by the groups, which run one after another.
"""
from __future__ import annotations

import torch

from . import binding as B


def _flat(nbytes: int, device) -> torch.Tensor:
    return B.workspace(nbytes, device)


class DecoderLayerSolver:
    """groups: sequence of (x_name, {tensor name: (d_out, d_in)}) in solve
    order; all tensors of a group share its input dimension d_in and thus one
    Hessian and one factor.  step(Ws, Xs) solves the whole layer: per group
    Hessian -> prepare -> quantize each tensor -> dequant -> layer error."""

    def __init__(self, groups, device="cuda", damp: float = 0.01,
                 out_dtype=torch.bfloat16, scale_rule="schur_replay"):
        dev = torch.device(device)
        self.device = dev
        self.damp = float(damp)
        self.params = B.solve_params(scale_rule)
        self.groups = [(x, dict(t)) for x, t in groups]
        for x, t in self.groups:
            d_ins = {s[1] for s in t.values()}
            if len(d_ins) != 1:
                raise ValueError(f"group {x}: tensors must share d_in, got {d_ins}")
        self.shapes = {n: s for _, t in self.groups for n, s in t.items()}
        dmax = max(s[1] for s in self.shapes.values())
        self.dmax = dmax
        self._H = torch.empty(dmax * dmax, dtype=torch.float32, device=dev)
        self._U = torch.empty(dmax * dmax, dtype=torch.float32, device=dev)
        self.dead = torch.empty(dmax, dtype=torch.uint8, device=dev)
        self.lam = torch.empty(1, dtype=torch.float32, device=dev)
        self.ws_prep = _flat(max(B.nvfp4_prepare_workspace_size(d)
                                 for d in {s[1] for s in self.shapes.values()}), dev)
        self.ws_quant = _flat(max(B.nvfp4_quantize_workspace_size(*s)
                                  for s in self.shapes.values()), dev)
        self.ws_err = _flat(max(B.nvfp4_layer_error_workspace_size(*s)
                                for s in self.shapes.values()), dev)
        self.codes, self.scales, self.s_g, self.err, self.layer_err, self.Q = {}, {}, {}, {}, {}, {}
        for n, (d_out, d_in) in self.shapes.items():
            self.codes[n] = torch.empty((d_out, d_in // 2), dtype=torch.uint8, device=dev)
            self.scales[n] = torch.empty((d_out, d_in // 16), dtype=torch.uint8, device=dev)
            self.s_g[n] = torch.empty(1, dtype=torch.float32, device=dev)
            self.err[n] = torch.empty(1, dtype=torch.float64, device=dev)
            self.layer_err[n] = torch.empty(1, dtype=torch.float64, device=dev)
            self.Q[n] = torch.empty((d_out, d_in), dtype=out_dtype, device=dev)

    def H(self, d):
        return self._H[:d * d].view(d, d)

    def U(self, d):
        return self._U[:d * d].view(d, d)

    def solve_group(self, tensors, W, stream=None, with_error=True):
        """Prepare the factor of the Hessian already in H(d), then quantize,
        dequantize (and measure) every tensor of the group."""
        d = self.shapes[tensors[0]][1]
        H, U = self.H(d), self.U(d)
        B.nvfp4_gptq_prepare(H, self.damp, U, self.dead[:d], self.lam, self.ws_prep, stream)
        for n in tensors:
            B.nvfp4_gptq_schur_replay_quantize(W[n], U, self.codes[n], self.scales[n],
                                               self.s_g[n], self.err[n], self.dead[:d],
                                               self.ws_quant, self.params, stream)
            B.nvfp4_dequant(self.codes[n], self.scales[n], self.s_g[n], self.Q[n], stream)
            if with_error:
                B.nvfp4_layer_error(W[n], self.codes[n], self.scales[n], self.s_g[n], H,
                                    self.layer_err[n], self.ws_err, stream)

    def step(self, W, X, stream=None, with_error=True):
        """W: {tensor name: device weights}, X: {x name: device tokens}."""
        for x, t in self.groups:
            d = next(iter(t.values()))[1]
            B.nvfp4_hessian_accumulate(self.H(d), X[x], 0, stream)
            self.solve_group(list(t), W, stream, with_error)

    def step_host(self, W_host, X_host, W_dev, chunk_tok=8192, stream=None, with_error=True,
                  out_host=None):
        """The same solve from host-resident (pinned) inputs, pipelined across
        the groups: the tokens of group g + 1 stream into a second Hessian
        buffer (the library's host-streamed Hessian, chunk_tok tokens per
        chunk, on a Hessian stream) while group g is factored and quantized on
        the caller's stream; a group's weights are copied into W_dev (device
        tensors of the same shapes) on a side stream once its tokens are on the
        device, beside its prepare.  With out_host = {name: (codes_h,
        scales_h, s_g_h)} the results are read back on the side stream as soon
        as each quantize has written them.  The caller's stream waits for all
        of it at the end.  (Groups alternate between the two Hessian buffers;
        H(d) afterwards holds group 0's, 2's, ... Hessian, not necessarily the
        last one.)"""
        st = stream if stream is not None else torch.cuda.current_stream(self.device)
        if not hasattr(self, "_side"):
            self._side = torch.cuda.Stream(self.device)   # weights in, results out
            self._hst = torch.cuda.Stream(self.device)    # tokens into the Hessians
            self._ev = {}
        if not hasattr(self, "_H2"):
            self._H2 = torch.empty_like(self._H)
        ev = self._ev

        def event(key):
            if key not in ev:
                ev[key] = torch.cuda.Event()
            return ev[key]

        key = int(chunk_tok)
        if getattr(self, "_ws_host_key", None) != key:
            self.ws_host = B.workspace(
                B.nvfp4_hessian_host_workspace_size(self.dmax, chunk_tok, torch.bfloat16),
                self.device)
            self._ws_host_key = key
        groups = self.groups
        dims = [next(iter(t.values()))[1] for _, t in groups]
        bufs = (self._H, self._H2)

        def hbuf(i):
            return bufs[i % 2][:dims[i] * dims[i]].view(dims[i], dims[i])

        # the Hessian stream starts after what the caller queued before
        event("start").record(st)
        self._hst.wait_event(event("start"))

        def hessian(i):
            if i >= 2:   # the buffer's last reader: group i - 2's layer errors
                self._hst.wait_event(event(("done", i - 2)))
            B.nvfp4_hessian_accumulate_host(hbuf(i), X_host[groups[i][0]], chunk_tok,
                                            self.ws_host, 0, self._hst)
            event(("h", i)).record(self._hst)

        hessian(0)
        for i, (x, t) in enumerate(groups):
            if i + 1 < len(groups):
                hessian(i + 1)
            d = dims[i]
            H, U = hbuf(i), self.U(d)
            self._side.wait_event(event(("h", i)))
            with torch.cuda.stream(self._side):
                for n in t:
                    W_dev[n].copy_(W_host[n], non_blocking=True)
                event(("w", i)).record(self._side)
            st.wait_event(event(("h", i)))
            B.nvfp4_gptq_prepare(H, self.damp, U, self.dead[:d], self.lam, self.ws_prep, st)
            st.wait_event(event(("w", i)))
            for n in t:
                B.nvfp4_gptq_schur_replay_quantize(W_dev[n], U, self.codes[n], self.scales[n],
                                                   self.s_g[n], self.err[n], self.dead[:d],
                                                   self.ws_quant, self.params, st)
                if out_host is not None:
                    event(("q", n)).record(st)
                    self._side.wait_event(event(("q", n)))
                    with torch.cuda.stream(self._side):
                        c_h, s_h, g_h = out_host[n]
                        c_h.copy_(self.codes[n], non_blocking=True)
                        s_h.copy_(self.scales[n], non_blocking=True)
                        g_h.copy_(self.s_g[n], non_blocking=True)
                B.nvfp4_dequant(self.codes[n], self.scales[n], self.s_g[n], self.Q[n], st)
                if with_error:
                    B.nvfp4_layer_error(W_dev[n], self.codes[n], self.scales[n], self.s_g[n], H,
                                        self.layer_err[n], self.ws_err, st)
            event(("done", i)).record(st)
        event("side").record(self._side)
        st.wait_event(event("side"))
        event("hst").record(self._hst)
        st.wait_event(event("hst"))

    def status(self, stream=None):
        return (B.nvfp4_workspace_status(self.ws_prep, stream),
                B.nvfp4_workspace_status(self.ws_quant, stream),
                B.nvfp4_hessian_status(stream))


class MoELayerSolver:
    """All experts of an MoE layer solved together through the batched
    calls: per expert a Hessian of its routed tokens for the expert input
    (shared by gate and up) and one for the down projection's input, the two
    factors, the three quantizations and their dequantizations.

    counts: routed tokens per expert; hidden / inter: the expert's model and
    intermediate widths."""

    def __init__(self, n_experts, hidden, inter, device="cuda", damp: float = 0.01,
                 out_dtype=torch.bfloat16, scale_rule="schur_replay"):
        dev = torch.device(device)
        self.device, self.damp = dev, float(damp)
        self.E, self.hidden, self.inter = int(n_experts), int(hidden), int(inter)
        self.params = B.solve_params(scale_rule)
        E = self.E
        # Hessians and factors: [in_0, mid_0, in_1, mid_1, ...]
        self.dims = [d for _ in range(E) for d in (hidden, inter)]
        self.H = [torch.empty((d, d), dtype=torch.float32, device=dev) for d in self.dims]
        self.U = [torch.empty((d, d), dtype=torch.float32, device=dev) for d in self.dims]
        self.ws_prep = _flat(B.nvfp4_prepare_batched_workspace_size(self.dims), dev)
        # weights: [gate_0, up_0, down_0, gate_1, ...]; factor index of each
        self.wshape = [s for _ in range(E) for s in ((inter, hidden), (inter, hidden),
                                                    (hidden, inter))]
        self.wfac = [2 * e + k for e in range(E) for k in (0, 0, 1)]
        self.codes = [torch.empty((o, i // 2), dtype=torch.uint8, device=dev) for o, i in self.wshape]
        self.scales = [torch.empty((o, i // 16), dtype=torch.uint8, device=dev)
                       for o, i in self.wshape]
        self.s_g = [torch.empty(1, dtype=torch.float32, device=dev) for _ in self.wshape]
        self.err = [torch.empty(1, dtype=torch.float64, device=dev) for _ in self.wshape]
        self.ws_quant = _flat(B.nvfp4_quantize_batched_workspace_size(self.wshape, self.params),
                              dev)
        self.Q = [torch.empty(s, dtype=out_dtype, device=dev) for s in self.wshape]
        self.layer_err = [torch.empty(1, dtype=torch.float64, device=dev) for _ in self.wshape]
        # the layer-error scratch reuses the prepare workspace behind its status
        # header (the per-problem status words the prepare leaves there stay
        # readable): the calls run one after another on one stream, and the
        # factors are done before the scratch is used
        n_err = B.nvfp4_layer_error_batched_workspace_size(self.wshape)
        hdr = (4 * (1 + len(self.dims)) + 255) // 256 * 256
        self.ws_err = (self.ws_prep[hdr:hdr + n_err] if hdr + n_err <= self.ws_prep.numel()
                       else _flat(n_err, dev))

    def step(self, Ws, Xs, stream=None, with_error=True):
        """Ws: [gate_0, up_0, down_0, ...] device weights; Xs: [X_in_0,
        X_mid_0, X_in_1, ...] device tokens."""
        B.nvfp4_hessian_accumulate_batched(self.H, Xs, 0, stream)
        B.nvfp4_gptq_prepare_batched(self.H, self.damp, self.U, ws=self.ws_prep, stream=stream)
        B.nvfp4_gptq_schur_replay_quantize_batched(
            Ws, [self.U[f] for f in self.wfac], self.codes, self.scales, self.s_g, self.err,
            ws=self.ws_quant, params=self.params, stream=stream)
        B.nvfp4_dequant_batched(self.codes, self.scales, self.s_g, self.Q, stream)
        if with_error:
            B.nvfp4_layer_error_batched(Ws, self.codes, self.scales, self.s_g,
                                        [self.H[f] for f in self.wfac], self.layer_err,
                                        self.ws_err, stream)

    def status(self, stream=None):
        """(prepare, quantize, layer-error, Hessian status): the first non-OK
        status of any problem of each batched call."""
        return (B.nvfp4_workspace_status(self.ws_prep, stream),
                B.nvfp4_workspace_status(self.ws_quant, stream),
                B.nvfp4_workspace_status(self.ws_err, stream),
                B.nvfp4_hessian_status(stream))
