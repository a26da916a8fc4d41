"""Benchmark of the NVFP4 GPTQ + Schur Replay layer solve on B200.

One step = one whole solve of a synthetic workload through the C ABI, inputs
already resident in HBM.  The default workload is the 70B-shaped dense decoder
layer (hidden 8192, kv 1024, intermediate 28672, 16384 calibration tokens per
Hessian): its linears solved in sequence with shared Hessians -- per group the
Hessian H = X^T X, damping + upper Cholesky factor of H_d^-1, then for every
tensor of the group the global scale + Schur Replay GPTQ (codes, E4M3 scales,
sum delta^2), dequantization to bf16 and the layer error
tr((W-Q) H (W-Q)^T).  The 128-expert MoE layer (every expert's Hessians,
factors and three projections through the batched calls) is measured beside
it and reported under "moe_128_experts".

Prints ONE JSON line (rank 0).  `value` is weights quantized per second over
the whole step, summed over ranks (each rank solves its own copy of the
workload: weak scaling, no collective on the data path).  `--impl reference`
times the fp64 CPU oracle instead, on a bounded sample of the same workload.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                       [--workload NAME] [--no-moe] [--no-cpu-baseline]
"""
from __future__ import annotations

import argparse
import json
import os
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "NVFP4 GPTQ+Schur Replay layer solve ms & weights/s; Hessian TFLOP/s"
UNIT = "weights/s"
DEFAULT_WORKLOAD = "dense_decoder_70b"
MOE_WORKLOAD = "moe_128_experts"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0}
N_SM = 148
N_PHASES = 9                # the library's profiling phases (nvfp4pw.h)
E2E_CHUNK_TOK = 8192        # tokens per host-to-device chunk of the end-to-end step
TF32_PER_BF16 = 1.1 / 2.25  # nominal dense tf32 : bf16 tensor rates
INT8_PER_BF16 = 4.5 / 2.25  # nominal dense int8 (= fp8) : bf16 tensor rates
# DRAM bytes (read + write) per launch of a phase's kernel, from an ncu
# capture of the current kernel source (what was averaged is named); a phase
# without an entry reports null, and an entry is dropped when its kernel
# changes.  factor_i8: ncu --metrics dram__bytes_read.sum,dram__bytes_write.sum
# over the 146 dgemm_i8_kernel launches of one 70B-decoder step (194.2 GB read,
# 70.4 GB written; about 150 GB if every byte moved once: 127 GB of it the fp64
# C of the trailing updates read and written, the rest slices and the
# doubling levels' blocks).
NCU_TRAFFIC = {
    "factor_i8": {
        "bytes": (194.2e9 + 70.4e9) / 146,
        "launch": "mean over the 146 dgemm_i8_kernel launches of one dense_decoder_70b step",
    },
}
I8_PAIRS = 21               # int8 slice products per fp64 MAC in the int8-slice GEMM (6 slices)
FP64_LANES_PER_SM = 64      # B200: 64 FP64 FMA lanes per SM
PHASE_NAMES = ["hessian", "prepare", "replay", "update", "dequant", "other", "factor_gemm",
               "panel", "factor_i8"]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        d["source"] = "measured"
        return d
    d = dict(PEAKS_FALLBACK)
    d["source"] = "fallback"
    return d


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    """Polls the SM clock and the clock-event (throttle) reasons of one GPU
    every 5 ms through NVML while the timed region runs."""
    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "hw_power_brake_slowdown": 0x80, "sw_power_cap": 0x4}

    def __init__(self, gpu_index):
        self.idx = gpu_index
        self.samples = []
        self.max_mhz = None
        self.err = None

    def _run(self):
        import pynvml as N
        h = N.nvmlDeviceGetHandleByIndex(self.idx)
        self.max_mhz = N.nvmlDeviceGetMaxClockInfo(h, N.NVML_CLOCK_SM)
        while not self._stop.is_set():
            self.samples.append((N.nvmlDeviceGetClockInfo(h, N.NVML_CLOCK_SM),
                                 N.nvmlDeviceGetCurrentClocksEventReasons(h)))
            self._stop.wait(0.005)

    def __enter__(self):
        import threading
        self._stop = threading.Event()
        try:
            import pynvml as N
            N.nvmlInit()
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            if vis:
                self.idx = int(vis.split(",")[self.idx])
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        except Exception as e:  # no NVML: report unsampled
            self.err = repr(e)
            self._t = None
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._t is not None:
            self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unsampled"],
                    "samples": 0}
        mask = 0
        for _, r in self.samples:
            mask |= r
        return {"sm_mhz": float(np.median([c for c, _ in self.samples])),
                "sm_max_mhz": self.max_mhz,
                "reasons": sorted(n for n, b in self.REASONS.items() if mask & b),
                "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# algorithmic work
# ---------------------------------------------------------------------------
def update_flops(d_out, d_in, batch=128):
    """W~[:, e:] -= Delta (d_out x 128) U[batch, e:], summed over the batches."""
    f = 0
    for c0 in range(0, d_in, batch):
        e = min(c0 + batch, d_in)
        f += 2 * d_out * (e - c0) * (d_in - e)
    return f


def phase_work(tensors, hessians, factors):
    """Algorithmic work per phase of one step (flops or bytes).
    tensors: [(d_out, d_in)] solved; hessians: [(n_tok, d)] accumulated;
    factors: [d] distinct factorisations."""
    w = {"hessian_flops": 0, "prepare_flops": 0, "update_flops": 0, "replay_flops": 0.0,
         "dequant_bytes": 0.0, "weights": 0}
    for n_tok, d in hessians:
        w["hessian_flops"] += n_tok * d * (d + 1)            # symmetric half, 2 flops per MAC
    for d in factors:
        w["prepare_flops"] += 2 * d ** 3 // 3                 # Cholesky 1/3 d^3 + trtri 1/3 d^3
    for d_out, d_in in tensors:
        w["update_flops"] += update_flops(d_out, d_in)
        nb = d_in // 16
        # fp64 flops of the Schur Replay per weight: 16 candidates x (scale,
        # residual, delta, score: 6 flops + 7.5 in-block update FMAs) plus the
        # in-batch update (3.5 later blocks of 16 columns on average)
        w["replay_flops"] += d_out * nb * 16 * (16 * (6 + 15) + 2 * 16 * 3.5)
        w["dequant_bytes"] += d_out * d_in * (0.5 + 2) + d_out * d_in / 16
        w["weights"] += d_out * d_in
    return w


def reduce_max(x, dist, device):
    """x maximised over all ranks (the step time of the slowest GPU)."""
    if not dist:
        return float(x)
    import torch
    import torch.distributed as tdist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    tdist.all_reduce(t, op=tdist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world, weights_per_rank, ms_per_step):
    """Whole-job weights/s: every rank solves its own layer in the step."""
    return world * weights_per_rank / (ms_per_step / 1e3)


# ---------------------------------------------------------------------------
# workloads (device side)
# ---------------------------------------------------------------------------
class SingleLayer:
    """One linear layer: Hessian, prepare, quantize, dequant, layer error."""

    def __init__(self, name, dev):
        import torch
        from nvfp4_post_weight_b200 import synth
        from nvfp4_post_weight_b200.layer import LayerSolver
        self.name = name
        W, X = synth.WORKLOADS[name]()
        self.W_host, self.X_host = W, X
        self.d_out, self.d_in = W.shape
        self.n_tok = X.shape[0]
        self.Wd, self.Xd = W.to(dev), X.to(dev)
        self.solver = LayerSolver(self.d_out, self.d_in, dev, out_dtype=torch.bfloat16)
        self.tensors = [(self.d_out, self.d_in)]
        self.hessians = [(self.n_tok, self.d_in)]
        self.factors = [self.d_in]
        self.dev = dev

    def config(self):
        return {"workload": self.name, "d_out": self.d_out, "d_in": self.d_in,
                "n_tok": self.n_tok}

    def step(self):
        self.solver.step(self.Wd, self.Xd)

    def status_ok(self):
        return self.solver.status() == (0, 0)

    def e2e_setup(self):
        import torch
        s = self.solver
        self.Wh, self.Xh = self.W_host.pin_memory(), self.X_host.pin_memory()
        self.W_e2e = torch.empty_like(self.Wd)
        self.out_h = (torch.empty(s.codes.shape, dtype=torch.uint8).pin_memory(),
                      torch.empty(s.scales.shape, dtype=torch.uint8).pin_memory(),
                      torch.empty(1, dtype=torch.float32).pin_memory())
        self.h2d = self.W_host.numel() * self.W_host.element_size() + \
            self.X_host.numel() * self.X_host.element_size()
        self.d2h = sum(t.numel() * t.element_size() for t in self.out_h)

    def e2e_step(self):
        self.solver.step_host(self.Wh, self.Xh, self.W_e2e, chunk_tok=E2E_CHUNK_TOK,
                              out_host=self.out_h)

    def layer_error_by_rule(self):
        from nvfp4_post_weight_b200 import binding as B
        s = self.solver
        out = {"schur_replay": s.layer_err.item()}
        sr = s.params
        for rule in ("amax", "block_mse"):
            s.params = B.solve_params(rule)
            s.quantize(self.Wd)
            s.layer_error(self.Wd)
            out[rule] = s.layer_err.item()
        s.params = sr
        return out


class DenseDecoder:
    """The 70B-shaped dense decoder layer, linears solved in sequence with
    shared Hessians: (q, k, v) from X_attn, o from X_o, (gate, up) from
    X_mlp, down from X_down."""

    def __init__(self, dev):
        import torch
        from nvfp4_post_weight_b200 import synth
        from nvfp4_post_weight_b200.decoder import DecoderLayerSolver
        self.name = DEFAULT_WORKLOAD
        self.dev = dev
        gen = synth.dense_decoder_layer()
        groups = [(x, {n: synth.DENSE_70B_SHAPES[n] for n in names})
                  for x, names in synth.DENSE_70B_GROUPS]
        self.groups = groups
        self.W_host, self.X_host, self.Wd, self.Xd = {}, {}, {}, {}
        for x, t in groups:
            self.X_host[x] = gen[x]()
            self.Xd[x] = self.X_host[x].to(dev)
            for n in t:
                self.W_host[n] = gen[n]()
                self.Wd[n] = self.W_host[n].to(dev)
        self.solver = DecoderLayerSolver(groups, dev, out_dtype=torch.bfloat16)
        self.tensors = [self.W_host[n].shape for _, t in groups for n in t]
        self.hessians = [tuple(self.X_host[x].shape) for x, _ in groups]
        self.factors = [self.X_host[x].shape[1] for x, _ in groups]

    def config(self):
        return {"workload": self.name, "hidden": 8192, "kv": 1024, "intermediate": 28672,
                "n_tok_per_hessian": 16384,
                "tensors": {n: list(self.W_host[n].shape) for n in self.W_host},
                "solve_order": [[x, list(t)] for x, t in self.groups]}

    def step(self):
        self.solver.step(self.Wd, self.Xd)

    def status_ok(self):
        p, q, h = self.solver.status()
        return p == 0 and q == 0 and h == 0

    def e2e_setup(self):
        import torch
        self.Wh = {n: w.pin_memory() for n, w in self.W_host.items()}
        self.Xh = {x: t.pin_memory() for x, t in self.X_host.items()}
        self.W_e2e = {n: torch.empty_like(w) for n, w in self.Wd.items()}
        s = self.solver
        self.out_h = {n: (torch.empty(s.codes[n].shape, dtype=torch.uint8).pin_memory(),
                          torch.empty(s.scales[n].shape, dtype=torch.uint8).pin_memory(),
                          torch.empty(1, dtype=torch.float32).pin_memory()) for n in self.Wd}
        self.h2d = sum(t.numel() * t.element_size()
                       for t in list(self.W_host.values()) + list(self.X_host.values()))
        self.d2h = sum(t.numel() * t.element_size() for o in self.out_h.values() for t in o)

    def e2e_step(self):
        self.solver.step_host(self.Wh, self.Xh, self.W_e2e, chunk_tok=E2E_CHUNK_TOK,
                              out_host=self.out_h)

    def layer_error_by_rule(self):
        from nvfp4_post_weight_b200 import binding as B
        s = self.solver
        out = {"schur_replay": {n: t.item() for n, t in s.layer_err.items()}}
        sr = s.params
        for rule in ("amax", "block_mse"):
            s.params = B.solve_params(rule)
            s.step(self.Wd, self.Xd)
            out[rule] = {n: t.item() for n, t in s.layer_err.items()}
        s.params = sr
        s.step(self.Wd, self.Xd)
        return out


class MoELayer:
    """128 experts (gate/up 4096 -> 1536, down 1536 -> 4096), Zipf(1.1)
    routed token counts 64..4096 (65536 in total); every phase (Hessian,
    prepare, quantize, dequant, layer error) one batched call over all
    experts."""

    def __init__(self, dev):
        import torch
        from nvfp4_post_weight_b200 import synth
        from nvfp4_post_weight_b200.decoder import MoELayerSolver
        self.name = MOE_WORKLOAD
        self.dev = dev
        counts, ex = synth.moe_all_experts()
        self.counts = counts
        self.W_host = [ex[e][n] for e in range(len(ex)) for n in ("gate", "up", "down")]
        self.X_host = [ex[e][n] for e in range(len(ex)) for n in ("X_in", "X_mid")]
        del ex
        self.Wd = [w.to(dev) for w in self.W_host]
        self.Xd = [x.to(dev) for x in self.X_host]
        self.solver = MoELayerSolver(len(counts), 4096, 1536, dev, out_dtype=torch.bfloat16)
        self.tensors = [tuple(w.shape) for w in self.W_host]
        self.hessians = [tuple(x.shape) for x in self.X_host]
        self.factors = [x.shape[1] for x in self.X_host]

    def config(self):
        return {"workload": self.name, "experts": len(self.counts), "hidden": 4096,
                "intermediate": 1536, "tokens_total": int(self.counts.sum()),
                "tokens_min": int(self.counts.min()), "tokens_max": int(self.counts.max())}

    def step(self):
        self.solver.step(self.Wd, self.Xd)

    def status_ok(self):
        return self.solver.status() == (0, 0, 0, 0)


WORKLOADS = {
    "dense_decoder_70b": DenseDecoder,
    "moe_128_experts": MoELayer,
    "attn_massive_4096x4096": lambda dev: SingleLayer("attn_massive_4096x4096", dev),
    "mlp_down_silu_4096x14336": lambda dev: SingleLayer("mlp_down_silu_4096x14336", dev),
    "small_outlier_256x256": lambda dev: SingleLayer("small_outlier_256x256", dev),
}


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def timed_steps(fn, steps, stream, flush, dist, dev, clocks=None):
    """Runs fn `steps` times, each bracketed by CUDA events on `stream`, L2
    flushed (untimed) before each; returns the mean step ms, max over ranks,
    and the number of library kernel launches."""
    import torch
    from nvfp4_post_weight_b200 import binding as B
    if dist:
        import torch.distributed as tdist
        tdist.barrier()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    n0 = B.lib().nvfp4_launch_count()
    for i in range(steps):
        flush.fill_(i & 0xFF)
        ev[i][0].record(stream)
        fn()
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    launches = B.lib().nvfp4_launch_count() - n0
    ms = reduce_max(sum(a.elapsed_time(b) for a, b in ev) / steps, dist, dev)
    if dist:
        tdist.barrier()
    return ms, launches


def profile_phases(wl, steps, flush):
    """The same steps again with the library's per-phase events on (they sit
    between the kernels, so this pass is not the one whose time is reported
    as the step time): per phase ms, launches and counted work per step."""
    import ctypes
    import torch
    from nvfp4_post_weight_b200 import binding as B
    B.lib().nvfp4_profile_begin()
    for i in range(steps):
        flush.fill_(i & 0xFF)
        wl.step()
    torch.cuda.synchronize()
    ms_ph = (ctypes.c_double * N_PHASES)()
    ln_ph = (ctypes.c_longlong * N_PHASES)()
    wk_ph = (ctypes.c_double * N_PHASES)()
    B.lib().nvfp4_profile_end(ms_ph, ln_ph, N_PHASES)
    B.lib().nvfp4_profile_work(wk_ph, N_PHASES)
    ph_ms = {n: ms_ph[i] / steps for i, n in enumerate(PHASE_NAMES) if n != "other"}
    ph_launch = {n: ln_ph[i] // steps for i, n in enumerate(PHASE_NAMES)}
    ph_work = {n: wk_ph[i] / steps for i, n in enumerate(PHASE_NAMES)}
    return ph_ms, ph_launch, ph_work


def rooflines(wk, ph_ms, ph_work, peaks):
    """Per-kernel-group roofline: what bounds each group in this build, its
    achieved rate from the algorithmic work and the phase's event time."""
    sm_ghz = peaks.get("sm_max_mhz", 1965.0) / 1e3
    fp64_peak = N_SM * FP64_LANES_PER_SM * 2 * sm_ghz / 1e3    # TFLOP/s, derived
    bf16_peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])   # inside a long step
    tf32_peak = bf16_peak * TF32_PER_BF16                        # nominal dense ratio
    int8_peak = bf16_peak * INT8_PER_BF16                        # nominal dense ratio
    hbm = peaks["hbm_gbs"]

    def rate(work, ms, scale):
        return work / (ms * scale) if ms > 0 else 0.0

    rl = {
        "hessian": ("tensor", rate(wk["hessian_flops"], ph_ms["hessian"], 1e9), bf16_peak,
                    "TFLOP/s", "hessian_tc_kernel (tcgen05 kind::f16)",
                    "measured bf16 sustained"),
        "factor_gemm": ("tensor", rate(ph_work["factor_gemm"], ph_ms["factor_gemm"], 1e9),
                        fp64_peak, "TFLOP/s",
                        "dgemm_nt_kernel (fp64 mma.sync m8n8k4, TMA-fed; narrow in-block updates)",
                        "derived fp64: 148 SMs x 64 lanes x 2 x max SM clock"),
        "factor_i8": ("tensor", rate(I8_PAIRS * ph_work["factor_i8"], ph_ms["factor_i8"], 1e9),
                      int8_peak, "TFLOP/s",
                      "dgemm_i8_kernel + slice_rows_kernel (fp64-accurate GEMM on tcgen05 "
                      "kind::i8; achieved counts the int8 ops: 21 slice products per fp64 MAC)",
                      "measured bf16 sustained x nominal int8/bf16 ratio"),
        "panel": ("alu", rate(ph_work["panel"], ph_ms["panel"], 1e9), fp64_peak, "TFLOP/s",
                  "chol_panel_kernel (fp64; bound by its serial 64-pivot chain per panel, "
                  "not by the fp64 rate)",
                  "derived fp64: 148 SMs x 64 lanes x 2 x max SM clock"),
        "update": ("tensor", rate(3 * wk["update_flops"], ph_ms["update"], 1e9), tf32_peak,
                   "TFLOP/s", "update_tc_kernel + gemm_nt_tc_kernel (tcgen05 kind::tf32, "
                   "3 products per MAC)",
                   "measured bf16 sustained x nominal tf32/bf16 ratio"),
        "replay": ("alu", rate(wk["replay_flops"], ph_ms["replay"], 1e9), fp64_peak, "TFLOP/s",
                   "schur_replay_batch_kernel (fp64 CUDA cores)",
                   "derived: 148 SMs x 64 fp64 lanes x 2 x max SM clock"),
        "dequant": ("hbm", rate(wk["dequant_bytes"], ph_ms["dequant"], 1e6), hbm, "GB/s",
                    "dequant_kernel", "measured HBM copy"),
    }
    return rl


def measure(wl, args, world, dist, dev, stream, flush, gpu_index, with_e2e=True,
            with_rules=True):
    """Warm-up, timed steps, phase profile, end to end: the workload's whole
    measurement as a dict of the bench line's keys."""
    import torch
    for _ in range(args.warmup):
        flush.fill_(1)
        wl.step()
    torch.cuda.synchronize()
    if not wl.status_ok():
        raise SystemExit(f"{wl.name}: device status after warm-up not ok")
    with ClockSampler(gpu_index) as clk:
        step_ms, launches = timed_steps(wl.step, args.steps, stream, flush, dist, dev)
    prof_steps = min(args.steps, args.profile_steps)
    ph_ms, ph_launch, ph_work = profile_phases(wl, prof_steps, flush)
    peaks = load_peaks()
    wk = phase_work(wl.tensors, wl.hessians, wl.factors)
    rl = rooflines(wk, ph_ms, ph_work, peaks)
    dom = max(rl, key=lambda n: ph_ms[n])
    bound, ach, peak, unit, kern, src = rl[dom]
    weights = wk["weights"]
    solve_ms = ph_ms["prepare"] + ph_ms["replay"] + ph_ms["update"]
    out = {
        "value": job_throughput(world, weights, step_ms), "ms_per_step": step_ms,
        "weights_per_step": weights,
        "layer_solve_ms": solve_ms,
        "solve_weights_per_s": weights / (solve_ms / 1e3) if solve_ms > 0 else None,
        "hessian_tflops": {
            "algorithmic_syrk_half": wk["hessian_flops"] / (ph_ms["hessian"] * 1e9),
            "conventional_2Nd2": 2 * sum(n * d * d for n, d in wl.hessians) /
            (ph_ms["hessian"] * 1e9)},
        "phase_ms": ph_ms, "phase_launches": ph_launch, "profile_steps": prof_steps,
        "phase_roofline": {n: {"bound": b, "achieved": a, "peak": p, "unit": u,
                               "frac": a / p, "kernels": k_, "peak_source": s_}
                           for n, (b, a, p, u, k_, s_) in rl.items()},
        "roofline": {"phase": dom, "kernel": kern, "bound": bound, "achieved": ach,
                     "peak": peak, "unit": unit, "frac": ach / peak,
                     "traffic": NCU_TRAFFIC.get(dom, {}).get("bytes"),
                     "traffic_launch": NCU_TRAFFIC.get(dom, {}).get("launch"),
                     "peak_source": f"{src} ({peaks['source']})"},
        "gpu_launches": launches,
        "clocks": clk.summary(),
    }
    if with_e2e and hasattr(wl, "e2e_setup"):
        wl.e2e_setup()
        wl.e2e_step()
        torch.cuda.synchronize()
        e2e_ms, _ = timed_steps(wl.e2e_step, args.steps, stream, flush, dist, dev)
        out["e2e"] = {"value": job_throughput(world, weights, e2e_ms), "unit": UNIT,
                      "ms_per_step": e2e_ms, "h2d_bytes_per_step": wl.h2d,
                      "d2h_bytes_per_step": wl.d2h}
    if with_rules and hasattr(wl, "layer_error_by_rule"):
        out["layer_error_by_scale_rule"] = wl.layer_error_by_rule()
        torch.cuda.synchronize()
    return out


def run_ours(args, rank, world, local_rank):
    import torch
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    dist = world > 1
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    wl = WORKLOADS[args.workload](dev)
    m = measure(wl, args, world, dist, dev, stream, flush, local_rank, with_rules=rank == 0)
    cfg = wl.config()
    cfg.update({"l2": "flushed between timed steps (256 MiB write, untimed)",
                "parallelism": f"{world} independent solves (one per GPU)"})
    out = {
        "metric": METRIC, "value": m.pop("value"), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": m.pop("ms_per_step"),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": ("bf16 in; f32 H; f64-accurate factor (int8-slice tensor cores + fp64 mma; "
                  "U stored f32); f64 working copy and replay; 3xTF32 update"),
        "data": "synthetic", "config": cfg,
    }
    out.update(m)
    if args.workload == DEFAULT_WORKLOAD and not args.no_moe:
        # the MoE layer beside the headline: freed first, then measured the
        # same way (its own warm-up and timed steps, no end-to-end pass)
        del wl
        torch.cuda.synchronize()
        torch.cuda.empty_cache()
        moe = MoELayer(dev)
        mm = measure(moe, args, world, dist, dev, stream, flush, local_rank, with_e2e=False,
                     with_rules=False)
        mm["config"] = moe.config()
        out[MOE_WORKLOAD] = mm
        del moe
    if rank != 0:
        return None
    if not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(args.workload)
        if MOE_WORKLOAD in out:
            out[MOE_WORKLOAD]["cpu_baseline"] = cpu_baseline(MOE_WORKLOAD)
    return out


# ---------------------------------------------------------------------------
# the oracle on the host cores (cpu_baseline and --impl reference)
# ---------------------------------------------------------------------------
def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return 1


class OracleSample:
    """A bounded sample of a workload for the fp64 oracle, and the model that
    scales its measured times to the whole workload by operation counts:
    the Hessian by n_tok d^2, the factor by d^3, and the solve (rows are
    independent given U) by rows x tau(d_in), the per-row time fitted as
    a d + b d^2 (replay per block, trailing updates) from the sampled rows
    solved at the sample's width d_s and at d_s / 2 (the leading columns,
    with the leading block of the same U: the time depends only on shapes).

    setup() times the sample's Hessian and factor once; step() times the
    solve + dequant of the sampled rows of the sample tensors, at both
    widths, and returns (seconds at d_s, seconds at d_s / 2)."""

    def __init__(self, name, n_rows):
        from nvfp4_post_weight_b200 import synth
        self.name = name
        rng = np.random.default_rng(7)
        if name == DEFAULT_WORKLOAD:
            # the attention group restricted to its first 4096 input channels
            # (the oracle's 8192-wide inverse alone takes tens of seconds)
            gen = synth.dense_decoder_layer()
            X = gen["X_attn"]()[:, :4096].contiguous()
            self.sample_tensors = {n: gen[n]()[:, :4096].contiguous() for n in ("q", "k", "v")}
            shapes = [synth.DENSE_70B_SHAPES[n] for _, t in synth.DENSE_70B_GROUPS for n in t]
            self.all_hessians = [(16384, 8192)] * 3 + [(16384, 28672)]
            self.all_factors = [8192, 8192, 8192, 28672]
            self.what = ("the attention group on its first 4096 input channels (X_attn[:, :4096]: "
                         "16384 tokens; q, k, v [:, :4096])")
        elif name == MOE_WORKLOAD:
            counts, make = synth.moe_layer()
            ex = make(0)
            X = ex["X_in"]
            self.sample_tensors = {n: ex[n] for n in ("gate", "up")}
            shapes = [s for _ in counts for s in ((1536, 4096), (1536, 4096), (4096, 1536))]
            self.all_hessians = [(int(n), d) for n in counts for d in (4096, 1536)]
            self.all_factors = [d for _ in counts for d in (4096, 1536)]
            self.what = f"expert 0's input group ({int(counts[0])} tokens x 4096; gate, up)"
        else:
            W, X = synth.WORKLOADS[name]()
            self.sample_tensors = {"W": W}
            shapes = [tuple(W.shape)]
            self.all_hessians = [tuple(X.shape)]
            self.all_factors = [X.shape[1]]
            self.what = f"the layer ({tuple(W.shape)})"
        self.X64 = X.double().numpy()
        self.W64 = {n: w.double().numpy() for n, w in self.sample_tensors.items()}
        self.rows = {n: np.sort(rng.choice(w.shape[0], min(n_rows, w.shape[0]), replace=False))
                     for n, w in self.W64.items()}
        self.n_rows = sum(len(r) for r in self.rows.values())
        self.all_tensors = shapes
        self.weights = int(sum(a * b for a, b in shapes))
        n_tok, d = self.X64.shape
        self.d_s = d
        self.d_h = max(16, (d // 2) // 16 * 16)
        self.r_hess = sum(n * dd * dd for n, dd in self.all_hessians) / (n_tok * d * d)
        self.r_fact = sum(dd ** 3 for dd in self.all_factors) / d ** 3

    def setup(self):
        import oracle as O
        t0 = time.perf_counter()
        H = O.hessian(self.X64)
        t1 = time.perf_counter()
        Hd, self.dead, _ = O.damp(H)
        self.U = O.inverse_cholesky_upper(Hd)
        t2 = time.perf_counter()
        self.sg = {n: O.global_scale(w) for n, w in self.W64.items()}
        self.t_hess, self.t_fact = t1 - t0, t2 - t1

    def step(self):
        import oracle as O
        t = []
        for width in (self.d_s, self.d_h):
            t0 = time.perf_counter()
            U = self.U[:width, :width]
            for n, w in self.W64.items():
                res = O.schur_replay_gptq(w[self.rows[n], :width], U, self.sg[n],
                                          self.dead[:width])
                O.dequant(res["codes"], res["scales"], self.sg[n], "bf16")
            t.append(time.perf_counter() - t0)
        return tuple(t)

    def solve_seconds(self, t_full, t_half):
        """The whole workload's solve time from the per-row fit."""
        ds, dh = float(self.d_s), float(self.d_h)
        tau1, tau2 = t_full / self.n_rows, t_half / self.n_rows
        b = (tau1 * dh - tau2 * ds) / (ds * ds * dh - dh * dh * ds)
        if b < 0:
            b = 0.0
        a = (tau1 - b * ds * ds) / ds
        if a < 0:
            a, b = 0.0, tau1 / (ds * ds)
        self.fit = (a, b)
        return sum(o * (a * i + b * i * i) for o, i in self.all_tensors)

    def full_seconds(self, t_full, t_half):
        return (self.t_hess * self.r_hess + self.t_fact * self.r_fact +
                self.solve_seconds(t_full, t_half))

    def describe(self, n_steps):
        rows = ", ".join(f"{len(r)} rows of {n}" for n, r in self.rows.items())
        return (f"{self.what}: fp64 Hessian ({self.t_hess:.1f} s) and factor "
                f"({self.t_fact:.1f} s) once, then per step the solve + dequant of {rows} "
                f"at widths {self.d_s} and {self.d_h} ({n_steps} step(s)); the whole "
                f"workload's time estimated by operation counts: Hessian x{self.r_hess:.2f} "
                f"(n_tok d^2), factor x{self.r_fact:.2f} (d^3), solve rows x (a d_in + b d_in^2) "
                f"fitted per row at the two widths")


def cpu_baseline(name, n_rows=16):
    s = OracleSample(name, n_rows)
    s.setup()
    t = s.step()
    full = s.full_seconds(*t)
    return {"value": s.weights / full, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": s.describe(1), "sample_wall_s": s.t_hess + s.t_fact + sum(t),
            "full_workload_s_est": full}


def run_reference(args):
    s = OracleSample(args.workload, args.ref_rows)
    s.setup()
    for _ in range(args.warmup):
        s.step()
    ts = np.array([s.step() for _ in range(args.steps)])
    t = float(ts.sum(axis=1).mean())
    full = s.full_seconds(*ts.mean(axis=0))
    v = s.weights / full
    return {
        "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": t * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "impl": "reference",
        "config": {"workload": args.workload, "l2": "n/a (CPU)"},
        "full_workload_ms_est": full * 1e3,
        "note": ("ms_per_step is the measured wall time of one sample step (the sampled "
                 "rows' solve at the two widths); value is the whole workload's weights per "
                 "second of the operation-count estimate full_workload_ms_est, which adds "
                 "the Hessian and factor timed once before the steps"),
        "cpu_baseline": {"value": v, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                         "sample": s.describe(args.steps)},
        "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(WORKLOADS))
    ap.add_argument("--ref-rows", type=int, default=8)
    ap.add_argument("--profile-steps", type=int, default=3)
    ap.add_argument("--no-moe", action="store_true",
                    help="skip the MoE layer measured beside the default workload")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return

    if world > 1:
        import datetime
        import torch
        import torch.distributed as tdist
        torch.cuda.set_device(local_rank)
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                 device_id=torch.device("cuda", local_rank))
    try:
        out = run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as tdist
            tdist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
