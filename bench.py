"""Benchmark of the per-layer NVFP4 GPTQ + Schur Replay solve on B200.

One step = one whole solve of a synthetic layer through the C ABI, inputs
already resident in HBM: Hessian H = X^T X, damping + upper Cholesky factor of
H_d^-1, global scale + Schur Replay GPTQ (codes, E4M3 scales, sum delta^2),
dequantization to bf16 and the layer error tr((W-Q) H (W-Q)^T).

Prints ONE JSON line (rank 0).  `value` is weights quantized per second over
the whole step, summed over ranks (each rank solves its own layer: weak
scaling, no collective on the data path).  `--impl reference` times the fp64
CPU oracle instead, on a bounded row sample of the same workload.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                       [--workload NAME]
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
DEFAULT_WORKLOAD = "attn_massive_4096x4096"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                  "sm_max_mhz": 1965.0}
N_SM = 148
N_PHASES = 9                # the library's profiling phases (nvfp4pw.h)
E2E_CHUNK_TOK = 1024        # tokens per host-to-device chunk of the end-to-end step
TF32_PER_BF16 = 1.1 / 2.25  # nominal dense tf32 : bf16 tensor rates
INT8_PER_BF16 = 4.5 / 2.25  # nominal dense int8 (= fp8) : bf16 tensor rates
# DRAM bytes (read + write) of one launch of a phase's kernel, from an ncu --set
# full capture of the current kernel source (this script with --steps 1
# --warmup 0 --no-cpu-baseline, the launch named); a phase without an entry
# reports null, and an entry is dropped when its kernel changes
NCU_TRAFFIC = {
    "panel": {"bytes": 1.824e6, "launch": "chol_panel_kernel, panel 11 of 64 (3328 rows below)"},
}
I8_PAIRS = 21               # int8 slice products per fp64 MAC in the int8-slice GEMM (6 slices)
FP64_LANES_PER_SM = 64      # B200: 64 FP64 FMA lanes per SM
FP32_LANES_PER_SM = 128


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


def workload(name):
    from nvfp4_post_weight_b200 import synth
    if name == "attn_massive_4096x4096":
        return synth.attn_massive()
    if name == "small_outlier_256x256":
        return synth.small_outlier()
    if name == "mlp_down_silu_4096x14336":
        return synth.mlp_down_silu()
    raise SystemExit(f"unknown workload {name}")


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
# our arm
# ---------------------------------------------------------------------------
def phase_work(d_out, d_in, n_tok):
    """Algorithmic work per phase of one step (flops or bytes)."""
    upd_flops = 0
    for c0 in range(0, d_in, 128):
        e = min(c0 + 128, d_in)
        # W~[:, e:] -= Delta (d_out x 128) U[batch, e:]
        upd_flops += 2 * d_out * (e - c0) * (d_in - e)
    nb = d_in // 16
    return {
        "hessian_flops": n_tok * d_in * (d_in + 1),          # symmetric half, 2 flops per MAC
        "prepare_flops": 2 * d_in ** 3 // 3,                  # Cholesky 1/3 d^3 + trtri 1/3 d^3
        "update_flops": upd_flops,
        # fp64 flops of the Schur Replay per weight: 16 candidates x (scale,
        # residual, delta, score: 6 flops + 7.5 in-block update FMAs) plus the
        # in-batch update (3.5 later blocks of 16 columns on average)
        "replay_flops": d_out * nb * 16 * (16 * (6 + 15) + 2 * 16 * 3.5),
        "dequant_bytes": d_out * d_in * (0.5 + 2) + d_out * d_in / 16,
    }


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


def run_ours(args, rank, world, local_rank):
    import torch
    from nvfp4_post_weight_b200 import binding as B
    from nvfp4_post_weight_b200.layer import LayerSolver

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    W, X = workload(args.workload)
    d_out, d_in = W.shape
    n_tok = X.shape[0]
    Wd, Xd = W.to(dev), X.to(dev)
    solver = LayerSolver(d_out, d_in, dev, out_dtype=torch.bfloat16)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        solver.step(Wd, Xd)

    for _ in range(args.warmup):
        flush.fill_(1)
        step()
    torch.cuda.synchronize()
    st = solver.status()
    if st != (0, 0):
        raise SystemExit(f"device status after warm-up: {st}")

    dist = world > 1
    if dist:
        import torch.distributed as tdist
        tdist.barrier()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(args.steps)]
    n0 = B.lib().nvfp4_launch_count()
    with ClockSampler(local_rank) as clk:
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
    launches = B.lib().nvfp4_launch_count() - n0
    step_ms = reduce_max(sum(a.elapsed_time(b) for a, b in ev) / args.steps, dist, dev)
    if dist:
        tdist.barrier()

    # phase breakdown: the same steps again with the library's per-phase
    # events on (they sit between the kernels, so this pass is not the one
    # whose time is reported as the step time)
    import ctypes
    B.lib().nvfp4_profile_begin()
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        step()
    torch.cuda.synchronize()
    ms_ph = (ctypes.c_double * N_PHASES)()
    ln_ph = (ctypes.c_longlong * N_PHASES)()
    wk_ph = (ctypes.c_double * N_PHASES)()
    B.lib().nvfp4_profile_end(ms_ph, ln_ph, N_PHASES)
    B.lib().nvfp4_profile_work(wk_ph, N_PHASES)

    # end to end through the C ABI from pinned host buffers: the tokens stream
    # from host memory into the Hessian in 1024-token chunks, W is copied
    # beside the prepare, then the solve; D2H of codes, scales and s_g beside
    # dequant and the layer error, waited for before the step's end event
    Wh, Xh = W.pin_memory(), X.pin_memory()
    W_e2e = torch.empty_like(Wd)
    codes_h = torch.empty(solver.codes.shape, dtype=torch.uint8).pin_memory()
    scales_h = torch.empty(solver.scales.shape, dtype=torch.uint8).pin_memory()
    sg_h = torch.empty(1, dtype=torch.float32).pin_memory()

    def e2e_step():
        solver.step_host(Wh, Xh, W_e2e, chunk_tok=E2E_CHUNK_TOK,
                         out_host=(codes_h, scales_h, sg_h))

    e2e_step()
    torch.cuda.synchronize()
    ev2 = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        ev2[i][0].record(stream)
        e2e_step()
        ev2[i][1].record(stream)
    torch.cuda.synchronize()
    e2e_ms = reduce_max(sum(a.elapsed_time(b) for a, b in ev2) / args.steps, dist, dev)

    if rank != 0:
        return None
    # untimed: the same layer's error tr((W-Q) H (W-Q)^T) under the
    # independent-block scale rules Schur Replay is compared with
    by_rule = {"schur_replay": solver.layer_err.item()}
    sr_params = solver.params
    for rule in ("amax", "block_mse"):
        solver.params = B.solve_params(rule)
        solver.quantize(Wd)
        solver.layer_error(Wd)
        by_rule[rule] = solver.layer_err.item()
    solver.params = sr_params
    torch.cuda.synchronize()
    peaks = load_peaks()
    wk = phase_work(d_out, d_in, n_tok)
    names = ["hessian", "prepare", "replay", "update", "dequant", "other", "factor_gemm",
             "panel", "factor_i8"]
    ph_ms = {n: ms_ph[i] / args.steps for i, n in enumerate(names) if n != "other"}
    ph_launch = {n: ln_ph[i] // args.steps for i, n in enumerate(names)}
    sm_ghz = peaks.get("sm_max_mhz", 1965.0) / 1e3
    fp64_peak = N_SM * FP64_LANES_PER_SM * 2 * sm_ghz / 1e3    # TFLOP/s, derived
    bf16_peak = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])   # inside a long step
    tf32_peak = bf16_peak * TF32_PER_BF16                        # nominal dense ratio
    int8_peak = bf16_peak * INT8_PER_BF16                        # nominal dense ratio
    hbm = peaks["hbm_gbs"]
    gemm_flops = wk_ph[6] / args.steps          # counted by the launcher from the shapes
    panel_flops = wk_ph[7] / args.steps
    i8_flops = wk_ph[8] / args.steps            # fp64-equivalent flops of the int8-slice GEMMs
    # per-kernel roofline (what bounds each kernel group in this build); the
    # prepare phase is the panel kernels plus the fp64 GEMMs
    rl = {
        "hessian": ("tensor", wk["hessian_flops"] / (ph_ms["hessian"] * 1e9), bf16_peak,
                    "TFLOP/s", "hessian_tc_kernel (tcgen05 kind::f16)",
                    "measured bf16 sustained"),
        "factor_gemm": ("tensor", gemm_flops / (ph_ms["factor_gemm"] * 1e9), fp64_peak,
                        "TFLOP/s", "dgemm_nt_kernel (fp64 mma.sync m8n8k4, TMA-fed; narrow "
                        "in-block updates)",
                        "derived fp64: 148 SMs x 64 lanes x 2 x max SM clock"),
        "factor_i8": ("tensor", I8_PAIRS * i8_flops / (ph_ms["factor_i8"] * 1e9), int8_peak,
                      "TFLOP/s", "dgemm_i8_kernel + slice_rows_kernel (fp64-accurate GEMM on "
                      "tcgen05 kind::i8; achieved counts the int8 ops: 21 slice products per "
                      "fp64 MAC)",
                      "measured bf16 sustained x nominal int8/bf16 ratio"),
        "panel": ("alu", panel_flops / (ph_ms["panel"] * 1e9), fp64_peak, "TFLOP/s",
                  "chol_panel_kernel (fp64; bound by its serial 64-pivot chain per panel, "
                  "not by the fp64 rate)",
                  "derived fp64: 148 SMs x 64 lanes x 2 x max SM clock"),
        "update": ("tensor", 3 * wk["update_flops"] / (ph_ms["update"] * 1e9), tf32_peak,
                   "TFLOP/s", "update_tc_kernel (tcgen05 kind::tf32, 3 products per MAC)",
                   "measured bf16 sustained x nominal tf32/bf16 ratio"),
        "replay": ("alu", wk["replay_flops"] / (ph_ms["replay"] * 1e9), fp64_peak, "TFLOP/s",
                   "schur_replay_batch_kernel (fp64 CUDA cores)",
                   "derived: 148 SMs x 64 fp64 lanes x 2 x max SM clock"),
        "dequant": ("hbm", wk["dequant_bytes"] / (ph_ms["dequant"] * 1e6), hbm, "GB/s",
                    "dequant_kernel", "measured HBM copy"),
    }
    dom = max(rl, key=lambda n: ph_ms[n])
    bound, ach, peak, unit, kern, _ = rl[dom]
    peak_src = {n: v[5] for n, v in rl.items()}
    solve_ms = ph_ms["prepare"] + ph_ms["replay"] + ph_ms["update"]
    weights = d_out * d_in
    out = {
        "metric": METRIC, "value": job_throughput(world, weights, step_ms), "unit": UNIT,
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": step_ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16 in; f32 H; f64-accurate factor (int8-slice tensor cores + fp64 mma; U stored f32); f64 working copy and replay; 3xTF32 update", "data": "synthetic",
        "config": {"workload": args.workload, "d_out": d_out, "d_in": d_in, "n_tok": n_tok,
                   "l2": "flushed between timed steps (256 MiB write, untimed)",
                   "parallelism": f"{world} independent layer solves (one per GPU)"},
        "layer_solve_ms": solve_ms,
        "solve_weights_per_s": weights / (solve_ms / 1e3),
        "hessian_tflops": {"algorithmic_syrk_half": wk["hessian_flops"] / (ph_ms["hessian"] * 1e9),
                           "conventional_2Nd2": 2 * n_tok * d_in * d_in / (ph_ms["hessian"] * 1e9)},
        "phase_ms": ph_ms, "phase_launches": ph_launch,
        "phase_roofline": {n: {"bound": b, "achieved": a, "peak": p, "unit": u, "frac": a / p,
                               "kernels": k_, "peak_source": src}
                           for n, (b, a, p, u, k_, src) in rl.items()},
        "roofline": {"phase": dom, "kernel": kern, "bound": bound, "achieved": ach, "peak": peak,
                     "unit": unit, "frac": ach / peak,
                     "traffic": NCU_TRAFFIC.get(dom, {}).get("bytes"),
                     "traffic_launch": NCU_TRAFFIC.get(dom, {}).get("launch"),
                     "peak_source": f"{peak_src[dom]} ({peaks['source']})"},
        "e2e": {"value": job_throughput(world, weights, e2e_ms), "unit": UNIT, "ms_per_step": e2e_ms,
                "h2d_bytes_per_step": W.numel() * W.element_size() + X.numel() * X.element_size(),
                "d2h_bytes_per_step": codes_h.numel() + scales_h.numel() + 4},
        "gpu_launches": launches,
        "layer_error_by_scale_rule": by_rule,
        "clocks": clk.summary(),
    }
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


def oracle_step(W64, X64, rows):
    """One bounded oracle sample: the full Hessian and factor, the solve and
    dequant of `rows`.  Returns (seconds, seconds scaled to the whole layer)."""
    import oracle as O
    t0 = time.perf_counter()
    H = O.hessian(X64)
    Hd, dead, lam = O.damp(H)
    U = O.inverse_cholesky_upper(Hd)
    sg = O.global_scale(W64)
    t1 = time.perf_counter()
    res = O.schur_replay_gptq(W64[rows], U, sg, dead)
    O.dequant(res["codes"], res["scales"], sg, "bf16")
    t2 = time.perf_counter()
    full = (t1 - t0) + (t2 - t1) * W64.shape[0] / len(rows)
    return t2 - t0, full


def oracle_inputs(name, n_rows):
    W, X = workload(name)
    W64 = W.double().numpy()
    X64 = X.double().numpy()
    rows = np.sort(np.random.default_rng(7).choice(W64.shape[0], min(n_rows, W64.shape[0]),
                                                   replace=False))
    return W64, X64, rows


def cpu_baseline(name, n_rows=128):
    W64, X64, rows = oracle_inputs(name, n_rows)
    wall, full = oracle_step(W64, X64, rows)
    return {"value": W64.size / full, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
            "sample": (f"full fp64 Hessian and factor; solve + dequant of {len(rows)} of "
                       f"{W64.shape[0]} rows, scaled by rows ({wall:.1f} s wall)")}


def run_reference(args):
    W64, X64, rows = oracle_inputs(args.workload, args.ref_rows)
    for _ in range(args.warmup):
        oracle_step(W64, X64, rows)
    fulls = [oracle_step(W64, X64, rows)[1] for _ in range(args.steps)]
    full = float(np.mean(fulls))
    v = W64.size / full
    d_out, d_in = W64.shape
    return {
        "metric": METRIC, "value": v, "unit": UNIT, "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": full * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "impl": "reference",
        "config": {"workload": args.workload, "d_out": d_out, "d_in": d_in,
                   "n_tok": X64.shape[0], "l2": "n/a (CPU)"},
        "cpu_baseline": {"value": v, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                         "sample": (f"each step: full fp64 Hessian and factor; solve + dequant "
                                    f"of {len(rows)} of {d_out} rows, scaled by rows")},
        "e2e": {"value": v, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--ref-rows", type=int, default=64)
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
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                 device_id=torch.device("cuda", local_rank))
    try:
        out = run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as tdist
            tdist.destroy_process_group()
    if rank == 0:
        if not args.no_cpu_baseline:
            out["cpu_baseline"] = cpu_baseline(args.workload)
        print(json.dumps(out), flush=True)


if __name__ == "__main__":
    main()
