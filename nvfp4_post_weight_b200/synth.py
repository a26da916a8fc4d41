"""Seeded synthetic layer inputs (weights W and calibration activations X).

This module only draws random numbers and rounds them to the storage dtype; it
holds none of the quantization arithmetic, so both the CUDA path and the fp64
oracle can be fed from it.  Every tensor gets its own child stream of
numpy.random.SeedSequence(seed), spawned in the order the tensors are listed.
Storage rounding to bf16 is round-to-nearest-even (torch's CPU cast).

Workloads (no trained model or calibration set is available, so these stand in
for the pages' LLM layers):
  small_outlier   fp32 W ~ N(0, 0.02^2) with 4 outlier input columns x20;
                  fp32 X ~ N(0,1) x per-channel lognormal(0, 1).
  attn_massive    bf16 W ~ N(0, 0.02^2) with 0.1% of entries replaced by
                  0.02 * Student-t(3); bf16 X ~ N(0,1) x lognormal(0, 1.5)
                  per channel, 8 "massive" channels x100.
  mlp_down_silu   bf16 W ~ N(0, 0.015^2); bf16 X = SiLU(A) * B, A, B ~ N(0,1).
  lognormal       bf16 W ~ N(0, 0.02^2); bf16 X ~ N(0,1) x lognormal(0, sigma)
                  per channel (the dense-decoder and MoE-expert layers; their
                  large tensors are drawn in float32 by row chunks, each chunk
                  from its own child stream, on a thread pool).
"""
from __future__ import annotations

import numpy as np
import torch


def _children(seed: int, n: int):
    return [np.random.default_rng(s) for s in np.random.SeedSequence(seed).spawn(n)]


def _bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)


def _f32(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))


def small_outlier(d_out=256, d_in=256, n_tok=512, seed=0):
    """fp32 layer with 4 outlier input columns (x20) and lognormal(0,1)
    channel scales on the activations."""
    g_w, g_o, g_x, g_s = _children(seed, 4)
    W = g_w.normal(0.0, 0.02, size=(d_out, d_in))
    cols = g_o.choice(d_in, size=min(4, d_in), replace=False)
    W[:, cols] *= 20.0
    X = g_x.standard_normal((n_tok, d_in))
    X *= g_s.lognormal(0.0, 1.0, size=d_in)[None, :]
    return _f32(W), _f32(X)


def attn_massive(d_out=4096, d_in=4096, n_tok=4096, seed=1, n_massive=8):
    """bf16 layer with 0.1% Student-t(3) weights and massive activation
    channels (x100) on top of lognormal(0, 1.5) channel scales."""
    g_w, g_p, g_t, g_x, g_s, g_m = _children(seed, 6)
    W = g_w.normal(0.0, 0.02, size=(d_out, d_in)).astype(np.float32)
    n_heavy = int(round(0.001 * d_out * d_in))
    pos = g_p.choice(d_out * d_in, size=n_heavy, replace=False)
    W.reshape(-1)[pos] = 0.02 * g_t.standard_t(3.0, size=n_heavy)
    X = g_x.standard_normal((n_tok, d_in), dtype=np.float32)
    scale = g_s.lognormal(0.0, 1.5, size=d_in).astype(np.float32)
    massive = g_m.choice(d_in, size=min(n_massive, d_in), replace=False)
    scale[massive] *= 100.0
    X *= scale[None, :]
    return _bf16(W), _bf16(X)


def mlp_down_silu(d_out=4096, d_in=14336, n_tok=8192, seed=2):
    """bf16 down-projection-shaped layer; activations are the SiLU-gated
    product of two N(0,1) streams."""
    g_w, g_a, g_b = _children(seed, 3)
    W = g_w.normal(0.0, 0.015, size=(d_out, d_in)).astype(np.float32)
    A = g_a.standard_normal((n_tok, d_in), dtype=np.float32)
    B = g_b.standard_normal((n_tok, d_in), dtype=np.float32)
    X = A / (1.0 + np.exp(-A)) * B
    return _bf16(W), _bf16(X)


def lognormal_acts(n_tok, d_in, sigma, rng_x, rng_s):
    X = rng_x.standard_normal((n_tok, d_in), dtype=np.float32)
    X *= rng_s.lognormal(0.0, sigma, size=d_in).astype(np.float32)[None, :]
    return _bf16(X)


def normal_weights(d_out, d_in, std, rng):
    return _bf16(rng.normal(0.0, std, size=(d_out, d_in)).astype(np.float32))


# Large tensors are drawn in row chunks of _CHUNK_ROWS rows, chunk c from the
# c-th child of the tensor's own SeedSequence, on a thread pool (numpy's
# generators release the GIL while they fill an array), in float32 precision.
_CHUNK_ROWS = 1024


def _pool():
    import concurrent.futures as cf
    import os
    return cf.ThreadPoolExecutor(max(1, min(32, len(os.sched_getaffinity(0)))))


def _fill_rows(out: np.ndarray, ss: np.random.SeedSequence, draw, pool=None) -> None:
    """out[r0:r1] = draw(rng_c, out[r0:r1]) for every row chunk c, rng_c the
    chunk's own generator; the chunks are independent, so the result does
    not depend on the number of threads.  pool: a thread pool, None (a new
    one) or "serial" (this thread)."""
    rows = out.shape[0]
    kids = ss.spawn((rows + _CHUNK_ROWS - 1) // _CHUNK_ROWS)

    def one(c):
        r0, r1 = c * _CHUNK_ROWS, min(rows, (c + 1) * _CHUNK_ROWS)
        draw(np.random.default_rng(kids[c]), out[r0:r1])

    if pool == "serial":
        for c in range(len(kids)):
            one(c)
    elif pool is None:
        with _pool() as p:
            list(p.map(one, range(len(kids))))
    else:
        list(pool.map(one, range(len(kids))))


def normal_weights_fast(d_out, d_in, std, ss, pool=None):
    """bf16 (d_out, d_in) ~ N(0, std^2), drawn in float32 by row chunks."""
    W = np.empty((d_out, d_in), dtype=np.float32)

    def draw(g, blk):
        g.standard_normal(out=blk, dtype=np.float32)
        blk *= np.float32(std)

    _fill_rows(W, ss, draw, pool)
    return _bf16(W)


def lognormal_acts_fast(n_tok, d_in, sigma, ss, pool=None):
    """bf16 (n_tok, d_in) activations: N(0,1) (float32, by row chunks of the
    first child of ss) times per-channel lognormal(0, sigma) scales (second
    child)."""
    ss_x, ss_s = ss.spawn(2)
    scale = np.random.default_rng(ss_s).lognormal(0.0, sigma, size=d_in).astype(np.float32)
    X = np.empty((n_tok, d_in), dtype=np.float32)

    def draw(g, blk):
        g.standard_normal(out=blk, dtype=np.float32)
        blk *= scale[None, :]

    _fill_rows(X, ss_x, draw, pool)
    return _bf16(X)


# The 70B-shaped dense decoder layer: its linears, each as (d_out, d_in), in
# the order they are solved; the Hessian groups share one factor.
DENSE_70B_SHAPES = {"q": (8192, 8192), "k": (1024, 8192), "v": (1024, 8192),
                    "o": (8192, 8192), "gate": (28672, 8192), "up": (28672, 8192),
                    "down": (8192, 28672)}
DENSE_70B_GROUPS = (("X_attn", ("q", "k", "v")), ("X_o", ("o",)), ("X_mlp", ("gate", "up")),
                    ("X_down", ("down",)))


def dense_decoder_layer(hidden=8192, kv=1024, inter=28672, n_tok=16384, seed=3):
    """70B-shaped dense decoder layer: q, k, v, o, gate, up, down weights
    (bf16 ~ N(0, 0.02^2)) and four independent calibration activations
    (attention input, o input, MLP input, down input: n_tok tokens,
    N(0,1) x lognormal(0, 1.5) channel scales).  Every tensor has its own
    child of SeedSequence(seed), in the order q, k, v, o, gate, up, down,
    X_attn, X_o, X_mlp, X_down.  Returned lazily as a dict of callables so
    that a caller can build one tensor at a time."""
    names = ["q", "k", "v", "o", "gate", "up", "down", "X_attn", "X_o", "X_mlp", "X_down"]
    kids = dict(zip(names, np.random.SeedSequence(seed).spawn(len(names))))
    shapes = {"q": (hidden, hidden), "k": (kv, hidden), "v": (kv, hidden),
              "o": (hidden, hidden), "gate": (inter, hidden), "up": (inter, hidden),
              "down": (hidden, inter)}
    out = {}
    for n, shp in shapes.items():
        out[n] = (lambda shp=shp, ss=kids[n]: normal_weights_fast(shp[0], shp[1], 0.02, ss))
    for x, d in (("attn", hidden), ("o", hidden), ("mlp", hidden), ("down", inter)):
        out["X_" + x] = (lambda d=d, ss=kids["X_" + x]: lognormal_acts_fast(n_tok, d, 1.5, ss))
    return out


def zipf_token_counts(n_experts=128, total=65536, alpha=1.1, lo=64, hi=4096):
    """Deterministic Zipf(alpha) routed-token counts that sum exactly to total:
    n_e = clamp(c * rank^-alpha, lo, hi) with c found by bisection, floored,
    the largest remainders taking the leftover tokens."""
    ranks = np.arange(1, n_experts + 1, dtype=np.float64)
    base = ranks ** (-alpha)

    def tot(c):
        return np.clip(c * base, lo, hi).sum()

    a, b = 0.0, float(total) * 10.0
    for _ in range(200):
        m = 0.5 * (a + b)
        if tot(m) < total:
            a = m
        else:
            b = m
    real = np.clip(b * base, lo, hi)
    n = np.floor(real).astype(np.int64)
    rem = real - n
    short = int(total - n.sum())
    order = np.argsort(-rem, kind="stable")
    n[order[:short]] += 1
    return n


def moe_layer(n_experts=128, hidden=4096, inter=1536, total_tokens=65536, seed=4):
    """MoE layer of independent experts (gate/up hidden->inter, down
    inter->hidden, bf16 ~ N(0, 0.02^2); activations N(0,1) x lognormal(0, 1)
    channel scales).  Returns (counts, make_expert) where make_expert(e)
    draws expert e's tensors from the children of the e-th child of
    SeedSequence(seed), in the order gate, up, down, X_in, X_mid."""
    counts = zipf_token_counts(n_experts, total_tokens)
    roots = np.random.SeedSequence(seed).spawn(n_experts)

    def make_expert(e, pool=None):
        g = roots[e].spawn(5)
        n = int(counts[e])
        return dict(
            gate=normal_weights_fast(inter, hidden, 0.02, g[0], pool),
            up=normal_weights_fast(inter, hidden, 0.02, g[1], pool),
            down=normal_weights_fast(hidden, inter, 0.02, g[2], pool),
            X_in=lognormal_acts_fast(n, hidden, 1.0, g[3], pool),
            X_mid=lognormal_acts_fast(n, inter, 1.0, g[4], pool),
        )

    return counts, make_expert


def moe_all_experts(n_experts=128, **kw):
    """counts and the list of every expert's tensors of moe_layer (drawn on
    one thread pool)."""
    counts, make = moe_layer(n_experts=n_experts, **kw)
    with _pool() as p:
        experts = list(p.map(lambda e: make(e, "serial"), range(n_experts)))
    return counts, experts


WORKLOADS = {
    "small_outlier_256x256": lambda: small_outlier(),
    "attn_massive_4096x4096": lambda: attn_massive(),
    "mlp_down_silu_4096x14336": lambda: mlp_down_silu(),
}
