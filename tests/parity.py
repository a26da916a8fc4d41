"""Comparison helpers for the GPU-vs-oracle parity tests.

The acceptance rule for the discrete outputs (E2M1 codes, E4M3 scales):
  * small layers: bit-exact;
  * larger layers: at least 99.9% of the 16-weight blocks identical, and in
    every row the FIRST block that differs must sit at a near-tie of the
    oracle -- its scale decision within 1e-5 relative of flipping (the top two
    candidate scores of a search rule; for the amax rule the block amax / 6 s_g
    against the nearest E4M3 rounding midpoint), or one of its
    codes within 1e-5 (relative to the grid step) of an E2M1 rounding
    midpoint.  Once a row has taken a different discrete decision its later
    blocks start from different weights (GPTQ carries every column's error
    forward), so the blocks after the first difference count towards the 0.1%
    budget but are not themselves required to be near-ties.
"""
from __future__ import annotations

import numpy as np

import oracle as O

NEAR_TIE = 1e-5


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    """(rows, d_in/2) packed bytes -> (rows, d_in) nibbles; the low nibble of
    byte c is column 2c."""
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty((p.shape[0], p.shape[1] * 2), dtype=np.int64)
    out[:, 0::2] = p & 0xF
    out[:, 1::2] = p >> 4
    return out


def pack_codes(codes: np.ndarray) -> np.ndarray:
    c = np.asarray(codes, dtype=np.uint8)
    return (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)


def top2_margin(scores: np.ndarray) -> np.ndarray:
    """(..., n_cand) scores -> relative gap between the two smallest."""
    s = np.sort(scores, axis=-1)
    return (s[..., 1] - s[..., 0]) / np.maximum(s[..., 0], 1e-300)


def midpoint_distance(v: np.ndarray, Ublk: np.ndarray, s: float) -> float:
    """Smallest distance, in units of the local E2M1 grid step, from any
    in-block GPTQ-updated value x_j / s of the replay at scale s to an E2M1
    rounding midpoint.  Replays with the oracle's own arithmetic."""
    v = np.array(v, dtype=np.float64, copy=True)
    best = np.inf
    mids = (O.E2M1_MAGNITUDE[:-1] + O.E2M1_MAGNITUDE[1:]) / 2.0
    steps = np.diff(O.E2M1_MAGNITUDE)
    for j in range(O.BLOCK):
        x = abs(v[j] / s)
        d = np.min(np.abs(x - mids) / steps)
        best = min(best, d)
        q = O.e2m1_value(O.e2m1_round(v[j] / s)) * s
        dj = (v[j] - q) / Ublk[j, j]
        v[j + 1:] -= dj * Ublk[j, j + 1:]
    return float(best)


def classify(ref: dict, U: np.ndarray, s_g: float, codes_gpu: np.ndarray,
             scales_gpu: np.ndarray, rows=None):
    """Compare GPU codes/scales with the oracle's (ref from
    oracle.schur_replay_gptq(..., return_diag=True)) on the given oracle rows.

    Returns a dict: n_blocks, n_mismatch, frac, rows_affected; for the first
    differing block of every affected row, which clause excused it:
    first_scale_tie (the oracle's top two scores within NEAR_TIE, the rule the
    acceptance criterion states) or first_midpoint (a replayed value within
    NEAR_TIE of an E2M1 rounding midpoint, this suite's reading of the same
    kind of event for the codes); and bad_first: list of (row, block, margin,
    midpoint_dist) for rows whose first differing block is neither."""
    oc = ref["codes"]
    os_ = ref["scales"]
    gc = codes_gpu
    gs = scales_gpu
    nb = os_.shape[1]
    blk_code_eq = (oc.reshape(oc.shape[0], nb, O.BLOCK) ==
                   gc.reshape(gc.shape[0], nb, O.BLOCK)).all(axis=2)
    blk_eq = blk_code_eq & (os_ == gs)
    mism = ~blk_eq
    res = dict(n_blocks=int(blk_eq.size), n_mismatch=int(mism.sum()),
               frac=float(mism.mean()) if blk_eq.size else 0.0,
               rows_affected=int(mism.any(axis=1).sum()), first_scale_tie=0,
               first_midpoint=0, bad_first=[])
    sg = float(np.float32(s_g))
    for r in np.nonzero(mism.any(axis=1))[0]:
        b = int(np.argmax(mism[r]))
        margin = float(ref["margin"][r, b]) if "margin" in ref else \
            float(top2_margin(ref["scores"][r, b]))
        if margin < NEAR_TIE:
            res["first_scale_tie"] += 1
            continue
        Ublk = U[16 * b:16 * b + 16, 16 * b:16 * b + 16]
        s_or = O.e4m3_value(os_[r, b]) * sg
        dist = midpoint_distance(ref["wblock"][r, b], Ublk, s_or)
        if gs[r, b] != os_[r, b]:
            s_gp = O.e4m3_value(gs[r, b]) * sg
            dist = min(dist, midpoint_distance(ref["wblock"][r, b], Ublk, s_gp))
        if dist < NEAR_TIE:
            res["first_midpoint"] += 1
            continue
        res["bad_first"].append((int(r if rows is None else rows[r]), b, margin, dist))
    return res


def report(label: str, c: dict) -> str:
    """One line of what a comparison found (printed by the parity tests; run
    pytest with -s to see them)."""
    line = (f"PARITY {label}: blocks={c['n_blocks']} mismatched={c['n_mismatch']} "
            f"({c['frac']:.2e}) rows_affected={c['rows_affected']} "
            f"first_excused_scale_tie={c['first_scale_tie']} "
            f"first_excused_midpoint={c['first_midpoint']} bad_first={len(c['bad_first'])}")
    print(line, flush=True)
    return line
