"""Plain fp64 CPU oracle for the per-layer NVFP4 GPTQ solve with Schur Replay.

TEST INFRASTRUCTURE ONLY.  This module is the slow, obviously-correct definition
that the CUDA path is checked against.  Only the tests, the smoke check and the
benchmark's CPU-baseline leg may import it; the product path never does, and it
shares no code, table or constant generator with the CUDA library.

Source of every step: "Replay the Curvature: Accurate and Scalable NVFP4
Quantization for Large Language Model Inference" (arXiv 2609.36654v1), Abstract.
The abstract fixes
  * the format: every 16 E2M1 weights share one E4M3 block scale (Abstract,
    sentence on NVFP4);
  * the setting: GPTQ, in which quantizing one column updates the columns that
    follow it (Abstract, sentence on why scale choice is hard);
  * the method: for each block scale, reproduce the GPTQ updates it causes and
    score the resulting block error after the compensation coming from the
    still-unquantized columns; keep the best scale (Abstract, sentence
    introducing Schur Replay).
It prints no equation, candidate set, rounding rule, damping constant or global
scale.  The readings taken where it is silent are marked READING below:

  READING R1  two-level scale: a per-tensor fp32 global scale
              s_g = fp32(amax|W| / (6 * 448)) (s_g = 1 when W == 0), dequant
              q = e2m1 * e4m3 * s_g.
  READING R2  E2M1 rounding is round-to-nearest, ties to the even code,
              saturating at 6; a code whose magnitude is 0 is stored as +0.
  READING R3  E4M3 (fn variant, bias 7, max 448, 0x7F = NaN) rounding is
              round-to-nearest-even with saturation.
  READING R4  candidate set: the 16 consecutive E4M3 codes k0-8 .. k0+7 around
              k0 = e4m3(amax_block / (6 s_g)) (k0 >= 1), shifted to stay inside
              codes 1..126.  For normal k0 this is every E4M3 value in
              [s0/2, 2 s0): one octave on each side of the amax-fitting scale.
  READING R5  the block amax is taken on the current, GPTQ-updated weights.
  READING R6  score = sum over the block's 16 columns of delta_j^2 with
              delta_j = (v_j - q_j) / U_jj (the GPTQ error term).  delta_j^2 is
              (v_j - q_j)^2 times 1/U_jj^2, and 1/U_jj^2 is the Schur complement
              of column j given the columns after it; the sum is the block's
              exact contribution to tr((W-Q) H_d (W-Q)^T).  Ties go to the
              lower code.  The choice is greedy, block by block.
  READING R7  damping lambda = 0.01 * mean(diag H); H_d = H + lambda I.  A
              column with H_ii == 0 is "dead": H_ii := 1 and W[:, i] := 0
              before anything else (the usual GPTQ convention).
  READING R8  U is the upper Cholesky factor of H_d^-1 (H_d^-1 = U^T U), the
              factor GPTQ updates with; no column reordering.
  READING R9  H = X^T X with no 1/N or factor 2 (codes are invariant to a
              scale of H because lambda scales with it).
  READING R14 export: the codes keep their row-major packed layout (two
              E2M1 nibbles per byte, low nibble = even column), which is the
              K-major data layout of an FP4 GEMM operand; the E4M3 block
              scales are re-tiled into the 128-row x 4-column, 512-byte tiles
              in which block-scaled tensor-core GEMMs read their scale operand
              (the public cuBLAS/CUTLASS layout for 16-element-block FP4
              operands); s_g becomes the GEMM's output scale.  The page only
              says that layers are exported.
  READING R10 the rules Schur Replay is set against (Abstract, sentence on
              why scale choice is hard: a block evaluated on its own can
              misestimate its final error) are taken as two independent-block
              rules run inside the same GPTQ sweep, same amax (R5) and same
              window (R4), so that only the scale decision differs:
                amax       k = k0, the scale that maps the block amax to 6;
                block_mse  k = argmin over the window of sum_j (v_j - q_j)^2
                           with every q_j = s * E2M1(v_j / s) taken on the
                           block's values before any in-block update, no
                           curvature weight; ties to the lower code.
              The block's codes always come from the GPTQ sweep at the chosen
              scale, as for Schur Replay.
"""
from __future__ import annotations

import numpy as np

# --------------------------------------------------------------------------
# Formats (Abstract, sentence on NVFP4: 16 E2M1 weights share one E4M3 scale)
# --------------------------------------------------------------------------

# E2M1 magnitudes by 3-bit magnitude index (bit 2..1 exponent, bit 0 mantissa).
E2M1_MAGNITUDE = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
E2M1_MAX = 6.0
E4M3_MAX = 448.0
BLOCK = 16            # weights per block scale
N_CAND = 16           # candidate block scales (READING R4)
CAND_LO = -8          # first candidate offset from k0 (READING R4)
DAMP = 0.01           # READING R7

# Block-scale rules (READING R6 for Schur Replay, R10 for the other two).
RULE_SCHUR_REPLAY = 0
RULE_AMAX = 1
RULE_BLOCK_MSE = 2
RULE_NAMES = {"schur_replay": RULE_SCHUR_REPLAY, "amax": RULE_AMAX,
              "block_mse": RULE_BLOCK_MSE}


def e4m3_value(code):
    """Value of a positive E4M3 (fn) code 0..126 (READING R3).

    code = (e << 3) | m.  e == 0: subnormal m * 2**-9.  Otherwise
    (1 + m/8) * 2**(e - 7).  0x7F is NaN and is never produced.
    """
    code = np.asarray(code, dtype=np.int64)
    e = code >> 3
    m = code & 7
    sub = m * 2.0 ** -9
    nrm = (1.0 + m / 8.0) * np.exp2(e - 7.0)
    return np.where(e == 0, sub, nrm)


E4M3_TABLE = e4m3_value(np.arange(127))   # strictly increasing, 0 .. 448


def e4m3_round_code(t):
    """Round non-negative t to the nearest E4M3 code, ties to the even code,
    saturating at 448 (code 126).  READING R3."""
    t = np.asarray(t, dtype=np.float64)
    t = np.minimum(t, E4M3_MAX)
    hi = np.searchsorted(E4M3_TABLE, t, side="left")        # first value >= t
    hi = np.clip(hi, 0, 126)
    lo = np.clip(hi - 1, 0, 126)
    d_lo = t - E4M3_TABLE[lo]
    d_hi = E4M3_TABLE[hi] - t
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    return np.where(pick_hi, hi, lo).astype(np.int64)


def e2m1_round(x):
    """Signed E2M1 code nibble of x: nearest grid value, ties to the even code
    (magnitude index with bit 0 clear), |x| >= 6 saturating to 6, and a zero
    magnitude stored as +0 (READING R2).  Returns int64 codes 0..15 where bit 3
    is the sign."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    mids = (E2M1_MAGNITUDE[:-1] + E2M1_MAGNITUDE[1:]) / 2.0   # 7 midpoints
    idx = np.zeros(a.shape, dtype=np.int64)
    for k, m in enumerate(mids):
        above = a > m
        tie_to_upper_even = (a == m) & (k % 2 == 1)   # index k odd -> k+1 even
        idx += (above | tie_to_upper_even).astype(np.int64)
    sign = ((x < 0) & (idx > 0)).astype(np.int64)
    return idx | (sign << 3)


def e2m1_value(code):
    """Value of a signed E2M1 code nibble."""
    code = np.asarray(code, dtype=np.int64)
    mag = E2M1_MAGNITUDE[code & 7]
    return np.where(code & 8, -mag, mag)


# --------------------------------------------------------------------------
# Second-order state (Abstract, sentences on GPTQ and on second-order state)
# --------------------------------------------------------------------------

def hessian(X):
    """H = X^T X in fp64 over the calibration tokens (rows of X).  READING R9."""
    X = np.asarray(X, dtype=np.float64)
    return X.T @ X


def damp(H, frac=DAMP):
    """Dead-column fix and damping (READING R7).

    Returns (H_d, dead, lam): dead[i] is True where H_ii == 0; those get
    H_ii = 1 before lambda = frac * mean(diag H) is added to the diagonal."""
    H = np.array(H, dtype=np.float64, copy=True)
    dead = np.diag(H) == 0.0
    H[dead, dead] = 1.0
    lam = frac * float(np.mean(np.diag(H)))
    H[np.diag_indices_from(H)] += lam
    return H, dead, lam


def inverse_cholesky_upper(H_d):
    """U upper with positive diagonal such that H_d^-1 = U^T U (READING R8).

    Route: explicit inverse, then the lower Cholesky factor L of it, U = L^T.
    (The CUDA path takes another route; the factor is unique.)  Raises
    numpy.linalg.LinAlgError when H_d is not positive definite."""
    Hinv = np.linalg.inv(np.asarray(H_d, dtype=np.float64))
    Hinv = (Hinv + Hinv.T) / 2.0
    L = np.linalg.cholesky(Hinv)
    return L.T.copy()


# --------------------------------------------------------------------------
# Global scale (READING R1)
# --------------------------------------------------------------------------

def global_scale(W):
    """s_g = fp32(amax|W| / (6 * 448)); 1.0 when W is all zero.

    W holds fp32-representable values, so the fp64 quotient rounded once to
    fp32 equals the correctly rounded fp32 division."""
    amax = float(np.max(np.abs(W))) if np.size(W) else 0.0
    if amax == 0.0:
        return np.float32(1.0)
    return np.float32(amax / (E2M1_MAX * E4M3_MAX))


def candidate_codes(k0, n_cand=N_CAND, cand_lo=CAND_LO):
    """The n_cand consecutive E4M3 codes starting at k0 + cand_lo, shifted to
    stay within 1..126 (READING R4).  k0 may be an array; returns
    k0.shape + (n_cand,)."""
    k0 = np.asarray(k0, dtype=np.int64)
    lo = np.clip(k0 + cand_lo, 1, 127 - n_cand)
    return lo[..., None] + np.arange(n_cand)


def block_center_code(amax_block, s_g):
    """k0 = e4m3(amax_block / (6 s_g)), at least 1 (READING R4)."""
    k0 = e4m3_round_code(np.asarray(amax_block, dtype=np.float64)
                         / (E2M1_MAX * float(s_g)))
    return np.maximum(k0, 1)


# --------------------------------------------------------------------------
# Schur Replay inside GPTQ (Abstract, sentence introducing Schur Replay)
# --------------------------------------------------------------------------

def replay_block(v, Ublk, s):
    """Replay the in-block GPTQ column updates for given block scales.

    v     (..., 16)  current (updated) weights of one block
    Ublk  (16, 16)   the block's diagonal block of U (upper)
    s     (...)      block scale(s) e4m3(k) * s_g, broadcast against v[..., 0]
    Returns (codes (...,16), q (...,16), delta (...,16), score (...)).

    Column j is quantized on its current value, its error divided by U_jj is
    delta_j, and the columns after it inside the block absorb delta_j * U[j, i]
    -- exactly the GPTQ update.  score = sum_j delta_j^2 (READING R6)."""
    v = np.array(v, dtype=np.float64, copy=True)
    s = np.asarray(s, dtype=np.float64)
    v, s = np.broadcast_arrays(v, s[..., None])
    v = v.copy()
    s = s[..., 0]
    codes = np.zeros(v.shape, dtype=np.int64)
    q = np.zeros(v.shape)
    delta = np.zeros(v.shape)
    for j in range(BLOCK):
        c = e2m1_round(v[..., j] / s)
        codes[..., j] = c
        q[..., j] = e2m1_value(c) * s
        delta[..., j] = (v[..., j] - q[..., j]) / Ublk[j, j]
        v[..., j + 1:] -= delta[..., j, None] * Ublk[j, j + 1:]
    score = np.sum(delta * delta, axis=-1)
    return codes, q, delta, score


def independent_block_error(v, s):
    """Squared error of rounding each of a block's values on its own at scale
    s, with no GPTQ update between the columns and no curvature weight
    (READING R10).  v (..., 16), s (...) -> (...)."""
    v = np.asarray(v, dtype=np.float64)
    s = np.asarray(s, dtype=np.float64)[..., None]
    q = e2m1_value(e2m1_round(v / s)) * s
    return np.sum((v - q) ** 2, axis=-1)


def e4m3_rounding_margin(t):
    """Relative distance of t >= 0 to the nearest E4M3 rounding boundary (the
    midpoint of two adjacent codes): how far the amax rule's k0 is from
    flipping.  Infinite for t == 0."""
    t = np.asarray(t, dtype=np.float64)
    mids = (E4M3_TABLE[:-1] + E4M3_TABLE[1:]) / 2.0
    d = np.min(np.abs(t[..., None] - mids), axis=-1)
    with np.errstate(divide="ignore", invalid="ignore"):
        return np.where(t > 0, d / t, np.inf)


def schur_replay_gptq(W, U, s_g, dead=None, n_cand=N_CAND, cand_lo=CAND_LO,
                      return_diag=False, rule=RULE_SCHUR_REPLAY):
    """GPTQ over the columns of W (d_out x d_in) with every 16-column block's
    E4M3 scale chosen by Schur Replay (rule = RULE_SCHUR_REPLAY), or by one of
    the independent-block rules of READING R10 (RULE_AMAX, RULE_BLOCK_MSE).

    Rows are independent given U.  For block b (columns c0..c0+15):
      a  = max |W~[r, block]| on the updated weights        (READING R5)
      k0 = e4m3(a / (6 s_g)), candidates k0-8 .. k0+7          (READING R4)
      each candidate: replay the in-block updates, score sum delta^2
      k* = argmin (lowest code on ties)                        (READING R6)
      emit k*'s codes; W~[r, c0+16:] -= delta^T U[block, c0+16:]
    A block whose amax is 0 emits scale code 0, codes 0, delta 0.

    Returns dict: codes (d_out, d_in) int64 nibbles, scales (d_out, d_in/16)
    int64 E4M3 codes, q (fp64 dequantized values), delta (d_out, d_in),
    err_sum = sum delta^2, and with return_diag: cand (d_out, nb, n_cand),
    scores (d_out, nb, n_cand) Schur Replay scores of every candidate (under
    any rule), wblock (updated W~ block inputs), margin (d_out, nb): how
    close the rule's decision is to flipping -- the relative gap of its two
    best scores, or for the amax rule e4m3_rounding_margin(a / (6 s_g))."""
    rule = RULE_NAMES.get(rule, rule)
    if rule not in (RULE_SCHUR_REPLAY, RULE_AMAX, RULE_BLOCK_MSE):
        raise ValueError(f"unknown scale rule {rule!r}")
    W = np.array(W, dtype=np.float64, copy=True)
    d_out, d_in = W.shape
    if d_in % BLOCK:
        raise ValueError("d_in must be a multiple of 16")
    if dead is not None and np.any(dead):
        W[:, dead] = 0.0
    nb = d_in // BLOCK
    s_g = float(np.float32(s_g))
    codes = np.zeros((d_out, d_in), dtype=np.int64)
    scales = np.zeros((d_out, nb), dtype=np.int64)
    q = np.zeros((d_out, d_in))
    delta = np.zeros((d_out, d_in))
    if return_diag:
        cand_all = np.zeros((d_out, nb, n_cand), dtype=np.int64)
        scores_all = np.zeros((d_out, nb, n_cand))
        win_all = np.zeros((d_out, nb, BLOCK))
        margin_all = np.full((d_out, nb), np.inf)
    for b in range(nb):
        c0, c1 = b * BLOCK, (b + 1) * BLOCK
        v = W[:, c0:c1]
        Ublk = U[c0:c1, c0:c1]
        amax = np.max(np.abs(v), axis=1)
        live = amax > 0.0
        k0 = block_center_code(np.where(live, amax, 1.0), s_g)
        cand = candidate_codes(k0, n_cand, cand_lo)           # (d_out, n_cand)
        s = e4m3_value(cand) * s_g                            # exact in fp64
        c_codes, c_q, c_delta, c_score = replay_block(v[:, None, :], Ublk, s)
        if rule == RULE_AMAX:
            best = k0 - cand[:, 0]                            # k0 is in the window
            margin = e4m3_rounding_margin(amax / (E2M1_MAX * s_g))
        else:
            sel = c_score if rule == RULE_SCHUR_REPLAY else \
                independent_block_error(v[:, None, :], s)
            best = np.argmin(sel, axis=1)                     # first = lowest code
            srt = np.sort(sel, axis=1)
            margin = (srt[:, 1] - srt[:, 0]) / np.maximum(srt[:, 0], 1e-300)
        rows = np.arange(d_out)
        blk_codes = c_codes[rows, best]
        blk_q = c_q[rows, best]
        blk_delta = c_delta[rows, best]
        blk_scale = cand[rows, best]
        blk_codes[~live] = 0
        blk_q[~live] = 0.0
        blk_delta[~live] = 0.0
        blk_scale[~live] = 0
        codes[:, c0:c1] = blk_codes
        q[:, c0:c1] = blk_q
        delta[:, c0:c1] = blk_delta
        scales[:, b] = blk_scale
        if return_diag:
            cand_all[:, b] = cand
            scores_all[:, b] = np.where(live[:, None], c_score, 0.0)
            win_all[:, b] = v
            margin_all[:, b] = np.where(live, margin, np.inf)
        if c1 < d_in:
            W[:, c1:] -= blk_delta @ U[c0:c1, c1:]
    out = dict(codes=codes, scales=scales, q=q, delta=delta,
               err_sum=float(np.sum(delta * delta)),
               row_err=np.sum(delta * delta, axis=1))
    if return_diag:
        out.update(cand=cand_all, scores=scores_all, wblock=win_all, margin=margin_all)
    return out


# --------------------------------------------------------------------------
# Dequantization and measurement
# --------------------------------------------------------------------------

def dequant(codes, scales, s_g, out_dtype=np.float32):
    """Q = e2m1(code) * e4m3(scale) * s_g: the product is exact in fp64
    (2 + 4 + 24 significant bits) and is rounded once to out_dtype."""
    codes = np.asarray(codes)
    d_out, d_in = codes.shape
    sv = e4m3_value(np.asarray(scales)).repeat(BLOCK, axis=1)
    exact = e2m1_value(codes) * sv * float(np.float32(s_g))
    if out_dtype == np.float32:
        return exact.astype(np.float32)
    if out_dtype == "bf16":
        return round_to_bf16(exact)
    raise ValueError(out_dtype)


# --------------------------------------------------------------------------
# Export layout (Abstract, infrastructure sentence: layers are exported before
# their full-precision weights are retired)
# --------------------------------------------------------------------------

SF_TILE_ROWS, SF_TILE_COLS = 128, 4   # one 512-byte tile of block scales


def scales_to_tiled(scales):
    """The block scales (rows x nb E4M3 codes, nb = d_in / 16) in the tiled
    layout that block-scaled tensor-core GEMMs read their scale operand in
    (READING R14): rows and scale columns padded with zero codes to multiples
    of 128 and 4; tile (R, C) of 128 rows x 4 scale columns is 512 contiguous
    bytes, tiles in row-major order over (R, C); inside a tile, the scale of
    row r and column c sits at byte (r % 32) * 16 + (r // 32) * 4 + c.
    Returns a flat uint8 array."""
    scales = np.asarray(scales, dtype=np.uint8)
    rows, nb = scales.shape
    rp = -(-rows // SF_TILE_ROWS) * SF_TILE_ROWS
    cp = -(-nb // SF_TILE_COLS) * SF_TILE_COLS
    padded = np.zeros((rp, cp), dtype=np.uint8)
    padded[:rows, :nb] = scales
    out = np.zeros(rp * cp, dtype=np.uint8)
    n_ct = cp // SF_TILE_COLS
    for r in range(rp):
        for c in range(cp):
            tile = (r // SF_TILE_ROWS) * n_ct + c // SF_TILE_COLS
            rr, cc = r % SF_TILE_ROWS, c % SF_TILE_COLS
            out[tile * 512 + (rr % 32) * 16 + (rr // 32) * 4 + cc] = padded[r, c]
    return out


def round_to_bf16(x):
    """Round fp64 values to bf16 (RN-even, one rounding straight from fp64),
    returned as float32 arrays holding the bf16 values.  Going through fp32
    first would round twice.  bf16 has fp32's exponent range: 8 significant
    bits in the binades from 2^-126 up, below that the fixed spacing 2^-133 of
    its subnormals; values from (2 - 2^-8) 2^127 up round to infinity."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                      # x = m * 2**e, 0.5 <= |m| < 1
    e = np.maximum(e, -125)                 # spacing 2^(e - 8) >= 2^-133
    r = np.rint(np.ldexp(x, 8 - e))         # ties to even
    with np.errstate(over="ignore"):
        return np.ldexp(r, e - 8).astype(np.float32)


def layer_error(W, Q, H):
    """tr((W - Q) H (W - Q)^T) in fp64 on the undamped H."""
    E = np.asarray(W, dtype=np.float64) - np.asarray(Q, dtype=np.float64)
    return float(np.einsum("ij,ij->", E @ np.asarray(H, dtype=np.float64), E))


def solve_layer(W, X=None, H=None, damp_frac=DAMP, n_cand=N_CAND,
                cand_lo=CAND_LO, return_diag=False, rule=RULE_SCHUR_REPLAY):
    """The whole per-layer solve: Hessian, damping, factor, global scale,
    Schur Replay GPTQ, dequant and layer error."""
    if H is None:
        H = hessian(X)
    H_d, dead, lam = damp(H, damp_frac)
    U = inverse_cholesky_upper(H_d)
    W = np.asarray(W, dtype=np.float64)
    Wz = W.copy()
    Wz[:, dead] = 0.0
    s_g = global_scale(Wz)
    res = schur_replay_gptq(Wz, U, s_g, dead, n_cand, cand_lo, return_diag, rule)
    Q = dequant(res["codes"], res["scales"], s_g)
    res.update(H=H, H_d=H_d, U=U, dead=dead, lam=lam, s_g=s_g, Q=Q,
               W=Wz, layer_error=layer_error(Wz, res["q"], H))
    return res
