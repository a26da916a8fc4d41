"""Pins for the fp64 oracle: checks against things other than the oracle itself.

* Format tables and rounding against ml_dtypes' independent float8_e4m3fn /
  float4_e2m1fn conversions (round-to-nearest-even on fp32 inputs).
* A textbook GPTQ written here in the Optimal-Brain-Surgeon form (explicit
  inverse, downdated column by column) with its own nearest-grid rounding; it
  shares no routine with the oracle's Cholesky-form replay.
* Brute force over every E4M3 code on tiny layers; closed forms for H = c I
  (GPTQ reduces to round-to-nearest) and diagonal H; the GPTQ loss identity
  tr((W-Q) H_d (W-Q)^T) = sum delta^2.

Method: "Replay the Curvature: Accurate and Scalable NVFP4 Quantization for
Large Language Model Inference", Abstract (NVFP4 format; GPTQ column updates;
Schur Replay scores each block scale by replaying the updates it causes).
"""
import ml_dtypes as md
import numpy as np
import pytest

import oracle as O

# --------------------------------------------------------------------------
# independent helpers (no oracle routine used)
# --------------------------------------------------------------------------
_E2M1_CODES = [c for c in range(16) if c != 8]          # +0 .. +6, -0.5 .. -6


def _e2m1_val(c):
    mags = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    return -mags[c & 7] if c & 8 else mags[c & 7]


def nearest_e2m1_code(x):
    """Nearest signed E2M1 value by exhaustive search; ties go to the code
    whose magnitude index is even.  Beyond +-6 the nearest value is +-6."""
    best, bd = None, None
    for c in _E2M1_CODES:
        d = abs(x - _e2m1_val(c))
        if bd is None or d < bd or (d == bd and (c & 1) == 0 and (best & 1) == 1):
            best, bd = c, d
    return best


def e4m3_val_md(code):
    return float(np.array([code], np.uint8).view(md.float8_e4m3fn).astype(np.float64)[0])


def e4m3_code_md(t):
    t = min(float(t), 448.0)
    return int(np.array([t], np.float32).astype(md.float8_e4m3fn).view(np.uint8)[0])


def obs_gptq_row(w, Hd, scale_of_block, start=0, stop=None, Hinv=None):
    """Textbook GPTQ on one row in Optimal-Brain-Surgeon form.

    Columns start..stop-1 are quantized in order: q_j = s * RN(w_j / s), the
    still-unquantized columns absorb (w_j - q_j) / Hinv_jj * Hinv[j, F], and the
    inverse is downdated to drop column j.  loss_j = (w_j - q_j)^2 / Hinv_jj.
    Returns (w, Hinv, q, loss) so that a caller can resume."""
    w = np.array(w, dtype=np.float64, copy=True)
    d = w.size
    stop = d if stop is None else stop
    if Hinv is None:
        Hinv = np.linalg.inv(Hd)
    Hinv = Hinv.copy()
    q = np.zeros(d)
    loss = np.zeros(d)
    for j in range(start, stop):
        s = scale_of_block(j // 16, w)
        q[j] = _e2m1_val(nearest_e2m1_code(w[j] / s)) * s
        h = Hinv[j, j]
        loss[j] = (w[j] - q[j]) ** 2 / h
        w[j + 1:] -= (w[j] - q[j]) / h * Hinv[j, j + 1:]
        Hinv = Hinv - np.outer(Hinv[:, j], Hinv[j, :]) / h
    return w, Hinv, q, loss


def window_md(amax, s_g):
    k0 = max(e4m3_code_md(amax / (6.0 * s_g)), 1)
    lo = min(max(k0 - 8, 1), 126 - 15)
    return list(range(lo, lo + 16))


def random_layer(rng, d_out, d_in, n_tok, outliers=True):
    W = rng.normal(0, 0.02, size=(d_out, d_in)).astype(np.float32).astype(np.float64)
    if outliers:
        W[:, rng.integers(0, d_in)] *= 20
    X = rng.standard_normal((n_tok, d_in)) * rng.lognormal(0, 1, size=d_in)
    X = X.astype(np.float32).astype(np.float64)
    return W, X


# --------------------------------------------------------------------------
# formats
# --------------------------------------------------------------------------

def test_e4m3_table_matches_ml_dtypes():
    ref = np.arange(127, dtype=np.uint8).view(md.float8_e4m3fn).astype(np.float64)
    np.testing.assert_array_equal(O.E4M3_TABLE, ref)
    assert O.E4M3_TABLE[126] == 448.0 and O.E4M3_TABLE[1] == 2.0 ** -9


def test_e4m3_round_matches_ml_dtypes_including_ties():
    rng = np.random.default_rng(1)
    t = np.concatenate([
        rng.uniform(0, 448, 20000), np.exp(rng.uniform(np.log(1e-4), np.log(448), 20000)),
        (O.E4M3_TABLE[:-1] + O.E4M3_TABLE[1:]) / 2.0, O.E4M3_TABLE]).astype(np.float32)
    ref = t.astype(md.float8_e4m3fn).view(np.uint8).astype(np.int64)
    np.testing.assert_array_equal(O.e4m3_round_code(t.astype(np.float64)), ref)


def test_e4m3_saturates():
    np.testing.assert_array_equal(O.e4m3_round_code([448.0, 460.0, 500.0, 1e9]), [126] * 4)


def test_e2m1_round_matches_ml_dtypes_including_ties():
    rng = np.random.default_rng(2)
    mids = (O.E2M1_MAGNITUDE[:-1] + O.E2M1_MAGNITUDE[1:]) / 2.0
    x = np.concatenate([rng.uniform(-8, 8, 50000), mids, -mids, O.E2M1_MAGNITUDE,
                        -O.E2M1_MAGNITUDE, [7.0, -7.0, 1e6, -1e6, 1e-30, -1e-30]]).astype(np.float32)
    ref = x.astype(md.float4_e2m1fn).view(np.uint8).astype(np.int64) & 0xF
    ref[ref == 8] = 0                              # -0 stored as +0 (READING R2)
    np.testing.assert_array_equal(O.e2m1_round(x.astype(np.float64)), ref)


def test_e2m1_tie_table():
    x = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 7.0, -0.25, -0.3, -5.0]
    want_vals = [0.0, 1.0, 1.0, 2.0, 2.0, 4.0, 4.0, 6.0, 0.0, -0.5, -4.0]
    got = O.e2m1_value(O.e2m1_round(x))
    np.testing.assert_array_equal(got, want_vals)
    assert O.e2m1_round(-0.25) == 0


def test_global_scale_is_correctly_rounded_fp32_division():
    rng = np.random.default_rng(3)
    for _ in range(200):
        W = (rng.standard_normal((8, 16)) * 10 ** rng.uniform(-4, 2)).astype(np.float32)
        want = np.float32(np.max(np.abs(W))) / np.float32(2688.0)
        assert O.global_scale(W) == want
    assert O.global_scale(np.zeros((4, 16))) == np.float32(1.0)


def test_candidate_window_edges():
    np.testing.assert_array_equal(O.candidate_codes(1), np.arange(1, 17))
    np.testing.assert_array_equal(O.candidate_codes(5), np.arange(1, 17))
    np.testing.assert_array_equal(O.candidate_codes(126), np.arange(111, 127))
    np.testing.assert_array_equal(O.candidate_codes(50), np.arange(42, 58))
    # one binade: codes k0-8 .. k0+7 span [s0/2, 2 s0) for normal k0
    v = O.e4m3_value(O.candidate_codes(60))
    assert v[0] == O.e4m3_value(60) / 2 and v[-1] < 2 * O.e4m3_value(60)


# --------------------------------------------------------------------------
# factor
# --------------------------------------------------------------------------

def test_inverse_cholesky_factor_identity_and_reversed_route():
    rng = np.random.default_rng(4)
    _, X = random_layer(rng, 4, 48, 96)
    H_d, _, _ = O.damp(X.T @ X)
    U = O.inverse_cholesky_upper(H_d)
    assert np.allclose(np.tril(U, -1), 0.0) and np.all(np.diag(U) > 0)
    np.testing.assert_allclose(U.T @ U @ H_d, np.eye(48), atol=1e-10)
    # another route to the same unique factor: H_d = R R^T with R upper
    # (Cholesky of the reversed matrix, reversed back), U = R^-1
    J = np.eye(48)[::-1]
    L = np.linalg.cholesky(J @ H_d @ J)
    R = J @ L @ J
    np.testing.assert_allclose(np.linalg.inv(R), U, rtol=1e-9, atol=1e-12)


def test_damping_and_dead_columns():
    rng = np.random.default_rng(5)
    W, X = random_layer(rng, 6, 32, 64)
    X[:, 7] = 0.0
    res = O.solve_layer(W, X)
    assert res["dead"][7] and res["dead"].sum() == 1
    H = X.T @ X
    Hc = H.copy()
    Hc[7, 7] = 1.0
    assert res["lam"] == pytest.approx(0.01 * np.mean(np.diag(Hc)), rel=1e-15)
    assert np.all(res["codes"][:, 7] == 0)


# --------------------------------------------------------------------------
# GPTQ bookkeeping and Schur Replay
# --------------------------------------------------------------------------

@pytest.mark.parametrize("seed,d_out,d_in", [(6, 5, 64), (7, 9, 48), (8, 3, 128)])
def test_gptq_loss_identity(seed, d_out, d_in):
    rng = np.random.default_rng(seed)
    W, X = random_layer(rng, d_out, d_in, 2 * d_in)
    res = O.solve_layer(W, X)
    E = res["W"] - res["q"]
    tr = np.einsum("ij,ij->", E @ res["H_d"], E)
    assert tr == pytest.approx(res["err_sum"], rel=1e-10)
    # layer error on the undamped H differs by lambda * ||E||^2
    assert res["layer_error"] == pytest.approx(tr - res["lam"] * np.sum(E * E), rel=1e-9)


def test_replay_score_equals_textbook_gptq_block_loss():
    rng = np.random.default_rng(9)
    W, X = random_layer(rng, 6, 64, 128)
    res = O.solve_layer(W, X, return_diag=True)
    s_g = float(res["s_g"])
    for r in range(W.shape[0]):
        scales = O.E4M3_TABLE[res["scales"][r]] * s_g
        _, _, q, loss = obs_gptq_row(res["W"][r], res["H_d"], lambda b, w: scales[b])
        np.testing.assert_allclose(q, res["q"][r], rtol=0, atol=1e-15)
        chosen = res["scores"][r][np.arange(4), res["scales"][r] - res["cand"][r][:, 0]]
        np.testing.assert_allclose(loss.reshape(4, 16).sum(1), chosen, rtol=1e-9)


def test_bruteforce_single_block_all_e4m3_codes():
    rng = np.random.default_rng(10)
    W, X = random_layer(rng, 8, 16, 64)
    res = O.solve_layer(W, X, return_diag=True)
    Hd, s_g = res["H_d"], float(res["s_g"])
    in_window = 0
    for r in range(8):
        tot = {}
        for k in range(1, 127):
            s = e4m3_val_md(k) * s_g
            _, _, q, _ = obs_gptq_row(res["W"][r], Hd, lambda b, w: s)
            e = res["W"][r] - q
            tot[k] = float(e @ Hd @ e)
        win = window_md(np.max(np.abs(res["W"][r])), s_g)
        best_in_win = min(win, key=lambda k: (tot[k], k))
        assert res["scales"][r, 0] == best_in_win
        assert res["scores"][r, 0].min() == pytest.approx(tot[best_in_win], rel=1e-10)
        in_window += min(tot, key=lambda k: (tot[k], k)) in win
    # the +-1 octave window should contain the global optimum nearly always
    assert in_window >= 7


def test_bruteforce_two_blocks_greedy():
    rng = np.random.default_rng(11)
    W, X = random_layer(rng, 3, 32, 64)
    res = O.solve_layer(W, X, return_diag=True)
    Hd, s_g = res["H_d"], float(res["s_g"])
    Hinv0 = np.linalg.inv(Hd)
    gaps = []
    for r in range(3):
        w0 = res["W"][r]
        win1 = window_md(np.max(np.abs(w0[:16])), s_g)
        block1 = {}
        allc = {}
        for k1 in win1:
            s1 = e4m3_val_md(k1) * s_g
            w1, Hinv1, q1, l1 = obs_gptq_row(w0, Hd, lambda b, w: s1, 0, 16, Hinv0)
            block1[k1] = l1[:16].sum()
            win2 = window_md(np.max(np.abs(w1[16:32])), s_g)
            for k2 in win2:
                s2 = e4m3_val_md(k2) * s_g
                _, _, q2, l2 = obs_gptq_row(w1, Hd, lambda b, w: s2, 16, 32, Hinv1)
                q = np.concatenate([q1[:16], q2[16:]])
                e = w0 - q
                total = float(e @ Hd @ e)
                assert total == pytest.approx(l1[:16].sum() + l2[16:].sum(), rel=1e-9)
                allc[(k1, k2)] = (total, l2[16:].sum())
        k1s, k2s = res["scales"][r]
        assert k1s == min(win1, key=lambda k: (block1[k], k))
        given = {k2: v for (k1, k2), v in allc.items() if k1 == k1s}
        assert k2s == min(given, key=lambda k: (given[k][1], k))
        assert k2s == min(given, key=lambda k: (given[k][0], k))
        gaps.append(allc[(k1s, k2s)][0] / min(v[0] for v in allc.values()) - 1.0)
    assert all(g >= -1e-12 for g in gaps)


def _rtn_mse_best(w, s_g, weights):
    """Independent scale search without updates: weighted squared error of
    round-to-nearest at each window code; ties to the lower code."""
    win = window_md(np.max(np.abs(w)), s_g)
    best = None
    for k in win:
        s = e4m3_val_md(k) * s_g
        q = np.array([_e2m1_val(nearest_e2m1_code(x / s)) * s for x in w])
        err = float(np.sum(weights * (w - q) ** 2))
        if best is None or err < best[0]:
            best = (err, k, q)
    return best


def test_identity_hessian_reduces_to_rtn():
    rng = np.random.default_rng(12)
    W = rng.normal(0, 0.02, size=(10, 48))
    res = O.solve_layer(W, H=3.5 * np.eye(48))
    np.testing.assert_allclose(res["U"], np.eye(48) / np.sqrt(3.5 * 1.01), rtol=1e-14)
    s_g = float(res["s_g"])
    for r in range(10):
        for b in range(3):
            w = res["W"][r, 16 * b:16 * b + 16]        # no updates with diagonal U
            err, k, q = _rtn_mse_best(w, s_g, np.ones(16))
            assert res["scales"][r, b] == k
            np.testing.assert_array_equal(res["q"][r, 16 * b:16 * b + 16], q)


def test_diagonal_hessian_weighted_rtn():
    rng = np.random.default_rng(13)
    W = rng.normal(0, 0.02, size=(8, 32))
    h = rng.lognormal(0, 1.5, size=32)
    res = O.solve_layer(W, H=np.diag(h))
    lam = 0.01 * h.mean()
    s_g = float(res["s_g"])
    for r in range(8):
        for b in range(2):
            sl = slice(16 * b, 16 * b + 16)
            err, k, q = _rtn_mse_best(res["W"][r, sl], s_g, h[sl] + lam)
            assert res["scales"][r, b] == k
            assert res["row_err"][r] >= 0
            np.testing.assert_array_equal(res["q"][r, sl], q)


def test_dequant_exact_and_codes_in_set():
    W, X = (t.double().numpy() for t in __import__(
        "nvfp4_post_weight_b200.synth", fromlist=["x"]).small_outlier(64, 64, 128, seed=0))
    res = O.solve_layer(W, X)
    Q = O.dequant(res["codes"], res["scales"], res["s_g"])
    assert Q.dtype == np.float32
    np.testing.assert_array_equal(Q, res["q"].astype(np.float32))
    assert np.all((res["codes"] >= 0) & (res["codes"] < 16) & (res["codes"] != 8))
    assert np.all((res["scales"] >= 0) & (res["scales"] <= 126))
    s = O.E4M3_TABLE[res["scales"]].repeat(16, 1) * float(res["s_g"])
    ratio = np.abs(res["q"]) / np.where(s > 0, s, 1)
    assert np.all(np.isin(ratio, O.E2M1_MAGNITUDE))
    Qb = O.dequant(res["codes"], res["scales"], res["s_g"], "bf16")
    np.testing.assert_array_equal(Qb, O.round_to_bf16(res["q"]))


def test_round_to_bf16_matches_ml_dtypes_on_fp32_values():
    rng = np.random.default_rng(14)
    x = (rng.standard_normal(10000) * 10 ** rng.uniform(-5, 3, 10000)).astype(np.float32)
    np.testing.assert_array_equal(O.round_to_bf16(x.astype(np.float64)),
                                  x.astype(md.bfloat16).astype(np.float32))
    # the ends of the range: bf16 subnormals (below 2^-126) and overflow
    lo = (rng.standard_normal(10000) * 10 ** rng.uniform(-44.5, -36, 10000)).astype(np.float32)
    with np.errstate(over="ignore"):   # some fp32 casts overflow to inf on purpose
        hi = (rng.standard_normal(10000) * 10 ** rng.uniform(37, 38.5, 10000)).astype(np.float32)
    for v in (lo, hi):
        with np.errstate(over="ignore"):
            want = v.astype(md.bfloat16).astype(np.float32)
        np.testing.assert_array_equal(O.round_to_bf16(v.astype(np.float64)), want)


def test_round_to_bf16_is_the_nearest_bf16_value():
    """Brute force over the whole bf16 grid: every finite bf16 value (all
    65536 bit patterns, the subnormals included), the nearest one to x, ties
    to the even bit pattern, overflow past the largest finite value plus half
    its spacing to infinity.  Inputs: exact products with up to 30
    significant bits (the dequant's e2m1 * e4m3 * s_g) across the range."""
    bits = np.arange(1 << 16, dtype=np.uint32)
    with np.errstate(invalid="ignore"):
        vals = (bits << 16).view(np.float32).astype(np.float64)
    fin = np.isfinite(vals) & (bits < 0x8000)           # non-negative finite values
    grid, gbits = vals[fin], bits[fin]
    order = np.argsort(grid, kind="stable")
    grid, gbits = grid[order], gbits[order]
    big = (2.0 - 2.0 ** -7) * 2.0 ** 127
    rng = np.random.default_rng(41)
    mant = rng.integers(1 << 29, 1 << 30, 3000).astype(np.float64)
    ex = rng.integers(-165, 100, 3000)
    xs = np.concatenate([np.ldexp(mant, ex - 29), np.ldexp(mant[:200], rng.integers(127, 130, 200) - 29),
                         grid[:40] + np.ldexp(1.0, -134), [0.0, big, big * (1 + 2.0 ** -9)]])
    got = O.round_to_bf16(xs)
    for x, g in zip(xs, got):
        i = np.searchsorted(grid, x)
        cands = [j for j in (i - 1, i) if 0 <= j < len(grid)]
        dist = [abs(grid[j] - x) for j in cands]
        best = min(dist)
        near = [j for j, dd in zip(cands, dist) if dd == best]
        j = near[0] if len(near) == 1 else min(near, key=lambda k: (int(gbits[k]) & 1, k))
        want = grid[j]
        if x >= big + 2.0 ** 119:   # half the top spacing past the largest value
            want = np.inf
        assert g == np.float32(want), (x, g, want)
        assert O.round_to_bf16(-x) == -g


def test_all_zero_row_and_block():
    rng = np.random.default_rng(15)
    W, X = random_layer(rng, 4, 32, 64, outliers=False)
    W[1, :] = 0.0
    W[2, :16] = 0.0
    X[:, :16] *= 0.0
    X[:, :16] += 1e-3 * rng.standard_normal((64, 16))   # keep columns alive
    res = O.solve_layer(W, X)
    assert np.all(res["codes"][1] == 0) and np.all(res["scales"][1] == 0)
    assert res["scales"][2, 0] == 0 and np.all(res["codes"][2, :16] == 0)


# --------------------------------------------------------------------------
# the independent-block rules Schur Replay is compared with ("Replay the
# Curvature", Abstract, sentence on why scale choice is hard in GPTQ)
# --------------------------------------------------------------------------

def _amax_scale_of_block(s_g):
    """Scale rule for obs_gptq_row: k = e4m3(amax / (6 s_g)) (>= 1) taken on
    the block's values when the sweep reaches its first column."""
    cache = {}

    def scale(b, w):
        if b not in cache:
            a = np.max(np.abs(w[16 * b:16 * b + 16]))
            cache[b] = (max(e4m3_code_md(a / (6.0 * s_g)), 1), e4m3_val_md(
                max(e4m3_code_md(a / (6.0 * s_g)), 1)) * s_g)
        return cache[b][1]
    return scale, cache


def _mse_scale_of_block(s_g):
    """Scale rule for obs_gptq_row: unweighted round-to-nearest squared error
    of the block's values as the sweep reaches it, minimised over the window."""
    cache = {}

    def scale(b, w):
        if b not in cache:
            err, k, _ = _rtn_mse_best(w[16 * b:16 * b + 16], s_g, np.ones(16))
            cache[b] = (k, e4m3_val_md(k) * s_g)
        return cache[b][1]
    return scale, cache


@pytest.mark.parametrize("rule", ["amax", "block_mse"])
def test_independent_rules_match_textbook_gptq(rule):
    """Every row of a 6 x 64 layer: the oracle's scales and values equal a
    textbook GPTQ sweep (explicit inverse, OBS downdates) that picks each
    block's scale by the rule when it reaches the block."""
    rng = np.random.default_rng(16)
    W, X = random_layer(rng, 6, 64, 128)
    res = O.solve_layer(W, X, rule=rule, return_diag=True)
    s_g = float(res["s_g"])
    for r in range(W.shape[0]):
        scale, cache = (_amax_scale_of_block if rule == "amax" else _mse_scale_of_block)(s_g)
        _, _, q, loss = obs_gptq_row(res["W"][r], res["H_d"], scale)
        assert [cache[b][0] for b in range(4)] == list(res["scales"][r])
        np.testing.assert_allclose(q, res["q"][r], rtol=0, atol=1e-15)
        np.testing.assert_allclose(loss.sum(), res["row_err"][r], rtol=1e-9)


@pytest.mark.parametrize("rule", ["amax", "block_mse"])
def test_independent_rules_loss_identity(rule):
    rng = np.random.default_rng(17)
    W, X = random_layer(rng, 7, 80, 96)
    res = O.solve_layer(W, X, rule=rule)
    E = res["W"] - res["q"]
    assert np.einsum("ij,jk,ik->", E, res["H_d"], E) == pytest.approx(res["err_sum"], rel=1e-10)


def test_identity_hessian_block_mse_equals_schur_replay_and_amax_is_rtn():
    """With H = c I nothing is updated and every column has the same Schur
    complement, so the replay score is the unweighted block error: the two
    search rules agree, and the amax rule is plain round-to-nearest at the
    scale that maps the block amax to 6."""
    rng = np.random.default_rng(18)
    W = rng.normal(0, 0.02, size=(12, 64))
    W[:, 5] *= 15
    H = 2.0 * np.eye(64)
    sr = O.solve_layer(W, H=H)
    mse = O.solve_layer(W, H=H, rule="block_mse")
    am = O.solve_layer(W, H=H, rule="amax")
    np.testing.assert_array_equal(sr["scales"], mse["scales"])
    np.testing.assert_array_equal(sr["codes"], mse["codes"])
    s_g = float(am["s_g"])
    for r in range(12):
        for b in range(4):
            w = am["W"][r, 16 * b:16 * b + 16]
            k = max(e4m3_code_md(np.max(np.abs(w)) / (6.0 * s_g)), 1)
            assert am["scales"][r, b] == k
            s = e4m3_val_md(k) * s_g
            q = [_e2m1_val(nearest_e2m1_code(x / s)) * s for x in w]
            np.testing.assert_array_equal(am["q"][r, 16 * b:16 * b + 16], q)


def test_schur_replay_never_worse_on_the_first_block_and_better_overall():
    """Given the same prefix (the first block of every row) Schur Replay's
    block error is the minimum over the window, so neither independent rule
    can beat it there.  Over a whole layer with outlier channels it should
    come out lower too, the improvement the method claims (Abstract); that
    part is a property of this seeded layer, not a theorem (the choice is
    greedy)."""
    rng = np.random.default_rng(19)
    W, X = random_layer(rng, 48, 256, 512)
    sr = O.solve_layer(W, X, return_diag=True)
    first = sr["scores"][:, 0]
    for rule in ("amax", "block_mse"):
        other = O.solve_layer(W, X, rule=rule, return_diag=True)
        k = other["scales"][:, 0] - other["cand"][:, 0, 0]
        np.testing.assert_array_equal(other["cand"][:, 0], sr["cand"][:, 0])
        assert np.all(first.min(axis=1) <= first[np.arange(48), k])
        np.testing.assert_allclose(other["scores"][:, 0], first, rtol=0, atol=0)
        assert sr["err_sum"] < other["err_sum"]
        assert sr["layer_error"] < other["layer_error"]


def test_amax_rule_margin_is_distance_to_e4m3_midpoint():
    t = np.array([1.0, 1.0625, 1.03125, 448.0, 500.0, 0.0])
    m = O.e4m3_rounding_margin(t)
    assert m[0] == pytest.approx(0.03125)            # 0.9375 and 1.0: midpoint 0.96875
    assert m[1] == 0.0                               # 1.0 and 1.125: midpoint 1.0625
    assert m[2] == pytest.approx(0.03125 / 1.03125)
    assert m[3] == pytest.approx(16.0 / 448.0)       # 416 and 448: midpoint 432
    assert m[5] == np.inf


# --------------------------------------------------------------------------
# export layout of the block scales (128 x 4 tiles of 512 bytes)
# --------------------------------------------------------------------------

def _tiled_by_reshape(scales):
    """The same tiling by reshapes: row r = 128 R + 32 b + a, column
    c4 = 4 C + c goes to tile (R, C), byte 16 a + 4 b + c."""
    rows, nb = scales.shape
    rp, cp = -(-rows // 128) * 128, -(-nb // 4) * 4
    p = np.zeros((rp, cp), dtype=np.uint8)
    p[:rows, :nb] = scales
    t = p.reshape(rp // 128, 4, 32, cp // 4, 4)        # (R, b, a, C, c)
    return t.transpose(0, 3, 2, 1, 4).reshape(-1)       # (R, C, a, b, c)


@pytest.mark.parametrize("rows,nb", [(1, 1), (7, 3), (128, 4), (200, 6), (300, 17)])
def test_export_tiling_matches_reshape_route_and_inverts(rows, nb):
    rng = np.random.default_rng(rows * 31 + nb)
    sc = rng.integers(1, 127, size=(rows, nb)).astype(np.uint8)
    t = O.scales_to_tiled(sc)
    np.testing.assert_array_equal(t, _tiled_by_reshape(sc))
    assert t.size == (-(-rows // 128) * 128) * (-(-nb // 4) * 4)
    assert np.count_nonzero(t) == rows * nb                # padding is zero codes
    assert sorted(t[t > 0].tolist()) == sorted(sc.reshape(-1).tolist())


def test_export_tiling_hand_position():
    sc = np.zeros((200, 6), dtype=np.uint8)
    sc[33, 5] = 77                     # tile (0, 1); r % 32 = 1, r // 32 = 1, c % 4 = 1
    t = O.scales_to_tiled(sc)
    assert np.nonzero(t)[0].tolist() == [512 + 16 + 4 + 1]
    sc = np.zeros((200, 6), dtype=np.uint8)
    sc[130, 2] = 9                     # tile (1, 0) of a 2 x 2 grid = third tile
    t = O.scales_to_tiled(sc)
    assert np.nonzero(t)[0].tolist() == [2 * 512 + 2 * 16 + 0 * 4 + 2]
