"""Plant plausible mistakes in the oracle (on the CPU only) and check that the
pins catch each one: a dropped in-block update, a wrong sign in the update, a
transposed factor, the wrong tie rule, the argmin taken on the wrong
quantity, and in the independent-block rules an L1 or truncating block error
or a centre code rounded up.  A pin set that let one of these through would not pin the oracle."""
import numpy as np
import pytest

import oracle as O
from oracle import nvfp4_oracle as M
import test_oracle_pins as P  # noqa: E402


def _replay_drop_update(v, Ublk, s):
    v = np.array(v, dtype=np.float64, copy=True)
    v, s = np.broadcast_arrays(v, np.asarray(s, dtype=np.float64)[..., None])
    v = v.copy()
    s = s[..., 0]
    codes = np.zeros(v.shape, np.int64)
    q = np.zeros(v.shape)
    delta = np.zeros(v.shape)
    for j in range(16):
        codes[..., j] = M.e2m1_round(v[..., j] / s)
        q[..., j] = M.e2m1_value(codes[..., j]) * s
        delta[..., j] = (v[..., j] - q[..., j]) / Ublk[j, j]
    return codes, q, delta, np.sum(delta * delta, -1)


def _replay_wrong_sign(v, Ublk, s):
    return M.__dict__["_orig_replay"](v, -Ublk + 2 * np.diag(np.diag(Ublk)), s)


def _replay_unweighted_score(v, Ublk, s):
    codes, q, delta, _ = M.__dict__["_orig_replay"](v, Ublk, s)
    vq = delta * np.diag(Ublk)                    # (v_j - q_j), not divided by U_jj
    return codes, q, delta, np.sum(vq * vq, -1)


def _inv_chol_transposed(H_d):
    return M.__dict__["_orig_invchol"](H_d).T.copy()


def _e2m1_ties_away(x):
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    mids = (M.E2M1_MAGNITUDE[:-1] + M.E2M1_MAGNITUDE[1:]) / 2
    idx = np.zeros(a.shape, np.int64)
    for m in mids:
        idx += (a >= m)
    return idx | (((x < 0) & (idx > 0)).astype(np.int64) << 3)


def _block_error_l1(v, s):
    v = np.asarray(v, dtype=np.float64)
    s = np.asarray(s, dtype=np.float64)[..., None]
    return np.sum(np.abs(v - M.e2m1_value(M.e2m1_round(v / s)) * s), axis=-1)


def _block_error_truncating(v, s):
    v = np.asarray(v, dtype=np.float64)
    s = np.asarray(s, dtype=np.float64)[..., None]
    x = v / s
    idx = np.searchsorted(M.E2M1_MAGNITUDE, np.minimum(np.abs(x), 6.0), side="right") - 1
    q = np.sign(x) * M.E2M1_MAGNITUDE[idx] * s
    return np.sum((v - q) ** 2, axis=-1)


def _center_code_ceil(amax_block, s_g):
    t = np.asarray(amax_block, dtype=np.float64) / (6.0 * float(s_g))
    return np.maximum(np.searchsorted(M.E4M3_TABLE, np.minimum(t, 448.0), side="left"), 1)


PINS = [
    P.test_replay_score_equals_textbook_gptq_block_loss,
    P.test_bruteforce_single_block_all_e4m3_codes,
    P.test_bruteforce_two_blocks_greedy,
    lambda: P.test_gptq_loss_identity(6, 5, 64),
    P.test_e2m1_round_matches_ml_dtypes_including_ties,
    P.test_e2m1_tie_table,
    P.test_inverse_cholesky_factor_identity_and_reversed_route,
    lambda: P.test_independent_rules_match_textbook_gptq("amax"),
    lambda: P.test_independent_rules_match_textbook_gptq("block_mse"),
]


def _caught(monkeypatch_ctx):
    for pin in PINS:
        try:
            pin()
        except (AssertionError, np.linalg.LinAlgError):
            return True
    return False


@pytest.mark.parametrize("mutation", ["drop_update", "wrong_sign", "transposed_U", "ties_away",
                                      "unweighted_score", "block_error_l1",
                                      "block_error_truncating", "center_code_ceil"])
def test_planted_mistake_is_caught(monkeypatch, mutation):
    monkeypatch.setitem(M.__dict__, "_orig_replay", M.replay_block)
    monkeypatch.setitem(M.__dict__, "_orig_invchol", M.inverse_cholesky_upper)
    if mutation == "drop_update":
        monkeypatch.setattr(M, "replay_block", _replay_drop_update)
    elif mutation == "wrong_sign":
        monkeypatch.setattr(M, "replay_block", _replay_wrong_sign)
    elif mutation == "transposed_U":
        monkeypatch.setattr(M, "inverse_cholesky_upper", _inv_chol_transposed)
    elif mutation == "unweighted_score":
        monkeypatch.setattr(M, "replay_block", _replay_unweighted_score)
    elif mutation == "ties_away":
        monkeypatch.setattr(M, "e2m1_round", _e2m1_ties_away)
    elif mutation == "block_error_l1":
        monkeypatch.setattr(M, "independent_block_error", _block_error_l1)
    elif mutation == "block_error_truncating":
        monkeypatch.setattr(M, "independent_block_error", _block_error_truncating)
    elif mutation == "center_code_ceil":
        monkeypatch.setattr(M, "block_center_code", _center_code_ceil)
    monkeypatch.setattr(O, "replay_block", M.replay_block, raising=False)
    monkeypatch.setattr(O, "inverse_cholesky_upper", M.inverse_cholesky_upper, raising=False)
    monkeypatch.setattr(O, "e2m1_round", M.e2m1_round, raising=False)
    assert _caught(monkeypatch), f"no pin caught the planted mistake {mutation}"
