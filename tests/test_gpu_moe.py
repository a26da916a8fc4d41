"""GPU parity of the batched calls on the mixture-of-experts workload: 128
experts, gate/up 4096 -> 1536 and down 1536 -> 4096 each, Zipf(1.1) routed
token counts of 64..4096 (65536 in total).

All 128 experts are solved in ONE batched call per phase: 256 Hessians (every
expert's input and intermediate activations), their 256 factors, the 384
quantizations (gate and up share the input factor) and the 384
dequantizations.  Checked:

* every problem's device status word;
* every result equals the single-problem call on the same inputs bit for bit
  (the Hessians, the factors, codes, scales, global scales and sums of
  delta^2 of all 384 weight matrices);
* every expert's two Hessians against the oracle's fp64 ones (1e-4 relative
  Frobenius);
* a spread of experts over the token range (every 8th and the last) against
  the oracle's whole solve from the same tokens, 64 sampled rows of each of
  gate, up and down, under
  the near-tie rule of parity.py, plus the rows' layer error within 1e-4:
  end to end (the library's Hessian and factor) where the Hessian has full
  rank (at least as many tokens as channels); where it has not, the solve is
  checked given the oracle's Hessian rounded to fp32 -- with fewer tokens
  than channels the damped Hessian's condition number reaches 1e4-1e5 and the
  fp32 storage of H alone (relative rounding 6e-8) moves the factor by up to
  ~1e-5, which can flip decisions that sit further than the 1e-5 near-tie
  bound from a tie.

Method: "Replay the Curvature", Abstract (a mixture-of-experts layer is
quantized expert by expert; each expert is a linear layer with its own
second-order state).
"""
import numpy as np
import pytest
import torch

import oracle as O
from nvfp4_post_weight_b200 import binding as B
from nvfp4_post_weight_b200 import synth
from parity import classify, report, unpack_codes

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
N_EXPERTS = 128
# every 8th expert and the last (4096 ... 97 tokens): 17 experts, their gate,
# up and down projections each on 64 seeded rows
ORACLE_EXPERTS = tuple(range(0, 128, 8)) + (127,)
ROWS = 64


def rel_frob(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


@pytest.fixture(scope="module")
def moe():
    counts, ex = synth.moe_all_experts(N_EXPERTS)
    assert counts.sum() == 65536 and counts.max() == 4096 and counts.min() >= 64
    # problems: per expert gate, up (sharing H_in) and down (H_mid)
    Xs, mats = [], []
    for e in range(N_EXPERTS):
        Xs += [ex[e]["X_in"], ex[e]["X_mid"]]
        mats += [(e, "gate", 2 * e), (e, "up", 2 * e), (e, "down", 2 * e + 1)]
    Xd = [x.to(DEV) for x in Xs]
    Hs = [torch.empty((x.shape[1], x.shape[1]), dtype=torch.float32, device=DEV) for x in Xs]
    launches = {}
    n0 = B.lib().nvfp4_launch_count()
    B.nvfp4_hessian_accumulate_batched(Hs, Xd)
    launches["hessian"] = B.lib().nvfp4_launch_count() - n0
    Us = [torch.empty_like(h) for h in Hs]
    wsp = B.workspace(B.nvfp4_prepare_batched_workspace_size([h.shape[0] for h in Hs]), DEV)
    n0 = B.lib().nvfp4_launch_count()
    B.nvfp4_gptq_prepare_batched(Hs, 0.01, Us, ws=wsp)
    launches["prepare"] = B.lib().nvfp4_launch_count() - n0
    status = [B.nvfp4_batched_workspace_status(wsp, len(Hs))]
    del wsp   # (each call's workspace is freed before the next one is made)
    Ws = [ex[e][name].to(DEV) for e, name, _ in mats]
    Uq = [Us[hi] for _, _, hi in mats]
    codes = [torch.empty((w.shape[0], w.shape[1] // 2), dtype=torch.uint8, device=DEV) for w in Ws]
    scales = [torch.empty((w.shape[0], w.shape[1] // 16), dtype=torch.uint8, device=DEV)
              for w in Ws]
    sgs = [torch.empty(1, dtype=torch.float32, device=DEV) for _ in Ws]
    errs = [torch.empty(1, dtype=torch.float64, device=DEV) for _ in Ws]
    wsq = B.workspace(B.nvfp4_quantize_batched_workspace_size([tuple(w.shape) for w in Ws]),
                      DEV)
    n0 = B.lib().nvfp4_launch_count()
    B.nvfp4_gptq_schur_replay_quantize_batched(Ws, Uq, codes, scales, sgs, errs, ws=wsq)
    launches["quantize"] = B.lib().nvfp4_launch_count() - n0
    status.append(B.nvfp4_batched_workspace_status(wsq, len(Ws)))
    del wsq
    Q = [torch.empty(w.shape, dtype=torch.float32, device=DEV) for w in Ws]
    n0 = B.lib().nvfp4_launch_count()
    B.nvfp4_dequant_batched(codes, scales, sgs, Q)
    launches["dequant"] = B.lib().nvfp4_launch_count() - n0
    Hq = [Hs[hi] for _, _, hi in mats]
    Ls = [torch.empty(1, dtype=torch.float64, device=DEV) for _ in Ws]
    wse = B.workspace(B.nvfp4_layer_error_batched_workspace_size([tuple(w.shape) for w in Ws]),
                      DEV)
    n0 = B.lib().nvfp4_launch_count()
    B.nvfp4_layer_error_batched(Ws, codes, scales, sgs, Hq, Ls, wse)
    launches["layer_error"] = B.lib().nvfp4_launch_count() - n0
    torch.cuda.synchronize()
    status.append(B.nvfp4_batched_workspace_status(wse, len(Ws)))
    del wse
    return dict(counts=counts, ex=ex, Xs=Xs, Xd=Xd, Hs=Hs, Us=Us, mats=mats, Ws=Ws, Uq=Uq,
                codes=codes, scales=scales, sgs=sgs, errs=errs, Q=Q, Hq=Hq, Ls=Ls,
                status=status, hstatus=B.nvfp4_hessian_status(), launches=launches)


def test_every_problem_status_ok(moe):
    assert moe["hstatus"] == 0
    for first, each in moe["status"]:
        assert first == 0 and all(s == 0 for s in each), [i for i, s in enumerate(each) if s]


def test_launches_grow_with_shapes_not_problems(moe):
    """Every launch of a batched call covers all problems of one shape: the
    128 experts take about as many launches as two single problems (one per
    shape), not 128 times as many."""
    L = moe["launches"]
    print(f"MOE launches per batched call: {L}")
    assert L["hessian"] == 2            # one per dimension (4096, 1536)
    assert L["dequant"] == 2            # one per shape
    # single calls, one problem of each shape, for comparison
    single = 0
    for hi in (0, 1):
        H = moe["Hs"][hi]
        d = H.shape[0]
        ws = B.workspace(B.nvfp4_prepare_workspace_size(d), DEV)
        n0 = B.lib().nvfp4_launch_count()
        B.nvfp4_gptq_prepare(H, 0.01, torch.empty_like(H), None, None, ws)
        single += B.lib().nvfp4_launch_count() - n0
    torch.cuda.synchronize()
    assert L["prepare"] <= single + 4, (L["prepare"], single)
    single = 0
    for i in (0, 2):
        W, U = moe["Ws"][i], moe["Uq"][i]
        d_out, d_in = W.shape
        ws = B.workspace(B.nvfp4_quantize_workspace_size(d_out, d_in), DEV)
        n0 = B.lib().nvfp4_launch_count()
        B.nvfp4_gptq_schur_replay_quantize(W, U, torch.empty_like(moe["codes"][i]),
                                           torch.empty_like(moe["scales"][i]),
                                           torch.empty(1, device=DEV), None, None, ws)
        single += B.lib().nvfp4_launch_count() - n0
    torch.cuda.synchronize()
    assert L["quantize"] <= single + 4, (L["quantize"], single)


def test_batched_equals_single_calls_every_problem(moe):
    for X, H in zip(moe["Xd"], moe["Hs"]):
        Hs = torch.empty_like(H)
        B.nvfp4_hessian_accumulate(Hs, X)
        torch.cuda.synchronize()
        assert torch.equal(Hs, H)
    for H, U in zip(moe["Hs"], moe["Us"]):
        d = H.shape[0]
        Us = torch.empty_like(U)
        ws = B.workspace(B.nvfp4_prepare_workspace_size(d), DEV)
        B.nvfp4_gptq_prepare(H, 0.01, Us, None, None, ws)
        torch.cuda.synchronize()
        assert torch.equal(Us, U)
    for i, (W, U) in enumerate(zip(moe["Ws"], moe["Uq"])):
        d_out, d_in = W.shape
        c = torch.empty_like(moe["codes"][i])
        s = torch.empty_like(moe["scales"][i])
        g = torch.empty(1, dtype=torch.float32, device=DEV)
        err = torch.empty(1, dtype=torch.float64, device=DEV)
        ws = B.workspace(B.nvfp4_quantize_workspace_size(d_out, d_in), DEV)
        B.nvfp4_gptq_schur_replay_quantize(W, U, c, s, g, err, None, ws)
        torch.cuda.synchronize()
        assert torch.equal(c, moe["codes"][i]) and torch.equal(s, moe["scales"][i]), i
        assert g.item() == moe["sgs"][i].item() and err.item() == moe["errs"][i].item(), i


def test_batched_layer_error_equals_single_calls(moe):
    assert moe["launches"]["layer_error"] <= 2 * 6   # a few launches per shape
    for i, W in enumerate(moe["Ws"]):
        d_out, d_in = W.shape
        L = torch.empty(1, dtype=torch.float64, device=DEV)
        ws = B.workspace(B.nvfp4_layer_error_workspace_size(d_out, d_in), DEV)
        B.nvfp4_layer_error(W, moe["codes"][i], moe["scales"][i], moe["sgs"][i], moe["Hq"][i],
                            L, ws)
        torch.cuda.synchronize()
        assert L.item() == moe["Ls"][i].item(), i


@pytest.mark.parametrize("e", (0, 64, 127))
def test_batched_layer_error_against_the_oracle(moe, e):
    """The library's tr((W - Q) H (W - Q)^T) of expert e's three tensors
    against the same quantity evaluated in fp64 on the host from the GPU's
    codes and the oracle's fp64 Hessian."""
    for i, (ee, name, hi) in enumerate(moe["mats"]):
        if ee != e:
            continue
        W64 = moe["ex"][e][name].double().numpy()
        H = O.hessian(moe["Xs"][hi].double().numpy())
        Q = moe["Q"][i].cpu().numpy().astype(np.float64)
        L = O.layer_error(W64, Q, H)
        assert abs(moe["Ls"][i].item() - L) <= 1e-4 * L, (e, name)


def test_every_expert_hessian(moe):
    for X, H in zip(moe["Xs"], moe["Hs"]):
        assert rel_frob(H.cpu().numpy().astype(np.float64), O.hessian(X.double().numpy())) < 1e-4


def check_rows(label, W64, rows, U, sg, codes, scales, H, Q_gpu):
    ref = O.schur_replay_gptq(W64[rows], U, sg, return_diag=True)
    c = classify(ref, U, sg, codes[rows], scales[rows], rows)
    report(f"moe_128_experts {label}: {len(rows)} rows", c)
    assert c["frac"] <= 1e-3, (label, c)
    assert not c["bad_first"], (label, c)
    Q = O.dequant(codes[rows], scales[rows], sg)
    assert np.array_equal(Q_gpu[rows].view(np.uint32), Q.view(np.uint32))
    L_gpu = O.layer_error(W64[rows], Q.astype(np.float64), H)
    L_ref = O.layer_error(W64[rows], ref["q"], H)
    assert abs(L_gpu - L_ref) <= 1e-4 * L_ref, label


def _given_hessian_solve(ex, names, H32):
    """The library's factor of the oracle's fp32 H and the quantize and
    dequant of the named weights with it."""
    d = H32.shape[0]
    Ug = torch.empty((d, d), dtype=torch.float32, device=DEV)
    ws = B.workspace(B.nvfp4_prepare_workspace_size(d), DEV)
    B.nvfp4_gptq_prepare(torch.from_numpy(H32).to(DEV), 0.01, Ug, None, None, ws)
    out = {}
    for name in names:
        W = ex[name].to(DEV)
        d_out = W.shape[0]
        c = torch.empty((d_out, d // 2), dtype=torch.uint8, device=DEV)
        s = torch.empty((d_out, d // 16), dtype=torch.uint8, device=DEV)
        g = torch.empty(1, dtype=torch.float32, device=DEV)
        wq = B.workspace(B.nvfp4_quantize_workspace_size(d_out, d), DEV)
        B.nvfp4_gptq_schur_replay_quantize(W, Ug, c, s, g, None, None, wq)
        Qg = torch.empty((d_out, d), dtype=torch.float32, device=DEV)
        B.nvfp4_dequant(c, s, g, Qg)
        torch.cuda.synchronize()
        assert B.nvfp4_workspace_status(wq) == 0
        out[name] = (c, s, g, Qg)
    assert B.nvfp4_workspace_status(ws) == 0
    return out


@pytest.mark.parametrize("e", ORACLE_EXPERTS)
def test_expert_against_oracle(moe, e):
    """Expert e's gate, up and down: end to end where its Hessian has full
    rank, else given the oracle's fp32-rounded Hessian."""
    n = int(moe["counts"][e])
    ex = moe["ex"][e]
    rng = np.random.default_rng(1000 + e)
    for x_name, names in (("X_in", ("gate", "up")), ("X_mid", ("down",))):
        H = O.hessian(ex[x_name].double().numpy())
        d = H.shape[0]
        full_rank = n >= d
        e2e = {name: (moe["codes"][i], moe["scales"][i], moe["sgs"][i], moe["Q"][i])
               for i, (ee, name, _) in enumerate(moe["mats"]) if ee == e and name in names}
        if full_rank:
            Href = H
            res = e2e
        else:
            # reported, not asserted: the batched end-to-end result against
            # the oracle's fp64 solve (the Hessian's fp32 rounding included)
            Hd, _, _ = O.damp(H)
            Uo = O.inverse_cholesky_upper(Hd)
            del Hd
            for name in names:
                c, s_, g, _ = e2e[name]
                W64 = ex[name].double().numpy()
                sg = O.global_scale(W64)
                rows = np.sort(np.random.default_rng(2000 + e).choice(W64.shape[0], ROWS,
                                                                       replace=False))
                ref = O.schur_replay_gptq(W64[rows], Uo, sg, return_diag=True)
                cc = classify(ref, Uo, sg, unpack_codes(c.cpu().numpy())[rows],
                              s_.cpu().numpy().astype(np.int64)[rows], rows)
                report(f"moe_128_experts expert {e} ({n} tokens) {name} end to end "
                       f"(rank {n} < {d}, reported only)", cc)
            H32 = H.astype(np.float32)
            Href = H32.astype(np.float64)
            res = _given_hessian_solve(ex, names, H32)
        Hd, _, _ = O.damp(Href)
        Uo = O.inverse_cholesky_upper(Hd)
        del Hd
        for name in names:
            c, s, g, Qg = res[name]
            W64 = ex[name].double().numpy()
            sg = O.global_scale(W64)
            assert np.float32(g.item()) == sg
            rows = np.sort(rng.choice(W64.shape[0], ROWS, replace=False))
            how = "end to end" if full_rank else "given H"
            check_rows(f"expert {e} ({n} tokens) {name} {how}", W64, rows, Uo, sg,
                       unpack_codes(c.cpu().numpy()), s.cpu().numpy().astype(np.int64), Href,
                       Qg.cpu().numpy())
