"""The row-sharded layer solve's orchestration on CPU: two gloo ranks on
127.0.0.1, each solving its half of the rows, against one process solving the
whole layer.  The per-rank compute is a test backend built from the oracle
(the CUDA backend needs a GPU; its row-shard entry points are checked against
the whole-layer call in tests/test_gpu_sharded.py).  The tokens are small
integers, so every partial Hessian and their all-reduced sum are exact in fp32
and both sides factor the same H.

Method: "Replay the Curvature", Abstract, infrastructure sentence (independent
output rows distributed across tensor-parallel ranks).
"""
import os
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
D_OUT, D_IN, N_TOK = 37, 64, 96


class OracleBackend:
    """Per-rank compute from the fp64 oracle (test infrastructure)."""

    def hessian(self, X):
        import oracle as O
        return torch.from_numpy(O.hessian(X.double().numpy()).astype(np.float32))

    def prepare(self, H):
        import oracle as O
        self.H = H.double().numpy()
        Hd, self.dead, _ = O.damp(self.H)
        self.U = O.inverse_cholesky_upper(Hd)

    def weight_amax(self, W):
        Wz = W.double().numpy().copy()
        Wz[:, self.dead] = 0.0
        return torch.tensor([np.abs(Wz).max() if Wz.size else 0.0], dtype=torch.float32)

    def quantize_rows(self, W, amax):
        import oracle as O
        W64 = W.double().numpy().copy()
        W64[:, self.dead] = 0.0
        sg = O.global_scale(np.array([[float(amax[0])]]))   # the layer's s_g
        res = O.schur_replay_gptq(W64, self.U, sg, self.dead)
        lerr = O.layer_error(W64, res["q"], self.H)
        return (torch.from_numpy(res["codes"]), torch.from_numpy(res["scales"]),
                torch.tensor([float(sg)]), torch.tensor([res["err_sum"]], dtype=torch.float64),
                torch.tensor([lerr], dtype=torch.float64))


def layer():
    rng = np.random.default_rng(5)
    W = torch.from_numpy(rng.normal(0, 0.02, size=(D_OUT, D_IN)).astype(np.float32))
    W[:, 3] *= 25
    X = torch.from_numpy(rng.integers(-2, 3, size=(N_TOK, D_IN)).astype(np.float32))
    return W, X


def _rank(rank, world, port, q):
    import torch.distributed as tdist
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from nvfp4_post_weight_b200.sharded import ShardedLayerSolver, row_range
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    tdist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        W, X = layer()
        s = ShardedLayerSolver(D_OUT, D_IN, backend=OracleBackend())
        t0, t1 = row_range(N_TOK, rank, world)         # this rank's tokens
        codes, scales, sg, err, lerr = s.step(W[s.r0:s.r1], X[t0:t1], tokens_split=True)
        all_codes, all_scales = s.gather()
        q.put((rank, s.r0, s.r1, all_codes.numpy(), all_scales.numpy(), float(sg[0]),
               float(err), float(lerr)))
        tdist.barrier()
    finally:
        tdist.destroy_process_group()


def test_row_range_partitions_the_rows():
    from nvfp4_post_weight_b200.sharded import row_range
    for d_out in (0, 1, 7, 37, 4096):
        for world in (1, 2, 3, 8):
            rr = [row_range(d_out, r, world) for r in range(world)]
            assert rr[0][0] == 0 and rr[-1][1] == d_out
            assert all(a[1] == b[0] for a, b in zip(rr, rr[1:]))
            sizes = [b - a for a, b in rr]
            assert max(sizes) - min(sizes) <= 1


@pytest.mark.parametrize("world", [2])
def test_two_ranks_equal_one_process(world):
    import oracle as O
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29700 + os.getpid() % 1000
    procs = [ctx.Process(target=_rank, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = sorted(q.get(timeout=300) for _ in range(world))
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    W, X = layer()
    ref = O.solve_layer(W.double().numpy(), X.double().numpy())
    for rank, r0, r1, codes, scales, sg, err, lerr in got:
        assert np.array_equal(codes, ref["codes"]) and np.array_equal(scales, ref["scales"])
        assert np.float32(sg) == ref["s_g"]
        assert err == pytest.approx(ref["err_sum"], rel=1e-12)
        assert lerr == pytest.approx(ref["layer_error"], rel=1e-12)
    # the shards' amax really is the layer's: the first shard alone has a smaller one
    assert np.abs(W[:D_OUT // 2].numpy()).max() <= np.abs(W.numpy()).max()
