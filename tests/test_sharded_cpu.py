"""Row-sharded EM orchestration on CPU: two and three gloo ranks, statistics from the oracle.

Each rank computes the fp64 statistics of its contiguous block of rows with the
oracle, the ranks all-gather them (soft_clustering_em_b200.sharded), and every
rank applies the M-step to the rank-ordered sum.  After three iterations all
ranks must hold identical parameters, equal (to fp64 rounding) to the oracle run
on all rows in one process.  This covers the host logic of the multi-GPU path;
on GPUs the same orchestration runs with gmm_estep_stats / gmm_mstep and NCCL.
"""
import multiprocessing as mp
import os
import socket

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _data():
    from soft_clustering_em_b200 import synth

    wl = synth.WORKLOADS["gauss8"]
    X, _ = synth.make_data(wl, 3001)
    return wl, X.astype(np.float64)


def _worker(rank, world, port, q):
    import sys

    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist

    import oracle
    from soft_clustering_em_b200 import sharded, synth

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl, X = _data()
        N, D, K = X.shape[0], X.shape[1], wl.K
        lo, hi = sharded.shard_rows(N, world, rank)
        Xs = X[lo:hi]
        w, mu, var = oracle.init(X, synth.init_rows(N, K, wl.init_seed), K, 0)
        if rank != 0:  # the broadcast must overwrite whatever other ranks hold
            w, mu, var = w * 0, mu * 0, var * 0 + 1
        tw, tmu, tvar = (torch.tensor(a) for a in (w, mu, var))
        sharded.broadcast_params(tw, tmu, tvar)
        state = {"w": tw.numpy(), "mu": tmu.numpy(), "var": tvar.numpy(), "ll": []}

        def estep():
            Nk, A, B, ll = oracle.estep_stats(Xs, state["w"], state["mu"], state["var"])
            return torch.tensor(np.concatenate([Nk, A.ravel(), B.ravel(), [ll]]))

        def mstep(gathered, n_total):
            tot = gathered[0].clone()
            for r in range(1, gathered.shape[0]):
                tot += gathered[r]
            t = tot.numpy()
            Nk, A = t[:K], t[K:K + K * D].reshape(K, D)
            B, ll = t[K + K * D:K + 2 * K * D].reshape(K, D), t[-1]
            state["w"], state["mu"], state["var"] = oracle.mstep(
                n_total, state["mu"], state["var"], Nk, A, B, wl.var_floor)
            state["ll"].append(ll)

        for _ in range(3):
            sharded.sharded_em_step(estep, mstep, N)
        q.put((rank, state["w"], state["mu"], state["var"], state["ll"]))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])  # 3001 rows: shards of 1000/1000/1001 at world 3
def test_sharded_em_matches_single_process(oracle_mod, world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = {}
    for _ in range(world):
        r, w, mu, var, ll = q.get(timeout=240)
        out[r] = (w, mu, var, ll)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # identical on every rank
    for r in range(1, world):
        for a, b in zip(out[0], out[r]):
            np.testing.assert_array_equal(np.asarray(a), np.asarray(b))
    # equal to one process over all rows
    wl, X = _data()
    from soft_clustering_em_b200 import synth

    w, mu, var = oracle_mod.init(X, synth.init_rows(X.shape[0], wl.K, wl.init_seed), wl.K, 0)
    w, mu, var, ll = oracle_mod.fit(X, w, mu, var, 3, wl.var_floor)
    np.testing.assert_allclose(out[0][0], w, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(out[0][1], mu, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(out[0][2], var, rtol=1e-10)
    np.testing.assert_allclose(out[0][3], ll, rtol=1e-12)


def test_shard_rows_cover_exactly():
    from soft_clustering_em_b200 import sharded

    for N in (1, 7, 1000, 10**8 + 3):
        for world in (1, 2, 3, 8):
            spans = [sharded.shard_rows(N, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == N
            assert all(spans[i][1] == spans[i + 1][0] for i in range(world - 1))
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1
