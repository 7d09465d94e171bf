"""IVF inverted lists on the GPU (gmm_ivf_build through the C ABI) against the oracle.

The build is integer work decided by a float32 comparison that both sides make
on the same float32 values, so on the same seeded top-m inputs the offsets and
the ids must be bit-identical to oracle/ivf.py.  The end-to-end case runs the
GPU's own top-m assignment first; there the GPU and oracle responsibilities
differ by rounding, so a point's lists may differ only where the oracle's
ranking or threshold decision is within the top-m tolerances.
"""
import numpy as np
import pytest

import oracle
from oracle import compare
from oracle import ivf
from soft_clustering_em_b200 import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def G():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from soft_clustering_em_b200 import build
    from soft_clustering_em_b200 import gmm

    build.build()
    gmm.load_library()
    return gmm


def _gpu_lists(G, idx, resp, K, tau):
    import torch

    N = idx.shape[0]
    ws = torch.zeros(G.gmm_ivf_workspace_size(N, K), dtype=torch.uint8, device="cuda")
    offsets, ids = G.gmm_ivf_build(torch.from_numpy(idx).cuda(), torch.from_numpy(resp).cuda(),
                                   K, tau, ws=ws)
    rc, flags = G.gmm_device_status(ws)
    off = offsets.cpu().numpy()
    return off, ids[:int(off[-1])].cpu().numpy(), rc, flags


@pytest.mark.parametrize("N,K,m,tau", [
    (1, 1, 1, 0.5),
    (37, 5, 3, 0.1),           # one ragged group of 32
    (100_003, 1024, 2, 0.1),   # K of the bf16 stream and sphere workloads, ragged chunks
    (300_000, 1024, 2, 0.0),   # every entry kept
    (300_000, 1024, 2, 1.5),   # a plain partition
    (1_000_000, 4096, 2, 0.05),
    (2_000_003, 65536, 8, 0.02),  # the largest K: the count matrix caps the chunks at 128
    (10_000_000, 4096, 2, 0.1),
])
def test_lists_are_bit_identical_to_oracle(G, N, K, m, tau):
    idx, resp = synth.topm_inputs(N, K, m, seed=N % 9973 + K, ties_at=tau)
    off, ids, rc, flags = _gpu_lists(G, idx, resp, K, tau)
    ref_off, ref_ids = ivf.ivf_lists(idx, resp, K, tau)
    assert rc == 0 and flags == 0
    np.testing.assert_array_equal(off, ref_off)
    np.testing.assert_array_equal(ids, ref_ids)


def test_invalid_entries_are_skipped_and_flagged(G):
    N, K, m = 100, 6, 3
    idx, resp = synth.topm_inputs(N, K, m, seed=5)
    idx = idx.copy()
    idx[3, 1] = K          # out of range
    idx[10, 2] = idx[10, 0]  # repeats the point's rank-1 index
    idx[50, 0] = -1        # negative, at rank 1
    valid = np.ones_like(idx, dtype=bool)
    valid[3, 1] = valid[10, 2] = valid[50, 0] = False
    off, ids, rc, flags = _gpu_lists(G, idx, resp, K, 0.0)  # tau 0: every valid entry kept
    assert rc == G.GMM_ERR_INVALID_ARG and flags == G.GMM_DEVFLAG_BAD_INDEX
    expect = [[n for n in range(N) if any(valid[n, j] and idx[n, j] == k for j in range(m))]
              for k in range(K)]
    assert [ids[off[k]:off[k + 1]].tolist() for k in range(K)] == expect


def _pairs(off, ids):
    lists = np.repeat(np.arange(len(off) - 1), np.diff(off))
    return set(zip(ids.tolist(), lists.tolist()))


def test_end_to_end_from_the_gpu_assignment(G):
    from test_parity_gpu import params_np, run_teacher_forced

    wl = synth.WORKLOADS["bf16stream"]
    N, K, m, tau = 30_001, 1024, 2, 0.05
    Xd, X64, (w, mu, var), _ = run_teacher_forced(G, wl, N, K, 2)
    th = params_np(w, mu, var)
    idx, resp = G.gmm_assign_topm(Xd, w, mu, var, m)
    off, ids, rc, flags = _gpu_lists(G, idx.cpu().numpy(), resp.cpu().numpy(), K, tau)
    assert rc == 0 and flags == 0
    for k in range(K):  # each list ascending, no point twice
        assert np.all(np.diff(ids[off[k]:off[k + 1]]) > 0)
    ridx, rresp = oracle.assign_topm(X64, *th, m + 1)
    ref_off, ref_ids = ivf.ivf_lists(ridx[:, :m], rresp[:, :m].astype(np.float32), K, tau)
    differ = sorted({n for n, _ in _pairs(off, ids) ^ _pairs(ref_off, ref_ids)})
    gaps = np.abs(np.diff(rresp, axis=1))  # rank j vs j+1, j = 0..m-1
    for n in differ:
        near_rank = bool(np.any(gaps[n, :m] < compare.TOPM_GAP))
        near_tau = bool(np.any(np.abs(rresp[n, 1:m] - tau) <= compare.REL * tau))
        assert near_rank or near_tau, (n, ridx[n], rresp[n])
    assert len(differ) <= N // 1000
