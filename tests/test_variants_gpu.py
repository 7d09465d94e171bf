"""Hard EM, spherical EM and k-means through the C ABI against the pinned numpy
oracle of oracle/variants.py (teacher-forced: both sides start from the same
stored parameters).

Spherical EM has soft responsibilities and is compared under the step
tolerances of oracle/compare.py.  Hard EM and k-means decide an integer per
point (its component) on the tensor-core log-joints, whose error is far below
1e-3 nats but not zero; where the oracle's two best components are that close,
either is correct.  So the labels must equal the oracle's wherever the gap is
wider, every label must be a valid choice (within the gap of the best), and
the M-step is compared with the oracle's M-step from the GPU's own labels.
"""
import numpy as np
import pytest

from oracle import compare
from oracle import variants as V
from soft_clustering_em_b200 import synth

pytestmark = pytest.mark.gpu

GAP = 1e-3  # nats of log-joint within which either of two components is a valid choice


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


def _data(name, N, K, seed=3):
    import torch

    wl = synth.WORKLOADS[name]
    X, _ = synth.make_data(wl, N)
    X64 = synth.x_as_f64(wl, X)
    Xd = (torch.from_numpy(X.view(np.int16)).view(torch.bfloat16) if wl.dtype == "bf16"
          else torch.from_numpy(X)).cuda()
    rows = np.random.default_rng(seed).choice(N, K, replace=False)
    return wl, X64, Xd, rows


def _np(*ts):
    return tuple(t.double().cpu().numpy() for t in ts)


def _check_labels(L, got):
    """L: oracle log-joints (or -distances), N x K; got: GPU labels."""
    order = np.argsort(-L, axis=1, kind="stable")
    best, second = L[np.arange(len(L)), order[:, 0]], L[np.arange(len(L)), order[:, 1]]
    wide = best - second >= GAP
    assert np.array_equal(got[wide], order[wide, 0]), int((got[wide] != order[wide, 0]).sum())
    assert np.all(best - L[np.arange(len(L)), got] < GAP)  # every label a valid choice
    return int((~wide).sum())


@pytest.mark.parametrize("name,N,K", [("gauss8", 5_003, 8), ("uint8img", 3_001, 64),
                                      ("bf16stream", 4_001, 128)])
def test_spherical_step_matches_oracle(G, name, N, K):
    import torch

    wl, X64, Xd, rows = _data(name, N, K)
    w = torch.full((K,), 1.0 / K, device="cuda")
    mu = Xd[torch.as_tensor(rows, device="cuda")].float().contiguous()
    s2 = torch.full((K,), float(X64.var(0).mean()), device="cuda")
    ws = G.workspace(G.problem_for(Xd, K))
    for t in range(3):
        th = _np(w, mu, s2)
        ll = torch.zeros(1, dtype=torch.float64, device="cuda")
        G.gmm_em_step_spherical(Xd, w, mu, s2, ll, ws=ws)
        rc, flags = G.gmm_device_status(ws)
        assert rc == 0, flags
        w2, mu2, s22, ll_ref, Nk = V.spherical_em_step(X64, *th)
        D = X64.shape[1]
        got = _np(w, mu, s2)
        rep = compare.compare_step((w2, mu2, np.repeat(s22[:, None], D, 1), ll_ref),
                                   (got[0], got[1], np.repeat(got[2][:, None], D, 1), ll.item()),
                                   Nk)
        assert rep["ok"], (t, rep)


@pytest.mark.parametrize("name,N,K", [("gauss8", 5_003, 8), ("uint8img", 3_001, 64),
                                      ("bf16stream", 4_001, 128)])
def test_hard_em_step_matches_oracle(G, name, N, K):
    import torch

    wl, X64, Xd, rows = _data(name, N, K)
    w = torch.full((K,), 1.0 / K, device="cuda")
    mu = Xd[torch.as_tensor(rows, device="cuda")].float().contiguous()
    var = torch.tensor(np.tile(np.maximum(X64.var(0), 1e-6), (K, 1)), dtype=torch.float32,
                       device="cuda")
    ws = G.workspace(G.problem_for(Xd, K))
    labels = torch.empty(N, dtype=torch.int32, device="cuda")
    for t in range(3):
        th = _np(w, mu, var)
        ll = torch.zeros(1, dtype=torch.float64, device="cuda")
        G.gmm_em_step_hard(Xd, w, mu, var, labels, ll, ws=ws)
        rc, flags = G.gmm_device_status(ws)
        assert rc == 0, flags
        z = labels.cpu().numpy().astype(np.int64)
        L = V.diag_logjoint(X64, *th)
        _check_labels(L, z)
        # the oracle's M-step from the GPU's own labels
        R = np.zeros_like(L)
        R[np.arange(N), z] = 1.0
        Nk, A, B = V._moments(X64, th[1], R)
        w2, mu2, var2 = Nk / N, th[1].copy(), th[2].copy()
        for k in range(K):
            if Nk[k] > 0:
                d = A[k] / Nk[k]
                mu2[k] = th[1][k] + d
                var2[k] = np.maximum(B[k] / Nk[k] - d * d, 1e-6)
        ll_ref = float(L[np.arange(N), z].sum())
        rep = compare.compare_step((w2, mu2, var2, ll_ref), (*_np(w, mu, var), ll.item()), Nk)
        assert rep["ok"], (t, rep)


@pytest.mark.parametrize("name,N,K", [("gauss8", 5_003, 8), ("uint8img", 3_001, 64),
                                      ("bf16stream", 4_001, 128)])
def test_kmeans_step_matches_oracle(G, name, N, K):
    import torch

    wl, X64, Xd, rows = _data(name, N, K)
    C = Xd[torch.as_tensor(rows, device="cuda")].float().contiguous()
    ws = G.workspace(G.problem_for(Xd, K))
    labels = torch.empty(N, dtype=torch.int32, device="cuda")
    scale = float(np.sqrt(X64.var(0).mean()))
    for t in range(3):
        C0 = C.double().cpu().numpy()
        inertia = torch.zeros(1, dtype=torch.float64, device="cuda")
        G.gmm_kmeans_step(Xd, C, labels, inertia, ws=ws)
        rc, flags = G.gmm_device_status(ws)
        assert rc == 0, flags
        z = labels.cpu().numpy().astype(np.int64)
        d2 = ((X64[:, None, :] - C0[None, :, :]) ** 2).sum(axis=2)
        # the GPU decides on log-joints -d2 / (2 v) with v the centres' spread
        v = float(((C0 - C0.mean(0)) ** 2).mean()) or 1.0
        _check_labels(-d2 / (2.0 * v), z)
        # centres: the mean of each centre's points under the GPU's labels
        ref = C0.copy()
        for k in range(K):
            if np.any(z == k):
                ref[k] = X64[z == k].mean(axis=0)
        got = C.double().cpu().numpy()
        assert np.all(np.abs(got - ref) <= 1e-4 * scale + 1e-6 * np.abs(ref)), \
            float(np.abs(got - ref).max() / scale)
        inertia_ref = float(d2[np.arange(N), z].sum())
        assert abs(inertia.item() - inertia_ref) <= 1e-4 * inertia_ref
        # and the oracle's own step agrees wherever no point was a near tie
        C2, z2, in2 = V.kmeans_step(X64, C0)
        assert abs(in2 - inertia_ref) <= 1e-4 * in2
