"""Parity of the CUDA path (through the C ABI) against the fp64 CPU oracle.

Every EM step is teacher-forced: the oracle starts from exactly the fp32
parameters the GPU started from, and the two results are compared under the
rules in oracle/compare.py.  Inputs are the seeded synthetic workloads of
soft_clustering_em_b200.synth, down-scaled in N so the oracle finishes in
seconds, with ragged N (not a multiple of any tile) and the degenerate cases.
"""
import numpy as np
import pytest

import oracle
from oracle import compare
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


def to_device(wl, X):
    import torch

    if wl.dtype == "bf16":
        return torch.from_numpy(X.view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(X).cuda()


def params_np(w, mu, var):
    return (w.double().cpu().numpy(), mu.double().cpu().numpy(), var.double().cpu().numpy())


def run_teacher_forced(G, wl, N, K, iters, rows=None):
    import torch

    X, _ = synth.make_data(wl, N)
    X64 = synth.x_as_f64(wl, X)
    Xd = to_device(wl, X)
    rows = synth.init_rows(N, K, wl.init_seed) if rows is None else rows
    mode = G.GMM_INIT_VAR_ONE if wl.var_init == "one" else G.GMM_INIT_VAR_DATA
    p = G.problem_for(Xd, K, wl.var_floor)
    ws = G.workspace(p)
    w, mu, var = G.gmm_init_rows(Xd, rows, K, mode, wl.var_floor, ws=ws)
    # init parity: gathered means exact, data variance to fp32 rounding
    rw, rmu, rvar = oracle.init(X64, rows, K, mode, wl.var_floor)
    gw, gmu, gvar = params_np(w, mu, var)
    np.testing.assert_array_equal(gmu, rmu)
    np.testing.assert_allclose(gw, rw, rtol=1e-7)
    np.testing.assert_allclose(gvar, rvar, rtol=1e-6)
    ll = torch.zeros(1, dtype=torch.float64, device="cuda")
    reports = []
    for t in range(iters):
        th = params_np(w, mu, var)
        G.gmm_em_step(Xd, w, mu, var, ll, wl.var_floor, ws=ws)
        torch.cuda.synchronize()
        rc, flags = G.gmm_device_status(ws)
        assert rc == 0 and flags == 0
        w2, mu2, var2, ll_ref, Nk = oracle.em_step(X64, *th, var_floor=wl.var_floor)
        got = (*params_np(w, mu, var), float(ll.item()))
        rep = compare.compare_step((w2, mu2, var2, ll_ref), got, Nk)
        reports.append(rep)
        assert rep["ok"], (t, rep)
    return Xd, X64, (w, mu, var), reports


CASES = [
    ("gauss8", 10_000, 8, 10),
    ("gauss8", 10_007, 8, 3),
    ("uint8img", 20_011, 256, 3),
    ("sphere768", 3_001, 1024, 2),
    ("sphere768", 50_000, 1024, 1),  # D = 768 streamed: 5 statistics groups, two row chunks
    ("gauss4096", 20_000, 4096, 2),  # two passes over 4 component groups of 8-CTA clusters
    ("gauss4096", 300_007, 1536, 1),  # two groups of 6 CTAs; two row chunks (2^18 + ragged)
    ("gauss4096", 20_000, 512, 2),  # D = 96 on the tensor cores: 3 feature chunks, 4-CTA clusters
    ("bf16stream", 40_001, 4096, 2),  # D = 32: two groups of 16-CTA clusters, bf16 rows
    ("bf16stream", 30_001, 1536, 2),  # 12-CTA clusters (non-portable size)
    ("bf16stream", 30_001, 2048, 2),  # 16-CTA clusters, the largest
    ("bf16stream", 50_001, 1024, 3),
]


@pytest.mark.parametrize("name,N,K,iters", CASES)
def test_em_steps_match_oracle(G, name, N, K, iters):
    run_teacher_forced(G, synth.WORKLOADS[name], N, K, iters)


@pytest.mark.parametrize("name,N,K", [("sphere768", 2_003, 1024), ("bf16stream", 30_001, 1024),
                                      ("gauss8", 1_001, 8), ("gauss4096", 20_000, 4096)])
def test_loglik_and_topm_match_oracle(G, name, N, K):
    wl = synth.WORKLOADS[name]
    Xd, X64, (w, mu, var), _ = run_teacher_forced(G, wl, N, K, 2)
    th = params_np(w, mu, var)
    ll = G.gmm_loglik(Xd, w, mu, var, wl.var_floor)
    ll_ref = oracle.loglik(X64, *th)
    assert abs(ll.item() - ll_ref) <= compare.LL_REL * abs(ll_ref)
    for m in (1, 2, 3):
        idx, resp = G.gmm_assign_topm(Xd, w, mu, var, m)
        ridx, rresp = oracle.assign_topm(X64, *th, min(m + 1, K))
        bad, worst = compare.compare_topm(ridx[:, :m], rresp[:, :m], idx.cpu().numpy(),
                                          resp.cpu().numpy(), rresp)
        assert bad == 0 and worst <= 1.0, (m, bad, worst)


@pytest.mark.parametrize("name,N,K", [("gauss8", 10_000, 8), ("uint8img", 20_011, 256),
                                      ("bf16stream", 30_001, 1024)])
def test_seeded_init_picks_the_oracles_rows(G, name, N, K):
    """gmm_init(seed) chooses its rows by SplitMix64-driven Floyd sampling on the
    host; the oracle's own implementation of those definitions picks the same
    rows, so the means are identical and the rest of the init agrees."""
    wl = synth.WORKLOADS[name]
    X, _ = synth.make_data(wl, N)
    X64 = synth.x_as_f64(wl, X)
    Xd = to_device(wl, X)
    mode = G.GMM_INIT_VAR_ONE if wl.var_init == "one" else G.GMM_INIT_VAR_DATA
    for seed in (wl.init_seed, 2**64 - 1):
        gw, gmu, gvar = params_np(*G.gmm_init(Xd, seed, K, mode, wl.var_floor))
        rw, rmu, rvar = oracle.init_seeded(X64, seed, K, mode, wl.var_floor)
        np.testing.assert_array_equal(gmu, rmu)
        np.testing.assert_allclose(gw, rw, rtol=1e-7)
        np.testing.assert_allclose(gvar, rvar, rtol=1e-6)


def _tiny(G, X, w, mu, var, floor=1e-6):
    import torch

    Xd = torch.tensor(X, dtype=torch.float32, device="cuda")
    wd = torch.tensor(w, dtype=torch.float32, device="cuda")
    mud = torch.tensor(mu, dtype=torch.float32, device="cuda")
    vard = torch.tensor(var, dtype=torch.float32, device="cuda")
    th = params_np(wd, mud, vard)
    ll = torch.zeros(1, dtype=torch.float64, device="cuda")
    G.gmm_em_step(Xd, wd, mud, vard, ll, floor)
    ref = oracle.em_step(np.asarray(X, dtype=np.float32).astype(np.float64), *th, var_floor=floor)
    return ref, (*params_np(wd, mud, vard), ll.item())


def test_single_point_single_component(G):
    ref, got = _tiny(G, [[1.0, 2.0, 3.0, 4.0]], [1.0], [[0.0] * 4], [[1.0] * 4])
    np.testing.assert_allclose(got[0], [1.0])
    np.testing.assert_allclose(got[1], [[1, 2, 3, 4]], rtol=1e-6)
    np.testing.assert_allclose(got[2], 1e-6, rtol=1e-6)  # one point: variance hits the floor
    assert abs(got[3] - ref[3]) <= 1e-6 * abs(ref[3])


def test_k1_closed_form_and_max_d(G):
    rng = np.random.default_rng(3)
    D = 1024
    X = (rng.normal(size=(777, D)) * 3 + 1).astype(np.float32)
    ref, got = _tiny(G, X, [1.0], rng.normal(size=(1, D)), np.ones((1, D)))
    X64 = X.astype(np.float64)
    np.testing.assert_allclose(got[1][0], X64.mean(0), rtol=0, atol=1e-3 * 3)
    np.testing.assert_allclose(got[2][0], X64.var(0), rtol=1e-3)
    assert compare.compare_step(ref[:4], got, ref[4])["ok"]


def test_ragged_k_and_dead_component(G):
    rng = np.random.default_rng(5)
    K, D, N = 300, 8, 4_099
    X = rng.normal(size=(N, D)).astype(np.float32) * 4
    w = rng.dirichlet(np.ones(K))
    w[7] = 0.0  # dead: responsibility 0 everywhere
    w = w / w.sum()
    mu = X[rng.choice(N, K, replace=False)]
    ref, got = _tiny(G, X, w, mu, np.ones((K, D)))
    assert got[0][7] == 0.0
    assert compare.compare_step(ref[:4], got, ref[4])["ok"]


def test_shapes_without_a_tensor_core_plan_are_rejected(G):
    """One backend: a shape the tensor-core kernel has no plan for is refused before any
    launch (D beyond 1024 at the argument check; K beyond what component groups of
    2-CTA clusters hold at D = 128), not run elsewhere."""
    import torch

    assert G.gmm_plan(G.problem(1000, 128, 16384))["tensor_cores"] == 1
    p = G.problem(1000, 128, 20000)
    assert G.gmm_plan(p)["tensor_cores"] == 0
    X = torch.zeros(1000, 128, device="cuda")
    K = 20000
    w = torch.full((K,), 1.0 / K, device="cuda")
    mu = torch.zeros(K, 128, device="cuda")
    var = torch.ones(K, 128, device="cuda")
    ll = torch.zeros(1, dtype=torch.float64, device="cuda")
    for call in (lambda: G.gmm_em_step(X, w, mu, var, ll),
                 lambda: G.gmm_loglik(X, w, mu, var)):
        with pytest.raises(G.GmmError) as e:
            call()
        assert e.value.status == G.GMM_ERR_UNSUPPORTED
    Xw = torch.zeros(100, 1028, device="cuda")
    with pytest.raises(G.GmmError) as e:
        G.gmm_em_step(Xw, w[:4] * 0 + 0.25, torch.zeros(4, 1028, device="cuda"),
                      torch.ones(4, 1028, device="cuda"), ll)
    assert e.value.status == G.GMM_ERR_UNSUPPORTED


def test_workspace_does_not_depend_on_n(G):
    for D, K, dt in ((128, 256, 0), (96, 4096, 0), (32, 1024, 1), (768, 1024, 0)):
        sizes = {G.gmm_workspace_size(G.problem(N, D, K, dt)) for N in (10_000, 10**6, 10**8)}
        assert len(sizes) == 1


def test_step_allocates_no_device_memory(G):
    import torch

    wl = synth.WORKLOADS["uint8img"]
    X, _ = synth.make_data(wl, 200_000)
    Xd = to_device(wl, X)
    p = G.problem_for(Xd, wl.K)
    ws = G.workspace(p)
    w, mu, var = G.gmm_init_rows(Xd, synth.init_rows(len(X), wl.K, 1), wl.K, ws=ws)
    ll = torch.zeros(1, dtype=torch.float64, device="cuda")
    G.gmm_em_step(Xd, w, mu, var, ll, ws=ws)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        G.gmm_em_step(Xd, w, mu, var, ll, ws=ws)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free0 == free1


def test_deterministic(G):
    import torch

    wl = synth.WORKLOADS["bf16stream"]
    X, _ = synth.make_data(wl, 40_000)
    Xd = to_device(wl, X)
    ws = G.workspace(G.problem_for(Xd, wl.K))
    w, mu, var = G.gmm_init_rows(Xd, synth.init_rows(len(X), wl.K, 9), wl.K, ws=ws)
    outs = []
    for _ in range(2):
        w2, mu2, var2 = w.clone(), mu.clone(), var.clone()
        ll = torch.zeros(1, dtype=torch.float64, device="cuda")
        G.gmm_em_step(Xd, w2, mu2, var2, ll, ws=ws)
        outs.append((w2.cpu(), mu2.cpu(), var2.cpu(), ll.cpu()))
    for a, b in zip(*outs):
        assert torch.equal(a, b)


def test_nonfinite_input_sets_device_flag(G):
    import torch

    rng = np.random.default_rng(1)
    X = rng.normal(size=(1000, 16)).astype(np.float32)
    X[123, 4] = np.nan
    Xd = torch.tensor(X, device="cuda")
    ws = G.workspace(G.problem_for(Xd, 4))
    w = torch.full((4,), 0.25, device="cuda")
    mu = torch.tensor(X[:4], device="cuda").nan_to_num()
    var = torch.ones(4, 16, device="cuda")
    G.gmm_em_step(Xd, w, mu, var, ws=ws)
    rc, flags = G.gmm_device_status(ws)
    assert rc == G.GMM_ERR_NUMERIC and flags & G.GMM_DEVFLAG_NONFINITE_X
    rc, flags = G.gmm_device_status(ws)  # cleared by the previous read
    assert rc == 0 and flags == 0
    Xd = torch.tensor(np.nan_to_num(X), device="cuda")
    var[2, 3] = 0.0
    G.gmm_em_step(Xd, w, mu, var, ws=ws)
    rc, flags = G.gmm_device_status(ws)
    assert rc == G.GMM_ERR_NUMERIC and flags & G.GMM_DEVFLAG_BAD_PARAMS


@pytest.mark.parametrize("name,N,K,iters", [("gauss8", 10_000, 8, 10), ("gauss8", 10_007, 8, 4),
                                            ("bf16stream", 8_001, 16, 3)])
def test_single_launch_fit_matches_oracle_each_iteration(G, name, N, K, iters):
    """gmm_fit on a problem that fits one cluster's shared memory runs every
    iteration in one launch.  Teacher-forced: each iteration run alone
    (gmm_fit with iters = 1, the same kernel) matches the oracle's step from the
    same parameters; and the one-launch fit over all iterations is bit-identical
    to those single iterations chained, LL history included."""
    import torch

    wl = synth.WORKLOADS[name]
    X, _ = synth.make_data(wl, N)
    X64 = synth.x_as_f64(wl, X)
    Xd = to_device(wl, X)
    ws = G.workspace(G.problem_for(Xd, K, wl.var_floor))
    mode = G.GMM_INIT_VAR_ONE if wl.var_init == "one" else G.GMM_INIT_VAR_DATA
    w, mu, var = G.gmm_init(Xd, wl.init_seed, K, mode, wl.var_floor, ws=ws)
    w1, mu1, var1 = w.clone(), mu.clone(), var.clone()
    hist = G.gmm_fit(Xd, w, mu, var, iters, wl.var_floor, ws=ws).cpu().numpy()
    rc, flags = G.gmm_device_status(ws)
    assert rc == 0 and flags == 0
    lls = []
    for t in range(iters):
        th = params_np(w1, mu1, var1)
        lls.append(G.gmm_fit(Xd, w1, mu1, var1, 1, wl.var_floor, ws=ws).item())
        w2, mu2, var2, ll_ref, Nk = oracle.em_step(X64, *th, var_floor=wl.var_floor)
        rep = compare.compare_step((w2, mu2, var2, ll_ref), (*params_np(w1, mu1, var1), lls[-1]),
                                   Nk)
        assert rep["ok"], (t, rep)
    assert torch.equal(w, w1) and torch.equal(mu, mu1) and torch.equal(var, var1)
    np.testing.assert_array_equal(hist, np.array(lls))
    # LL of the trajectory is monotone up to fp32 rounding
    assert np.all(np.diff(hist) >= -1e-6 * np.abs(hist[1:]))


def test_single_launch_fit_agrees_with_the_fused_step(G):
    """The one-launch fit (direct form on the CUDA cores) and gmm_em_step (the
    tensor-core pass) take the same EM step within the parity tolerances."""
    import torch

    wl = synth.WORKLOADS["gauss8"]
    X, _ = synth.make_data(wl)
    Xd = to_device(wl, X)
    ws = G.workspace(G.problem_for(Xd, wl.K))
    w, mu, var = G.gmm_init(Xd, wl.init_seed, wl.K, G.GMM_INIT_VAR_ONE, ws=ws)
    G.gmm_fit(Xd, w, mu, var, 3, ws=ws)
    a = [w.clone(), mu.clone(), var.clone()]
    b = [w.clone(), mu.clone(), var.clone()]
    lla = G.gmm_fit(Xd, *a, 1, ws=ws).item()
    llb = torch.zeros(1, dtype=torch.float64, device="cuda")
    G.gmm_em_step(Xd, *b, llb, ws=ws)
    rep = compare.compare_step((*params_np(*b), llb.item()), (*params_np(*a), lla),
                               a[0].double().cpu().numpy() * len(X))
    assert rep["ok"], rep


@pytest.mark.parametrize("name,N,K,fit_iters", [("uint8img", 20_011, 256, 8),
                                                 ("bf16stream", 60_001, 1024, 6),
                                                 ("gauss8", 10_000, 8, 6),
                                                 ("uint8img", 1_000_000, 256, 6),
                                                 ("bf16stream", 1_000_000, 1024, 4),
                                                 ("gauss4096", 100_000, 4096, 3)])
def test_late_iteration_step_matches_oracle(G, name, N, K, fit_iters):
    """Teacher-forced step from parameters the oracle has already fitted for a
    few iterations: the variances have shrunk, so the expanded form's
    cancellation (mu~^2 / var up to ~650 on uint8img) is at its worst here.  The
    N = 1e6 cases are the full uint8img workload and a million bf16stream rows:
    about a hundred tiles per cluster, so the every-8-tiles drain cadence and
    the tight components of a fitted mixture are both reached."""
    import torch

    wl = synth.WORKLOADS[name]
    X, _ = synth.make_data(wl, N)
    X64 = synth.x_as_f64(wl, X)
    Xd = to_device(wl, X)
    rows = synth.init_rows(N, K, wl.init_seed)
    mode = 0 if wl.var_init == "one" else 1
    th = oracle.init(X64, rows, K, mode, wl.var_floor)
    th = oracle.fit(X64, *th, fit_iters, wl.var_floor)[:3]
    w = torch.tensor(th[0], dtype=torch.float32, device="cuda")
    mu = torch.tensor(th[1], dtype=torch.float32, device="cuda")
    var = torch.tensor(th[2], dtype=torch.float32, device="cuda")
    th32 = params_np(w, mu, var)
    ll = torch.zeros(1, dtype=torch.float64, device="cuda")
    ws = G.workspace(G.problem_for(Xd, K, wl.var_floor))
    G.gmm_em_step(Xd, w, mu, var, ll, wl.var_floor, ws=ws)
    rc, flags = G.gmm_device_status(ws)
    assert rc == 0, flags
    w2, mu2, var2, ll_ref, Nk = oracle.em_step(X64, *th32, var_floor=wl.var_floor)
    rep = compare.compare_step((w2, mu2, var2, ll_ref), (*params_np(w, mu, var), ll.item()), Nk)
    assert rep["ok"], rep


@pytest.mark.parametrize("name,N,K", [("uint8img", 20_011, 256), ("bf16stream", 30_001, 1024),
                                      ("sphere768", 2_003, 1024), ("gauss4096", 20_000, 4096)])
def test_estep_statistics_match_oracle(G, name, N, K):
    """gmm_estep_stats returns [N_k | A | B | LL] about the input means, the
    same quantities (and layout) as the oracle's E-step statistics."""
    import torch

    wl = synth.WORKLOADS[name]
    X, _ = synth.make_data(wl, N)
    X64 = synth.x_as_f64(wl, X)
    Xd = to_device(wl, X)
    ws = G.workspace(G.problem_for(Xd, K, wl.var_floor))
    w, mu, var = G.gmm_init_rows(Xd, synth.init_rows(N, K, wl.init_seed), K, 1, wl.var_floor, ws=ws)
    G.gmm_em_step(Xd, w, mu, var, None, wl.var_floor, ws=ws)
    th = params_np(w, mu, var)
    st = G.gmm_estep_stats(Xd, w, mu, var, None, wl.var_floor, ws=ws).cpu().numpy()
    Nk, A, B, ll = oracle.estep_stats(X64, *th)
    D = X.shape[1]
    gN, gA = st[:K], st[K:K + K * D].reshape(K, D)
    gB, gll = st[K + K * D:K + 2 * K * D].reshape(K, D), st[-1]
    # N_k at the weight tolerance: 1e-3 relative plus 1e-9 of N
    assert np.all(np.abs(gN - Nk) <= 1e-3 * Nk + compare.W_ABS * N)
    gate = Nk >= 10
    # a sum of deviations is judged against its natural scale sqrt(N_k * B)
    scale = np.sqrt(np.maximum(Nk[:, None] * B, 1e-300))
    assert np.all(np.abs(gA - A)[gate] <= 1e-3 * scale[gate] + 1e-9)
    # the second moments through the M-step they feed, under the step tolerances
    ref = oracle.mstep(N, th[1], th[2], Nk, A, B, wl.var_floor)
    got = oracle.mstep(N, th[1], th[2], gN, gA, gB, wl.var_floor)
    rep = compare.compare_step((*ref, ll), (*got, gll), Nk, N)
    assert rep["ok"], rep
    assert abs(gll - ll) <= compare.LL_REL * abs(ll)


@pytest.mark.parametrize("name,N,K,shards", [("uint8img", 40_000, 256, 3),
                                             ("bf16stream", 50_000, 1024, 2)])
def test_row_shards_sum_to_the_full_step(G, name, N, K, shards):
    """Statistics of disjoint row blocks, summed by gmm_mstep in shard order,
    give the same M-step as one gmm_em_step over all rows."""
    import torch

    from soft_clustering_em_b200 import sharded

    wl = synth.WORKLOADS[name]
    X, _ = synth.make_data(wl, N)
    Xd = to_device(wl, X)
    ws = G.workspace(G.problem_for(Xd, K, wl.var_floor))
    w, mu, var = G.gmm_init_rows(Xd, synth.init_rows(N, K, wl.init_seed), K, 1, wl.var_floor, ws=ws)
    full = [w.clone(), mu.clone(), var.clone()]
    ll_full = torch.zeros(1, dtype=torch.float64, device="cuda")
    G.gmm_em_step(Xd, *full, ll_full, wl.var_floor, ws=ws)
    parts = []
    for r in range(shards):
        lo, hi = sharded.shard_rows(N, shards, r)
        Xs = Xd[lo:hi]
        wss = G.workspace(G.problem_for(Xs, K, wl.var_floor))
        parts.append(G.gmm_estep_stats(Xs, w, mu, var, None, wl.var_floor, ws=wss))
    ll_sh = torch.zeros(1, dtype=torch.float64, device="cuda")
    sh = [w.clone(), mu.clone(), var.clone()]
    G.gmm_mstep(torch.stack(parts), N, *sh, ll_sh, wl.var_floor, G.xdtype_of(Xd))
    nk = full[0].double().cpu().numpy() * N
    rep = compare.compare_step((*params_np(*full), ll_full.item()), (*params_np(*sh), ll_sh.item()),
                               nk)
    assert rep["ok"], rep


def _kappa(w, mu, var):
    """kappa_k = sum_d (mu^^2 + 1)/var^ in the whitened units of the tensor-core path
    (centring at the mixture mean, s = 2^(round(log2 std) + 1)); recomputed here only
    to show that a case reaches the split thresholds."""
    w, mu, var = (np.asarray(a, dtype=np.float64) for a in (w, mu, var))
    m = (w[:, None] * mu).sum(0) / w.sum()
    v = (w[:, None] * (var + mu ** 2)).sum(0) / w.sum() - m ** 2
    s = 2.0 ** (np.rint(0.5 * np.log2(v)) + 1)
    return ((((mu - m) / s) ** 2 + 1) / (var / s ** 2)).sum(1)


def _split_case():
    """A component collapsed onto 40 rows identical in 4 dimensions, and a tight
    20-point component; see test_split_dimensions_match_oracle."""
    rng = np.random.default_rng(11)
    N, D, K = 6_001, 16, 12
    centers = rng.uniform(-20, 20, size=(K, D))
    z = rng.integers(2, K, size=N)
    X = (centers[z] + rng.normal(size=(N, D))).astype(np.float32)
    X[:40, :4] = 7.0  # 40 rows identical in dimensions 0-3
    X[:40, 4:] = (centers[0, 4:] + rng.normal(size=(40, D - 4))).astype(np.float32)
    # 3.2 from the mixture mean (0.1 in x^ units), spread 0.2: mu^^2/var^ stays ~200,
    # and x^^2 of its points stays in fp16's normal range
    centers[1] = centers[2:].mean(0) + 3.2
    X[40:60] = (centers[1] + 0.2 * rng.normal(size=(20, D))).astype(np.float32)
    w = np.full(K, 1.0 / K)
    w[0], w[1] = 40.0 / N, 20.0 / N
    w = w / w.sum()
    mu = centers.copy()
    mu[0, :4] = 7.0
    mu[0, 4:] = X[:40, 4:].mean(0)
    mu[1] = X[40:60].mean(0)
    var = np.ones((K, D))
    var[0, :4] = 1e-6
    var[1] = 0.05
    return X, w, mu, var


def test_split_dimensions_deterministic(G):
    """The split dimensions' direct-form moments are summed as fixed-point
    integers, so two runs of the same step give bit-identical results whatever
    the order in which rows and clusters add them."""
    import torch

    X, w, mu, var = _split_case()
    Xd = torch.tensor(X, device="cuda")
    ws = G.workspace(G.problem_for(Xd, len(w)))
    outs = []
    for _ in range(3):
        t = [torch.tensor(a, dtype=torch.float32, device="cuda") for a in (w, mu, var)]
        ll = torch.zeros(1, dtype=torch.float64, device="cuda")
        st = G.gmm_estep_stats(Xd, *t, None, ws=ws)
        G.gmm_em_step(Xd, *t, ll, ws=ws)
        outs.append([a.cpu() for a in (*t, ll, st)])
    for run in outs[1:]:
        for a, b in zip(outs[0], run):
            assert torch.equal(a, b)


def test_split_dimensions_match_oracle(G):
    """A component collapsed onto rows that share exact values in some dimensions
    (variance at the floor there: kappa far above 1e7), and a tight component
    expecting 20 points (kappa between 6e3 and 1e7): both take exact log-joints in
    direct form for the rows near them, and the moments of their dimensions with
    kappa_kd > 500 in direct form too.  (The tight
    component sits 0.1 from the centring point in x^ units: far from it, mu^^2/var^ of
    its kept dimensions would bound its variance's precision at about that ratio times
    2^-22; right at it, x^^2 of its points would fall below fp16's normal range -- the
    tensor-core statistics' two limits.)"""
    X, w, mu, var = _split_case()
    N = len(X)
    kap = _kappa(np.float32(w), np.float32(mu), np.float32(var))
    # component 0 by kappa alone, component 1 only because it expects few points
    assert kap[0] > 1e7 and w[1] * N < 50 and 2e4 < kap[1] < 1e7, kap[:2]
    ref, got = _tiny(G, X, w, mu, var)
    rep = compare.compare_step(ref[:4], got, ref[4])
    assert rep["ok"], rep
    # the collapsed component keeps its 40 points and its zero spread in dimensions 0-3
    assert abs(got[0][0] * N - 40.0) < 0.05
    np.testing.assert_allclose(got[2][0][:4], 1e-6, rtol=1e-6)


@pytest.mark.parametrize("D,K", [(48, 200), (96, 300), (260, 200), (1024, 130)])
def test_padded_and_odd_feature_chunks(G, D, K):
    """2D not a multiple of 64 (D = 48: two chunks, the second half padding), an odd
    chunk count (D = 96: three chunks), and streamed features (D = 260: nine chunks in
    statistics groups of five and four; D = 1024, the largest: 32 chunks in seven
    groups), with ragged K and N."""
    rng = np.random.default_rng(D)
    N = 5_003
    centers = rng.uniform(-6, 6, size=(K, D))
    z = rng.integers(0, K, size=N)
    X = (centers[z] + rng.normal(size=(N, D))).astype(np.float32)
    w = rng.dirichlet(np.ones(K))
    mu = X[rng.choice(N, K, replace=False)]
    ref, got = _tiny(G, X, w, mu, np.ones((K, D)))
    rep = compare.compare_step(ref[:4], got, ref[4])
    assert rep["ok"], rep
