"""Pins for the CPU oracle against what the mathematics fixes (no GPU).

The pages ("Flash-GMM: A Memory-Efficient Kernel for Scalable Soft Clustering",
review page section 3, and the abstract) name EM for a Gaussian mixture but
print no formulas or worked values, so each pin below comes from the
definition of EM: a closed-form worked case, brute-force enumeration of all
labellings, the K = 1 closed form, invariants (row sums, monotone
log-likelihood), symmetric special cases, recovery of well-separated mixtures
and an independent library implementation (scikit-learn).
"""
import json
import math
import os

import numpy as np
import pytest

from oracle import brute
from soft_clustering_em_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_problem(rng, N, D, K, spread=2.0):
    X = rng.normal(size=(N, D)) * spread
    w = rng.dirichlet(np.ones(K))
    mu = rng.normal(size=(K, D)) * spread
    var = rng.uniform(0.3, 3.0, size=(K, D))
    return X, w, mu, var


def test_golden_two_point_symmetric(oracle_mod):
    g = json.load(open(os.path.join(GOLDEN, "two_point_symmetric.json")))
    w2, mu2, var2, ll, _ = oracle_mod.em_step(g["X"], g["w"], g["mu"], g["var"], var_floor=0.0)
    e, tol = g["expect"], g["tol"]
    np.testing.assert_allclose(w2, e["w"], rtol=0, atol=tol)
    np.testing.assert_allclose(mu2, e["mu"], rtol=0, atol=tol)
    np.testing.assert_allclose(var2, e["var"], rtol=0, atol=tol)
    assert abs(ll - e["loglik"]) < tol
    R, _ = oracle_mod.responsibilities(g["X"], g["w"], g["mu"], g["var"])
    np.testing.assert_allclose(R[0], e["r_row0"], rtol=0, atol=tol)


@pytest.mark.parametrize("seed", range(12))
def test_brute_force_enumeration(oracle_mod, seed):
    rng = np.random.default_rng(seed)
    N = int(rng.integers(1, 7))
    K = int(rng.integers(1, 4))
    D = int(rng.integers(1, 3))
    X, w, mu, var = _rand_problem(rng, N, D, K)
    bw, bmu, bvar, bll, bR = brute.em_step(X, w, mu, var, var_floor=0.0)
    w2, mu2, var2, ll, _ = oracle_mod.em_step(X, w, mu, var, var_floor=0.0)
    R, lse = oracle_mod.responsibilities(X, w, mu, var)
    np.testing.assert_allclose(R, bR, rtol=1e-11, atol=1e-300)
    np.testing.assert_allclose(w2, bw, rtol=1e-11)
    np.testing.assert_allclose(mu2, bmu, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(var2, bvar, rtol=1e-10)
    assert abs(ll - bll) <= 1e-12 * max(1.0, abs(bll))
    assert abs(lse.sum() - bll) <= 1e-12 * max(1.0, abs(bll))


@pytest.mark.parametrize("seed", range(4))
def test_row_sums_are_one(oracle_mod, seed):
    rng = np.random.default_rng(100 + seed)
    X, w, mu, var = _rand_problem(rng, 500, 5, 7, spread=1.0)
    R, _ = oracle_mod.responsibilities(X, w, mu, var)
    assert np.all(R >= 0)
    np.testing.assert_allclose(R.sum(axis=1), 1.0, rtol=0, atol=1e-12)


def test_k1_closed_form(oracle_mod):
    rng = np.random.default_rng(7)
    X = rng.normal(size=(3000, 6)) * rng.uniform(0.5, 4, size=6) + rng.normal(size=6) * 5
    w, mu, var = np.ones(1), rng.normal(size=(1, 6)), rng.uniform(0.5, 2, size=(1, 6))
    w2, mu2, var2, _, _ = oracle_mod.em_step(X, w, mu, var, var_floor=1e-6)
    np.testing.assert_allclose(w2, [1.0], rtol=0, atol=1e-15)
    np.testing.assert_allclose(mu2[0], X.mean(axis=0), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(var2[0], X.var(axis=0), rtol=1e-10)
    # LL at the fitted single Gaussian: -(N/2) sum_d (log(2 pi var_d) + 1)
    ll1 = oracle_mod.loglik(X, w2, mu2, var2)
    expect = -0.5 * X.shape[0] * np.sum(np.log(2 * np.pi * var2[0]) + 1.0)
    assert abs(ll1 - expect) <= 1e-11 * abs(expect)


def test_identical_components(oracle_mod):
    rng = np.random.default_rng(11)
    X = rng.normal(size=(400, 3)) * 2 + 1
    K = 5
    w = rng.dirichlet(np.ones(K))
    mu = np.tile(rng.normal(size=3), (K, 1))
    var = np.tile(rng.uniform(0.5, 2, size=3), (K, 1))
    R, _ = oracle_mod.responsibilities(X, w, mu, var)
    np.testing.assert_allclose(R, np.tile(w, (X.shape[0], 1)), rtol=1e-13)
    w2, mu2, var2, _, _ = oracle_mod.em_step(X, w, mu, var)
    np.testing.assert_allclose(w2, w, rtol=1e-12)
    for k in range(K):
        np.testing.assert_allclose(mu2[k], X.mean(axis=0), rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(var2[k], X.var(axis=0), rtol=1e-11)


@pytest.mark.parametrize("name", list(synth.WORKLOADS))
def test_loglik_monotone(oracle_mod, name):
    wl = synth.WORKLOADS[name]
    n = {1: 10_000, 2: 4000, 3: 1500, 4: 6000, 5: 20_000}[wl.number]
    K = min(wl.K, {1: 8, 2: 64, 3: 32, 4: 128, 5: 128}[wl.number])
    X, _ = synth.make_data(wl, n)
    X = synth.x_as_f64(wl, X)
    rows = synth.init_rows(n, K, wl.init_seed)
    w, mu, var = oracle_mod.init(X, rows, K, 0 if wl.var_init == "one" else 1, wl.var_floor)
    _, _, _, ll = oracle_mod.fit(X, w, mu, var, 8, wl.var_floor)
    assert np.all(np.isfinite(ll))
    assert np.all(np.diff(ll) >= -1e-12 * np.abs(ll[1:])), ll


def test_separated_recovery(oracle_mod):
    wl = synth.WORKLOADS["gauss8"]
    X32, z = synth.make_data(wl)
    X = X32.astype(np.float64)
    pi_t, mu_t, sd_t, _ = synth.true_params(wl)
    rows = np.array([np.flatnonzero(z == k)[0] for k in range(wl.K)])
    w, mu, var = oracle_mod.init(X, rows, wl.K, 0, wl.var_floor)
    w, mu, var, ll = oracle_mod.fit(X, w, mu, var, wl.iters, wl.var_floor)
    counts = np.bincount(z, minlength=wl.K)
    # means within 5 standard errors of the generating means
    assert np.all(np.abs(mu - mu_t) <= 5 * sd_t / np.sqrt(counts)[:, None])
    assert np.all(np.abs(w - pi_t) <= 5 * np.sqrt(pi_t * (1 - pi_t) / X.shape[0]))
    assert np.all(np.abs(var - 1.0) <= 5 * np.sqrt(2.0 / counts)[:, None])


def test_sklearn_one_step(oracle_mod):
    mixture = pytest.importorskip("sklearn.mixture")
    import warnings

    rng = np.random.default_rng(5)
    X, w, mu, var = _rand_problem(rng, 2000, 4, 3, spread=1.5)
    gm = mixture.GaussianMixture(n_components=3, covariance_type="diag", reg_covar=0.0,
                                 max_iter=1, tol=0.0, weights_init=w, means_init=mu,
                                 precisions_init=1.0 / var, init_params="random")
    with warnings.catch_warnings():
        warnings.simplefilter("ignore")
        gm.fit(X)
    w2, mu2, var2, ll, _ = oracle_mod.em_step(X, w, mu, var, var_floor=0.0)
    np.testing.assert_allclose(w2, gm.weights_, rtol=1e-9)
    np.testing.assert_allclose(mu2, gm.means_, rtol=1e-9, atol=1e-10)
    np.testing.assert_allclose(var2, gm.covariances_, rtol=1e-8)
    # score() averages LL over points, at the updated parameters
    ll_new = oracle_mod.loglik(X, w2, mu2, var2)
    assert abs(ll_new / X.shape[0] - gm.score(X)) < 1e-10


def test_topm_matches_sorted_brute_force(oracle_mod):
    rng = np.random.default_rng(21)
    for _ in range(6):
        N, D, K = 5, 2, 3
        X, w, mu, var = _rand_problem(rng, N, D, K, spread=1.0)
        *_, bR = brute.em_step(X, w, mu, var)
        bR = np.array(bR)
        for m in (1, 2, 3):
            idx, resp = oracle_mod.assign_topm(X, w, mu, var, m)
            for n in range(N):
                order = np.lexsort((np.arange(K), -bR[n]))[:m]
                assert list(idx[n]) == list(order)
                np.testing.assert_allclose(resp[n], bR[n][order], rtol=1e-11)


def test_topm_ties_take_lower_index(oracle_mod):
    X = np.array([[0.0, 0.0], [3.0, 1.0]])
    w = np.full(4, 0.25)
    mu = np.zeros((4, 2))
    var = np.ones((4, 2))
    idx, resp = oracle_mod.assign_topm(X, w, mu, var, 3)
    assert idx.tolist() == [[0, 1, 2], [0, 1, 2]]
    np.testing.assert_allclose(resp, 0.25, rtol=1e-15)


def test_init_modes(oracle_mod):
    rng = np.random.default_rng(3)
    X = rng.normal(size=(300, 4)) * [1, 2, 3, 4]
    rows = np.array([5, 17, 250])
    w, mu, var = oracle_mod.init(X, rows, 3, 1, 1e-6)
    np.testing.assert_array_equal(mu, X[rows])
    np.testing.assert_allclose(w, 1 / 3, rtol=1e-15)
    np.testing.assert_allclose(var, np.tile(X.var(axis=0), (3, 1)), rtol=1e-12)
    w, mu, var = oracle_mod.init(X, rows, 3, 0, 1e-6)
    np.testing.assert_array_equal(var, 1.0)
    # constant data: the variance init hits the floor
    w, mu, var = oracle_mod.init(np.ones((10, 2)), [0, 1], 2, 1, 1e-6)
    np.testing.assert_array_equal(var, 1e-6)


def test_empty_and_dead_components(oracle_mod):
    rng = np.random.default_rng(9)
    X = rng.normal(size=(200, 2))
    w = np.array([0.5, 0.3, 0.2, 0.0])
    mu = np.array([[0.0, 0.0], [1.0, 0.0], [1e4, 1e4], [0.5, 0.5]])
    var = np.ones((4, 2))
    w2, mu2, var2, ll, Nk = oracle_mod.em_step(X, w, mu, var)
    # component 2 is so far away that every responsibility underflows to zero
    assert Nk[2] == 0.0 and w2[2] == 0.0
    np.testing.assert_array_equal(mu2[2], mu[2])
    np.testing.assert_array_equal(var2[2], var[2])
    # component 3 has pi = 0: it is dead, and the LL equals that of the mixture without it
    assert Nk[3] == 0.0 and w2[3] == 0.0
    ll3 = oracle_mod.loglik(X, w[:3], mu[:3], var[:3])
    assert abs(ll - ll3) <= 1e-13 * abs(ll3)


def test_variance_floor(oracle_mod):
    # a component sitting on one isolated point collapses onto it: var -> floor
    X = np.array([[0.0], [0.1], [-0.1], [50.0]])
    w = np.array([0.75, 0.25])
    mu = np.array([[0.0], [50.0]])
    var = np.array([[1.0], [1.0]])
    w2, mu2, var2, _, _ = oracle_mod.em_step(X, w, mu, var, var_floor=1e-6)
    assert var2[1, 0] == 1e-6
    assert abs(mu2[1, 0] - 50.0) < 1e-12
    np.testing.assert_allclose(var2[0, 0], np.var([0.0, 0.1, -0.1]), rtol=1e-12)


def test_determinism_across_threads(oracle_mod):
    import subprocess
    import sys

    code = ("import numpy as np, oracle; rng=np.random.default_rng(1);"
            "X=rng.normal(size=(5000,8)); w=np.full(6,1/6); mu=rng.normal(size=(6,8));"
            "var=np.ones((6,8)); r=oracle.em_step(X,w,mu,var);"
            "print(repr(r[3]), repr(float(r[1].sum())), repr(float(r[2].sum())))")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    outs = []
    for t in ("1", "3"):
        env = dict(os.environ, OMP_NUM_THREADS=t)
        outs.append(subprocess.check_output([sys.executable, "-c", code], cwd=root, env=env))
    assert outs[0] == outs[1]
