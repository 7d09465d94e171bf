"""Pins of the spherical, hard-EM and k-means oracle (oracle/variants.py), on the CPU.

Each form is tied to something other than its own formula:
  * spherical EM: scikit-learn's GaussianMixture(covariance_type="spherical")
    one step; the C diagonal oracle with every variance of a component equal
    (same log-likelihood and N_k; the spherical variance is the dimension
    average of the unfloored diagonal one);
  * hard EM: closed form on separated clusters (per-cluster np.mean / np.var),
    the weights deciding an equidistant point, ties and empty components, and
    the classification log-likelihood never decreasing;
  * k-means: scikit-learn's KMeans one Lloyd step, inertia never increasing,
    ties, empty clusters, and the k-means limit of hard EM (equal weights, one
    shared spherical variance) giving the same labels and centres.
A mutant test plants plausible mistakes in a copy of the oracle and checks that
some pin fails for each.
"""
import inspect
import types
import warnings

import numpy as np
import pytest

from oracle import variants


def _blobs(rng, N, D, K, spread):
    centres = rng.uniform(-spread, spread, size=(K, D))
    z = rng.integers(0, K, N)
    return centres[z] + rng.standard_normal((N, D)), centres, z


# ---------------------------------------------------------------- spherical

def pin_spherical_sklearn(V):
    mixture = pytest.importorskip("sklearn.mixture")
    rng = np.random.default_rng(7)
    X, centres, _ = _blobs(rng, 1500, 5, 3, 2.0)
    w = np.array([0.2, 0.5, 0.3])
    mu = centres + 0.3 * rng.standard_normal(centres.shape)
    s2 = np.array([0.8, 1.3, 2.1])
    gm = mixture.GaussianMixture(n_components=3, covariance_type="spherical", reg_covar=0.0,
                                 max_iter=1, tol=0.0, weights_init=w, means_init=mu,
                                 precisions_init=1.0 / s2, init_params="random")
    with warnings.catch_warnings():
        warnings.simplefilter("ignore")
        gm.fit(X)
    w2, mu2, s22, _, _ = V.spherical_em_step(X, w, mu, s2, var_floor=0.0)
    np.testing.assert_allclose(w2, gm.weights_, rtol=1e-9)
    np.testing.assert_allclose(mu2, gm.means_, rtol=1e-9, atol=1e-10)
    np.testing.assert_allclose(s22, gm.covariances_, rtol=1e-8)
    # score() is the mean LL at the updated parameters
    _, _, _, ll_new, _ = V.spherical_em_step(X, w2, mu2, s22, var_floor=0.0)
    assert abs(ll_new / X.shape[0] - gm.score(X)) < 1e-10


def pin_spherical_is_diag_with_equal_variances(V):
    import oracle

    rng = np.random.default_rng(8)
    X, centres, _ = _blobs(rng, 800, 4, 3, 1.5)
    w = np.array([0.5, 0.3, 0.2])
    mu = centres + 0.2
    s2 = np.array([0.7, 1.0, 1.6])
    var = np.repeat(s2[:, None], 4, axis=1)
    w2, mu2, s22, ll, Nk = V.spherical_em_step(X, w, mu, s2, var_floor=0.0)
    dw, dmu, dvar, dll, dNk = oracle.em_step(X, w, mu, var, var_floor=0.0)
    assert abs(ll - dll) <= 1e-12 * abs(dll)
    np.testing.assert_allclose(Nk, dNk, rtol=1e-12)
    np.testing.assert_allclose(mu2, dmu, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(s22, dvar.mean(axis=1), rtol=1e-12)


def pin_spherical_floor(V):
    X = np.array([[1.0, 2.0], [1.0, 2.0], [1.0, 2.0]])
    w2, mu2, s22, _, _ = V.spherical_em_step(X, [1.0], [[0.0, 0.0]], [1.0], var_floor=0.25)
    np.testing.assert_allclose(mu2, [[1.0, 2.0]])
    assert s22[0] == 0.25 and w2[0] == 1.0


# ---------------------------------------------------------------- hard EM

def pin_hard_separated_closed_form(V):
    rng = np.random.default_rng(9)
    K, D = 3, 4
    centres = np.array([[-30.0] * D, [0.0] * D, [30.0] * D])
    z = rng.integers(0, K, 900)
    X = centres[z] + rng.standard_normal((900, D)) * np.array([0.5, 1.0, 1.5, 2.0])
    w2, mu2, var2, _, labels = V.hard_em_step(X, np.full(K, 1 / K), centres + 0.1,
                                              np.ones((K, D)), var_floor=0.0)
    np.testing.assert_array_equal(labels, z)
    for k in range(K):
        np.testing.assert_allclose(mu2[k], X[z == k].mean(axis=0), rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(var2[k], X[z == k].var(axis=0), rtol=1e-10)
        assert w2[k] == np.count_nonzero(z == k) / 900


def pin_hard_weights_decide_equidistant_point(V):
    X = np.array([[0.0]])
    _, _, _, cl, labels = V.hard_em_step(X, [0.3, 0.7], [[-1.0], [1.0]], [[1.0], [1.0]])
    assert labels[0] == 1
    assert abs(cl - (np.log(0.7) - 0.5 * (np.log(2 * np.pi) + 1.0))) < 1e-14


def pin_hard_ties_and_empty(V):
    X = np.array([[0.0, 1.0], [0.5, 1.5], [2.0, 2.0]])
    mu = np.array([[1.0, 1.0], [1.0, 1.0]])
    var = np.array([[2.0, 3.0], [5.0, 7.0]])
    var[1] = var[0]  # identical components: everything goes to the lower index
    w2, mu2, var2, _, labels = V.hard_em_step(X, [0.5, 0.5], mu, var, var_floor=0.0)
    np.testing.assert_array_equal(labels, [0, 0, 0])
    assert w2[1] == 0.0
    np.testing.assert_array_equal(mu2[1], mu[1])  # the empty one keeps its parameters
    np.testing.assert_array_equal(var2[1], var[1])


def pin_hard_objective_monotone(V):
    rng = np.random.default_rng(10)
    X, centres, _ = _blobs(rng, 2000, 3, 5, 2.5)
    K = 5
    w, mu, var = np.full(K, 1 / K), X[rng.choice(2000, K, replace=False)], np.ones((K, 3))
    last = -np.inf
    for _ in range(10):
        w, mu, var, cl, _ = V.hard_em_step(X, w, mu, var, var_floor=1e-6)
        assert cl >= last - 1e-9 * abs(cl)
        last = cl


# ---------------------------------------------------------------- k-means

def pin_kmeans_sklearn(V):
    cluster = pytest.importorskip("sklearn.cluster")
    rng = np.random.default_rng(11)
    X, centres, _ = _blobs(rng, 1200, 3, 4, 4.0)
    C = centres + 0.5 * rng.standard_normal(centres.shape)
    km = cluster.KMeans(n_clusters=4, init=C, n_init=1, max_iter=1, tol=0.0,
                        algorithm="lloyd")
    with warnings.catch_warnings():
        warnings.simplefilter("ignore")
        km.fit(X)
    C2, _, inertia = V.kmeans_step(X, C)
    np.testing.assert_allclose(C2, km.cluster_centers_, rtol=1e-10, atol=1e-10)
    _, labels2, inertia2 = V.kmeans_step(X, C2)
    np.testing.assert_array_equal(labels2, km.labels_)
    assert abs(inertia2 - km.inertia_) <= 1e-9 * inertia2


def pin_kmeans_monotone_ties_empty(V):
    rng = np.random.default_rng(12)
    X, _, _ = _blobs(rng, 1000, 2, 6, 3.0)
    C = X[rng.choice(1000, 6, replace=False)]
    last = np.inf
    for _ in range(8):
        C, _, inertia = V.kmeans_step(X, C)
        assert inertia <= last + 1e-9 * last
        last = inertia
    # an equidistant point goes to the lower index; a centre with no point stays put
    C2, labels, _ = V.kmeans_step(np.array([[0.0, 0.0]]),
                                  np.array([[-1.0, 0.0], [1.0, 0.0], [50.0, 50.0]]))
    assert labels[0] == 0
    np.testing.assert_array_equal(C2[1:], [[1.0, 0.0], [50.0, 50.0]])


def pin_kmeans_is_the_hard_em_limit(V):
    rng = np.random.default_rng(13)
    X, _, _ = _blobs(rng, 1500, 4, 5, 2.0)
    C = X[rng.choice(1500, 5, replace=False)]
    C2, labels, inertia = V.kmeans_step(X, C)
    _, mu2, _, cl, hlabels = V.hard_em_step(X, np.full(5, 0.2), C, np.full((5, 4), 0.5))
    np.testing.assert_array_equal(labels, hlabels)
    np.testing.assert_allclose(mu2, C2, rtol=1e-12, atol=1e-12)
    # with variance 1/2 in every dimension, l_nk = log(1/5) - (D/2) log(pi) - |x - c_k|^2
    assert abs(cl - (1500 * (np.log(0.2) - 2 * np.log(np.pi)) - inertia)) <= 1e-9 * inertia


PINS = [pin_spherical_sklearn, pin_spherical_is_diag_with_equal_variances, pin_spherical_floor,
        pin_hard_separated_closed_form, pin_hard_weights_decide_equidistant_point,
        pin_hard_ties_and_empty, pin_hard_objective_monotone, pin_kmeans_sklearn,
        pin_kmeans_monotone_ties_empty, pin_kmeans_is_the_hard_em_limit]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_oracle_meets_pin(pin):
    pin(variants)


MUTANTS = {
    "spherical_sum_over_d": ("np.mean(B[k] / Nk[k] - delta * delta)",
                             "np.sum(B[k] / Nk[k] - delta * delta)"),
    "spherical_logdet_once": ("- 0.5 * D * np.log(2.0 * np.pi * s2)",
                              "- 0.5 * np.log(2.0 * np.pi * s2)"),
    "spherical_about_old_mean": ("np.mean(B[k] / Nk[k] - delta * delta)",
                                 "np.mean(B[k] / Nk[k])"),
    "spherical_no_floor": ("max(float(np.mean(B[k] / Nk[k] - delta * delta)), var_floor)",
                           "float(np.mean(B[k] / Nk[k] - delta * delta))"),
    "hard_argmin": ("z = np.argmax(L, axis=1)", "z = np.argmin(L, axis=1)"),
    "hard_no_weights": ("return logw[None, :] - 0.5 * (logdet[None, :] + q)",
                        "return -0.5 * (logdet[None, :] + q)"),
    "hard_ties_high": ("z = np.argmax(L, axis=1)",
                       "z = L.shape[1] - 1 - np.argmax(L[:, ::-1], axis=1)"),
    "hard_weights_unnormalised": ("w2, mu2, var2 = Nk / N, mu.copy(), var.copy()",
                                  "w2, mu2, var2 = Nk, mu.copy(), var.copy()"),
    "kmeans_empty_to_zero": ("C2 = C.copy()", "C2 = np.zeros_like(C)"),
    "kmeans_ties_high": ("z = np.argmin(d2, axis=1)",
                         "z = d2.shape[1] - 1 - np.argmin(d2[:, ::-1], axis=1)"),
    "kmeans_median": ("C2[k] = members.mean(axis=0)", "C2[k] = np.median(members, axis=0)"),
}


def _mutant(name):
    src = inspect.getsource(variants)
    old, new = MUTANTS[name]
    assert src.count(old) == 1, name
    mod = types.ModuleType("variants_" + name)
    exec(compile(src.replace(old, new), "variants_" + name, "exec"), mod.__dict__)
    return mod


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name):
    V = _mutant(name)
    caught = 0
    for pin in PINS:
        try:
            with warnings.catch_warnings():
                warnings.simplefilter("ignore")
                pin(V)
        except (AssertionError, IndexError, ValueError, FloatingPointError):
            caught += 1
    assert caught >= 1, f"no pin noticed mutant {name}"
