"""Plant plausible mistakes in a copy of the CPU oracle and check the pins catch each.

Every mutant is a one-token edit of the oracle source (a dropped term, a wrong
sign, a transposed index, a missing normaliser ...), compiled on the CPU into a
temporary library.  The pins of test_oracle_pins (closed-form golden case,
brute-force enumeration, K = 1 closed form, top-m order) are re-run against the
mutant; at least one of them must fail, otherwise the pins would not have
noticed that mistake in the real oracle.
"""
import ctypes
import json
import os
import subprocess

import numpy as np
import pytest

import oracle
from oracle import brute

SRC = os.path.join(os.path.dirname(oracle.__file__), "gmm_oracle.c")
GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "two_point_symmetric.json")

MUTANTS = {
    "drop_logdet": ("c->logw[k] - 0.5 * (c->logdet[k] + q)", "c->logw[k] - 0.5 * (q)"),
    "sign_quadratic": ("c->logw[k] - 0.5 * (c->logdet[k] + q)",
                       "c->logw[k] - 0.5 * (c->logdet[k] - q)"),
    "drop_logw": ("c->logw[k] - 0.5 * (c->logdet[k] + q)", "-0.5 * (c->logdet[k] + q)"),
    "logdet_no_2pi": ("s += log(2.0 * M_PI * v);", "s += log(v);"),
    "ivar_transposed": ("c->ivar[(size_t)k * D + d] = 1.0 / v;",
                        "c->ivar[(size_t)d * K + k] = 1.0 / v;"),
    "lse_drop_max": ("return m + log(s);", "return log(s);"),
    "resp_unnormalised": ("double r = exp(l[k] - lse);", "double r = exp(l[k]);"),
    "second_moment_linear": ("bk[d] += r * e * e;", "bk[d] += r * e;"),
    "mean_wrong_sign": ("mu_out[i] = mu[i] + delta;", "mu_out[i] = mu[i] - delta;"),
    "var_drop_delta2": ("const double v = B[i] / nk - delta * delta;",
                        "const double v = B[i] / nk;"),
    "weight_unnormalised": ("w_out[k] = nk / (double)N;", "w_out[k] = nk;"),
    "topm_ties_high": ("if (best < 0 || l[k] > l[best]) best = k;",
                       "if (best < 0 || l[k] >= l[best]) best = k;"),
    "topm_ascending": ("if (best < 0 || l[k] > l[best]) best = k;",
                       "if (best < 0 || l[k] < l[best]) best = k;"),
}


def _pins(lib_mod):
    """Run the oracle pins on the given module; raise AssertionError on any mismatch."""
    g = json.load(open(GOLDEN))
    w2, mu2, var2, ll, _ = lib_mod.em_step(g["X"], g["w"], g["mu"], g["var"], var_floor=0.0)
    e, tol = g["expect"], g["tol"]
    np.testing.assert_allclose(w2, e["w"], rtol=0, atol=tol)
    np.testing.assert_allclose(mu2, e["mu"], rtol=0, atol=tol)
    np.testing.assert_allclose(var2, e["var"], rtol=0, atol=tol)
    assert abs(ll - e["loglik"]) < tol
    rng = np.random.default_rng(0)
    for _ in range(4):
        N, D, K = 4, 2, 3
        X = rng.normal(size=(N, D)) * 2
        w = rng.dirichlet(np.ones(K))
        mu = rng.normal(size=(K, D)) * 2
        var = rng.uniform(0.3, 3.0, size=(K, D))
        bw, bmu, bvar, bll, bR = brute.em_step(X, w, mu, var)
        w2, mu2, var2, ll, _ = lib_mod.em_step(X, w, mu, var, var_floor=0.0)
        np.testing.assert_allclose(w2, bw, rtol=1e-10)
        np.testing.assert_allclose(mu2, bmu, rtol=1e-9, atol=1e-12)
        np.testing.assert_allclose(var2, bvar, rtol=1e-9)
        assert abs(ll - bll) <= 1e-12 * max(1.0, abs(bll))
        bR = np.array(bR)
        idx, resp = lib_mod.assign_topm(X, w, mu, var, 2)
        for n in range(N):
            order = np.lexsort((np.arange(K), -bR[n]))[:2]
            assert list(idx[n]) == list(order)
    # ties go to the lower index
    idx, _ = lib_mod.assign_topm(np.zeros((1, 2)), np.full(3, 1 / 3), np.zeros((3, 2)),
                                 np.ones((3, 2)), 2)
    assert idx.tolist() == [[0, 1]]


class _Swap:
    """Temporarily point the oracle module at another compiled library."""

    def __init__(self, lib):
        self.lib = lib

    def __enter__(self):
        self.saved = oracle._lib
        oracle._lib = self.lib
        return oracle

    def __exit__(self, *exc):
        oracle._lib = self.saved


def test_unmutated_oracle_passes_pins(oracle_mod):
    _pins(oracle_mod)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(oracle_mod, tmp_path, name):
    before, after = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(before) == 1, f"mutation site for {name} not unique"
    mut = tmp_path / f"{name}.c"
    mut.write_text(src.replace(before, after))
    so = tmp_path / f"{name}.so"
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fPIC", "-shared",
                           "-std=c11", "-D_DEFAULT_SOURCE", "-o", str(so), str(mut), "-lm"])
    lib = oracle.bind(ctypes.CDLL(str(so)))
    with _Swap(lib) as mod:
        with pytest.raises(AssertionError):
            _pins(mod)
