"""Brute-force EM step by enumerating every joint labelling (TEST INFRASTRUCTURE ONLY).

An independent route to the same numbers as the oracle, for tiny inputs
(N <= 6, K <= 3).  For a mixture the joint density of the data and a labelling
z in {0..K-1}^N is

    p(X, z) = prod_n pi_{z_n} * prod_d Normal(x_nd; mu_{z_n d}, var_{z_n d}).

Summing it over all K^N labellings gives p(X) (so LL = log p(X)); the posterior
marginal P(z_n = k | X) is the responsibility r_nk; and the M-step is the
weighted mean and weighted (biased) variance under those posteriors.  Nothing
here uses the log-sum-exp factorisation, the moments-about-the-old-mean form or
any code of the C oracle: densities are evaluated in the linear domain with
pure Python floats.
"""
import itertools
import math


def _normal_pdf(x, mu, var):
    return math.exp(-0.5 * (x - mu) ** 2 / var) / math.sqrt(2.0 * math.pi * var)


def em_step(X, w, mu, var, var_floor=0.0):
    """Returns (w', mu', var', LL, R) with R the N x K posterior marginals."""
    X = [list(map(float, row)) for row in X]
    w = list(map(float, w))
    mu = [list(map(float, row)) for row in mu]
    var = [list(map(float, row)) for row in var]
    N, D, K = len(X), len(X[0]), len(w)
    assert K ** N <= 10 ** 6, "brute force is for tiny inputs only"
    dens = [[w[k] * math.prod(_normal_pdf(X[n][d], mu[k][d], var[k][d]) for d in range(D))
             for k in range(K)] for n in range(N)]
    total = 0.0
    marg = [[0.0] * K for _ in range(N)]
    for z in itertools.product(range(K), repeat=N):
        p = math.prod(dens[n][z[n]] for n in range(N))
        total += p
        for n in range(N):
            marg[n][z[n]] += p
    R = [[marg[n][k] / total for k in range(K)] for n in range(N)]
    Nk = [sum(R[n][k] for n in range(N)) for k in range(K)]
    w2 = [Nk[k] / N for k in range(K)]
    mu2 = [[sum(R[n][k] * X[n][d] for n in range(N)) / Nk[k] for d in range(D)]
           for k in range(K)]
    var2 = [[max(sum(R[n][k] * (X[n][d] - mu2[k][d]) ** 2 for n in range(N)) / Nk[k], var_floor)
             for d in range(D)] for k in range(K)]
    return w2, mu2, var2, math.log(total), R
