"""CPU oracle for diagonal-covariance GMM EM (TEST INFRASTRUCTURE ONLY).

Plain fp64 implementation written from the definition of EM for a Gaussian
mixture ("Flash-GMM: A Memory-Efficient Kernel for Scalable Soft Clustering",
review page, section 3: an E-step over data tiles, statistics accumulated
globally, then the M-step).  The formulas are written out in
``gmm_oracle.c``'s header.  Only the tests, the smoke check and the benchmark's
CPU-baseline leg may import this package; the CUDA product path never does.

Every function takes float64 numpy arrays (inputs of other dtypes are converted
exactly, fp32 and bf16 values being representable in fp64) and returns float64
results.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def bind(lib):
    """Declare the C signatures on a loaded oracle library and return it."""
    P = ctypes.c_void_p
    I64, I32, F64 = ctypes.c_int64, ctypes.c_int, ctypes.c_double
    lib.oracle_estep_stats.argtypes = [I64, I32, I32, P, P, P, P, P, P, P, P]
    lib.oracle_em_step.argtypes = [I64, I32, I32, P, P, P, P, F64, P, P, P, P, P]
    lib.oracle_loglik.argtypes = [I64, I32, I32, P, P, P, P, P]
    lib.oracle_responsibilities.argtypes = [I64, I32, I32, P, P, P, P, P, P]
    lib.oracle_assign_topm.argtypes = [I64, I32, I32, P, P, P, P, I32, P, P]
    lib.oracle_init.argtypes = [I64, I32, I32, P, P, I32, F64, P, P, P]
    lib.oracle_fit.argtypes = [I64, I32, I32, P, I32, F64, P, P, P, P]
    lib.oracle_mstep.argtypes = [I64, I32, I32, P, P, P, P, P, F64, P, P, P]
    lib.oracle_mstep.restype = None
    lib.oracle_num_threads.restype = I32
    return lib


def _load():
    global _lib
    if _lib is None:
        _lib = bind(ctypes.CDLL(_build.build()))
    return _lib


def _f64(a):
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def _check(rc, what):
    if rc != 0:
        raise RuntimeError(f"oracle {what} failed (rc={rc})")


def num_threads() -> int:
    """OpenMP threads the oracle will use (OMP_NUM_THREADS or all cores)."""
    return int(_load().oracle_num_threads())


def _shapes(X, w, mu, var):
    X, w, mu, var = _f64(X), _f64(w), _f64(mu), _f64(var)
    N, D = X.shape
    K = w.shape[0]
    assert mu.shape == (K, D) and var.shape == (K, D)
    return X, w, mu, var, N, D, K


def estep_stats(X, w, mu, var):
    """Sufficient statistics about the old means: (N_k, A, B, LL)."""
    X, w, mu, var, N, D, K = _shapes(X, w, mu, var)
    Nk = np.zeros(K)
    A = np.zeros((K, D))
    B = np.zeros((K, D))
    ll = ctypes.c_double(0.0)
    _check(_load().oracle_estep_stats(N, D, K, _p(X), _p(w), _p(mu), _p(var), _p(Nk), _p(A),
                                      _p(B), ctypes.byref(ll)), "estep_stats")
    return Nk, A, B, ll.value


def mstep(N, mu, var, Nk, A, B, var_floor):
    """M-step from statistics about the old means: (w', mu', var')."""
    mu, var, Nk, A, B = _f64(mu), _f64(var), _f64(Nk), _f64(A), _f64(B)
    K, D = mu.shape
    w2, mu2, var2 = np.zeros(K), np.zeros((K, D)), np.zeros((K, D))
    _load().oracle_mstep(int(N), D, K, _p(mu), _p(var), _p(Nk), _p(A), _p(B), float(var_floor),
                         _p(w2), _p(mu2), _p(var2))
    return w2, mu2, var2


def em_step(X, w, mu, var, var_floor=1e-6):
    """One EM step.  Returns (w', mu', var', LL(theta_in), N_k)."""
    X, w, mu, var, N, D, K = _shapes(X, w, mu, var)
    w2, mu2, var2, Nk = np.zeros(K), np.zeros((K, D)), np.zeros((K, D)), np.zeros(K)
    ll = ctypes.c_double(0.0)
    _check(_load().oracle_em_step(N, D, K, _p(X), _p(w), _p(mu), _p(var), float(var_floor),
                                  _p(w2), _p(mu2), _p(var2), ctypes.byref(ll), _p(Nk)), "em_step")
    return w2, mu2, var2, ll.value, Nk


def loglik(X, w, mu, var):
    """LL(theta) = sum_n log sum_k pi_k N(x_n | mu_k, diag var_k)."""
    X, w, mu, var, N, D, K = _shapes(X, w, mu, var)
    ll = ctypes.c_double(0.0)
    _check(_load().oracle_loglik(N, D, K, _p(X), _p(w), _p(mu), _p(var), ctypes.byref(ll)),
           "loglik")
    return ll.value


def responsibilities(X, w, mu, var):
    """Full N x K responsibility matrix and per-row LSE (small N only)."""
    X, w, mu, var, N, D, K = _shapes(X, w, mu, var)
    R = np.zeros((N, K))
    lse = np.zeros(N)
    _check(_load().oracle_responsibilities(N, D, K, _p(X), _p(w), _p(mu), _p(var), _p(R),
                                           _p(lse)), "responsibilities")
    return R, lse


def assign_topm(X, w, mu, var, m):
    """Top-m components per point by responsibility (ties -> lower index)."""
    X, w, mu, var, N, D, K = _shapes(X, w, mu, var)
    idx = np.zeros((N, m), dtype=np.int32)
    resp = np.zeros((N, m))
    _check(_load().oracle_assign_topm(N, D, K, _p(X), _p(w), _p(mu), _p(var), int(m), _p(idx),
                                      _p(resp)), "assign_topm")
    return idx, resp


def init(X, rows, K, var_mode, var_floor=1e-6):
    """Initial (w, mu, var): means = X[rows], w = 1/K, var = 1 or data variance."""
    X = _f64(X)
    N, D = X.shape
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    assert rows.shape == (K,)
    w, mu, var = np.zeros(K), np.zeros((K, D)), np.zeros((K, D))
    _check(_load().oracle_init(N, D, K, _p(X), _p(rows), int(var_mode), float(var_floor), _p(w),
                               _p(mu), _p(var)), "init")
    return w, mu, var


def init_seeded(X, seed, K, var_mode, var_floor=1e-6):
    """init() at the K rows the library's gmm_init picks from `seed`
    (SplitMix64-driven Floyd sampling, oracle/sampling.py)."""
    from .sampling import floyd_rows

    return init(X, floyd_rows(len(X), K, seed), K, var_mode, var_floor)


def fit(X, w, mu, var, iters, var_floor=1e-6):
    """iters EM steps; returns (w, mu, var, ll_history) with ll[t] = LL(theta_t)."""
    X, w, mu, var, N, D, K = _shapes(X, w, mu, var)
    w, mu, var = w.copy(), mu.copy(), var.copy()
    ll = np.zeros(iters)
    _check(_load().oracle_fit(N, D, K, _p(X), int(iters), float(var_floor), _p(w), _p(mu),
                              _p(var), _p(ll)), "fit")
    return w, mu, var, ll
