"""CPU oracle for the hard-assignment and spherical variants of the mixture EM step
(TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU
baseline may use it; the CUDA product path never does).

The pages present soft GMM clustering as a drop-in replacement for k-means in an
IVF coarse quantizer ("Flash-GMM: A Memory-Efficient Kernel for Scalable Soft
Clustering": abstract; review page, section 3, where k-means is the baseline).
Three neighbours of the diagonal EM step follow from the same E-step/M-step
structure; the pages print none of them, so these are the textbook forms:

  spherical EM   one variance s2_k per component (covariance s2_k * I):
                 l_nk = log pi_k - (D/2) log(2 pi s2_k) - |x_n - mu_k|^2 / (2 s2_k),
                 soft responsibilities, and the M-step variance is the average
                 over dimensions of the per-dimension variance about the new mean,
                 floored: s2_k' = max((1/D) sum_d (B_kd/N_k - delta_kd^2), floor).
  hard EM        (classification EM) the diagonal model, but each point is given
                 wholly to its most probable component (ties to the lower index);
                 the M-step is the diagonal one with 0/1 responsibilities.  Its
                 objective is the classification log-likelihood sum_n max_k l_nk.
  k-means        the hard-EM limit with equal weights and one shared spherical
                 variance: each point to its nearest centre in squared Euclidean
                 distance (ties to the lower index), each centre to the mean of its
                 points.  Objective: the sum of squared distances (inertia).

In all three a component with no mass (N_k <= 1e-12 N; for hard assignments, no
point) keeps its mean and variance, as in the diagonal oracle.  Statistics are
moments about the old means (A = sum r (x - mu), B = sum r (x - mu)^2), so the
new variance never cancels.  Plain numpy in float64, the N x K matrices formed
in full: for the small sizes the tests use.
"""
import numpy as np

EMPTY_FRACTION = 1e-12


def _f64(a):
    return np.asarray(a, dtype=np.float64)


def _lse_rows(L):
    """Row-wise log-sum-exp of an N x K matrix (rows of -inf give -inf)."""
    m = L.max(axis=1)
    safe = np.where(np.isfinite(m), m, 0.0)
    return safe + np.log(np.exp(L - safe[:, None]).sum(axis=1))


def _moments(X, mu, R):
    """N_k, A_kd = sum_n r_nk (x_nd - mu_kd), B_kd = sum_n r_nk (x_nd - mu_kd)^2."""
    Nk = R.sum(axis=0)
    K, D = mu.shape
    A = np.empty((K, D))
    B = np.empty((K, D))
    for k in range(K):
        E = X - mu[k]
        A[k] = R[:, k] @ E
        B[k] = R[:, k] @ (E * E)
    return Nk, A, B


def spherical_logjoint(X, w, mu, s2):
    """l_nk for covariance s2_k * I (pi_k = 0 gives -inf)."""
    X, w, mu, s2 = _f64(X), _f64(w), _f64(mu), _f64(s2)
    D = X.shape[1]
    sq = ((X[:, None, :] - mu[None, :, :]) ** 2).sum(axis=2)
    with np.errstate(divide="ignore"):
        logw = np.log(w)
    return logw[None, :] - 0.5 * D * np.log(2.0 * np.pi * s2)[None, :] - sq / (2.0 * s2[None, :])


def spherical_em_step(X, w, mu, s2, var_floor=1e-6):
    """One soft EM step with spherical covariances.

    Returns (w', mu', s2', LL of the input parameters, N_k)."""
    X, mu, s2 = _f64(X), _f64(mu), _f64(s2)
    N, D = X.shape
    L = spherical_logjoint(X, w, mu, s2)
    lse = _lse_rows(L)
    R = np.exp(L - lse[:, None])
    Nk, A, B = _moments(X, mu, R)
    w2, mu2, s22 = Nk / N, mu.copy(), s2.copy()
    for k in range(len(Nk)):
        if Nk[k] > EMPTY_FRACTION * N:
            delta = A[k] / Nk[k]
            mu2[k] = mu[k] + delta
            s22[k] = max(float(np.mean(B[k] / Nk[k] - delta * delta)), var_floor)
    return w2, mu2, s22, float(lse.sum()), Nk


def diag_logjoint(X, w, mu, var):
    """l_nk for diagonal covariances (pi_k = 0 gives -inf)."""
    X, w, mu, var = _f64(X), _f64(w), _f64(mu), _f64(var)
    q = (((X[:, None, :] - mu[None, :, :]) ** 2) / var[None, :, :]).sum(axis=2)
    logdet = np.log(2.0 * np.pi * var).sum(axis=1)
    with np.errstate(divide="ignore"):
        logw = np.log(w)
    return logw[None, :] - 0.5 * (logdet[None, :] + q)


def hard_em_step(X, w, mu, var, var_floor=1e-6):
    """One classification-EM step of the diagonal model.

    Returns (w', mu', var', classification log-likelihood of the input
    parameters, labels)."""
    X, mu, var = _f64(X), _f64(mu), _f64(var)
    N = X.shape[0]
    L = diag_logjoint(X, w, mu, var)
    z = np.argmax(L, axis=1)  # the first maximum: ties go to the lower index
    R = np.zeros_like(L)
    R[np.arange(N), z] = 1.0
    Nk, A, B = _moments(X, mu, R)
    w2, mu2, var2 = Nk / N, mu.copy(), var.copy()
    for k in range(len(Nk)):
        if Nk[k] > 0:
            delta = A[k] / Nk[k]
            mu2[k] = mu[k] + delta
            var2[k] = np.maximum(B[k] / Nk[k] - delta * delta, var_floor)
    return w2, mu2, var2, float(L[np.arange(N), z].sum()), z


def kmeans_step(X, C):
    """One Lloyd step: (new centres, labels, inertia of the input centres)."""
    X, C = _f64(X), _f64(C)
    d2 = ((X[:, None, :] - C[None, :, :]) ** 2).sum(axis=2)
    z = np.argmin(d2, axis=1)  # the first minimum: ties go to the lower index
    C2 = C.copy()
    for k in range(C.shape[0]):
        members = X[z == k]
        if len(members):
            C2[k] = members.mean(axis=0)
    return C2, z, float(d2[np.arange(X.shape[0]), z].sum())
