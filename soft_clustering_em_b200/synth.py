"""Seeded synthetic workloads for the EM step (inputs only, no EM arithmetic).

Five mixture workloads, each drawn from numpy's PCG64 with data seed
1000*c + 1 and init seed 1000*c + 2 for workload number c:

  1. gauss8     N=1e4,  D=16,  K=8     fp32  means U[-10,10], std 1, equal weights
  2. uint8img   N=1e6,  D=128, K=256   fp32  means U[0,255], std U[5,40],
                                             Dirichlet(1) weights, clipped to
                                             [0,255] and rounded to integers
  3. sphere768  N=1e6,  D=768, K=1024  fp32  means on the unit sphere, std
                                             U[0.01,0.05], weights ~ (k+1)^-1.1,
                                             samples L2-normalised
  4. gauss4096  N=1e7,  D=96,  K=4096  fp32  means N(0,I), std U[0.1,0.5],
                                             equal weights
  5. bf16stream N=1e8,  D=32,  K=1024  bf16  means U[-1,1], std U[0.02,0.2],
                                             Dirichlet(0.5) weights

Labels z_n ~ Categorical(weights); x_n = mu_{z_n} + std_{z_n} * eps_n with
eps_n ~ N(0, I).  ``make_data(wl, N=n)`` returns the first n rows of the same
stream (same per-component parameters), which gives down-scaled cases that the
oracle finishes in seconds.

The initial means are K distinct data rows drawn with the init seed
(``init_rows``); the EM method draws no other random numbers.
"""
from dataclasses import dataclass

import numpy as np


@dataclass(frozen=True)
class Workload:
    name: str
    number: int
    N: int
    D: int
    K: int
    dtype: str  # "f32" or "bf16": storage type of X
    iters: int
    var_init: str  # "one" or "data"
    topm: int  # 0: no assignment pass
    var_floor: float = 1e-6

    @property
    def data_seed(self) -> int:
        return 1000 * self.number + 1

    @property
    def init_seed(self) -> int:
        return 1000 * self.number + 2


WORKLOADS = {
    "gauss8": Workload("gauss8", 1, 10_000, 16, 8, "f32", 10, "one", 0),
    "uint8img": Workload("uint8img", 2, 1_000_000, 128, 256, "f32", 20, "data", 0),
    "sphere768": Workload("sphere768", 3, 1_000_000, 768, 1024, "f32", 10, "data", 2),
    "gauss4096": Workload("gauss4096", 4, 10_000_000, 96, 4096, "f32", 5, "data", 0),
    "bf16stream": Workload("bf16stream", 5, 100_000_000, 32, 1024, "bf16", 3, "data", 2),
}


def true_params(wl: Workload):
    """Generating (weights, means, stds) of workload ``wl`` (float64)."""
    rng = np.random.Generator(np.random.PCG64(wl.data_seed))
    K, D = wl.K, wl.D
    if wl.number == 1:
        mu = rng.uniform(-10.0, 10.0, size=(K, D))
        sd = np.ones((K, D))
        pi = np.full(K, 1.0 / K)
    elif wl.number == 2:
        mu = rng.uniform(0.0, 255.0, size=(K, D))
        sd = rng.uniform(5.0, 40.0, size=(K, D))
        pi = rng.dirichlet(np.ones(K))
    elif wl.number == 3:
        g = rng.standard_normal(size=(K, D))
        mu = g / np.linalg.norm(g, axis=1, keepdims=True)
        sd = rng.uniform(0.01, 0.05, size=(K, D))
        pi = (np.arange(K) + 1.0) ** -1.1
        pi = pi / pi.sum()
    elif wl.number == 4:
        mu = rng.standard_normal(size=(K, D))
        sd = rng.uniform(0.1, 0.5, size=(K, D))
        pi = np.full(K, 1.0 / K)
    elif wl.number == 5:
        mu = rng.uniform(-1.0, 1.0, size=(K, D))
        sd = rng.uniform(0.02, 0.2, size=(K, D))
        pi = rng.dirichlet(np.full(K, 0.5))
    else:
        raise ValueError(wl)
    return pi, mu, sd, rng


def _finish(wl: Workload, x: np.ndarray) -> np.ndarray:
    if wl.number == 2:
        x = np.rint(np.clip(x, 0.0, 255.0))
    elif wl.number == 3:
        x = x / np.linalg.norm(x, axis=1, keepdims=True)
    return x


def bf16_round(x32: np.ndarray) -> np.ndarray:
    """Round fp32 to the nearest bf16 (ties to even); returns the bf16 bits as uint16."""
    u = np.ascontiguousarray(x32, dtype=np.float32).view(np.uint32)
    lsb = (u >> 16) & 1
    return ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)


def bf16_to_f32(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32)


def make_data(wl: Workload, N: int = None, chunk: int = 1 << 16, start: int = 0):
    """Sample rows [start, start + N) of workload ``wl``'s data stream.

    Returns (X, labels).  X is float32, or uint16 bf16 bit patterns when
    wl.dtype == "bf16".  The stream is cut into chunks of ``chunk`` rows, each
    drawn from its own seeded generator, so any block of rows is the same
    whatever else is generated: make_data(wl, n) is a prefix of
    make_data(wl, N) for n <= N, and make_data(wl, n, start=s) equals rows
    s .. s+n-1 of a longer draw (one block of rows per rank).
    """
    N = wl.N if N is None else int(N)
    pi, mu, sd, rng = true_params(wl)
    out_dtype = np.uint16 if wl.dtype == "bf16" else np.float32
    X = np.empty((N, wl.D), dtype=out_dtype)
    labels = np.empty(N, dtype=np.int32)
    cdf = np.cumsum(pi)
    cdf[-1] = 1.0
    stop = start + N
    for ci in range(start // chunk, (stop + chunk - 1) // chunk):
        c0 = ci * chunk
        crng = np.random.Generator(np.random.PCG64([wl.data_seed, ci]))
        z = np.searchsorted(cdf, crng.random(chunk), side="right").astype(np.int32)
        z = np.minimum(z, wl.K - 1)
        lo, hi = max(start, c0), min(stop, c0 + chunk)
        # draw the whole chunk so its rows do not depend on the block requested
        eps = crng.standard_normal(size=(hi - c0, wl.D))[lo - c0:]
        zz = z[lo - c0:hi - c0]
        x = _finish(wl, mu[zz] + sd[zz] * eps).astype(np.float32)
        X[lo - start:hi - start] = bf16_round(x) if wl.dtype == "bf16" else x
        labels[lo - start:hi - start] = zz
    return X, labels


def x_as_f64(wl: Workload, X: np.ndarray) -> np.ndarray:
    """The exact values of X in float64 (bf16 bit patterns decoded)."""
    if wl.dtype == "bf16":
        return bf16_to_f32(X).astype(np.float64)
    return X.astype(np.float64)


def init_rows(N: int, K: int, seed: int) -> np.ndarray:
    """K distinct row indices in [0, N), drawn uniformly with PCG64(seed)."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return np.sort(rng.choice(N, size=K, replace=False)).astype(np.int64)


def topm_inputs(N: int, K: int, m: int, seed: int, ties_at: float = None):
    """A seeded stand-in for a top-m assignment: (idx N x m int32, resp N x m float32).

    Each row holds m distinct component indices.  The first is skewed towards
    low indices (u^2 scaling), so list sizes are uneven like those of a mixture
    with unequal weights.  The others step forward from it modulo K.  resp is
    descending along a row and sums to at most 1.  With ``ties_at`` set, about
    one entry in 16 of ranks 2..m is then overwritten with exactly
    float32(ties_at), which can break that order.
    """
    assert 1 <= m <= K
    rng = np.random.Generator(np.random.PCG64(seed))
    first = np.minimum(K - 1, (K * rng.random(N) ** 2).astype(np.int64))
    idx = np.empty((N, m), dtype=np.int64)
    idx[:, 0] = first
    if m > 1:
        steps = rng.integers(1, (K - 1) // (m - 1) + 1, size=(N, m - 1))
        idx[:, 1:] = (first[:, None] + np.cumsum(steps, axis=1)) % K
    resp = np.empty((N, m), dtype=np.float64)
    resp[:, 0] = rng.uniform(0.3, 1.0, N)
    rest = 1.0 - resp[:, 0]
    for j in range(1, m):
        resp[:, j] = rest * rng.random(N)
        rest = rest - resp[:, j]
    if m > 1:
        resp[:, 1:] = -np.sort(-resp[:, 1:], axis=1)
        resp[:, 1:] = np.minimum(resp[:, 1:], resp[:, :1])
    resp = resp.astype(np.float32)
    if ties_at is not None and m > 1:
        hit = rng.random((N, m - 1)) < 1.0 / 16
        resp[:, 1:][hit] = np.float32(ties_at)
    return idx.astype(np.int32), resp
