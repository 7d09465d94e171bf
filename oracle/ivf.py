"""CPU oracle for the IVF inverted lists built from a top-m assignment
(TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU
baseline may use it; the CUDA product path never does).

"Flash-GMM: A Memory-Efficient Kernel for Scalable Soft Clustering", abstract:
the mixture serves as the coarse quantizer of an IVF index, and its
responsibilities put a vector that lies near a cluster border into more than
one cluster's list.  The pages give no rule for that choice.  The reading taken
here, the plainest one:

    point n is filed in the list of its most responsible component always, and
    in the list of its rank-j component (j = 2..m) when that component's
    responsibility is at least tau.

The decision is taken on the float32 responsibilities that the top-m
assignment returns, against float32(tau).  The lists come back in
compressed-row form: list k is ids[offsets[k]:offsets[k+1]], with the point
indices ascending inside each list.

This is the definition written out with numpy primitives (a boolean mask, a
lexicographic sort and a bincount); nothing is blocked or fused.
"""
import numpy as np


def ivf_lists(idx, resp, K, tau):
    """(offsets (K+1,) int64, ids (total,) int64) for a valid top-m assignment.

    idx: N x m component indices in [0, K), distinct within a row, ordered by
    responsibility (rank 1 first); resp: the matching responsibilities.
    """
    idx = np.asarray(idx)
    resp = np.asarray(resp, dtype=np.float32)
    N, m = idx.shape
    assert resp.shape == (N, m) and idx.min(initial=0) >= 0 and idx.max(initial=0) < K
    rank_one = np.zeros((N, m), dtype=bool)
    rank_one[:, 0] = True
    keep = rank_one | (resp >= np.float32(tau))
    points = np.broadcast_to(np.arange(N, dtype=np.int64)[:, None], (N, m))[keep]
    lists = idx[keep].astype(np.int64)
    order = np.lexsort((points, lists))  # by list, then by point
    offsets = np.zeros(K + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(np.bincount(lists, minlength=K))
    return offsets, points[order]
