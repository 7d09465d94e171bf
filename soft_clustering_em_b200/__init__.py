"""Fused EM for diagonal-covariance Gaussian mixtures on B200 (sm_100a).

``soft_clustering_em_b200.gmm`` is the Python binding of the C ABI in
include/gmm.h; ``soft_clustering_em_b200.sharded`` runs row-sharded EM over
torch.distributed (one process per GPU); ``soft_clustering_em_b200.synth``
holds the seeded synthetic workloads.  The CUDA library is loaded on first use
and every call raises if it is not built.
"""
