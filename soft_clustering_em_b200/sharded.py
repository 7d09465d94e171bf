"""Row-sharded EM across processes (one per GPU), over torch.distributed.

EM over the rows of X splits exactly: given the parameters, every row's
responsibilities are independent, and the M-step needs only the sums of the
per-row statistics ("Flash-GMM: A Memory-Efficient Kernel for Scalable Soft
Clustering", review page, section 3: statistics computed per data tile and
accumulated globally).  Each rank holds a block of rows; one EM iteration is

    local statistics (gmm_estep_stats)  ->  all-gather of the K(2D+1)+1
    fp64 statistics of every rank  ->  M-step on every rank (gmm_mstep, which
    sums the gathered shards in rank order inside the library).

Every rank therefore ends the iteration with bit-identical parameters, and the
result does not depend on how the collective schedules its transfers.  The
exchange is an all-gather rather than an all-reduce for exactly that reason; it
moves world_size x K(2D+1)+1 doubles per iteration (1.6 MB per rank for K=1024,
D=96).
"""
import torch
import torch.distributed as dist


def gather_stats(stats: torch.Tensor, group=None) -> torch.Tensor:
    """All-gather each rank's statistics into a (world_size, S) tensor, rank-ordered."""
    world = dist.get_world_size(group)
    out = torch.empty(world * stats.numel(), dtype=stats.dtype, device=stats.device)
    dist.all_gather_into_tensor(out, stats.contiguous().view(-1), group=group)
    return out.view(world, stats.numel())


def broadcast_params(w, mu, var, src=0, group=None):
    """Make every rank start from rank `src`'s parameters."""
    for t in (w, mu, var):
        dist.broadcast(t, src=src, group=group)


def sharded_em_step(estep_stats, mstep, N_total, group=None):
    """One row-sharded EM iteration.

    estep_stats() -> this rank's statistics tensor (S,); mstep(gathered, N_total)
    applies the M-step from the (world_size, S) rank-ordered statistics.  Both
    are callables so the same orchestration serves the CUDA library and, in
    tests, the CPU oracle.  Returns the gathered statistics.
    """
    local = estep_stats()
    gathered = gather_stats(local, group)
    mstep(gathered, N_total)
    return gathered


def shard_rows(N_total: int, world: int, rank: int):
    """[start, stop) of this rank's contiguous block of rows (sizes differ by at most 1)."""
    return (N_total * rank) // world, (N_total * (rank + 1)) // world
