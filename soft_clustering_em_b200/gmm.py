"""Thin Python binding of the C ABI in include/gmm.h (argument marshalling only).

Every entry point keeps its C name.  Arrays are torch CUDA tensors; the binding
passes their device pointers and the current CUDA stream to the library and
does no arithmetic of its own.  The library must be built
(``python -m soft_clustering_em_b200.build``); if it is missing every call
raises -- there is no fallback implementation.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libscem_gmm.so")

GMM_OK, GMM_ERR_INVALID_ARG, GMM_ERR_UNSUPPORTED, GMM_ERR_CUDA = 0, 1, 2, 3
GMM_ERR_NUMERIC, GMM_ERR_TIMEOUT, GMM_ERR_WORKSPACE = 4, 5, 6
GMM_F32, GMM_BF16 = 0, 1
GMM_INIT_VAR_ONE, GMM_INIT_VAR_DATA = 0, 1
GMM_DEVFLAG_NONFINITE_X, GMM_DEVFLAG_BAD_PARAMS, GMM_DEVFLAG_WAIT_TIMEOUT = 0x1, 0x2, 0x4
GMM_DEVFLAG_X_RANGE, GMM_DEVFLAG_BAD_INDEX = 0x8, 0x10

EXPORTS = ("gmm_workspace_size", "gmm_plan", "gmm_init", "gmm_init_rows", "gmm_em_step",
           "gmm_em_step_hard", "gmm_em_step_spherical", "gmm_kmeans_step", "gmm_em_step_noalloc",
           "gmm_host_staging_size", "gmm_em_step_host",
           "gmm_estep_stats", "gmm_mstep", "gmm_fit", "gmm_loglik",
           "gmm_assign_topm", "gmm_ivf_workspace_size", "gmm_ivf_build", "gmm_device_status",
           "gmm_trace_fused", "gmm_set_wait_budget", "gmm_launch_count", "gmm_status_string")


class gmm_problem(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int64), ("D", ctypes.c_int32), ("K", ctypes.c_int32),
                ("xdtype", ctypes.c_int32), ("var_floor", ctypes.c_float)]


class gmm_plan_info(ctypes.Structure):
    _fields_ = [("tensor_cores", ctypes.c_int32), ("cluster_ctas", ctypes.c_int32),
                ("groups", ctypes.c_int32), ("fit_one_launch", ctypes.c_int32),
                ("chunk_rows", ctypes.c_int64)]


class GmmError(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


_lib = None


def load_library(path: str = LIB_PATH):
    """Load the CUDA library and declare its signatures (raises if not built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"CUDA library {path} is not built; run "
                           "`python -m soft_clustering_em_b200.build`")
    lib = ctypes.CDLL(path)
    P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    PP = ctypes.POINTER(gmm_problem)
    lib.gmm_workspace_size.argtypes = [PP, ctypes.POINTER(SZ)]
    lib.gmm_plan.argtypes = [PP, ctypes.POINTER(gmm_plan_info)]
    lib.gmm_init.argtypes = [PP, P, ctypes.c_uint64, I32, P, P, P, P, SZ, P]
    lib.gmm_init_rows.argtypes = [PP, P, ctypes.POINTER(I64), I32, P, P, P, P, SZ, P]
    lib.gmm_em_step.argtypes = [PP, P, P, P, P, P, P, SZ, P]
    lib.gmm_em_step_noalloc.argtypes = [PP, P, P, P, P, P, P, P]
    lib.gmm_em_step_hard.argtypes = [PP, P, P, P, P, P, P, P, SZ, P]
    lib.gmm_em_step_spherical.argtypes = [PP, P, P, P, P, P, P, SZ, P]
    lib.gmm_kmeans_step.argtypes = [PP, P, P, P, P, P, SZ, P]
    lib.gmm_host_staging_size.argtypes = [PP, I64, ctypes.POINTER(SZ)]
    lib.gmm_em_step_host.argtypes = [PP, P, I64, P, SZ, P, P, P, P, P, SZ, P, P]
    lib.gmm_estep_stats.argtypes = [PP, P, P, P, P, P, P, SZ, P]
    lib.gmm_mstep.argtypes = [PP, P, I32, P, P, P, P, P]
    lib.gmm_fit.argtypes = [PP, P, I32, P, P, P, P, P, SZ, P]
    lib.gmm_loglik.argtypes = [PP, P, P, P, P, P, P, SZ, P]
    lib.gmm_assign_topm.argtypes = [PP, P, P, P, P, I32, P, P, P, SZ, P]
    lib.gmm_ivf_workspace_size.argtypes = [I64, I32, ctypes.POINTER(SZ)]
    lib.gmm_ivf_build.argtypes = [I64, I32, I32, P, P, ctypes.c_float, P, P, I64, P, SZ, P]
    lib.gmm_device_status.argtypes = [P, SZ, P, ctypes.POINTER(ctypes.c_uint32), I32]
    lib.gmm_trace_fused.argtypes = [P, P]
    lib.gmm_set_wait_budget.argtypes = [ctypes.c_uint64]
    lib.gmm_launch_count.argtypes = [ctypes.POINTER(ctypes.c_uint64)]
    lib.gmm_status_string.argtypes = [ctypes.c_int]
    lib.gmm_status_string.restype = ctypes.c_char_p
    for name in EXPORTS[:-1]:
        getattr(lib, name).restype = ctypes.c_int
    _lib = lib
    return lib


def status_string(s: int) -> str:
    return load_library().gmm_status_string(int(s)).decode()


def _check(rc, what):
    if rc != GMM_OK:
        raise GmmError(rc, what)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def xdtype_of(X) -> int:
    if X.dtype == torch.float32:
        return GMM_F32
    if X.dtype == torch.bfloat16:
        return GMM_BF16
    raise TypeError(f"X must be float32 or bfloat16, got {X.dtype}")


def problem(N, D, K, xdtype=GMM_F32, var_floor=1e-6) -> gmm_problem:
    return gmm_problem(int(N), int(D), int(K), int(xdtype), float(var_floor))


def problem_for(X, K, var_floor=1e-6) -> gmm_problem:
    N, D = X.shape
    return problem(N, D, K, xdtype_of(X), var_floor)


def gmm_workspace_size(p: gmm_problem) -> int:
    n = ctypes.c_size_t(0)
    _check(load_library().gmm_workspace_size(ctypes.byref(p), ctypes.byref(n)),
           "gmm_workspace_size")
    return int(n.value)


def gmm_plan(p: gmm_problem) -> dict:
    """How the library runs problem p on the current device."""
    info = gmm_plan_info()
    _check(load_library().gmm_plan(ctypes.byref(p), ctypes.byref(info)), "gmm_plan")
    return {f: int(getattr(info, f)) for f, _ in gmm_plan_info._fields_}


def workspace(p: gmm_problem, device=None) -> torch.Tensor:
    """A zero-filled device workspace for problem p (caller-owned, reusable)."""
    return torch.zeros(gmm_workspace_size(p), dtype=torch.uint8, device=device or "cuda")


def _ws(p, ws, device):
    return workspace(p, device) if ws is None else ws


def _init_out(X, K):
    w = torch.empty(K, dtype=torch.float32, device=X.device)
    mu = torch.empty(K, X.shape[1], dtype=torch.float32, device=X.device)
    return w, mu, torch.empty_like(mu)


def gmm_init(X, seed, K, init_var=GMM_INIT_VAR_DATA, var_floor=1e-6, ws=None, stream=None):
    """Initial (w, mu, var): means at K distinct rows of X chosen from `seed`."""
    p = problem_for(X, K, var_floor)
    ws = _ws(p, ws, X.device)
    w, mu, var = _init_out(X, K)
    _check(load_library().gmm_init(ctypes.byref(p), _ptr(X), int(seed) & ((1 << 64) - 1),
                                   int(init_var), _ptr(w), _ptr(mu), _ptr(var), _ptr(ws),
                                   ws.numel(), _stream(stream)), "gmm_init")
    return w, mu, var


def gmm_init_rows(X, rows, K, init_var=GMM_INIT_VAR_DATA, var_floor=1e-6, ws=None, stream=None):
    """Initial (w, mu, var) from the K chosen rows of X (host int64 indices)."""
    p = problem_for(X, K, var_floor)
    ws = _ws(p, ws, X.device)
    rows = (ctypes.c_int64 * K)(*[int(r) for r in rows])
    w, mu, var = _init_out(X, K)
    _check(load_library().gmm_init_rows(ctypes.byref(p), _ptr(X), rows, int(init_var), _ptr(w),
                                        _ptr(mu), _ptr(var), _ptr(ws), ws.numel(),
                                        _stream(stream)), "gmm_init_rows")
    return w, mu, var


def gmm_em_step(X, w, mu, var, loglik=None, var_floor=1e-6, ws=None, stream=None):
    """One fused EM iteration in place; loglik (1 double, device) gets LL of the input."""
    p = problem_for(X, w.numel(), var_floor)
    ws = _ws(p, ws, X.device)
    _check(load_library().gmm_em_step(ctypes.byref(p), _ptr(X), _ptr(w), _ptr(mu), _ptr(var),
                                      _ptr(loglik), _ptr(ws), ws.numel(), _stream(stream)),
           "gmm_em_step")


def gmm_em_step_hard(X, w, mu, var, labels=None, loglik=None, var_floor=1e-6, ws=None,
                     stream=None):
    """One classification-EM step in place; labels (N int32) and loglik optional outputs."""
    p = problem_for(X, w.numel(), var_floor)
    ws = _ws(p, ws, X.device)
    _check(load_library().gmm_em_step_hard(ctypes.byref(p), _ptr(X), _ptr(w), _ptr(mu),
                                           _ptr(var), _ptr(labels), _ptr(loglik), _ptr(ws),
                                           ws.numel(), _stream(stream)), "gmm_em_step_hard")


def gmm_em_step_spherical(X, w, mu, s2, loglik=None, var_floor=1e-6, ws=None, stream=None):
    """One soft EM step in place with covariances s2_k * I (s2: K floats)."""
    p = problem_for(X, w.numel(), var_floor)
    ws = _ws(p, ws, X.device)
    _check(load_library().gmm_em_step_spherical(ctypes.byref(p), _ptr(X), _ptr(w), _ptr(mu),
                                                _ptr(s2), _ptr(loglik), _ptr(ws), ws.numel(),
                                                _stream(stream)), "gmm_em_step_spherical")


def gmm_kmeans_step(X, centers, labels=None, inertia=None, ws=None, stream=None):
    """One Lloyd step in place on centers (K x D); optional labels (N int32) and inertia."""
    p = problem_for(X, centers.shape[0])
    ws = _ws(p, ws, X.device)
    _check(load_library().gmm_kmeans_step(ctypes.byref(p), _ptr(X), _ptr(centers), _ptr(labels),
                                          _ptr(inertia), _ptr(ws), ws.numel(), _stream(stream)),
           "gmm_kmeans_step")


_copy_streams = {}


def copy_stream_for(device):
    """A side stream per device for gmm_em_step_host's host-to-device copies."""
    key = torch.device(device).index if torch.device(device).index is not None else \
        torch.cuda.current_device()
    if key not in _copy_streams:
        _copy_streams[key] = torch.cuda.Stream(device=key)
    return _copy_streams[key]


def gmm_host_staging_size(p: gmm_problem, chunk_rows) -> int:
    n = ctypes.c_size_t(0)
    _check(load_library().gmm_host_staging_size(ctypes.byref(p), int(chunk_rows),
                                                ctypes.byref(n)), "gmm_host_staging_size")
    return int(n.value)


def gmm_em_step_host(X_host, w, mu, var, loglik=None, chunk_rows=1 << 18, var_floor=1e-6,
                     staging=None, ws=None, stream=None, copy_stream=None):
    """One EM iteration in place with X in host memory (pinned for overlap).

    X_host: contiguous CPU tensor, float32 or bfloat16, N x D.  The rows are
    copied chunk_rows at a time through device staging on copy_stream (default:
    a side stream of the parameters' device) while the E-step runs on stream.
    """
    if X_host.is_cuda or not X_host.is_contiguous():
        raise ValueError("X_host must be a contiguous host tensor")
    p = problem_for(X_host, w.numel(), var_floor)
    ws = _ws(p, ws, w.device)
    if staging is None:
        staging = torch.empty(gmm_host_staging_size(p, chunk_rows), dtype=torch.uint8,
                              device=w.device)
    cs = copy_stream_for(w.device) if copy_stream is None else copy_stream
    _check(load_library().gmm_em_step_host(ctypes.byref(p), ctypes.c_void_p(X_host.data_ptr()),
                                           int(chunk_rows), _ptr(staging), staging.numel(),
                                           _ptr(w), _ptr(mu), _ptr(var), _ptr(loglik), _ptr(ws),
                                           ws.numel(), _stream(stream), _stream(cs)),
           "gmm_em_step_host")


def stats_size(K, D) -> int:
    """Doubles in a statistics buffer: [N_k (K) | A (K x D) | B (K x D) | LL]."""
    return int(K) * (2 * int(D) + 1) + 1


def gmm_estep_stats(X, w, mu, var, stats=None, var_floor=1e-6, ws=None, stream=None):
    """E-step statistics of the rows of X (fp64 device tensor [N_k | A | B | LL])."""
    p = problem_for(X, w.numel(), var_floor)
    ws = _ws(p, ws, X.device)
    if stats is None:
        stats = torch.empty(stats_size(w.numel(), X.shape[1]), dtype=torch.float64,
                            device=X.device)
    _check(load_library().gmm_estep_stats(ctypes.byref(p), _ptr(X), _ptr(w), _ptr(mu), _ptr(var),
                                          _ptr(stats), _ptr(ws), ws.numel(), _stream(stream)),
           "gmm_estep_stats")
    return stats


def gmm_mstep(stats, N_total, w, mu, var, loglik=None, var_floor=1e-6, xdtype=GMM_F32,
              stream=None):
    """M-step in place from the statistics of row shards holding N_total points.

    stats: fp64 device tensor of shape (S,) or (nshards, S), S = stats_size(K, D);
    the shards are summed in order inside the library."""
    K, D = mu.shape
    nshards = 1 if stats.dim() == 1 else stats.shape[0]
    p = problem(N_total, D, K, xdtype, var_floor)
    _check(load_library().gmm_mstep(ctypes.byref(p), _ptr(stats.contiguous()), int(nshards),
                                    _ptr(w), _ptr(mu), _ptr(var), _ptr(loglik), _stream(stream)),
           "gmm_mstep")


def gmm_em_step_noalloc(X, w, mu, var, loglik=None, dev_flags=None, var_floor=1e-6,
                        stream=None):
    """gmm_em_step on the library's built-in scratch: no workspace, no device allocation.

    For callers that may not obtain device memory (see include/gmm.h).  dev_flags
    (1 int32 device tensor, optional) receives the call's device status bits.
    """
    p = problem_for(X, w.numel(), var_floor)
    _check(load_library().gmm_em_step_noalloc(ctypes.byref(p), _ptr(X), _ptr(w), _ptr(mu),
                                              _ptr(var), _ptr(loglik), _ptr(dev_flags),
                                              _stream(stream)), "gmm_em_step_noalloc")


def gmm_fit(X, w, mu, var, iters, var_floor=1e-6, ws=None, stream=None):
    """iters EM iterations in place; returns the device LL history (iters doubles)."""
    p = problem_for(X, w.numel(), var_floor)
    ws = _ws(p, ws, X.device)
    ll = torch.zeros(max(int(iters), 1), dtype=torch.float64, device=X.device)
    _check(load_library().gmm_fit(ctypes.byref(p), _ptr(X), int(iters), _ptr(w), _ptr(mu),
                                  _ptr(var), _ptr(ll), _ptr(ws), ws.numel(), _stream(stream)),
           "gmm_fit")
    return ll[:iters]


def gmm_loglik(X, w, mu, var, var_floor=1e-6, ws=None, stream=None):
    """LL of the given parameters as a 1-element device double tensor."""
    p = problem_for(X, w.numel(), var_floor)
    ws = _ws(p, ws, X.device)
    ll = torch.zeros(1, dtype=torch.float64, device=X.device)
    _check(load_library().gmm_loglik(ctypes.byref(p), _ptr(X), _ptr(w), _ptr(mu), _ptr(var),
                                     _ptr(ll), _ptr(ws), ws.numel(), _stream(stream)),
           "gmm_loglik")
    return ll


def gmm_assign_topm(X, w, mu, var, m, var_floor=1e-6, ws=None, stream=None):
    """(idx N x m int32, resp N x m float32): the m most responsible components per point."""
    p = problem_for(X, w.numel(), var_floor)
    ws = _ws(p, ws, X.device)
    N = X.shape[0]
    idx = torch.empty(N, int(m), dtype=torch.int32, device=X.device)
    resp = torch.empty(N, int(m), dtype=torch.float32, device=X.device)
    _check(load_library().gmm_assign_topm(ctypes.byref(p), _ptr(X), _ptr(w), _ptr(mu), _ptr(var),
                                          int(m), _ptr(idx), _ptr(resp), _ptr(ws), ws.numel(),
                                          _stream(stream)), "gmm_assign_topm")
    return idx, resp


def gmm_ivf_workspace_size(N, K) -> int:
    n = ctypes.c_size_t(0)
    _check(load_library().gmm_ivf_workspace_size(int(N), int(K), ctypes.byref(n)),
           "gmm_ivf_workspace_size")
    return int(n.value)


def gmm_ivf_build(idx, resp, K, tau, ws=None, stream=None):
    """(offsets (K+1) int64, ids (N*m) int64): IVF lists from a top-m assignment.

    idx (N x m int32) and resp (N x m float32) as gmm_assign_topm returns them.
    List k is ids[offsets[k]:offsets[k+1]]; entries past offsets[K] are unused.
    ws: a zeroed uint8 device tensor of gmm_ivf_workspace_size(N, K) bytes
    (allocated here when None); its first word is the device status word.
    """
    if idx.dtype != torch.int32 or resp.dtype != torch.float32:
        raise TypeError("idx must be int32 and resp float32")
    if idx.dim() != 2 or resp.shape != idx.shape or not (idx.is_contiguous()
                                                       and resp.is_contiguous()):
        raise ValueError("idx and resp must be contiguous N x m tensors of the same shape")
    N, m = idx.shape
    if ws is None:
        ws = torch.zeros(gmm_ivf_workspace_size(N, K), dtype=torch.uint8, device=idx.device)
    offsets = torch.empty(int(K) + 1, dtype=torch.int64, device=idx.device)
    ids = torch.empty(N * m, dtype=torch.int64, device=idx.device)
    _check(load_library().gmm_ivf_build(int(N), int(K), int(m), _ptr(idx), _ptr(resp),
                                        float(tau), _ptr(offsets), _ptr(ids), N * m, _ptr(ws),
                                        ws.numel(), _stream(stream)), "gmm_ivf_build")
    return offsets, ids


def gmm_device_status(ws, clear=True, stream=None):
    """(status, flags): waits for the stream and reads the workspace's device status word."""
    f = ctypes.c_uint32(0)
    rc = load_library().gmm_device_status(_ptr(ws), ws.numel(), _stream(stream), ctypes.byref(f),
                                          int(bool(clear)))
    return rc, int(f.value)


def gmm_trace_fused(start=None, stop=None):
    """Record torch.cuda.Event start/stop around every later fused-kernel launch (None: off)."""
    if start is None:
        _check(load_library().gmm_trace_fused(None, None), "gmm_trace_fused")
        return
    for e in (start, stop):
        if not e.cuda_event:
            e.record()  # torch creates the CUDA event lazily, on its first record
    _check(load_library().gmm_trace_fused(ctypes.c_void_p(start.cuda_event),
                                          ctypes.c_void_p(stop.cuda_event)), "gmm_trace_fused")


def gmm_set_wait_budget(ns=0):
    """Budget of every device-side wait in nanoseconds (0: the default, one second)."""
    _check(load_library().gmm_set_wait_budget(int(ns)), "gmm_set_wait_budget")


def gmm_launch_count() -> int:
    """Kernels the library has enqueued in this process so far."""
    c = ctypes.c_uint64(0)
    _check(load_library().gmm_launch_count(ctypes.byref(c)), "gmm_launch_count")
    return int(c.value)
