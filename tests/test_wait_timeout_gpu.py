"""The bounded device-side waits give up, report GMM_ERR_TIMEOUT and leave the
context usable.

Every spin of the tensor-core EM kernel is an mbarrier wait with a time budget.
These tests make such waits run out in the two allowed ways -- a barrier that
nothing completes, and a budget shorter than the work being waited for -- and
check that the status comes back and that the device still works afterwards.
"""
import ctypes
import os
import subprocess

import numpy as np
import pytest

import oracle
from oracle import compare
from soft_clustering_em_b200 import synth

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


@pytest.fixture(scope="module")
def probe():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    src = os.path.join(HERE, "csrc", "wait_probe.cu")
    so = os.path.join(HERE, "csrc", "_wait_probe.so")
    if not os.path.exists(so) or os.path.getmtime(so) < os.path.getmtime(src):
        subprocess.check_call([
            os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc"), "-gencode",
            "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-Xcompiler", "-fPIC",
            "-shared", "-I", os.path.join(ROOT, "soft_clustering_em_b200", "csrc"), "-I",
            os.path.join(ROOT, "include"), "-o", so, src])
    lib = ctypes.CDLL(so)
    P = ctypes.c_void_p
    lib.wait_probe_run.argtypes = [ctypes.c_ulonglong, ctypes.c_int, P, P, P]
    return lib


def _probe(probe, budget_ns, arrive):
    import torch

    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.zeros(2, dtype=torch.int64, device="cuda")
    rc = probe.wait_probe_run(budget_ns, arrive, status.data_ptr(), out.data_ptr(),
                              torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    return int(status.item()), int(out[0].item()), int(out[1].item())


def test_wait_on_a_barrier_nothing_completes_gives_up(probe):
    from soft_clustering_em_b200 import gmm as G

    status, done, ns = _probe(probe, 1_000_000, arrive=0)  # 1 ms budget
    assert done == 0 and status == G.GMM_DEVFLAG_WAIT_TIMEOUT
    assert 1_000_000 <= ns < 200_000_000, ns
    # the same wait with an arrival completes and raises nothing
    status, done, ns = _probe(probe, 1_000_000, arrive=1)
    assert done == 1 and status == 0


@pytest.fixture(scope="module")
def G():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from soft_clustering_em_b200 import build
    from soft_clustering_em_b200 import gmm

    build.build()
    gmm.load_library()
    return gmm


@pytest.mark.parametrize("name,N,K", [("uint8img", 20_011, 256), ("bf16stream", 30_001, 1024)])
def test_step_with_a_short_budget_times_out_and_the_next_step_is_exact(G, name, N, K):
    import torch

    wl = synth.WORKLOADS[name]
    X, _ = synth.make_data(wl, N)
    X64 = synth.x_as_f64(wl, X)
    Xd = (torch.from_numpy(X.view(np.int16)).view(torch.bfloat16) if wl.dtype == "bf16"
          else torch.from_numpy(X)).cuda()
    ws = G.workspace(G.problem_for(Xd, K, wl.var_floor))
    w, mu, var = G.gmm_init_rows(Xd, synth.init_rows(N, K, wl.init_seed), K, G.GMM_INIT_VAR_DATA,
                            wl.var_floor, ws=ws)
    theta = (w.clone(), mu.clone(), var.clone())
    try:
        G.gmm_set_wait_budget(1)  # 1 ns: the first wait that has to wait at all gives up
        G.gmm_em_step(Xd, w, mu, var, None, wl.var_floor, ws=ws)
        rc, flags = G.gmm_device_status(ws)
    finally:
        G.gmm_set_wait_budget(0)
    assert rc == G.GMM_ERR_TIMEOUT and flags & G.GMM_DEVFLAG_WAIT_TIMEOUT, (rc, flags)
    # the flag was cleared by the read; the context still runs a correct step
    for t, t0 in zip((w, mu, var), theta):
        t.copy_(t0)
    ll = torch.zeros(1, dtype=torch.float64, device="cuda")
    G.gmm_em_step(Xd, w, mu, var, ll, wl.var_floor, ws=ws)
    rc, flags = G.gmm_device_status(ws)
    assert rc == 0 and flags == 0
    th = tuple(t.double().cpu().numpy() for t in theta)
    w2, mu2, var2, ll_ref, Nk = oracle.em_step(X64, *th, var_floor=wl.var_floor)
    got = tuple(t.double().cpu().numpy() for t in (w, mu, var)) + (ll.item(),)
    rep = compare.compare_step((w2, mu2, var2, ll_ref), got, Nk)
    assert rep["ok"], rep
