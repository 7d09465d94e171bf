"""gmm_em_step_noalloc: the EM step for callers that may not allocate device memory.

Some callers cannot obtain device memory at all -- a plug-in inside an
application that owns the whole device budget, or a loop that must not call
cudaMalloc because it blocks the device.  This entry point runs the same EM
step on a fixed scratch array built into the library.  The test calls it
through the C ABI twice in a row and checks each result against gmm_em_step
on a caller-provided workspace, under the same tolerances as the other parity
tests, and checks that no device memory was taken.  It lives in a file of its
own so that it runs last.
"""
import numpy as np
import pytest

from oracle import compare
from soft_clustering_em_b200 import synth

pytestmark = pytest.mark.gpu


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


def _np(*ts):
    return tuple(t.double().cpu().numpy() for t in ts)


@pytest.mark.parametrize("name,N", [("gauss8", 10_007), ("uint8img", 60_001),
                                    ("bf16stream", 40_003)])
def test_noalloc_matches_workspace_step_twice(G, name, N):
    import torch

    wl = synth.WORKLOADS[name]
    X, _ = synth.make_data(wl, N)
    if wl.dtype == "bf16":
        Xd = torch.from_numpy(X.view(np.int16)).view(torch.bfloat16).cuda()
    else:
        Xd = torch.from_numpy(X).cuda()
    ws = G.workspace(G.problem_for(Xd, wl.K, wl.var_floor))
    mode = G.GMM_INIT_VAR_ONE if wl.var_init == "one" else G.GMM_INIT_VAR_DATA
    w, mu, var = G.gmm_init_rows(Xd, synth.init_rows(N, wl.K, wl.init_seed), wl.K, mode,
                            wl.var_floor, ws=ws)
    ref = [w.clone(), mu.clone(), var.clone()]
    got = [w.clone(), mu.clone(), var.clone()]
    ll_ref = torch.zeros(1, dtype=torch.float64, device="cuda")
    ll_got = torch.zeros(1, dtype=torch.float64, device="cuda")
    flags = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    for call in range(2):
        G.gmm_em_step(Xd, *ref, ll_ref, wl.var_floor, ws=ws)
        torch.cuda.synchronize()
        free0, _ = torch.cuda.mem_get_info()
        G.gmm_em_step_noalloc(Xd, *got, ll_got, flags, wl.var_floor)
        torch.cuda.synchronize()
        free1, _ = torch.cuda.mem_get_info()
        assert free0 == free1, "the no-allocation step changed free device memory"
        assert int(flags.item()) == 0
        # the workspace path's N_k for gating: recover it from its weights
        nk = ref[0].double().cpu().numpy() * N
        rep = compare.compare_step((*_np(*ref), ll_ref.item()), (*_np(*got), ll_got.item()), nk)
        assert rep["ok"], (call, rep)


def test_noalloc_rejects_problems_beyond_its_scratch(G):
    import torch

    X = torch.zeros(64, 1024, device="cuda")
    K = 8192  # one statistics slot alone is 8192 * 2049 * 8 bytes, far above the scratch
    w = torch.full((K,), 1.0 / K, device="cuda")
    mu = torch.zeros(K, 1024, device="cuda")
    var = torch.ones(K, 1024, device="cuda")
    with pytest.raises(G.GmmError) as e:
        G.gmm_em_step_noalloc(X, w, mu, var)
    assert e.value.status == G.GMM_ERR_UNSUPPORTED
