"""gmm_em_step_host: EM with X in (pinned) host memory, streamed to the device in
chunks, against the oracle (teacher-forced, the rules of oracle/compare.py) and
against the same step on device-resident X.
"""
import numpy as np
import pytest

import oracle
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


def _params_np(w, mu, var):
    return (w.double().cpu().numpy(), mu.double().cpu().numpy(), var.double().cpu().numpy())


def _setup(G, name, N, K):
    import torch

    wl = synth.WORKLOADS[name]
    X, _ = synth.make_data(wl, N)
    Xh = torch.from_numpy(X.view(np.int16)).view(torch.bfloat16) if wl.dtype == "bf16" else \
        torch.from_numpy(X)
    Xh = Xh.pin_memory()
    Xd = Xh.cuda()
    mode = G.GMM_INIT_VAR_ONE if wl.var_init == "one" else G.GMM_INIT_VAR_DATA
    w, mu, var = G.gmm_init_rows(Xd, synth.init_rows(N, K, wl.init_seed), K, mode, wl.var_floor)
    return wl, Xh, Xd, synth.x_as_f64(wl, X), (w, mu, var)


@pytest.mark.parametrize("name,N,K,chunk", [
    ("uint8img", 20_001, 256, 3_000),    # 7 chunks, ragged last one; tensor cores
    ("bf16stream", 30_001, 1024, 4_096),  # bf16 rows, 8-CTA clusters
    ("gauss8", 1_001, 8, 7),             # 143 chunks of 7 rows
    ("gauss8", 1_000, 8, 1_000),         # exactly one chunk
    ("gauss8", 999, 8, 5_000),           # chunk larger than N
    ("sphere768", 2_003, 1024, 500),     # D = 768: streamed features, 5 statistics groups
    ("gauss4096", 20_000, 4096, 6_000),  # component groups: two passes per host chunk
])
def test_host_streamed_step_matches_oracle(G, name, N, K, chunk):
    import torch

    wl, Xh, _, X64, (w, mu, var) = _setup(G, name, N, K)
    p = G.problem_for(Xh, K, wl.var_floor)
    ws = G.workspace(p)
    ll = torch.zeros(1, dtype=torch.float64, device="cuda")
    for t in range(2):
        th = _params_np(w, mu, var)
        G.gmm_em_step_host(Xh, w, mu, var, ll, chunk, wl.var_floor, ws=ws)
        torch.cuda.synchronize()
        rc, flags = G.gmm_device_status(ws)
        assert rc == 0 and flags == 0
        w2, mu2, var2, ll_ref, Nk = oracle.em_step(X64, *th, var_floor=wl.var_floor)
        rep = compare.compare_step((w2, mu2, var2, ll_ref),
                                   (*_params_np(w, mu, var), float(ll.item())), Nk)
        assert rep["ok"], (t, rep)


def test_host_streamed_step_agrees_with_resident_step(G):
    import torch

    wl, Xh, Xd, _, theta = _setup(G, "uint8img", 20_001, 256)
    runs = {}
    for how in ("resident", "side_stream", "one_stream"):
        w, mu, var = (t.clone() for t in theta)
        ll = torch.zeros(1, dtype=torch.float64, device="cuda")
        if how == "resident":
            G.gmm_em_step(Xd, w, mu, var, ll, wl.var_floor)
        else:
            cs = torch.cuda.current_stream() if how == "one_stream" else None
            G.gmm_em_step_host(Xh, w, mu, var, ll, 4_096, wl.var_floor, copy_stream=cs)
        torch.cuda.synchronize()
        runs[how] = (*_params_np(w, mu, var), float(ll.item()))
    # the copy stream changes only timing: bit-identical
    for a, b in zip(runs["side_stream"], runs["one_stream"]):
        np.testing.assert_array_equal(a, b)
    # chunking changes only the order of the statistics' sums
    res, host = runs["resident"], runs["side_stream"]
    Nk = res[0] * 20_001
    assert compare.compare_step(res, host, Nk)["ok"]
    assert abs(host[3] - res[3]) <= 1e-9 * abs(res[3])
