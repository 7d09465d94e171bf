"""The C-ABI library loads, exports every symbol include/gmm.h declares, and
rejects bad arguments on the host before touching the device (no GPU needed)."""
import ctypes
import os
import re

import pytest

from soft_clustering_em_b200 import gmm as G

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from soft_clustering_em_b200 import build

    build.build()
    return G.load_library()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "gmm.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(gmm_[a-z_]+)\s*\(", text)))


def test_header_declares_the_calls():
    names = declared_functions()
    for n in ("gmm_plan", "gmm_init", "gmm_init_rows", "gmm_em_step_hard",
              "gmm_em_step_spherical", "gmm_kmeans_step", "gmm_em_step", "gmm_em_step_noalloc",
              "gmm_estep_stats", "gmm_mstep", "gmm_set_wait_budget",
              "gmm_fit", "gmm_loglik",
              "gmm_assign_topm", "gmm_ivf_workspace_size", "gmm_ivf_build",
              "gmm_host_staging_size", "gmm_em_step_host",
              "gmm_workspace_size", "gmm_device_status", "gmm_trace_fused",
              "gmm_launch_count", "gmm_status_string"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for n in declared_functions():
        assert hasattr(lib, n), n
    assert set(declared_functions()) == set(G.EXPORTS)  # the binding declares exactly the ABI


def test_status_strings(lib):
    assert G.status_string(0) == "GMM_OK"
    assert G.status_string(G.GMM_ERR_WORKSPACE) == "GMM_ERR_WORKSPACE"
    assert G.status_string(99) == "GMM_ERR_UNKNOWN"


def _call_em(lib, p, X=16, w=16, mu=16, var=16):
    P = ctypes.c_void_p
    return lib.gmm_em_step(ctypes.byref(p), P(X), P(w), P(mu), P(var), P(0), P(256), 1 << 30,
                           P(0))


@pytest.mark.parametrize("N,D,K,dt,floor,code", [
    (0, 4, 2, 0, 1e-6, G.GMM_ERR_INVALID_ARG),
    (10, 0, 2, 0, 1e-6, G.GMM_ERR_INVALID_ARG),
    (10, 4, 0, 0, 1e-6, G.GMM_ERR_INVALID_ARG),
    (10, 4, 2, 7, 1e-6, G.GMM_ERR_INVALID_ARG),
    (10, 4, 2, 0, float("nan"), G.GMM_ERR_INVALID_ARG),
    (10, 4, 2, 0, -1.0, G.GMM_ERR_INVALID_ARG),
    (10, 2, 2, 0, 1e-6, G.GMM_ERR_UNSUPPORTED),   # 8-byte rows: not a TMA-legal row pitch
    (10, 4, 2, 1, 1e-6, G.GMM_ERR_UNSUPPORTED),   # bf16 rows must be 16-byte multiples too
    (10, 4096, 2, 0, 1e-6, G.GMM_ERR_UNSUPPORTED),
])
def test_em_step_rejects_bad_problems(lib, N, D, K, dt, floor, code):
    assert _call_em(lib, G.problem(N, D, K, dt, floor)) == code


def test_null_and_misaligned_pointers(lib):
    p = G.problem(10, 4, 2)
    assert _call_em(lib, p, X=0) == G.GMM_ERR_INVALID_ARG
    assert _call_em(lib, p, X=8) == G.GMM_ERR_UNSUPPORTED
    assert _call_em(lib, p, w=0) == G.GMM_ERR_INVALID_ARG
    assert _call_em(lib, p, var=0) == G.GMM_ERR_INVALID_ARG
    assert lib.gmm_workspace_size(ctypes.byref(p), None) == G.GMM_ERR_INVALID_ARG
    assert lib.gmm_workspace_size(None, ctypes.byref(ctypes.c_size_t())) == G.GMM_ERR_INVALID_ARG


def test_topm_and_init_argument_checks(lib):
    P = ctypes.c_void_p
    p = G.problem(10, 4, 3)
    for m in (0, 4, 9):
        rc = lib.gmm_assign_topm(ctypes.byref(p), P(16), P(16), P(16), P(16), m, P(16), P(16),
                                 P(256), 1 << 30, P(0))
        assert rc == G.GMM_ERR_INVALID_ARG, m
    rows = (ctypes.c_int64 * 3)(0, 5, 10)  # 10 is out of range for N = 10
    rc = lib.gmm_init_rows(ctypes.byref(p), P(16), rows, 1, P(16), P(16), P(16), P(256), 1 << 30, P(0))
    assert rc == G.GMM_ERR_INVALID_ARG
    rows = (ctypes.c_int64 * 3)(0, 5, 9)
    rc = lib.gmm_init_rows(ctypes.byref(p), P(16), rows, 2, P(16), P(16), P(16), P(256), 1 << 30, P(0))
    assert rc == G.GMM_ERR_INVALID_ARG
    rc = lib.gmm_fit(ctypes.byref(p), P(16), -1, P(16), P(16), P(16), P(0), P(256), 1 << 30, P(0))
    assert rc == G.GMM_ERR_INVALID_ARG
    # seeded init: K distinct rows need K <= N; the variance mode is checked too
    few = G.problem(2, 4, 3)
    rc = lib.gmm_init(ctypes.byref(few), P(16), 5, 1, P(16), P(16), P(16), P(256), 1 << 30, P(0))
    assert rc == G.GMM_ERR_INVALID_ARG
    rc = lib.gmm_init(ctypes.byref(p), P(16), 5, 2, P(16), P(16), P(16), P(256), 1 << 30, P(0))
    assert rc == G.GMM_ERR_INVALID_ARG


def test_no_device_is_a_cuda_error_not_a_crash(lib):
    import torch

    if torch.cuda.is_available():
        pytest.skip("a device is present")
    p = G.problem(1000, 16, 8)
    n = ctypes.c_size_t(0)
    assert lib.gmm_workspace_size(ctypes.byref(p), ctypes.byref(n)) == G.GMM_ERR_CUDA
    assert _call_em(lib, p) == G.GMM_ERR_CUDA


def test_trace_hook_arguments(lib):
    P = ctypes.c_void_p
    assert lib.gmm_trace_fused(P(16), None) == G.GMM_ERR_INVALID_ARG
    assert lib.gmm_trace_fused(None, None) == G.GMM_OK


def test_split_step_argument_checks(lib):
    P = ctypes.c_void_p
    p = G.problem(10, 4, 3)
    assert lib.gmm_estep_stats(ctypes.byref(p), P(16), P(16), P(16), P(16), P(0), P(256), 1 << 30,
                               P(0)) == G.GMM_ERR_INVALID_ARG
    assert lib.gmm_mstep(ctypes.byref(p), P(0), 1, P(16), P(16), P(16), P(0), P(0)) == \
        G.GMM_ERR_INVALID_ARG
    assert lib.gmm_mstep(ctypes.byref(p), P(16), 0, P(16), P(16), P(16), P(0), P(0)) == \
        G.GMM_ERR_INVALID_ARG
    bad = G.problem(0, 4, 3)
    assert lib.gmm_mstep(ctypes.byref(bad), P(16), 1, P(16), P(16), P(16), P(0), P(0)) == \
        G.GMM_ERR_INVALID_ARG


def _ivf_ws(lib, N, K):
    n = ctypes.c_size_t(0)
    rc = lib.gmm_ivf_workspace_size(N, K, ctypes.byref(n))
    return rc, n.value


def test_ivf_workspace_grows_with_n_up_to_a_cap(lib):
    assert _ivf_ws(lib, 0, 4)[0] == G.GMM_ERR_INVALID_ARG
    assert _ivf_ws(lib, 10, 0)[0] == G.GMM_ERR_INVALID_ARG
    assert _ivf_ws(lib, 10, 65537)[0] == G.GMM_ERR_UNSUPPORTED
    assert _ivf_ws(lib, (1 << 40) + 1, 4)[0] == G.GMM_ERR_UNSUPPORTED
    assert lib.gmm_ivf_workspace_size(10, 4, None) == G.GMM_ERR_INVALID_ARG
    sizes = [_ivf_ws(lib, N, 1024)[1] for N in (1, 10**4, 10**6, 10**8, 10**10)]
    assert sizes == sorted(sizes) and sizes[-2] == sizes[-1]  # capped chunk count
    for K in (1024, 4096, 65536):
        assert _ivf_ws(lib, 10**9, K)[1] <= (64 << 20) + 8 * K + 1024


def test_ivf_build_argument_checks(lib):
    P = ctypes.c_void_p
    N, K, m = 100, 16, 2
    ok_ws = _ivf_ws(lib, N, K)[1]

    def call(N=N, K=K, m=m, idx=16, resp=16, tau=0.1, off=16, ids=16, cap=N * m, ws=256,
             ws_bytes=ok_ws):
        return lib.gmm_ivf_build(N, K, m, P(idx), P(resp), tau, P(off), P(ids), cap, P(ws),
                                 ws_bytes, P(0))

    assert call(N=0) == G.GMM_ERR_INVALID_ARG
    assert call(K=0) == G.GMM_ERR_INVALID_ARG
    assert call(K=65537) == G.GMM_ERR_UNSUPPORTED
    for bad_m in (0, 9):
        assert call(m=bad_m) == G.GMM_ERR_INVALID_ARG
    assert call(K=1, m=2) == G.GMM_ERR_INVALID_ARG  # m > K
    for name in ("idx", "resp", "off", "ids"):
        assert call(**{name: 0}) == G.GMM_ERR_INVALID_ARG, name
    assert call(tau=float("nan")) == G.GMM_ERR_INVALID_ARG
    assert call(cap=N * m - 1) == G.GMM_ERR_INVALID_ARG
    assert call(ws=0) == G.GMM_ERR_WORKSPACE
    assert call(ws=128) == G.GMM_ERR_WORKSPACE
    assert call(ws_bytes=ok_ws - 1) == G.GMM_ERR_WORKSPACE


def _staging(lib, p, rows):
    n = ctypes.c_size_t(0)
    rc = lib.gmm_host_staging_size(ctypes.byref(p), rows, ctypes.byref(n))
    return rc, n.value


def test_host_staging_size_is_two_chunks_and_two_stats_buffers(lib):
    def up(x):
        return (x + 255) // 256 * 256

    for N, D, K, dt, rows in ((10**6, 128, 256, 0, 65_536), (10**8, 32, 1024, 1, 1 << 20),
                              (7, 4, 3, 0, 3)):
        p = G.problem(N, D, K, dt)
        rc, n = _staging(lib, p, rows)
        S = K * (2 * D + 1) + 1
        assert rc == G.GMM_OK and n == 2 * up(rows * D * (2 if dt else 4)) + 2 * up(S * 8)
    assert _staging(lib, G.problem(10, 4, 2), 0)[0] == G.GMM_ERR_INVALID_ARG
    assert _staging(lib, G.problem(0, 4, 2), 5)[0] == G.GMM_ERR_INVALID_ARG
    assert lib.gmm_host_staging_size(ctypes.byref(G.problem(10, 4, 2)), 5, None) == \
        G.GMM_ERR_INVALID_ARG


def test_em_step_host_argument_checks(lib):
    P = ctypes.c_void_p
    p = G.problem(100, 4, 2)
    need = _staging(lib, p, 10)[1]

    def call(X=16, rows=10, staging=256, sbytes=need, w=16):
        return lib.gmm_em_step_host(ctypes.byref(p), P(X), rows, P(staging), sbytes, P(w), P(16),
                                    P(16), P(0), P(256), 1 << 30, P(0), P(0))

    assert call(X=0) == G.GMM_ERR_INVALID_ARG
    assert call(w=0) == G.GMM_ERR_INVALID_ARG
    assert call(rows=0) == G.GMM_ERR_INVALID_ARG
    assert call(staging=0) == G.GMM_ERR_WORKSPACE
    assert call(staging=128) == G.GMM_ERR_WORKSPACE
    assert call(sbytes=need - 1) == G.GMM_ERR_WORKSPACE
    bad = G.problem(100, 2, 2)  # 8-byte rows: not a legal row pitch for the staged copy
    assert lib.gmm_em_step_host(ctypes.byref(bad), P(16), 10, P(256), 1 << 20, P(16), P(16),
                                P(16), P(0), P(256), 1 << 30, P(0), P(0)) == \
        G.GMM_ERR_UNSUPPORTED


def test_header_is_plain_c99_and_the_c_example_links(lib, tmp_path):
    """include/gmm.h compiles as pedantic C99, and a plain C program using the
    ABI builds, links and runs: without a device it reports GMM_ERR_CUDA cleanly."""
    import shutil
    import subprocess

    import torch

    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("gcc not available")
    inc = os.path.join(ROOT, "include")
    hdr = tmp_path / "hdr.c"
    hdr.write_text('#include "gmm.h"\nint main(void) { return gmm_status_string(GMM_OK) == 0; }\n')
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic", "-I", inc, "-c",
                    str(hdr), "-o", str(tmp_path / "hdr.o")], check=True, capture_output=True)
    cuda = "/usr/local/cuda"
    libdir = os.path.dirname(G.LIB_PATH)
    exe = str(tmp_path / "c_abi_example")
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-Werror", "-I", inc, "-I",
                    os.path.join(cuda, "include"), "-o", exe,
                    os.path.join(ROOT, "tests", "csrc", "c_abi_example.c"), "-L", libdir,
                    "-lscem_gmm", "-L", os.path.join(cuda, "lib64"), "-lcudart",
                    "-Wl,-rpath," + libdir, "-Wl,-rpath," + os.path.join(cuda, "lib64")],
                   check=True, capture_output=True)
    out = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    if torch.cuda.is_available():
        assert out.returncode == 0 and out.stdout.startswith("LL(theta_9)"), out.stdout
    else:
        assert out.returncode == 0 and "GMM_ERR_CUDA" in out.stdout, out.stdout
