"""Host-side logic on the CPU: the input generator's guarantees, the parity rules
the GPU tests judge by, and the bench's gating of stored ncu traffic."""
import json
import os

import numpy as np
import pytest

from oracle import compare
from soft_clustering_em_b200 import synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


# ---------------------------------------------------------------- generator

@pytest.mark.parametrize("name", ["uint8img", "bf16stream"])
def test_row_blocks_are_the_same_whatever_else_is_drawn(name):
    wl = synth.WORKLOADS[name]
    start, n = 65_000, 1_200  # crosses the 65,536-row chunk boundary
    full, zf = synth.make_data(wl, start + n)
    block, zb = synth.make_data(wl, n, start=start)
    np.testing.assert_array_equal(block, full[start:])
    np.testing.assert_array_equal(zb, zf[start:])
    small, _ = synth.make_data(wl, 500)
    np.testing.assert_array_equal(small, full[:500])


def test_workload_value_structure():
    X, _ = synth.make_data(synth.WORKLOADS["uint8img"], 3_000)
    assert X.dtype == np.float32 and X.min() >= 0 and X.max() <= 255
    np.testing.assert_array_equal(X, np.rint(X))  # integers, exact in fp32
    S, _ = synth.make_data(synth.WORKLOADS["sphere768"], 200)
    np.testing.assert_allclose(np.linalg.norm(S.astype(np.float64), axis=1), 1.0, atol=1e-6)
    B, _ = synth.make_data(synth.WORKLOADS["bf16stream"], 2_000)
    assert B.dtype == np.uint16
    f = synth.x_as_f64(synth.WORKLOADS["bf16stream"], B)
    assert np.all(np.abs(f) < 4.0)  # means in [-1, 1], std <= 0.2


def test_bf16_rounding_is_to_nearest_even():
    one, next_up = 1.0, 1.0 + 2.0 ** -7  # adjacent bf16 values
    x = np.array([one + 2.0 ** -8,            # halfway: ties to the even (1.0)
                  next_up + 2.0 ** -8,        # halfway above an odd mantissa: up
                  one + 2.0 ** -8 + 2.0 ** -20,  # just above halfway: up
                  -(one + 2.0 ** -9)], dtype=np.float32)
    got = synth.bf16_to_f32(synth.bf16_round(x))
    np.testing.assert_array_equal(got, np.array([one, next_up + 2.0 ** -7, next_up, -one],
                                                dtype=np.float32))


def test_init_rows_are_distinct_sorted_and_in_range():
    rows = synth.init_rows(10_000, 256, 2002)
    assert rows.shape == (256,) and len(np.unique(rows)) == 256
    assert np.all(np.diff(rows) > 0) and rows[0] >= 0 and rows[-1] < 10_000
    np.testing.assert_array_equal(rows, synth.init_rows(10_000, 256, 2002))


# ---------------------------------------------------------------- parity rules

def _step(K=4, D=3, N=10_000.0):
    w = np.array([0.5, 0.3, 0.2 - 5e-4, 5e-4])  # the last component: 5 points
    mu = np.arange(K * D, dtype=np.float64).reshape(K, D) - 4.0
    var = np.full((K, D), 2.0)
    Nk = w * N
    return (w, mu, var, -1234.5), Nk, N


def test_weight_rule_is_relative_plus_1e9():
    """|dpi| <= 1e-3 pi + 1e-9, for a 5000-point and a 5-point component alike
    (no floor at ten points); the looser 10-point reading is reported beside it."""
    ref, Nk, N = _step()
    for k in (0, 3):  # 5000 points; 5 points
        scale = 1e-3 * ref[0][k] + 1e-9
        for frac, ok in ((0.9, True), (1.1, False)):
            w = ref[0].copy()
            w[k] += frac * scale
            rep = compare.compare_step(ref, (w, *ref[1:]), Nk, N)
            assert rep["ok"] is ok, (k, frac, rep)
            assert rep["w"] == pytest.approx(frac, rel=1e-6)
            floor = 1e-3 * max(ref[0][k], 10 / N)
            assert rep["w_floor10"] == pytest.approx(frac * scale / floor, rel=1e-6)


def test_mean_rule_scales_with_max_of_mean_and_sigma():
    ref, Nk, N = _step()
    sigma = np.sqrt(2.0)
    for (k, d), scale in (((1, 1), sigma), ((3, 2), 7.0)):  # mu = 0: sigma wins; mu = 7 wins
        mu = ref[1].copy()
        mu[k, d] += 0.9e-3 * scale
        rep = compare.compare_step(ref, (ref[0], mu, *ref[2:]), Nk, N)
        gated = Nk[k] >= compare.MIN_NK
        assert rep["ok"], rep
        assert (rep["mu"] if gated else rep["mu_ungated"]) == pytest.approx(0.9, rel=1e-6)
    mu = ref[1].copy()
    mu[1, 1] += 1.1e-3 * sigma
    assert not compare.compare_step(ref, (ref[0], mu, *ref[2:]), Nk, N)["ok"]


def test_mean_and_variance_are_gated_at_ten_points():
    ref, Nk, N = _step()
    var = ref[2].copy()
    var[3] *= 1.5  # the 5-point component: reported, not judged
    rep = compare.compare_step(ref, (ref[0], ref[1], var, ref[3]), Nk, N)
    assert rep["ok"] and rep["var_ungated"] == pytest.approx(500.0)
    assert rep["gated_components"] == 3
    var = ref[2].copy()
    var[2, 0] *= 1.0011  # a 1995-point component: judged at 1e-3 relative
    assert not compare.compare_step(ref, (ref[0], ref[1], var, ref[3]), Nk, N)["ok"]


def test_loglik_rule_is_relative_1e4():
    ref, Nk, N = _step()
    for frac, ok in ((0.9, True), (1.1, False)):
        ll = ref[3] + frac * 1e-4 * abs(ref[3])
        assert compare.compare_step(ref, (*ref[:3], ll), Nk, N)["ok"] is ok


def test_topm_mismatch_is_excused_only_within_the_gap():
    idx_ref = np.array([[0, 1], [2, 3]])
    resp_ref = np.array([[0.6, 0.39], [0.5, 0.49]])
    R_sorted = np.array([[0.6, 0.39, 0.01], [0.5, 0.49999, 0.00001]])
    # row 1's rank-1 candidate (0.49999) and the next one (0.00001) are far apart:
    # returning another index there is a real mismatch
    idx_got = np.array([[0, 1], [2, 4]])
    bad, worst = compare.compare_topm(idx_ref, resp_ref, idx_got, resp_ref, R_sorted)
    assert bad == 1
    # ...and excused when the two are within 1e-5
    R_close = np.array([[0.6, 0.39, 0.01], [0.5, 0.499995, 0.499990]])
    bad, _ = compare.compare_topm(idx_ref, resp_ref, idx_got, resp_ref, R_close)
    assert bad == 0
    resp_got = resp_ref * np.array([[1.0009, 1.0], [1.0, 1.0]])
    _, worst = compare.compare_topm(idx_ref, resp_ref, idx_ref, resp_got, R_sorted)
    assert worst == pytest.approx(0.9, rel=1e-6)


# ---------------------------------------------------------------- bench

def test_stored_traffic_is_used_only_for_the_source_it_was_measured_on(monkeypatch):
    import bench

    path = os.path.join(ROOT, "profiles", "traffic.json")
    stored = json.load(open(path))["uint8img"]
    monkeypatch.setattr(bench, "fused_source_sha", lambda: stored["source_sha"])
    assert bench.ncu_traffic("uint8img") == stored["dram_bytes_per_launch"]
    assert bench.ncu_traffic("bf16stream") is None
    monkeypatch.setattr(bench, "fused_source_sha", lambda: "0" * 16)
    assert bench.ncu_traffic("uint8img") is None


def test_reference_arm_prints_one_contract_line():
    import subprocess
    import sys

    cmd = [sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
           "--workload", "gauss8", "--steps", "2", "--warmup", "1"]
    out = subprocess.run(cmd, capture_output=True, text=True, timeout=300, check=True,
                         env={**os.environ, "RANK": "0"})
    lines = [ln for ln in out.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["steps"] == 2 and d["value"] > 0
    assert d["config"]["workload"] == "gauss8"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"
    assert d["cpu_baseline"]["cores"] >= 1
    # ranks other than 0 print nothing and exit 0
    quiet = subprocess.run(cmd, capture_output=True, text=True, timeout=120, check=True,
                           env={**os.environ, "RANK": "1"})
    assert quiet.stdout.strip() == ""


def test_tensor_core_shape_limits_and_f_buffers(tmp_path):
    """The tensor-core kernel's shape rule and F-buffer choice, from the host-side
    layout code itself (compiled for the host with nvcc; no device needed)."""
    import subprocess

    nvcc = "/usr/local/cuda/bin/nvcc"
    if not os.path.exists(nvcc):
        pytest.skip("nvcc not available")
    exe = str(tmp_path / "tc_layout_check")
    subprocess.run([nvcc, "-gencode", "arch=compute_100a,code=sm_100a", "-O1", "-std=c++17",
                    "--expt-relaxed-constexpr", "-I", os.path.join(ROOT, "include"),
                    "-I", os.path.join(ROOT, "soft_clustering_em_b200", "csrc"), "-o", exe,
                    os.path.join(ROOT, "tests", "csrc", "tc_layout_check.cu")],
                   check=True, capture_output=True, timeout=600)
    rows = [list(map(int, ln.split())) for ln in
            subprocess.run([exe], check=True, capture_output=True, text=True).stdout.split("\n")
            if ln.strip()]
    assert [r[0] for r in rows] == list(range(4, 129, 4))
    for D, maxk, nfb256, nfb1024, nfbmax, c4096, g4096 in rows:
        assert maxk == (2048 if D <= 64 else 1280 if D <= 96 else 256), D
        # K = 4096 takes component groups of one cluster each, of at most 4 CTAs
        assert (c4096, g4096) == ((4, 8) if D <= 96 else (2, 16)), D
        if D <= 32:  # two F buffers at every K
            assert (nfb256, nfb1024, nfbmax) == (2, 2, 2), D
        elif D <= 64:  # two only at small K, where the cluster is small enough
            assert (nfb256, nfb1024, nfbmax) == (2, 1, 1), D
        else:
            assert nfb256 == 1 and nfbmax == 1 and nfb1024 == (1 if D <= 96 else 0), D
    # streamed features (D > 128): every case has a plan that fits 227 KB of shared
    # memory, statistics groups of five chunks, chunk buffers within 256 MiB, and
    # r^ images only where there is more than one statistics group
    out = subprocess.run([exe, "streamed"], check=True, capture_output=True, text=True).stdout
    for ln in out.strip().split("\n"):
        D, K, C, G, nch, nfg, NFG, R, smem, fhi, rbuf = map(int, ln.split())
        assert C > 0 and G > 0, (D, K)
        assert nch == (2 * D + 63) // 64 and nfg == 5 and NFG == (nch + 4) // 5, (D, K)
        assert smem <= 232448, (D, K, smem)
        assert R >= 128 and R % 128 == 0, (D, K, R)
        assert 2 * fhi <= (256 << 20) + 512, (D, K, fhi)  # hi and lo feature planes
        if NFG == 1:
            assert rbuf == 0, (D, K)
        else:
            assert (R // 128) * G * C * 65536 <= rbuf <= (256 << 20) + 256, (D, K, rbuf)
    # the largest K with a tensor-core plan: 37 groups of 4-CTA clusters (one cluster
    # per group at least on 148 SMs), or 64 groups of 2 at D = 100..128
    out = subprocess.run([exe, "maxk"], check=True, capture_output=True, text=True).stdout
    for ln in out.strip().split("\n"):
        D, maxk = map(int, ln.split())
        assert maxk == (16384 if 100 <= D <= 128 else 18944), (D, maxk)
