"""The sm_100a building blocks of the tensor-core EM kernel, checked against torch.

tests/csrc/tc_probe.cu runs one CTA that writes bf16 operands into the
128-byte-swizzled shared-memory layout (by threads, and by TMA), multiplies
them with tcgen05.mma (K-major and MN-major operand descriptors, N = 16..256)
into tensor memory and reads the accumulator back with tcgen05.ld.  Products of
bf16 values are exact in fp32, so the result must match a float64 matmul of
the same bf16 values to fp32 accumulation rounding.
"""
import ctypes
import os
import subprocess

import numpy as np
import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)


@pytest.fixture(scope="module")
def probe():
    import torch

    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    src = os.path.join(HERE, "csrc", "tc_probe.cu")
    so = os.path.join(HERE, "csrc", "_tc_probe.so")
    if not os.path.exists(so) or os.path.getmtime(so) < os.path.getmtime(src):
        subprocess.check_call([
            os.environ.get("NVCC", "/usr/local/cuda/bin/nvcc"), "-gencode",
            "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17", "-lineinfo", "-Xcompiler",
            "-fPIC", "-shared", "-I", os.path.join(ROOT, "soft_clustering_em_b200", "csrc"),
            "-I", os.path.join(ROOT, "include"), "-o", so, src])
    lib = ctypes.CDLL(so)
    P = ctypes.c_void_p
    lib.tc_probe_run.argtypes = [ctypes.c_int, ctypes.c_int, P, P, P, P, P]
    return lib


def _run(probe, mode, N, A, B, out_shape):
    import torch

    out = torch.full(out_shape, float("nan"), dtype=torch.float32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    Bp = B.data_ptr() if B is not None else 0
    rc = probe.tc_probe_run(mode, N, A.data_ptr(), Bp, out.data_ptr(), status.data_ptr(),
                            torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    assert status.item() == 0
    return out.cpu().double().numpy()


def _bf16(shape, seed):
    import torch

    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * 2).to(torch.bfloat16).cuda()


@pytest.mark.parametrize("N", [16, 64, 128, 256])
def test_kmajor_mma_with_tma_operand(probe, N):
    A = _bf16((128, 64), 1)
    B = _bf16((N, 64), 2)
    got = _run(probe, 0, N, A, B, (128, N))
    ref = A.double().cpu().numpy() @ B.double().cpu().numpy().T
    np.testing.assert_allclose(got, ref, rtol=1e-5, atol=1e-4)


def test_mn_major_operands(probe):
    At = _bf16((128, 128), 3)  # [K rows x M]
    Bt = _bf16((128, 64), 4)   # [K rows x N]
    got = _run(probe, 1, 64, At, Bt, (128, 64))
    ref = At.double().cpu().numpy().T @ Bt.double().cpu().numpy()
    np.testing.assert_allclose(got, ref, rtol=1e-5, atol=1e-4)


def test_column_sums_through_ones_operand(probe):
    At = _bf16((128, 128), 5)
    got = _run(probe, 2, 16, At, None, (128, 16))
    ref = At.double().cpu().numpy().sum(axis=0)
    for j in range(16):
        np.testing.assert_allclose(got[:, j], ref, rtol=1e-5, atol=1e-4)
