"""tcgen05 operand layouts and descriptors (sm100.cuh) against a plain matmul.

Each case puts A (128 x K) and B (N x K) in one of the layouts the KDA kernels
use, runs one chain of tcgen05.mma and compares D = A B^T with torch's matmul of
the same bf16 values (fp32 accumulation on both sides)."""
import ctypes
import os
import subprocess

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "csrc", "umma_selftest.cu")
SO = os.path.join(ROOT, "_build", "libumma_selftest.so")


def build_selftest() -> str:
    os.makedirs(os.path.dirname(SO), exist_ok=True)
    cmd = ["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O2", "-std=c++17",
           "-shared", "-Xcompiler", "-fPIC",
           "-I", os.path.join(ROOT, "gated_delta_rule_74_b200", "csrc"),
           "-I", os.path.join(ROOT, "include"), SRC, "-o", SO]
    subprocess.run(cmd, check=True)
    return SO


@pytest.fixture(scope="module")
def lib():
    L = ctypes.CDLL(build_selftest())
    L.umma_selftest.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int] * 4 + [ctypes.c_void_p] * 2
    L.umma_selftest.restype = ctypes.c_int
    return L


CASES = [
    # (a_layout, b_layout, N, K)       use in the prefill kernel
    (1, 2, 16, 128), (1, 2, 32, 128), (1, 2, 48, 128), (1, 2, 64, 128),   # Gram: L x R^(a)
    (2, 0, 64, 64),                                                       # W^T = Kbar^T (T beta)^T
    (1, 0, 64, 64),                                                       # U^T = V^T (T beta)^T
    (2, 1, 64, 128),                                                      # P = S^T W^T, O^T = S^T Qbar^T
    (2, 0, 128, 64),                                                      # S^T += Delta^T Kend
    (0, 1, 128, 128),                                                     # segment combine: X S
    (0, 0, 128, 128), (0, 1, 64, 128), (2, 2, 32, 64),                    # other combinations
]


@pytest.mark.parametrize("a_layout,b_layout,N,K", CASES)
def test_umma_layout(lib, a_layout, b_layout, N, K):
    g = torch.Generator(device="cuda").manual_seed(N * 1000 + K + 10 * a_layout + b_layout)
    A = torch.randn(128, K, device="cuda", generator=g).to(torch.bfloat16)
    B = torch.randn(N, K, device="cuda", generator=g).to(torch.bfloat16)
    D = torch.full((128, N), float("nan"), device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = lib.umma_selftest(A.data_ptr(), B.data_ptr(), D.data_ptr(), N, K, a_layout, b_layout,
                           status.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    assert int(status.item()) == 0, "MMA completion wait timed out"
    ref = A.float() @ B.float().T
    err = (D - ref).abs().max().item()
    assert err <= 1e-3 * ref.abs().max().item(), (a_layout, b_layout, N, K, err)
