"""The library's tcgen05 GEMM (csrc/tc_gemm.cuh) against a plain PyTorch FP32 matmul of
the same bf16 operands, for every operand-major combination the loss uses, ragged
tile edges and split K."""

import ctypes
import os
import subprocess

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "tc_gemm_harness.cu")
CSRC = os.path.join(ROOT, "speculative_decoding_draft_vocab_b200", "csrc")


@pytest.fixture(scope="module")
def harness(tmp_path_factory):
    out = str(tmp_path_factory.mktemp("tcgemm") / "libtcgemm.so")
    subprocess.run(["/usr/local/cuda/bin/nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
                    "-shared", "-Xcompiler", "-fPIC", "-cudart", "static", "-I", CSRC,
                    "-I", os.path.join(ROOT, "include"), SRC, "-o", out], check=True)
    lib = ctypes.CDLL(out)
    lib.tc_gemm_test.restype = ctypes.c_int
    lib.tc_gemm_test.argtypes = [ctypes.c_void_p] * 3 + [ctypes.c_int] * 7 + [ctypes.c_void_p]
    return lib


@pytest.mark.parametrize("a_mn,b_mn,bn", [(0, 0, 256), (0, 1, 256), (1, 0, 256), (1, 1, 256), (0, 0, 128), (1, 1, 128)])
@pytest.mark.parametrize("M,N,K,ksplit", [(128, 256, 64, 1), (304, 520, 448, 1), (256, 256, 4096, 3)])
def test_tc_gemm_matches_fp32_matmul(harness, a_mn, b_mn, bn, M, N, K, ksplit):
    g = torch.Generator(device="cuda").manual_seed(M * 7 + N + K + 31 * a_mn + 17 * b_mn + bn)
    A = torch.randn(M, K, generator=g, device="cuda").to(torch.bfloat16)
    B = torch.randn(N, K, generator=g, device="cuda").to(torch.bfloat16)
    a_arg = A.t().contiguous() if a_mn else A  # [K][M] when MN-major
    b_arg = B.t().contiguous() if b_mn else B
    ks = max(1, min(ksplit, (K + 63) // 64))
    D = torch.full((ks, M, N), float("nan"), device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = harness.tc_gemm_test(a_arg.data_ptr(), b_arg.data_ptr(), D.data_ptr(), M, N, K, a_mn, b_mn, bn, ksplit,
                              status.data_ptr())
    assert rc == 0
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    ref = A.float() @ B.float().t()
    got = D.sum(0)
    err = (got - ref).abs().max().item()
    # fp32 accumulation of exact bf16 products: the error is FP32 summation order only
    assert err <= 1e-5 * K ** 0.5 * ref.abs().max().item() + 1e-4, err
