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


@pytest.fixture(scope="module")
def gather_harness(harness):
    harness.tc_gemm_gather_test.restype = ctypes.c_int
    harness.tc_gemm_gather_test.argtypes = ([ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_void_p,
                                             ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_int,
                                             ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_void_p])
    return harness


@pytest.mark.parametrize("a_mn", [0, 1])
@pytest.mark.parametrize("src_rows,cols,n_list,positions,ksplit", [(300, 512, 200, 256, 1), (300, 640, 77, 256, 3),
                                                                     (64, 1024, 0, 128, 2), (1000, 448, 513, 640, 1)])
def test_tc_gemm_gathered_rows(gather_harness, a_mn, src_rows, cols, n_list, positions, ksplit):
    """A's rows fetched by index (four-row gathers), the count on the device: positions at
    or past the count read as zero rows; with A's rows as K indices the contraction is also
    cut at the count (a list of length 0 gives an all-zero product)."""
    g = torch.Generator(device="cuda").manual_seed(src_rows + cols + n_list + 7 * a_mn)
    src = torch.randn(src_rows, cols, generator=g, device="cuda").to(torch.bfloat16)
    perm = torch.randperm(src_rows, generator=g, device="cuda")[:n_list].to(torch.int32)
    lst = torch.zeros(positions, dtype=torch.int32, device="cuda")
    lst[:n_list] = perm
    length = torch.tensor([n_list], dtype=torch.int32, device="cuda")
    N = 256
    gathered = torch.zeros(positions, cols, device="cuda")
    gathered[:n_list] = src[perm.long()].float()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    if a_mn == 0:
        B = torch.randn(N, cols, generator=g, device="cuda").to(torch.bfloat16)
        ks = max(1, min(ksplit, (cols + 63) // 64))
        D = torch.zeros((ks, positions, N), device="cuda")
        rc = gather_harness.tc_gemm_gather_test(src.data_ptr(), src_rows, cols, lst.data_ptr(), length.data_ptr(),
                                                positions, B.data_ptr(), N, D.data_ptr(), 0, ksplit,
                                                status.data_ptr())
        ref = gathered @ B.float().t()
        got = D.sum(0)
        rows = (n_list + 127) // 128 * 128  # tiles past the count are skipped (left as they were)
        ref, got = ref[:min(rows, positions)], got[:min(rows, positions)]
    else:
        B = torch.randn(positions, N, generator=g, device="cuda").to(torch.bfloat16)
        Bz = B.float().clone()
        Bz[n_list:] = 0  # positions past the count contribute nothing
        D = torch.full((1, cols, N), float("nan"), device="cuda")
        rc = gather_harness.tc_gemm_gather_test(src.data_ptr(), src_rows, cols, lst.data_ptr(), length.data_ptr(),
                                                positions, B.data_ptr(), N, D.data_ptr(), 1, 1, status.data_ptr())
        # whole 64-position chunks up to the count take part: rows of A past the count
        # are zero, so the product is the sum over the listed rows only
        ref = gathered.t() @ Bz
        got = D.sum(0)
    assert rc == 0
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    assert torch.isfinite(got).all()
    err = (got - ref).abs().max().item() if ref.numel() else 0.0
    assert err <= 1e-5 * max(cols, positions) ** 0.5 * max(ref.abs().max().item() if ref.numel() else 0.0, 1.0) + 1e-4
