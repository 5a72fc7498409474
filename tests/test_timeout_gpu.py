"""The device-timeout path, in the form this pool allows: a bounded wait that runs out
because nothing ever arrives (no trap, no fault, nothing in flight toward the waiting
CTA).  The harness is built with a wait limit of a few milliseconds; the kernel must
give up, record the timeout in the workspace header the way the library's kernels do,
and return, after which the library's dspark_check_status reports
DSPARK_ERR_DEVICE_TIMEOUT and the context stays usable."""

import ctypes
import os
import subprocess

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "timeout_harness.cu")
CSRC = os.path.join(ROOT, "speculative_decoding_draft_vocab_b200", "csrc")
LIMIT_NS = 5_000_000  # 5 ms


@pytest.fixture(scope="module")
def harness(tmp_path_factory):
    out = str(tmp_path_factory.mktemp("timeout") / "libtimeout.so")
    subprocess.run(["/usr/local/cuda/bin/nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-std=c++17",
                    "-shared", "-Xcompiler", "-fPIC", "-cudart", "static", f"-DDSPARK_WAIT_LIMIT_NS={LIMIT_NS}ull",
                    "-I", CSRC, "-I", os.path.join(ROOT, "include"), SRC, "-o", out], check=True)
    lib = ctypes.CDLL(out)
    lib.timeout_harness_run.restype = ctypes.c_int
    lib.timeout_harness_run.argtypes = [ctypes.c_void_p] * 4
    lib.timeout_harness_limit_ns.restype = ctypes.c_uint64
    return lib


def test_a_wait_that_nothing_arms_times_out_and_is_reported(harness):
    from speculative_decoding_draft_vocab_b200 import abi, build, torch_api
    from speculative_decoding_draft_vocab_b200.synthetic import make_inputs
    build.build()
    assert harness.timeout_harness_limit_ns() == LIMIT_NS
    ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    waited = torch.zeros(1, dtype=torch.int32, device="cuda")
    ns = torch.zeros(1, dtype=torch.int64, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    assert harness.timeout_harness_run(ws.data_ptr(), waited.data_ptr(), ns.data_ptr(), stream) == 0
    st = abi.dspark_check_status(ctypes.c_void_p(ws.data_ptr()), ctypes.c_void_p(stream))
    assert st == abi.DSPARK_ERR_DEVICE_TIMEOUT
    assert int(waited.item()) == 1
    assert LIMIT_NS <= int(ns.item()) < 1_000_000_000  # gave up after the limit, well before 1 s
    # the context is still usable: a fused call runs and reports no error
    inp = make_inputs("tiny", device="cuda", seed=5)
    call = torch_api.Call(inp)
    call.launch()
    torch.cuda.synchronize()
    assert call.check_status() == 0
