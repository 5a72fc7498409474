"""dspark_loss_fwd_noalloc: the fused forward + backward with the library's fixed
device scratch in place of a caller workspace, for callers that cannot allocate
device memory.  It must give what dspark_loss_fwd gives on the same inputs, call after
call (the scratch is shared and reused), and refuse micro-batches above its size.

Kept in the last-collected file so that a run stopping at the first failure has run
every other test already."""

import ctypes

import numpy as np
import pytest
import torch

from speculative_decoding_draft_vocab_b200.synthetic import make_inputs

pytestmark = pytest.mark.gpu


def _noalloc(call, abi):
    st = abi.dspark_loss_fwd_noalloc(ctypes.byref(call.prob), ctypes.byref(call.prm),
                                     ctypes.byref(call.fwd), ctypes.byref(call.grads),
                                     ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    abi.check(st, "dspark_loss_fwd_noalloc")


def _bf16_close(a: torch.Tensor, b: torch.Tensor):
    """The dlogits rule of the parity tests: max(2e-3 relative, one bf16 ulp)."""
    x = a.float().cpu().double().numpy()
    y = b.float().cpu().double().numpy()
    ay = np.abs(y)
    _, e = np.frexp(np.where(ay > 0, ay, 1.0))
    ulp = np.where(ay > 0, np.ldexp(1.0, e - 8), 0.0)
    tol = np.maximum(2e-3 * ay, ulp) + 1e-6 * ay.max(initial=0.0)
    assert np.all(np.abs(x - y) <= tol)


def test_no_alloc_entry_point_matches_workspace_entry_point():
    from speculative_decoding_draft_vocab_b200 import build
    build.build()
    from speculative_decoding_draft_vocab_b200 import abi, torch_api
    assert torch.cuda.is_available()

    inp = make_inputs("recipe", device="cuda", B=2, N=8, K=7, V=151936, conf="given",
                      mask_holes=True, seed=21)
    ref = torch_api.Call(inp)
    ref.launch()
    torch.cuda.synchronize()
    assert ref.check_status() == 0

    fixed = torch_api.Call(inp)  # its own output buffers; its workspace is not used
    for _ in range(2):           # two calls in a row on the shared scratch
        fixed.out.dlogits.fill_(3.0)
        fixed.out.report.fill_(-1.0)
        _noalloc(fixed, abi)
        torch.cuda.synchronize()
        assert int(fixed.out.num_tokens.item()) == int(ref.out.num_tokens.item())
        r, f = ref.out.report.cpu().double().numpy(), fixed.out.report.cpu().double().numpy()
        assert np.array_equal(r[:, 1], f[:, 1])
        assert np.all(np.abs(r[:, 0] - f[:, 0]) <= 1e-4 * np.abs(r[:, 0]) + 1e-6 * np.maximum(r[:, 1], 1.0))
        assert abs(float(ref.out.loss_num.item()) - float(fixed.out.loss_num.item())) <= \
            1e-4 * abs(float(ref.out.loss_num.item()))
        np.testing.assert_allclose(fixed.out.l1_rows.cpu().numpy(), ref.out.l1_rows.cpu().numpy(), atol=1e-3)
        np.testing.assert_allclose(fixed.out.dconf.cpu().numpy(), ref.out.dconf.cpu().numpy(), rtol=1e-4, atol=1e-6)
        _bf16_close(fixed.out.dlogits, ref.out.dlogits)


def test_no_alloc_entry_point_refuses_oversized_batches():
    from speculative_decoding_draft_vocab_b200 import abi, torch_api
    inp = make_inputs("recipe", device="cuda", B=2, N=8, K=7, V=1024, seed=22)
    call = torch_api.Call(inp)
    call.prob.N = (abi.NOALLOC_MAX_ROWS // (inp.B * inp.K)) + 1  # rows above the limit
    st = abi.dspark_loss_fwd_noalloc(ctypes.byref(call.prob), ctypes.byref(call.prm),
                                     ctypes.byref(call.fwd), ctypes.byref(call.grads), None)
    assert st == abi.DSPARK_ERR_WORKSPACE


def _sentinel_outputs(call):
    """Fill every output the call could write with a marker value; returns a checker that
    the outputs still hold it (nothing was enqueued)."""
    bufs = [t for t in (call.out.loss_num, call.out.report, call.out.dlogits, call.out.dconf, call.out.dW2,
                        call.out.dconf_w) if t is not None]
    for t in bufs:
        t.fill_(7.0)
    call.out.num_tokens.fill_(-5)
    torch.cuda.synchronize()

    def untouched():
        torch.cuda.synchronize()
        assert int(call.out.num_tokens.item()) == -5
        for t in bufs:
            assert bool((t.float() == 7.0).all())
    return untouched


@pytest.mark.parametrize("kind", ["markov", "conf_head_448_rows", "teacher_from_hidden"])
def test_no_alloc_entry_point_refuses_problems_larger_than_its_scratch(kind):
    """Problems whose workspace exceeds the fixed array return DSPARK_ERR_WORKSPACE and
    leave every output untouched: the Markov head and the teacher from hidden states
    (4*V bytes per row of FP32 vocabulary rows) and a confidence head on the 448-row
    recipe micro-batch (its dL/dproj partial sums)."""
    from speculative_decoding_draft_vocab_b200 import abi, torch_api
    if kind == "markov":
        inp = make_inputs("recipe_heads", device="cuda", B=1, N=4, K=7, V=8192, conf=None, seed=31)
    elif kind == "conf_head_448_rows":
        inp = make_inputs("recipe", device="cuda", B=4, N=16, K=7, V=1024, conf="head", seed=32)
    else:
        inp = make_inputs("lm_head_teacher", device="cuda", B=1, N=4, K=7, V=8192, conf=None, markov=False,
                          target_hidden_size=256, seed=33)
    call = torch_api.Call(inp)
    assert abi.dspark_workspace_size(ctypes.byref(call.prob)) > abi.NOALLOC_BYTES
    untouched = _sentinel_outputs(call)
    st = abi.dspark_loss_fwd_noalloc(ctypes.byref(call.prob), ctypes.byref(call.prm), ctypes.byref(call.fwd),
                                     ctypes.byref(call.grads),
                                     ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == abi.DSPARK_ERR_WORKSPACE
    untouched()


def test_no_alloc_entry_point_serves_a_small_confidence_head():
    """A confidence head on 224 rows fits the array and matches dspark_loss_fwd."""
    from speculative_decoding_draft_vocab_b200 import abi, torch_api
    inp = make_inputs("recipe", device="cuda", B=2, N=16, K=7, V=16384, conf="head", seed=34)
    ref = torch_api.Call(inp)
    assert abi.dspark_workspace_size(ctypes.byref(ref.prob)) <= abi.NOALLOC_BYTES
    ref.launch()
    torch.cuda.synchronize()
    assert ref.check_status() == 0
    fixed = torch_api.Call(inp)
    for _ in range(2):
        fixed.out.dlogits.fill_(3.0)
        fixed.out.dconf_w.fill_(5.0)
        _noalloc(fixed, abi)
        torch.cuda.synchronize()
        assert int(fixed.out.num_tokens.item()) == int(ref.out.num_tokens.item())
        r, f = ref.out.report.cpu().double().numpy(), fixed.out.report.cpu().double().numpy()
        assert np.array_equal(r[:, 1], f[:, 1])
        assert np.all(np.abs(r[:, 0] - f[:, 0]) <= 1e-4 * np.abs(r[:, 0]) + 1e-6 * np.maximum(r[:, 1], 1.0))
        np.testing.assert_allclose(fixed.out.conf_rows.cpu().numpy(), ref.out.conf_rows.cpu().numpy(),
                                   rtol=1e-4, atol=1e-5)
        np.testing.assert_allclose(fixed.out.dconf_w.cpu().numpy(), ref.out.dconf_w.cpu().numpy(),
                                   rtol=1e-4, atol=1e-6)
        _bf16_close(fixed.out.dlogits, ref.out.dlogits)
        _bf16_close(fixed.out.dhidden, ref.out.dhidden)
