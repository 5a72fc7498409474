"""GPU parity of the teacher computed from the target's final hidden states
(t = lm_head . h on the tensor cores, one chunk of at most 512 supervised rows at a
time) against the FP64 oracle, alone and with the Markov and confidence heads, in the
fused call and in the separate backward, with one and with several chunks."""

import numpy as np
import pytest
import torch

from speculative_decoding_draft_vocab_b200.synthetic import make_inputs
from tests.parity_util import check_heads, compare, oracle_run

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from speculative_decoding_draft_vocab_b200 import build
    build.build()
    assert torch.cuda.is_available(), "the GPU tests need a CUDA device"


def _check(inp, call, ref, mode=0):
    compare(inp, call, ref)
    if inp.markov_w2 is not None or inp.conf_w is not None:
        check_heads(inp, call, ref, mode)


def _run(inp, mode=0):
    from speculative_decoding_draft_vocab_b200 import torch_api
    call = torch_api.Call(inp, grads=True, invalid_row_mode=mode)
    call.launch()
    torch.cuda.synchronize()
    assert call.check_status() == 0
    ref = oracle_run(inp, invalid_row_mode=mode)
    _check(inp, call, ref, mode)
    return call, ref


def test_teacher_from_hidden_alone():
    inp = make_inputs("lm_head_teacher", device="cuda", seed=41, B=2, N=4, K=7, V=8192, target_hidden_size=256,
                      markov=False, conf=None, mask_holes=True)
    _run(inp)


@pytest.mark.parametrize("mode", [0, 1])
def test_teacher_from_hidden_with_heads(mode):
    inp = make_inputs("lm_head_teacher", device="cuda", seed=42 + mode, B=2, N=4, K=7, V=8192,
                      target_hidden_size=320, hidden=256, rank=64, target_vocab=2000, markov_std=0.3,
                      conf_bias=0.2, valid_p=0.75)
    _run(inp, mode)


def test_teacher_given_confidence_logits():
    inp = make_inputs("lm_head_teacher", device="cuda", seed=44, B=2, N=3, K=7, V=4096, target_hidden_size=128,
                      markov=False, conf="given")
    _run(inp)


@pytest.mark.parametrize("prefix", [(5, 8), (1, 3)])
def test_several_teacher_chunks(prefix):
    """1024 rows: with long prefixes more than 512 supervised rows (two chunks, the
    second ragged); with short ones fewer (the second chunk is empty)."""
    inp = make_inputs("lm_head_teacher", device="cuda", seed=45 + prefix[0], B=4, N=32, K=8, V=2048,
                      target_hidden_size=128, markov=True, rank=64, target_vocab=700, markov_std=0.3,
                      conf="head", hidden=64, prefix=prefix)
    call, ref = _run(inp)
    n = ref["num_tokens"]
    assert (n > 512) == (prefix[0] >= 5)


@pytest.mark.parametrize("chunks", [1, 2])
def test_separate_backward_teacher_from_hidden(chunks):
    """Forward without grads, then dspark_loss_bwd: a single chunk is reused from the
    workspace, several are recomputed."""
    from speculative_decoding_draft_vocab_b200 import torch_api
    shape = dict(B=2, N=4, K=7, V=8192) if chunks == 1 else dict(B=4, N=32, K=8, V=2048, prefix=(5, 8))
    inp = make_inputs("lm_head_teacher", device="cuda", seed=47 + chunks, target_hidden_size=192, hidden=128,
                      rank=64, target_vocab=900, markov_std=0.3, grad_scale=0.75, **shape)
    call = torch_api.Call(inp, grads=True)
    fwd_only = torch_api.Call(inp, out=call.out, grads=False)
    call.out.dlogits.fill_(5.0)
    fwd_only.launch()
    call.backward()
    torch.cuda.synchronize()
    assert call.check_status() == 0
    ref = oracle_run(inp)
    _check(inp, call, ref)


def test_lm_head_teacher_config_every_row():
    """4 x 16 x 7 rows, V = 151936, teacher from 4096-wide hidden states, Markov rank
    256 and the confidence head."""
    inp = make_inputs("lm_head_teacher", device="cuda")
    call, ref = _run(inp)
    assert np.all(ref["l1"][ref["rows"]] > 0)


@pytest.mark.parametrize("heads", [False, True])
def test_teacher_from_prenorm_hidden(heads):
    """Pre-norm teacher hidden states: the target's final RMS norm is applied in the
    gather before the teacher GEMM."""
    kw = dict(markov=False, conf=None) if not heads else dict(rank=64, target_vocab=900, markov_std=0.3, hidden=128)
    inp = make_inputs("lm_head_teacher", device="cuda", seed=51 + heads, B=2, N=4, K=7, V=8192,
                      target_hidden_size=256, target_prenorm=True, **kw)
    assert inp.target_norm_weight is not None
    _run(inp)


def test_prenorm_teacher_config_every_row():
    """The lm_head teacher shape (4 x 16 x 7 rows, lm_head 151936 x 4096) with pre-norm
    4096-wide hidden states."""
    inp = make_inputs("lm_head_teacher", device="cuda", seed=53, target_prenorm=True)
    _run(inp)
