"""GPU parity of the Markov head and the confidence head (forward, dlogits and every
weight gradient) against the FP64 oracle; the tolerances of the weight gradients are
derived in tests/parity_util.py."""

import numpy as np
import pytest
import torch

from oracle import dspark_oracle as O
from speculative_decoding_draft_vocab_b200.synthetic import make_inputs
from tests.parity_util import check_heads, compare, np32, oracle_run

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from speculative_decoding_draft_vocab_b200 import build
    build.build()
    assert torch.cuda.is_available(), "the GPU tests need a CUDA device"


def _call(inp, mode=0, grads=True, accumulate=False):
    from speculative_decoding_draft_vocab_b200 import torch_api
    call = torch_api.Call(inp, grads=grads, invalid_row_mode=mode, accumulate=accumulate)
    return call


def _run(inp, mode=0):
    call = _call(inp, mode)
    call.launch()
    torch.cuda.synchronize()
    assert call.check_status() == 0
    ref = oracle_run(inp, invalid_row_mode=mode)
    compare(inp, call, ref)
    return call, ref, check_heads(inp, call, ref, mode)


SMALL = dict(B=2, N=4, K=7, V=8192, hidden=512, rank=64, target_vocab=3000, markov_std=0.3,
             conf_bias=0.25, valid_p=0.7, mask_holes=True)


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("with_markov", [True, False])
def test_heads_small(mode, with_markov):
    """Both invalid-row readings, confidence input with and without the Markov
    embedding; previous ids of invalid slots set to -1 (they must not be read)."""
    inp = make_inputs("recipe_heads", device="cuda", seed=21 + mode + 2 * with_markov,
                      conf_with_markov=with_markov, **SMALL)
    inp.prev_ids = torch.where(inp.valid != 0, inp.prev_ids, torch.full_like(inp.prev_ids, -1))
    _run(inp, mode)


def test_heads_ragged_rank_and_sizes():
    """rank 72 (a ragged tensor-core tile), V = 5000, hidden 200, 3 x 5 x 6 rows."""
    inp = make_inputs("recipe_heads", device="cuda", seed=31, B=3, N=5, K=6, V=5000, hidden=200, rank=72,
                      target_vocab=777, markov_std=0.3, conf_bias=-0.5, valid_p=0.8)
    _run(inp, 0)


def test_confidence_head_without_markov():
    inp = make_inputs("recipe", device="cuda", seed=32, B=2, N=4, K=7, V=4096, conf="head", hidden=256,
                      conf_bias=0.1)
    _run(inp, 0)


def test_markov_head_without_confidence():
    inp = make_inputs("recipe_heads", device="cuda", seed=33, B=2, N=4, K=7, V=12288, conf=None, rank=128,
                      target_vocab=500, markov_std=0.3)
    _run(inp, 0)


def test_markov_head_ce_only():
    """No teacher: the corrected rows feed CE alone."""
    inp = make_inputs("recipe_heads", device="cuda", seed=34, B=2, N=3, K=7, V=4096, conf=None, rank=64,
                      markov_std=0.3, no_target=True)
    _run(inp, 0)


def test_separate_backward_with_heads():
    """Forward without grads, then dspark_loss_bwd from the saved corrected rows."""
    inp = make_inputs("recipe_heads", device="cuda", seed=35, grad_scale=0.5, **SMALL)
    from speculative_decoding_draft_vocab_b200 import torch_api
    call = _call(inp, 0)
    fwd_only = torch_api.Call(inp, out=call.out, grads=False)
    call.out.dlogits.fill_(3.0)
    fwd_only.launch()
    call.backward()
    torch.cuda.synchronize()
    assert call.check_status() == 0
    ref = oracle_run(inp)
    compare(inp, call, ref)
    check_heads(inp, call, ref, 0)


def test_weight_gradients_accumulate():
    """accumulate=1: dW2, dconf_w and dconf_b add to what is there; dW1 always adds."""
    inp = make_inputs("recipe_heads", device="cuda", seed=36, **SMALL)
    one = _call(inp)
    one.launch()
    two = _call(inp, accumulate=True)
    two.launch()
    two.launch()
    torch.cuda.synchronize()
    for name in ("dW1", "dW2", "dconf_w", "dconf_b"):
        a, b = getattr(one.out, name), getattr(two.out, name)
        assert torch.allclose(b, 2 * a, rtol=1e-5, atol=1e-7), name
    # overwrite mode: a second call leaves dW2, dconf_w, dconf_b as after one call,
    # while dW1 keeps adding
    kept = {n: getattr(one.out, n).clone() for n in ("dW2", "dconf_w", "dconf_b")}
    one.launch()
    torch.cuda.synchronize()
    for n, v in kept.items():
        assert torch.equal(getattr(one.out, n), v), n
    assert torch.allclose(one.out.dW1, two.out.dW1, rtol=1e-5, atol=1e-7)


def test_recipe_heads_every_row():
    """4 x 16 x 7 rows, V = 151936, rank 256, hidden 4096, init-scale weights."""
    inp = make_inputs("recipe_heads", device="cuda")
    _, _, st = _run(inp, 0)
    assert st["dW2_frob_err"] <= 1.0 and st["dW1_frob_err"] <= 1.0


def test_recipe_heads_visible_correction():
    """The same shape with Markov tables large enough to move the logits by O(1)."""
    inp = make_inputs("recipe_heads", device="cuda", seed=37, markov_std=0.25, conf_bias=0.3)
    _run(inp, 1)


def test_large_config():
    """8 x 64 x 16 rows (8192), V = 151936, heads on, ragged prefixes with empty blocks.
    The oracle runs on every row (report, per-row terms, dL/dc, every weight gradient,
    dW2 and dW1 checked element-wise); dlogits are compared on every row of 64 whole
    blocks drawn at random and on 1024 more supervised rows drawn at random (the oracle
    run a chunk of rows at a time: rows are independent), and every unsupervised row must
    be exactly zero."""
    from tests.parity_util import check_dlogit_row
    inp = make_inputs("large", device="cuda")
    call = _call(inp, 0)
    call.launch()
    torch.cuda.synchronize()
    assert call.check_status() == 0
    m = O.prefix_supervision_mask(np32(inp.eval_mask), np32(inp.block_keep)).reshape(-1)
    sup = np.nonzero(m)[0]
    rng = np.random.default_rng(5)
    blocks = rng.choice(inp.B * inp.N, size=64, replace=False)
    in_blocks = {int(b) * inp.K + k for b in blocks for k in range(inp.K)}
    extra = set(rng.choice(sup, size=min(1024, len(sup)), replace=False).tolist())
    rows = sorted(r for r in (in_blocks | extra) if m[r])
    ref = oracle_run(inp, keep_rows=rows[:64])
    compare(inp, call, ref)
    check_heads(inp, call, ref, 0, elementwise=True)
    g = call.out.dlogits.view(inp.R, inp.V)
    for c0 in range(64, len(rows), 128):
        chunk = rows[c0:c0 + 128]
        part = oracle_run(inp, rows=np.array(chunk), keep_rows=chunk)
        for r in chunk:
            check_dlogit_row(g[r].float().cpu().double().numpy(), part["dlogits"][r], part["sign_amb"][r],
                             inp.dtype, tag=f"row {r}")
    unsup_in_blocks = [r for r in in_blocks if not m[r]]
    if unsup_in_blocks:
        assert bool((g[torch.tensor(unsup_in_blocks, device=g.device)] == 0).all())
    assert ref["report"]["tau"][1] < inp.B * inp.N  # some blocks are empty
