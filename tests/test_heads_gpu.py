"""GPU parity of the Markov head and the confidence head (forward, dlogits and every
weight gradient) against the FP64 oracle.

The head gradients dW2 = sum_r dz_r (x) e_r and dE_r = W2^T dz_r are contracted on the
tensor cores from the bf16 dlogits the sweep writes, so they carry the bf16 rounding of
dz (unit roundoff u = 2^-8, one rounding per element, errors independent across
elements).  Their tolerance is derived from that: the error of a sum of n rounded
products is bounded in distribution by u/sqrt(3) * sqrt(sum_k (dz_k x_k)^2); the tests
allow 4u * sqrt(sum_k (dz_k x_k)^2), about seven standard deviations, plus 1e-5 of the
magnitude for FP32 accumulation.  A vocabulary entry j where some row's sign(p_j - q_j)
is undecided at FP32 precision (either sign is a valid sub-gradient) is left out of the
element-wise check of dW2 (and a row with such an entry out of the check of dE); those
are counted, must be rare, and the whole matrix must still agree to 2e-3 in relative
Frobenius norm.
"""

import numpy as np
import pytest
import torch

from oracle import dspark_oracle as O
from speculative_decoding_draft_vocab_b200.synthetic import make_inputs
from tests.parity_util import compare, np32, oracle_run, round_to, bf16_ulp

pytestmark = pytest.mark.gpu

U_BF16 = 2.0 ** -8


@pytest.fixture(scope="module", autouse=True)
def _built():
    from speculative_decoding_draft_vocab_b200 import build
    build.build()
    assert torch.cuda.is_available(), "the GPU tests need a CUDA device"


def _call(inp, mode=0, grads=True, accumulate=False):
    from speculative_decoding_draft_vocab_b200 import torch_api
    call = torch_api.Call(inp, grads=grads, invalid_row_mode=mode, accumulate=accumulate)
    return call


def _live_rows(inp, ref):
    valid = np32(inp.valid).reshape(-1)
    sup = ref["rows"]
    return np.array([int(r) for r in sup if valid[r] != 0], dtype=np.int64)


def _frob_rel(got, want):
    n = np.linalg.norm(want)
    return np.linalg.norm(got - want) / n if n > 0 else np.linalg.norm(got)


def check_heads(inp, call, ref, mode, elementwise=True):
    """Confidence logits, dL/dc and the head weight gradients of a finished call.
    ``elementwise`` False (the oracle returned dlogits for a sample of rows only)
    checks dW1 and dW2 in relative Frobenius norm alone."""
    out = call.out
    R = inp.R
    valid = np32(inp.valid).reshape(-1)
    # confidence logits of every row (0 on invalid slots)
    if inp.conf_w is not None:
        c = out.conf_rows.cpu().double().numpy()
        np.testing.assert_allclose(c, ref["conf"], rtol=1e-4, atol=1e-5)
    np.testing.assert_allclose(out.dconf.cpu().double().numpy(), ref["dconf"], rtol=1e-4, atol=2e-6)
    live = _live_rows(inp, ref)
    amb_cols = np.zeros(inp.V, dtype=bool)
    amb_rows = set()
    for r in live:
        a = ref["sign_amb"].get(int(r))
        if a is not None and a.any():
            amb_cols |= a
            amb_rows.add(int(r))
    stats = {}
    if inp.markov_w2 is not None and not elementwise:
        assert _frob_rel(out.dW2.cpu().double().numpy(), ref["dW2"]) <= 2e-3
        gotw1 = out.dW1.cpu().double().numpy()
        ids = sorted(ref["dW1"])
        assert _frob_rel(gotw1[ids], np.stack([ref["dW1"][i] for i in ids])) <= 2e-3
        untouched = np.ones(gotw1.shape[0], dtype=bool)
        untouched[ids] = False
        assert np.all(gotw1[untouched] == 0.0)
    elif inp.markov_w2 is not None:
        w2 = np32(inp.markov_w2).astype(np.float64)
        prev = np32(inp.prev_ids).reshape(-1).astype(np.int64)
        e_live = O.markov_embedding(prev[live], np32(inp.markov_w1)) if len(live) else np.zeros((0, w2.shape[1]))
        Dz = np.stack([ref["dlogits"][int(r)] for r in live]) if len(live) else np.zeros((0, inp.V))
        # dW2
        got = out.dW2.cpu().double().numpy()
        want = ref["dW2"]
        bound = 4 * U_BF16 * np.sqrt((Dz ** 2).T @ (e_live ** 2)) + 1e-5 * np.abs(want) + 1e-7 * np.abs(want).max()
        bad = (np.abs(got - want) > bound) & ~amb_cols[:, None]
        assert not bad.any(), f"dW2: {int(bad.sum())} entries off; worst {np.max(np.abs(got - want) - bound)}"
        assert _frob_rel(got, want) <= 2e-3
        stats["dW2_amb_cols"] = int(amb_cols.sum())
        # dW1: sums of dE over rows sharing a previous token
        gotw1 = out.dW1.cpu().double().numpy()
        proj_e = None
        if inp.conf_w is not None and inp.conf_with_markov:
            proj_e = np32(inp.conf_w).reshape(-1).astype(np.float64)[inp.draft_hidden.shape[-1]:]
        bound_e = {}
        for i, r in enumerate(live):
            b = 4 * U_BF16 * np.sqrt((Dz[i] ** 2) @ (w2 ** 2))
            if proj_e is not None:
                b = b + 1e-5 * np.abs(ref["dconf"][r] * proj_e)
            pid = int(prev[r])
            bound_e[pid] = bound_e.get(pid, 0.0) + b
        skip_ids = {int(prev[r]) for r in amb_rows}
        touched = np.zeros(gotw1.shape[0], dtype=bool)
        for pid, want_row in ref["dW1"].items():
            touched[pid] = True
            err = np.abs(gotw1[pid] - want_row)
            tol = bound_e[pid] + 1e-5 * np.abs(want_row) + 1e-9
            if pid not in skip_ids:
                assert np.all(err <= tol), f"dW1[{pid}]: worst {np.max(err - tol)}"
        assert np.all(gotw1[~touched] == 0.0), "dW1 rows of untouched ids must stay zero"
        if ref["dW1"]:
            ids = sorted(ref["dW1"])
            assert _frob_rel(gotw1[ids], np.stack([ref["dW1"][i] for i in ids])) <= 2e-3
        stats["dE_amb_rows"] = len(amb_rows)
    if inp.conf_w is not None:
        H = inp.draft_hidden.shape[-1]
        h = np32(inp.draft_hidden).reshape(R, H).astype(np.float64)
        sup = np.zeros(R, dtype=bool)
        sup[ref["rows"]] = True
        dcl = np.where(sup & (valid != 0), ref["dconf"], 0.0)
        x = h
        if inp.conf_with_markov:
            prev = np32(inp.prev_ids).reshape(-1).astype(np.int64)
            e_all = np.zeros((R, inp.markov_w1.shape[1]))
            lv = np.nonzero(sup & (valid != 0))[0]
            e_all[lv] = O.markov_embedding(prev[lv], np32(inp.markov_w1))
            x = np.concatenate([h, e_all], axis=1)
        got = out.dconf_w.cpu().double().numpy()
        tol = 1e-4 * (np.abs(dcl) @ np.abs(x)) + 1e-9
        assert np.all(np.abs(got - ref["dconf_w"]) <= tol), np.max(np.abs(got - ref["dconf_w"]) - tol)
        gb = float(out.dconf_b.item())
        assert abs(gb - ref["dconf_b"]) <= 1e-4 * np.sum(np.abs(dcl)) + 1e-9
        dh = out.dhidden.float().cpu().double().numpy().reshape(R, H)
        want = ref["dhidden"]
        want_o = round_to(want, "bf16")
        tol = np.maximum(1e-4 * np.abs(want_o), bf16_ulp(want_o)) + 1e-12
        assert np.all(np.abs(dh - want_o) <= tol)
    return stats


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
    assert st["dW2_amb_cols"] < 2000 and st["dE_amb_rows"] <= inp.R


def test_recipe_heads_visible_correction():
    """The same shape with Markov tables large enough to move the logits by O(1)."""
    inp = make_inputs("recipe_heads", device="cuda", seed=37, markov_std=0.25, conf_bias=0.3)
    _run(inp, 1)


def test_large_config():
    """8 x 64 x 16 rows (8192), V = 151936, heads on, ragged prefixes with empty blocks.
    The oracle runs on every row (report, per-row terms, dL/dc, every weight
    gradient); dlogits are compared on 256 sampled supervised rows plus every row of
    the first four blocks, and every unsupervised row must be exactly zero."""
    inp = make_inputs("large", device="cuda")
    call = _call(inp, 0)
    call.launch()
    torch.cuda.synchronize()
    assert call.check_status() == 0
    m = O.prefix_supervision_mask(np32(inp.eval_mask), np32(inp.block_keep)).reshape(-1)
    sup = np.nonzero(m)[0]
    rng = np.random.default_rng(5)
    sample = sorted(set(rng.choice(sup, size=min(256, len(sup)), replace=False).tolist())
                    | {int(r) for r in sup if r < 4 * inp.K})
    ref = oracle_run(inp, keep_rows=sample)
    compare(inp, call, ref)
    check_heads(inp, call, ref, 0, elementwise=False)
    assert ref["report"]["tau"][1] < inp.B * inp.N  # some blocks are empty
