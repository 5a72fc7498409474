"""Pins for the FP64 oracle: facts fixed by the pages and by mathematics, not by the
oracle's own formulas.  CPU only.

Each test states what it pins.  Together they are chosen so that a plausible slip
in the oracle (a dropped term, a wrong sign or index, a transposed operand, the
rejected 1/2 factor) fails at least one of them; ``test_planted_mistakes`` plants
such slips in the oracle and checks that.
"""

import json
import math
import os

import numpy as np
import scipy.special
import pytest

from oracle import dspark_oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "pages_values.json")


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


def _rand_problem(rng, B=2, N=3, K=4, V=24, scale=2.0, full=True):
    draft = rng.normal(0, scale, (B, N, K, V))
    target = draft * 0.7 + rng.normal(0, 1.0, (B, N, K, V))
    ids = rng.integers(0, V, (B, N, K))
    if full:
        ev = np.ones((B, N, K), dtype=np.uint8)
    else:
        L = rng.integers(0, K + 1, (B, N))
        ev = (np.arange(K)[None, None, :] < L[..., None]).astype(np.uint8)
    return draft, target, ids, ev


# ------------------------------------------------------------------ masks / weights
def test_prefix_mask_matches_leading_run_brute_force():
    """m is 1 exactly on the leading run of ones of each block (pure-Python scan)."""
    rng = np.random.default_rng(0)
    ev = (rng.random((5, 7, 9)) < 0.7).astype(np.uint8)
    keep = (rng.random((5, 7)) < 0.8).astype(np.uint8)
    m = O.prefix_supervision_mask(ev, keep)
    for b in range(5):
        for n in range(7):
            alive = keep[b, n] == 1
            for k in range(9):
                alive = alive and ev[b, n, k] == 1
                assert m[b, n, k] == (1 if alive else 0)
    assert m.dtype == np.int64


def test_weights_slot0_is_one_and_decay_ratio_constant():
    """Slot 0 (the first prediction) has weight 1; each later slot is exp(-1/gamma)
    times the previous one; gamma=None gives the bare mask."""
    m = np.ones((1, 1, 7), dtype=np.int64)
    w = O.loss_weights(m, 4.0)
    assert w[0, 0, 0] == 1.0
    ratios = w[0, 0, 1:] / w[0, 0, :-1]
    assert np.allclose(ratios, math.exp(-0.25), rtol=1e-15, atol=0)
    assert np.array_equal(O.loss_weights(m, None), m.astype(np.float64))
    m2 = np.array([[[1, 1, 0, 0]]])
    assert np.array_equal(O.loss_weights(m2, 2.0)[0, 0, 2:], [0.0, 0.0])


# ---------------------------------------------------------------- row-term identities
def test_identical_rows_give_zero_l1_accept_one_tau_k_plus_one():
    """Identical draft and teacher: L1 = 0, accept = 1, tau = K + 1 on a full mask and
    the BCE reduces to log(1 + exp(-c)) (label 1)."""
    rng = np.random.default_rng(1)
    B, N, K, V = 2, 2, 5, 40
    d = rng.normal(0, 3, (B, N, K, V))
    c = rng.normal(0, 1, (B, N, K))
    ids = rng.integers(0, V, (B, N, K))
    res = O.dspark_loss(d, ids, np.ones((B, N, K)), target_logits=d.copy(), confidence_logits=c)
    assert np.all(res["l1"] == 0.0)
    assert np.all(res["accept"] == 1.0)
    assert np.all(res["tau_blocks"] == K + 1)
    bce_ref = np.array([math.log1p(math.exp(-x)) for x in c.reshape(-1)])
    assert np.allclose(res["bce"], bce_ref, rtol=1e-14, atol=1e-15)


def test_disjoint_saturated_rows_match_the_pages_values():
    """Two disjoint saturated distributions: raw L1 = 2.0 (TV 1.0), accept 0, tau 1,
    and BCE(c, 0) = log(1 + exp(c)).  The L1 and TV values are the ones printed by the
    pages; the training term keeps the raw L1."""
    g = _golden()["disjoint_saturated"]
    V, K = 16, 3
    d = np.full((1, 1, K, V), -100.0)
    t = np.full((1, 1, K, V), -100.0)
    for k in range(K):
        d[0, 0, k, k] = 100.0
        t[0, 0, k, k + 5] = 100.0
    c = np.array([[[0.3, -1.2, 2.0]]])
    res = O.dspark_loss(d, np.zeros((1, 1, K), dtype=np.int64), np.ones((1, 1, K)),
                        target_logits=t, confidence_logits=c, gamma=None)
    assert np.allclose(res["l1"], g["raw_l1"], rtol=0, atol=1e-12)
    assert np.allclose(0.5 * res["l1"], g["total_variation"], rtol=0, atol=1e-12)
    assert np.allclose(res["accept"], 0.0, atol=1e-12)
    assert res["tau_blocks"][0, 0] == pytest.approx(1.0, abs=1e-12)
    sp = np.array([math.log1p(math.exp(x)) for x in c.reshape(-1)])
    assert np.allclose(res["bce"], sp, rtol=1e-12)
    # the l1 report numerator carries the raw L1 (weights 1 with gamma None)
    assert res["report"]["l1"][0] == pytest.approx(2.0 * K, abs=1e-10)


def test_l1_closed_forms_uniform_vs_onehot_and_two_point():
    """Uniform draft against a saturated one-hot teacher: L1 = 2 (1 - 1/V).
    V = 2: L1 = 2 |sigmoid(z0 - z1) - sigmoid(t0 - t1)|."""
    for V in (2, 7, 100):
        z = np.zeros(V)
        t = np.full(V, -800.0)
        t[3 % V] = 0.0
        rt = O.row_terms(z, t, 0)
        assert rt["l1"] == pytest.approx(2.0 * (1.0 - 1.0 / V), rel=1e-13)
    rng = np.random.default_rng(2)
    for _ in range(20):
        z = rng.normal(0, 2, 2)
        t = rng.normal(0, 2, 2)
        s = lambda x: 1.0 / (1.0 + math.exp(-x))
        rt = O.row_terms(z, t, 1)
        assert rt["l1"] == pytest.approx(2 * abs(s(z[0] - z[1]) - s(t[0] - t[1])), rel=1e-12)


def test_ce_matches_brute_force_negative_log_softmax():
    """CE = -log(exp(z_tid) / sum_j exp(z_j)), summed with math.fsum and no shift;
    uniform logits give CE = log V."""
    rng = np.random.default_rng(3)
    for V in (5, 33, 257):
        z = rng.normal(0, 2, V)
        tid = int(rng.integers(0, V))
        ref = -math.log(math.exp(z[tid]) / math.fsum(math.exp(x) for x in z))
        assert O.row_terms(z, None, tid)["ce"] == pytest.approx(ref, rel=1e-13, abs=1e-13)
        assert O.row_terms(np.full(V, 1.7), None, tid)["ce"] == pytest.approx(math.log(V), rel=1e-14)


def test_bounds_on_random_rows():
    """0 <= L1 <= 2, 0 <= accept <= 1, 1 <= tau <= K + 1, CE >= 0."""
    rng = np.random.default_rng(4)
    d, t, ids, ev = _rand_problem(rng, B=3, N=4, K=6, V=50, full=False)
    res = O.dspark_loss(d, ids, ev, target_logits=t)
    sup = res["m"] == 1
    assert np.all(res["l1"][sup] >= 0) and np.all(res["l1"][sup] <= 2)
    assert np.all(res["ce"][sup] >= 0)
    assert np.all((res["accept"] >= 0) & (res["accept"] <= 1))
    assert np.all((res["tau_blocks"] >= 1) & (res["tau_blocks"] <= 7))


# ------------------------------------------------------------------------ acceptance
@pytest.mark.parametrize("K", [1, 4, 7, 16])
def test_tau_constant_accept_closed_form(K):
    """Constant accept a on a full mask: tau = 1 + sum_{k=1..K} a^k
    = (1 - a^(K+1)) / (1 - a); K = 1 gives 1 + a."""
    for a in (0.0, 0.3, 0.77, 1.0):
        l1 = np.full((2, 3, K), 2 * (1 - a))
        rep = O.acceptance_report(l1, np.ones((2, 3, K), dtype=np.int64))
        ref = K + 1.0 if a == 1.0 else (1 - a ** (K + 1)) / (1 - a)
        assert np.allclose(rep["tau_blocks"], ref, rtol=1e-14)
        assert rep["tau"][1] == 6.0
        assert rep["tau"][0] == pytest.approx(6 * ref, rel=1e-13)
        assert rep["accept"] == pytest.approx((6 * K * a, 6 * K), rel=1e-13, abs=1e-13)


def test_tau_stops_at_first_unsupervised_slot_and_keep_weights():
    """A masked slot ends the running product; dropped blocks leave both tau terms."""
    l1 = np.zeros((1, 2, 4))
    m = np.array([[[1, 1, 0, 0], [1, 1, 1, 1]]])
    rep = O.acceptance_report(l1, m, block_keep=np.array([[1, 0]]))
    assert rep["tau_blocks"][0, 0] == 3.0 and rep["tau_blocks"][0, 1] == 5.0
    assert rep["tau"] == (3.0, 1.0)


# ------------------------------------------------------------------------ masking
def test_all_masked_batch_contributes_nothing():
    rng = np.random.default_rng(5)
    d, t, ids, _ = _rand_problem(rng)
    res = O.dspark_loss(d, ids, np.zeros(ids.shape), target_logits=t,
                        confidence_logits=rng.normal(size=ids.shape))
    assert res["loss_num"] == 0.0 and res["num_tokens"] == 0
    assert res["dlogits"] == {} and np.all(res["dconf"] == 0)
    assert all(res["report"][k][0] == 0.0 for k in ("loss", "ce", "l1", "conf", "accept"))
    # every block still scores its verified anchor: tau = 1 per kept block
    assert res["report"]["tau"] == (float(ids.shape[0] * ids.shape[1]),) * 2


def test_masked_inputs_do_not_leak():
    """NaN/Inf in unsupervised rows never reach the sums (masked rows are skipped)."""
    rng = np.random.default_rng(6)
    d, t, ids, ev = _rand_problem(rng, full=False)
    ev[0, 0, :] = 0
    d[0, 0] = np.nan
    t[0, 0] = np.inf
    res = O.dspark_loss(d, ids, ev, target_logits=t)
    assert np.isfinite(res["loss_num"]) and all(np.isfinite(v[0]) for v in res["report"].values())


def test_no_teacher_means_ce_only_and_errors_otherwise():
    rng = np.random.default_rng(7)
    d, _, ids, ev = _rand_problem(rng)
    res = O.dspark_loss(d, ids, ev, l1_alpha=0.0)
    assert np.all(res["l1"] == 0) and np.all(res["accept"] == 1.0)
    with pytest.raises(ValueError):
        O.dspark_loss(d, ids, ev)
    with pytest.raises(ValueError):
        O.dspark_loss(d, ids, ev, l1_alpha=0.0, confidence_logits=np.zeros(ids.shape))


def test_report_never_divides_and_microbatches_add_up():
    """Splitting the blocks into micro-batches with unequal token counts and summing the
    pairs reproduces the one-shot pairs, while the mean of per-micro-batch means does
    not (the bias the return contract avoids)."""
    rng = np.random.default_rng(8)
    d, t, ids, ev = _rand_problem(rng, B=4, N=3, K=5, V=20, full=False)
    ev[0] = 1
    ev[1:, :, 1:] = 0
    c = rng.normal(size=ids.shape)
    full = O.dspark_loss(d, ids, ev, target_logits=t, confidence_logits=c)
    parts = [O.dspark_loss(d[i:i + 1], ids[i:i + 1], ev[i:i + 1], target_logits=t[i:i + 1],
                           confidence_logits=c[i:i + 1]) for i in range(4)]
    for key in O.REPORT_KEYS:
        num = sum(p["report"][key][0] for p in parts)
        den = sum(p["report"][key][1] for p in parts)
        assert num == pytest.approx(full["report"][key][0], rel=1e-12, abs=1e-12)
        assert den == full["report"][key][1]
    assert sum(p["num_tokens"] for p in parts) == full["num_tokens"]
    mean_of_means = np.mean([p["loss_num"] / p["num_tokens"] for p in parts])
    assert abs(mean_of_means - full["loss_num"] / full["num_tokens"]) > 1e-3


# -------------------------------------------------------------------------- heads
def test_markov_bias_matches_explicit_loops_and_zero_w2_reduces():
    """z_j = base_j + sum_i W2[j, i] W1[prev, i] (triple loop), invalid rows all zero;
    W2 = 0 gives back the no-Markov loss."""
    rng = np.random.default_rng(9)
    V, r, Vt = 11, 3, 13
    w1 = rng.normal(0, 0.5, (Vt, r))
    w2 = rng.normal(0, 0.5, (V, r))
    base = rng.normal(0, 1, (4, V))
    prev = np.array([0, 12, 5, 5])
    valid = np.array([1, 1, 0, 1])
    z = O.markov_corrected_rows(base, O.markov_embedding(prev, w1), valid, w2)
    for row in range(4):
        for j in range(V):
            ref = 0.0 if not valid[row] else base[row, j] + sum(w2[j, i] * w1[prev[row], i] for i in range(r))
            assert z[row, j] == pytest.approx(ref, abs=1e-14)
    z1 = O.markov_corrected_rows(base, O.markov_embedding(prev, w1), valid, w2, invalid_row_mode=1)
    assert np.array_equal(z1[2], base[2])
    d, t, ids, ev = _rand_problem(rng, B=1, N=2, K=2, V=V)
    pv = rng.integers(0, Vt, ids.shape)
    a = O.dspark_loss(d, ids, ev, target_logits=t, prev_ids=pv, valid=np.ones(ids.shape),
                      markov_w1=w1, markov_w2=np.zeros_like(w2))
    b = O.dspark_loss(d, ids, ev, target_logits=t)
    assert a["loss_num"] == pytest.approx(b["loss_num"], rel=1e-14)


def test_confidence_head_matches_explicit_sum():
    rng = np.random.default_rng(10)
    H, r = 6, 3
    h = rng.normal(size=(5, H))
    e = rng.normal(size=(5, r))
    proj = rng.normal(size=(1, H + r))
    valid = np.array([1, 0, 1, 1, 0])
    c = O.confidence_head_logits(h, e, proj, [0.25], valid)
    for i in range(5):
        ref = 0.0 if not valid[i] else (sum(proj[0, j] * h[i, j] for j in range(H))
                                        + sum(proj[0, H + j] * e[i, j] for j in range(r)) + 0.25)
        assert c[i] == pytest.approx(ref, abs=1e-14)


def test_bce_special_values_and_derivative():
    assert O.bce_with_logits(0.0, 0.37) == pytest.approx(math.log(2.0), rel=1e-15)
    for c in (-3.0, -0.2, 0.0, 1.5, 30.0):
        for y in (0.0, 0.25, 1.0):
            h = 1e-6
            fd = (O.bce_with_logits(c + h, y) - O.bce_with_logits(c - h, y)) / (2 * h)
            assert fd == pytest.approx(1.0 / (1.0 + math.exp(-c)) - y, abs=1e-8)


# ---------------------------------------------------------------- gradients
def test_gradient_row_sums_vanish():
    """sum_j dCE/dz_j = 0 and sum_j dL1/dz_j = 0 (softmax calculus)."""
    rng = np.random.default_rng(11)
    d, t, ids, ev = _rand_problem(rng, V=64)
    for ce_a, l1_a in ((1.0, 0.0), (0.0, 1.0), (0.1, 0.9)):
        res = O.dspark_loss(d, ids, ev, target_logits=t, ce_alpha=ce_a, l1_alpha=l1_a)
        for row in res["dlogits"].values():
            assert abs(row.sum()) < 1e-14


def _fd_problem(seed=12, markov=True, conf="head"):
    rng = np.random.default_rng(seed)
    B, N, K, V, r, H = 1, 2, 3, 9, 3, 5
    d, t, ids, ev = _rand_problem(rng, B, N, K, V, scale=1.5)
    ev[0, 1, 2] = 0
    kw = dict(target_logits=t, gamma=4.0, grad_scale=0.7, ce_alpha=0.3, l1_alpha=0.9, conf_alpha=1.1)
    if markov:
        kw.update(prev_ids=rng.integers(0, 7, ids.shape), valid=np.array([[[1, 1, 0], [1, 1, 1]]]),
                  markov_w1=rng.normal(0, 0.4, (7, r)), markov_w2=rng.normal(0, 0.4, (V, r)))
    if conf == "head":
        kw.update(draft_hidden=rng.normal(size=(B, N, K, H)), conf_w=rng.normal(0, 0.3, (1, H + (r if markov else 0))),
                  conf_b=np.array([0.1]), conf_with_markov=markov)
        if not markov:
            kw["valid"] = np.array([[[1, 1, 0], [1, 1, 1]]])
    elif conf == "given":
        kw["confidence_logits"] = rng.normal(size=ids.shape)
    return d, ids, ev, kw


def _central(f, x, idx, h=1e-6):
    old = x[idx]
    x[idx] = old + h
    fp = f()
    x[idx] = old - h
    fm = f()
    x[idx] = old
    return (fp - fm) / (2 * h)


@pytest.mark.parametrize("markov,conf", [(False, "given"), (True, "head"), (False, "head"), (True, None)])
def test_finite_differences_all_gradients(markov, conf):
    """Central differences of grad_scale * loss (BCE label held fixed, as detached)
    against dlogits, dconf, dW1, dW2, dconf_w, dconf_b and dhidden."""
    d, ids, ev, kw = _fd_problem(markov=markov, conf=conf)
    base = O.dspark_loss(d, ids, ev, **kw)
    y0 = base["label"]
    g = kw["grad_scale"]

    def L():
        return g * O.dspark_loss(d, ids, ev, want_grads=False, fixed_label=y0, **kw)["loss_num"]

    R = ids.size
    V = d.shape[-1]
    # no ties anywhere (the L1 is smooth there)
    for r, amb in base["sign_amb"].items():
        assert not amb.any()
    dfl = d.reshape(R, V)
    for r in range(R):
        for j in range(V):
            fd = _central(L, d.reshape(-1), r * V + j)
            an = base["dlogits"].get(r, np.zeros(V))[j]
            assert fd == pytest.approx(an, abs=2e-8), (r, j)
    if conf == "given":
        c = kw["confidence_logits"]
        for r in range(R):
            fd = _central(L, c.reshape(-1), r)
            assert fd == pytest.approx(base["dconf"][r], abs=2e-8)
    if markov:
        w2, w1 = kw["markov_w2"], kw["markov_w1"]
        for idx in np.ndindex(w2.shape):
            assert _central(L, w2, idx) == pytest.approx(base["dW2"][idx], abs=2e-8)
        for idx in np.ndindex(w1.shape):
            an = base["dW1"].get(idx[0], np.zeros(w1.shape[1]))[idx[1]]
            assert _central(L, w1, idx) == pytest.approx(an, abs=2e-8)
    if conf == "head":
        pw, pb, h = kw["conf_w"], kw["conf_b"], kw["draft_hidden"]
        for idx in np.ndindex(pw.shape):
            assert _central(L, pw, idx) == pytest.approx(base["dconf_w"][idx[1]], abs=2e-8)
        assert _central(L, pb, (0,)) == pytest.approx(base["dconf_b"], abs=2e-8)
        hr = h.reshape(R, -1)
        for r in range(R):
            for j in range(hr.shape[1]):
                assert _central(L, h.reshape(-1), r * hr.shape[1] + j) == pytest.approx(
                    base["dhidden"][r, j], abs=2e-8)
    del dfl


def test_teacher_from_hidden_equals_given_teacher():
    rng = np.random.default_rng(13)
    B, N, K, V, Ht = 1, 2, 3, 10, 6
    h = rng.normal(size=(B, N, K, Ht))
    lm = rng.normal(0, 0.5, (V, Ht))
    t = np.einsum("bnkh,vh->bnkv", h, lm)
    d, _, ids, ev = _rand_problem(rng, B, N, K, V)
    a = O.dspark_loss(d, ids, ev, target_hidden=h, lm_head=lm)
    b = O.dspark_loss(d, ids, ev, target_logits=t)
    assert a["loss_num"] == pytest.approx(b["loss_num"], rel=1e-13)
    for r in a["dlogits"]:
        assert np.allclose(a["dlogits"][r], b["dlogits"][r], rtol=1e-12, atol=1e-15)


def test_reference_scale_tensor_size_from_pages():
    """The pages' 2.03 GiB for one FP32 [.., 512, 7, vocab] tensor pins vocab ~ 151936."""
    g = _golden()["reference_scale_fp32_tensor_gib"]
    gib = g["num_blocks"] * g["block_size"] * g["vocab"] * 4 / 2 ** 30
    assert round(gib, 2) == g["value"]

def _bf16(x):
    import torch
    return torch.from_numpy(np.asarray(x, dtype=np.float64)).to(torch.bfloat16).double().numpy()


def test_target_final_norm_closed_forms():
    """RMS norm: a constant row c*1 normalises to sign(c) * w (eps = 0); with w = 1 and
    eps = 0 every row has unit mean square (to bf16 rounding); scaling a row by a power
    of two changes nothing; an all-zero row stays zero with eps > 0."""
    rng = np.random.default_rng(31)
    Ht = 64
    w = _bf16(rng.normal(1.0, 0.2, Ht))
    for c in (3.0, -0.25, 17.5):
        y = O.target_final_norm(np.full((1, Ht), c), w, 0.0)
        np.testing.assert_array_equal(y[0], np.sign(c) * w)
    x = rng.normal(0, 2.0, (5, Ht))
    y = O.target_final_norm(x, np.ones(Ht), 0.0)
    np.testing.assert_allclose(np.mean(y * y, axis=1), 1.0, rtol=2 * 2.0 ** -8)
    np.testing.assert_array_equal(O.target_final_norm(4.0 * x, w, 0.0), O.target_final_norm(x, w, 0.0))
    np.testing.assert_array_equal(O.target_final_norm(np.zeros((2, Ht)), w, 1e-6), 0.0)
    # by hand for one row: w * x / sqrt(mean(x^2) + eps), rounded to bf16
    xr = np.array([[1.0, -2.0, 3.0, 0.5]])
    wr = np.array([1.0, 0.5, 2.0, -1.0])
    ms = (1.0 + 4.0 + 9.0 + 0.25) / 4.0
    want = _bf16(wr * xr[0] / math.sqrt(ms + 0.1))
    np.testing.assert_array_equal(O.target_final_norm(xr, wr, 0.1)[0], want)


def test_teacher_from_prenorm_hidden_equals_normed_teacher():
    """The loss on pre-norm hidden states with the norm weight equals the loss on the
    normed states given directly."""
    rng = np.random.default_rng(32)
    B, N, K, V, Ht = 1, 2, 3, 12, 16
    h = rng.normal(0, 3.0, (B, N, K, Ht))
    w = _bf16(rng.normal(1.0, 0.3, Ht))
    lm = rng.normal(0, 0.3, (V, Ht))
    d, _, ids, ev = _rand_problem(rng, B, N, K, V)
    a = O.dspark_loss(d, ids, ev, target_hidden=h, lm_head=lm, target_norm_weight=w, target_norm_eps=1e-5)
    hn = O.target_final_norm(h.reshape(-1, Ht), w, 1e-5).reshape(h.shape)
    b = O.dspark_loss(d, ids, ev, target_hidden=hn, lm_head=lm)
    assert a["loss_num"] == b["loss_num"]
    for r in a["dlogits"]:
        np.testing.assert_array_equal(a["dlogits"][r], b["dlogits"][r])


# ------------------------------------------------------ vocabulary-parallel form
def _random_bounds(rng, V, T):
    """T contiguous shards of [0, V), some of them empty."""
    cuts = np.sort(rng.integers(0, V + 1, size=T - 1))
    return [0, *cuts.tolist(), V]


def test_lse_partials_merge_to_library_logsumexp():
    """Shard partials merged in order give scipy's logsumexp of the whole row, for
    rows far from 0, with large spreads, and with empty shards (the merge's identity)."""
    rng = np.random.default_rng(41)
    for V, T, loc, scale in [(1, 1, 0.0, 1.0), (17, 3, -1e4, 3.0), (1000, 8, 80.0, 10.0),
                             (4096, 5, 0.0, 40.0), (333, 16, -50.0, 0.5)]:
        x = loc + scale * rng.standard_normal(V)
        bounds = _random_bounds(rng, V, T)
        parts = [O.lse_partial(x[a:b]) for a, b in zip(bounds[:-1], bounds[1:])]
        want = float(scipy.special.logsumexp(x))
        assert abs(O.merge_lse_partials(parts) - want) <= 1e-12 * max(1.0, abs(want))
        assert O.merge_lse_partials(parts + [(-math.inf, 0.0)]) == O.merge_lse_partials(parts)
    assert O.lse_partial(np.zeros(0)) == (-math.inf, 0.0)
    # two equal halves: log(2) above each half's logsumexp
    h = rng.standard_normal(64)
    one = O.lse_partial(h)
    assert abs(O.merge_lse_partials([one, one]) - (scipy.special.logsumexp(h) + math.log(2.0))) <= 1e-12


def test_tp_row_terms_closed_forms():
    """Disjoint saturated rows in different shards: L1 = 2, S = 1.  Identical rows:
    L1 = 0, S = 0.  A flat draft row against a saturated teacher: L1 = 2 (1 - 1/V)."""
    V = 96
    z = np.full(V, -60.0); z[5] = 60.0
    t = np.full(V, -60.0); t[70] = 60.0
    for bounds in ([0, 32, 64, 96], [0, 6, 6, 96], [0, 96]):
        r = O.tp_row_terms(z, t, 5, bounds)
        assert abs(r["l1"] - 2.0) <= 1e-12 and abs(r["S"] - 1.0) <= 1e-12
        assert abs(r["ce"]) <= 1e-12
        r = O.tp_row_terms(z, z.copy(), 70, bounds)
        assert r["l1"] == 0.0 and r["S"] == 0.0 and abs(r["ce"] - 120.0) <= 1e-9
        r = O.tp_row_terms(np.zeros(V), t, 0, bounds)
        assert abs(r["l1"] - 2.0 * (1.0 - 1.0 / V)) <= 1e-12
        assert abs(r["ce"] - math.log(V)) <= 1e-12


def test_tp_row_terms_match_brute_force_for_any_split():
    """Every split of a row (1 to 9 shards, empty ones included) gives the brute-force
    softmax sums of the whole row, written out here without any shift."""
    rng = np.random.default_rng(43)
    for trial in range(20):
        V = int(rng.integers(1, 300))
        z = 2.0 * rng.standard_normal(V)
        t = 0.8 * z + 1.5 * rng.standard_normal(V)
        tid = int(rng.integers(0, V))
        ez, et = np.exp(z), np.exp(t)
        p, q = ez / ez.sum(), et / et.sum()
        l1 = sum(abs(p[j] - q[j]) for j in range(V))
        S = sum(p[j] * np.sign(p[j] - q[j]) for j in range(V))
        ce = -math.log(p[tid])
        for T in (1, 2, 3, 9):
            r = O.tp_row_terms(z, t, tid, _random_bounds(rng, V, T))
            assert abs(r["l1"] - l1) <= 1e-12 and abs(r["S"] - S) <= 1e-12
            assert abs(r["ce"] - ce) <= 1e-11


# --------------------------------------------------------------- planted mistakes
def _mutant_half_l1(z, t, tid, _orig=O.row_terms):
    out = _orig(z, t, tid)
    out["l1"] *= 0.5
    return out


def _mutant_no_S(z, t, tid, _orig=O.row_terms):
    out = _orig(z, t, tid)
    out["S"] = 0.0
    return out


def _mutant_sign_flip(z, t, tid, _orig=O.row_terms):
    out = _orig(z, t, tid)
    if out["s"] is not None:
        out["s"] = -out["s"]
        out["S"] = -out["S"]
    return out


def _mutant_decay_index(m, gamma, _orig=O.loss_weights):
    w = _orig(m, gamma)
    if gamma is None:
        return w
    return w * math.exp(-1.0 / gamma)


def _mutant_w2_transposed(base_rows, e_rows, valid_rows, w2, invalid_row_mode=0,
                          _orig=O.markov_corrected_rows):
    w2 = np.asarray(w2)
    if w2.shape[0] == w2.shape[1]:
        w2 = w2.T
    return _orig(base_rows, e_rows, valid_rows, w2[:, ::-1], invalid_row_mode)


def _mutant_norm_no_square(hidden_rows, weight, eps, _orig=O.target_final_norm):
    x = np.asarray(hidden_rows, dtype=np.float64)
    return _orig(np.abs(x) ** 0.5 * np.sign(x), weight, eps)


def _mutant_merge_no_rescale(parts, _orig=O.merge_lse_partials):
    M = max(m for m, _ in parts)
    return M + math.log(sum(s for m, s in parts if m != -math.inf))


def _mutant_l1_shard_normalised(z_shard, t_shard, lse_d, lse_t, _orig=O.l1_partial):
    z = np.asarray(z_shard, dtype=np.float64)
    t = np.asarray(t_shard, dtype=np.float64)
    if z.size == 0:
        return (0.0, 0.0)
    return _orig(z, t, float(scipy.special.logsumexp(z)), float(scipy.special.logsumexp(t)))


@pytest.mark.parametrize("target,mutant,pins", [
    ("row_terms", _mutant_half_l1, [test_disjoint_saturated_rows_match_the_pages_values]),
    ("row_terms", _mutant_no_S, [lambda: test_finite_differences_all_gradients(False, "given")]),
    ("row_terms", _mutant_sign_flip, [lambda: test_finite_differences_all_gradients(False, "given")]),
    ("loss_weights", _mutant_decay_index, [test_weights_slot0_is_one_and_decay_ratio_constant]),
    ("target_final_norm", _mutant_norm_no_square, [test_target_final_norm_closed_forms]),
    ("markov_corrected_rows", _mutant_w2_transposed,
     [test_markov_bias_matches_explicit_loops_and_zero_w2_reduces]),
    ("merge_lse_partials", _mutant_merge_no_rescale, [test_lse_partials_merge_to_library_logsumexp]),
    ("l1_partial", _mutant_l1_shard_normalised, [test_tp_row_terms_match_brute_force_for_any_split]),
])
def test_planted_mistakes(monkeypatch, target, mutant, pins):
    """Each planted slip in the oracle makes at least one pin fail."""
    monkeypatch.setattr(O, target, mutant)
    failed = 0
    for pin in pins:
        try:
            pin()
        except AssertionError:
            failed += 1
    assert failed >= 1


def test_subgradient_swing_on_ties_and_none_elsewhere():
    """Identical draft and teacher rows tie on every element: each |p_j - q_j| takes any
    sub-gradient in [-1, 1], so the valid dz_j span 2 g w l1_alpha p_j with p the plain
    softmax; rows far from ties have no such interval, and the per-row sums agree."""
    rng = np.random.default_rng(21)
    B, N, K, V = 1, 2, 3, 50
    d = rng.normal(0, 2, (B, N, K, V))
    ev = np.ones((B, N, K), dtype=np.int64)
    ids = rng.integers(0, V, (B, N, K))
    res = O.dspark_loss(d, ids, ev, target_logits=d.copy(), grad_scale=0.6, l1_alpha=0.9, gamma=4.0)
    for r, sw in res["dlogit_swing"].items():
        k = r % K
        p = scipy.special.softmax(d.reshape(-1, V)[r])
        np.testing.assert_allclose(sw, 2 * 0.6 * np.exp(-k / 4.0) * 0.9 * p, rtol=1e-12)
        assert abs(res["swing_sum"][r] - sw.sum()) < 1e-12
        assert abs(res["dz_norm2"][r] - np.dot(res["dlogits"][r], res["dlogits"][r])) < 1e-15
    # a teacher far from the draft: no undecided signs
    t = d + rng.normal(0, 1, d.shape)
    res = O.dspark_loss(d, ids, ev, target_logits=t)
    assert all(not sw.any() for sw in res["dlogit_swing"].values())
    assert np.all(res["swing_sum"] == 0.0)


def test_weight_gradient_tolerance_sums_equal_their_definitions():
    """The sums the weight-gradient tolerances are built from, written out per element from
    the rows' own dlogits, swings and embeddings: sum over the Markov-live rows of
    dz^2 (x) e^2 and swing (x) |e| for dW2, and per row (dz^2) . W2^2 and swing . |W2| for dE.
    Rows tie on purpose (the teacher equals the draft on one block) so the swing terms
    are not all zero."""
    rng = np.random.default_rng(31)
    B, N, K, V, r = 1, 2, 3, 11, 4
    d, t, ids, ev = _rand_problem(rng, B, N, K, V, scale=1.5)
    prev = rng.integers(1, 6, ids.shape)
    valid = np.array([[[1, 0, 1], [1, 1, 1]]])
    w1, w2 = rng.normal(0, 0.4, (6, r)), rng.normal(0, 0.4, (V, r))
    # block 0: a zero embedding (no bias) and a teacher equal to the draft, so every sign
    # there is undecided
    w1[0] = 0.0
    prev[0, 0] = 0
    t[0, 0] = d[0, 0]
    res = O.dspark_loss(d, ids, ev, target_logits=t, prev_ids=prev, valid=valid, markov_w1=w1, markov_w2=w2,
                        grad_scale=0.8, gamma=4.0)
    live = [int(x) for x in res["rows"] if valid.reshape(-1)[int(x)]]
    assert live and any(res["dlogit_swing"][x].any() for x in live)
    rss2 = np.zeros((V, r))
    swing = np.zeros((V, r))
    for x in live:
        e = w1[prev.reshape(-1)[x]]
        for j in range(V):
            for c in range(r):
                rss2[j, c] += res["dlogits"][x][j] ** 2 * e[c] ** 2
                swing[j, c] += res["dlogit_swing"][x][j] * abs(e[c])
        de_rss2 = [sum(res["dlogits"][x][j] ** 2 * w2[j, c] ** 2 for j in range(V)) for c in range(r)]
        de_swing = [sum(res["dlogit_swing"][x][j] * abs(w2[j, c]) for j in range(V)) for c in range(r)]
        np.testing.assert_allclose(res["tol_dE_rss2"][x], de_rss2, rtol=1e-12, atol=1e-300)
        np.testing.assert_allclose(res["tol_dE_swing"][x], de_swing, rtol=1e-12, atol=1e-300)
    assert set(res["tol_dE_rss2"]) == set(live)
    np.testing.assert_allclose(res["tol_dW2_rss2"], rss2, rtol=1e-12, atol=1e-300)
    np.testing.assert_allclose(res["tol_dW2_swing"], swing, rtol=1e-12, atol=1e-300)
