"""DSpark loss oracle: TEST INFRASTRUCTURE, not product code.

A plain, slow, FP64 CPU statement of what the DSpark draft-training loss sweep
computes, written from the pages that define it.  It exists so the CUDA path can be
checked against something independent of it.  Only ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` leg of ``bench.py`` may import
it; the product path never does.  It shares no code, table or constant with the
CUDA library, and nothing in it is derived from that library's results.

Sources (cited by page title and section throughout):
  [MB-API]  Megatron-Bridge API doc, ``bridge.training.post_training.dspark.loss``
            (module docstring "Return contract"; ``_loss_weight_mask``,
            ``_chunk_terms``, ``_ce_and_l1_per_token``, ``dspark_loss``,
            ``_acceptance_report``).
  [MB-PR]   Megatron-Bridge pull request #5241 (closing comment on the rejected
            "TV half-factor" change; the masked-input merge note).
  [TS-PR]   TorchSpec pull request #132 (DSpark scope list: cumprod prefix mask,
            anchor-seeded Markov previous token, Markov bias == W2(W1[prev]),
            target LM head applied to the final hidden state).
  [RL-HEADS] NeMo RL design doc "DSpark Auxiliary Heads" (head inputs/outputs,
            zero on invalid slots, checkpoint shapes).

Readings taken where the pages leave a step open (each is listed with its reason in
the design notes of the repository):
  * L1 is the raw probability L1 in the training term (no 1/2); the 1/2 appears
    only in the acceptance label 1 - 0.5*L1 [MB-API module docstring; MB-PR].
  * k in exp(-k/gamma) is the 0-based block position.
  * the mask is always reduced to its contiguous prefix (cumprod), then
    multiplied by block_keep.
  * the BCE label y = clamp(1 - 0.5*L1, 0, 1) is detached.
  * sign(0) = 0 in the L1 sub-gradient.
  * an invalid Markov slot has an all-zero corrected row (mode 0) or, as a
    switch, keeps its base row with the bias removed (mode 1).
  * confidence proj input is [hidden ; markov_embedding] in that order.
  * report pairs: loss/ce/l1/conf = [sum w*term, num_tokens];
    accept = [sum m*a, num_tokens]; tau = [sum keep*tau_blk, sum keep].
  * without target logits: L1 = 0 (so accept = 1), CE only.
  * vocabulary-parallel ranks ([RL-HEADS] Tensor Parallelism) combine per-shard
    partials: logsumexp partials (m, s) merged in rank order, then (L1, S) partials
    summed in rank order.
  * pre-norm target hidden states (the vLLM case of the [TS-PR] review) get the
    target's final RMS norm, y = w * x / sqrt(mean(x^2) + eps), before lm_head; the
    normed state is rounded to bf16 once, as the norm's output in the model's dtype.

Every function below is pinned by ``tests/test_oracle_pins.py`` against closed
forms, invariants, brute force and finite differences.
"""

from __future__ import annotations

import math
from typing import Optional

import numpy as np

# Report pair order (fixed).
REPORT_KEYS = ("loss", "ce", "l1", "conf", "accept", "tau")


# --------------------------------------------------------------------------- masks
def prefix_supervision_mask(eval_mask, block_keep=None) -> np.ndarray:
    """m[b,n,k] = prod_{j<=k} eval[b,n,j], times keep[b,n] when given.

    [TS-PR] scope list: the eval mask is cut to its leading run of ones by a
    cumulative product; [MB-API] ``DSparkForwardOutput.eval_mask`` (supervision
    covers an unbroken prefix of each block) and ``block_keep_mask`` (which
    anchors are kept).
    Integer arithmetic: the result is exact.
    """
    e = (np.asarray(eval_mask) != 0).astype(np.int64)
    m = np.cumprod(e, axis=-1)
    if block_keep is not None:
        m = m * (np.asarray(block_keep) != 0).astype(np.int64)[..., None]
    return m


def loss_weights(m: np.ndarray, gamma: Optional[float]) -> np.ndarray:
    """w[b,n,k] = m[b,n,k] * exp(-k / gamma); gamma None disables the decay.

    [MB-API] ``_loss_weight_mask`` and the module docstring: the float supervision
    mask times a decay that falls off exponentially with block position k, at
    rate 1/loss_decay_gamma.
    """
    m = np.asarray(m, dtype=np.float64)
    if gamma is None:
        return m.copy()
    K = m.shape[-1]
    decay = np.array([math.exp(-k / gamma) for k in range(K)], dtype=np.float64)
    return m * decay


# ----------------------------------------------------------------------- row terms
def log_sum_exp(x: np.ndarray) -> float:
    """log sum_j exp(x_j), shifted by the maximum so nothing overflows."""
    M = float(np.max(x))
    return M + math.log(float(np.sum(np.exp(x - M))))


def row_terms(z: np.ndarray, t: Optional[np.ndarray], tid: int) -> dict:
    """Cross-entropy and raw probability L1 of one row, plus what the backward needs.

    [MB-API] ``_chunk_terms`` (both terms from one normalised draft distribution),
    ``dspark_loss`` (ce = cross-entropy against the target's next token; l1 =
    ||p_draft - p_target||_1, no 1/2).  ``S = sum_j p_j * sign(p_j - q_j)`` is the
    row scalar of the L1 derivative.  Without a target row, L1 = 0 ([MB-API]
    ``_ce_and_l1_per_token``: the L1 output is then zeros).
    """
    z = np.asarray(z, dtype=np.float64)
    lse_d = log_sum_exp(z)
    p = np.exp(z - lse_d)
    out = dict(lse_d=lse_d, ce=lse_d - float(z[tid]), p=p)
    if t is None:
        out.update(lse_t=0.0, q=None, s=None, l1=0.0, S=0.0)
        return out
    t = np.asarray(t, dtype=np.float64)
    lse_t = log_sum_exp(t)
    q = np.exp(t - lse_t)
    s = np.sign(p - q)
    out.update(lse_t=lse_t, q=q, s=s, l1=float(np.sum(np.abs(p - q))), S=float(np.sum(p * s)))
    return out


# ---------------------------------------------------- vocabulary-parallel form
# [RL-HEADS] Tensor Parallelism: each tensor-parallel rank holds the base logits of
# its own contiguous shard of the draft vocabulary.  A full-vocabulary row term then
# needs the shards' partial sums.  The reading taken here: a rank reduces its
# columns to a logsumexp partial (m, s); the ranks' partials are merged in rank
# order; then each rank reduces its columns to an (L1, S) partial against the merged
# normalisers, and those are summed in rank order.
def lse_partial(x_shard: np.ndarray) -> tuple:
    """(m, s) of one shard: m = max_j x_j, s = sum_j exp(x_j - m); (-inf, 0) if empty."""
    x = np.asarray(x_shard, dtype=np.float64)
    if x.size == 0:
        return (-math.inf, 0.0)
    m = float(np.max(x))
    return (m, float(np.sum(np.exp(x - m))))


def merge_lse_partials(parts) -> float:
    """log sum_j exp(x_j) of the whole row from its shards' (m, s) partials:
    M = max_k m_k, lse = M + log sum_k s_k exp(m_k - M) (empty shards add nothing)."""
    M = max(m for m, _ in parts)
    total = sum(s * math.exp(m - M) for m, s in parts if m != -math.inf)
    return M + math.log(total)


def l1_partial(z_shard: np.ndarray, t_shard: np.ndarray, lse_d: float, lse_t: float) -> tuple:
    """(sum_j |p_j - q_j|, sum_j p_j sign(p_j - q_j)) over one shard's columns, with
    p = exp(z - lse_d) and q = exp(t - lse_t) normalised over the whole row."""
    p = np.exp(np.asarray(z_shard, dtype=np.float64) - lse_d)
    q = np.exp(np.asarray(t_shard, dtype=np.float64) - lse_t)
    return (float(np.sum(np.abs(p - q))), float(np.sum(p * np.sign(p - q))))


def tp_row_terms(z: np.ndarray, t: Optional[np.ndarray], tid: int, bounds) -> dict:
    """CE, L1 and S of one row computed shard by shard: ``bounds`` = [v_0 = 0, v_1, ...,
    v_T = V] splits the columns into T contiguous shards (empty ones allowed).  Same
    quantities as ``row_terms``, reached through the partials above."""
    z = np.asarray(z, dtype=np.float64)
    shards = [(bounds[k], bounds[k + 1]) for k in range(len(bounds) - 1)]
    lse_d = merge_lse_partials([lse_partial(z[a:b]) for a, b in shards])
    out = dict(lse_d=lse_d, ce=lse_d - float(z[tid]))
    if t is None:
        out.update(lse_t=0.0, l1=0.0, S=0.0)
        return out
    t = np.asarray(t, dtype=np.float64)
    lse_t = merge_lse_partials([lse_partial(t[a:b]) for a, b in shards])
    parts = [l1_partial(z[a:b], t[a:b], lse_d, lse_t) for a, b in shards]
    out.update(lse_t=lse_t, l1=float(sum(l for l, _ in parts)), S=float(sum(s for _, s in parts)))
    return out


def sign_ambiguity(p: np.ndarray, q: np.ndarray, rel: float = 3e-5) -> np.ndarray:
    """Elements where sign(p - q) is not decided at FP32 working precision.

    There either sign is a valid L1 sub-gradient; comparisons skip them.
    """
    return np.abs(p - q) <= rel * np.maximum(p, q)


def bce_with_logits(c, y):
    """-[y log sigmoid(c) + (1 - y) log(1 - sigmoid(c))], written with softplus.

    [MB-API] module docstring: confidence is binary cross-entropy of the confidence
    head's logit, with the analytical acceptance value as its label.  -log sigmoid(c) = softplus(-c) and
    -log(1 - sigmoid(c)) = softplus(c).
    """
    c = np.asarray(c, dtype=np.float64)
    y = np.asarray(y, dtype=np.float64)
    return y * np.logaddexp(0.0, -c) + (1.0 - y) * np.logaddexp(0.0, c)


def sigmoid(c):
    c = np.asarray(c, dtype=np.float64)
    return 0.5 * (1.0 + np.tanh(0.5 * c))


def acceptance_label(l1):
    """a = clamp(1 - 0.5 * L1, 0, 1): [MB-API] module docstring and
    ``_acceptance_report``; the clamp to [0, 1] follows the [MB-PR] merge note."""
    return np.clip(1.0 - 0.5 * np.asarray(l1, dtype=np.float64), 0.0, 1.0)


# --------------------------------------------------------------------------- heads
def markov_embedding(prev_ids, w1) -> np.ndarray:
    """e[r] = markov_w1[prev_ids[r]]: the previous-token embedding ([RL-HEADS]
    "Inputs and Outputs"; checkpoint key markov_head.markov_w1.weight of shape
    [target_vocab, rank])."""
    return np.asarray(w1, dtype=np.float64)[np.asarray(prev_ids, dtype=np.int64)]


def markov_corrected_rows(base_rows, e_rows, valid_rows, w2, invalid_row_mode=0) -> np.ndarray:
    """z = base + markov_w2 @ e on valid slots; invalid slots -> 0 (mode 0) or base (mode 1).

    [RL-HEADS] "Inputs and Outputs": a valid slot gets a low-rank bias, built from
    its previous token, added to its base logits, and an invalid slot's head output
    is zero; [TS-PR] test list: the bias is W2 applied to the W1 row of the previous
    token.  The bias uses a library matmul and is not rounded.
    """
    base_rows = np.asarray(base_rows, dtype=np.float64)
    w2 = np.asarray(w2, dtype=np.float64)
    bias = np.asarray(e_rows, dtype=np.float64) @ w2.T
    z = base_rows + bias
    inv = np.asarray(valid_rows) == 0
    if invalid_row_mode == 0:
        z[inv] = 0.0
    else:
        z[inv] = base_rows[inv]
    return z


def target_final_norm(hidden_rows, weight, eps) -> np.ndarray:
    """The target's final RMS norm on pre-norm hidden states ([TS-PR] review of the
    vLLM path: its stored last hidden states precede the final norm, which must be
    applied before lm_head): y = w * x / sqrt(mean_h(x^2) + eps), each row on its own,
    computed in FP64 and converted to bf16 through FP32 by torch's cast (the dtype in
    which the norm hands its output to the lm_head product)."""
    import torch
    x = np.asarray(hidden_rows, dtype=np.float64)
    w = np.asarray(weight, dtype=np.float64).reshape(-1)
    y = w * x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + float(eps))
    return torch.from_numpy(y).to(torch.bfloat16).double().numpy()


def confidence_head_logits(hidden_rows, e_rows, proj, bias, valid_rows) -> np.ndarray:
    """c = proj . [h ; e] + bias on valid slots, 0 on invalid ones ([RL-HEADS]
    "Inputs and Outputs" and "Checkpoint Contract": a single float logit per slot,
    proj of shape [1, hidden_size + markov_rank], zero output on invalid slots).
    ``e_rows`` None means with_markov=False (proj [1, hidden_size])."""
    h = np.asarray(hidden_rows, dtype=np.float64)
    proj = np.asarray(proj, dtype=np.float64).reshape(-1)
    H = h.shape[-1]
    c = h @ proj[:H]
    if e_rows is not None:
        c = c + np.asarray(e_rows, dtype=np.float64) @ proj[H:]
    c = c + float(np.asarray(bias, dtype=np.float64).reshape(-1)[0])
    c[np.asarray(valid_rows) == 0] = 0.0
    return c


# -------------------------------------------------------------------- acceptance
def acceptance_report(l1_rows, m, block_keep=None) -> dict:
    """Accept-rate and tau pairs of [MB-API] ``_acceptance_report``.

    accept a = 1 - 0.5*L1 on supervised slots; a drafted token counts only when all
    tokens before it in the block were accepted, hence the running product, and the
    anchor token adds one: tau_blk = 1 + sum_k prod_{j<=k} a_j m_j.  Pairs: accept [sum m*a, sum m];
    tau [sum keep*tau_blk, sum keep].
    """
    m = np.asarray(m, dtype=np.int64)
    B, N, K = m.shape
    a = acceptance_label(np.asarray(l1_rows, dtype=np.float64).reshape(B, N, K))
    am = np.where(m != 0, a, 0.0)
    tau = np.ones((B, N), dtype=np.float64)
    for b in range(B):
        for n in range(N):
            run = 1.0
            for k in range(K):
                run *= am[b, n, k]
                tau[b, n] += run
    keep = np.ones((B, N)) if block_keep is None else (np.asarray(block_keep) != 0).astype(np.float64)
    return dict(accept_rows=am, tau_blocks=tau,
                accept=(float(np.sum(am)), float(np.sum(m))),
                tau=(float(np.sum(keep * tau)), float(np.sum(keep))))


# ------------------------------------------------------------------------- driver
def _as_rows(x, R):
    if x is None:
        return None
    return np.asarray(x).reshape(R, -1)


def _matmul_rows_by_table(rows, table, vchunk=16384):
    """rows @ table.T in FP64, converting the table to FP64 a slab at a time."""
    rows = np.asarray(rows, dtype=np.float64)
    V = table.shape[0]
    out = np.empty((rows.shape[0], V))
    for v0 in range(0, V, vchunk):
        out[:, v0:v0 + vchunk] = rows @ np.asarray(table[v0:v0 + vchunk], dtype=np.float64).T
    return out


def dspark_loss(draft_logits, target_ids, eval_mask, *, target_logits=None, block_keep=None,
                confidence_logits=None, prev_ids=None, valid=None, markov_w1=None,
                markov_w2=None, draft_hidden=None, conf_w=None, conf_b=None,
                conf_with_markov=False, target_hidden=None, lm_head=None,
                target_norm_weight=None, target_norm_eps=1e-6,
                ce_alpha=0.1, l1_alpha=0.9, conf_alpha=1.0, gamma: Optional[float] = 4.0,
                grad_scale=1.0, invalid_row_mode=0, want_grads=True,
                rows: Optional[np.ndarray] = None, keep_rows: Optional[np.ndarray] = None,
                fixed_label: Optional[np.ndarray] = None, row_chunk: int = 64) -> dict:
    """The DSpark objective of [MB-API] ``dspark_loss`` and its gradient, in FP64.

    Returns ``loss_num`` (unnormalised weighted numerator), ``num_tokens``,
    ``report`` (key -> (numerator, denominator); nothing divided), per-row
    ``ce``, ``l1``, ``S``, ``lse_d``, ``lse_t``, ``conf`` (c), ``bce``, ``accept``,
    masks ``m`` and ``w``, and with ``want_grads``: ``dlogits`` (row -> dL/dbase
    row), ``sign_amb`` (row -> mask), ``dlogit_swing`` (row -> width of the interval of
    valid dz_j where sign(p_j - q_j) is undecided, 0 elsewhere), per-row sums over
    every supervised row ``dz_norm2`` [R] (sum_j dlogits_j^2) and ``swing_sum`` [R],
    ``dconf`` [R], and for the heads ``dW2``,
    ``dE`` (row -> dL/de), ``dW1`` (id -> row), ``dconf_w``, ``dconf_b``, ``dhidden``,
    plus the sums a tolerance on the weight gradients needs, over every row the Markov
    contractions take (so no caller has to keep every row's dlogits):
    ``tol_dW2_rss2`` = sum_r dz_r^2 (x) e_r^2 and ``tol_dW2_swing`` = sum_r swing_r (x) |e_r|
    ([V, rank]), and per row ``tol_dE_rss2`` = (dz_r^2) . (W2^2) and ``tol_dE_swing`` =
    swing_r . |W2| ([rank]); swing_r is the ``dlogit_swing`` row.

    The loss is sum_r w_r (ce_alpha*CE_r + l1_alpha*L1_r + conf_alpha*BCE_r) where
    the BCE term exists only with a confidence source, and the L1 and BCE terms need
    the teacher ([MB-API] ``dspark_loss``, Raises: ValueError without
    aligned_target_logits).  Gradients are of grad_scale * loss with the BCE label
    detached.  Rows are independent ([MB-API] ``_ce_and_l1_per_token``: every row
    is reduced on its own), so they are visited ``row_chunk`` at a time only to
    bound memory.

    ``rows`` restricts the per-row work to a subset of supervised rows (the head
    weight gradients are then partial sums over those rows); ``keep_rows`` limits
    which rows' dlogits are returned.  ``fixed_label`` replaces the BCE label (the
    finite-difference tests hold it constant, as the detach does).
    """
    eval_mask = np.asarray(eval_mask)
    B, N, K = eval_mask.shape
    R = B * N * K
    has_teacher = target_logits is not None or lm_head is not None
    has_conf = confidence_logits is not None or conf_w is not None
    if not has_teacher and (l1_alpha != 0.0 or has_conf):
        raise ValueError("the L1 term and the confidence head need the target distribution")
    has_markov = markov_w2 is not None

    m = prefix_supervision_mask(eval_mask, block_keep)
    w = loss_weights(m, gamma)
    m_r, w_r = m.reshape(R), w.reshape(R)
    tids = np.asarray(target_ids, dtype=np.int64).reshape(R)
    valid_r = None if valid is None else np.asarray(valid).reshape(R)
    draft_r = _as_rows(draft_logits, R)
    target_r = _as_rows(target_logits, R)
    V = draft_r.shape[1]

    e_all = markov_embedding(np.asarray(prev_ids).reshape(R), markov_w1) if has_markov else None
    w2 = np.asarray(markov_w2, dtype=np.float64) if has_markov else None
    c_rows = np.zeros(R)
    if confidence_logits is not None:
        c_rows = np.asarray(confidence_logits, dtype=np.float64).reshape(R).copy()
    elif conf_w is not None:
        c_rows = confidence_head_logits(_as_rows(draft_hidden, R),
                                        e_all if conf_with_markov else None,
                                        conf_w, conf_b, valid_r)

    sup = np.nonzero(m_r)[0] if rows is None else np.asarray(rows, dtype=np.int64)
    keep = set(int(r) for r in (sup if keep_rows is None else keep_rows))
    ce = np.zeros(R); l1 = np.zeros(R); S = np.zeros(R); lse_d = np.zeros(R); lse_t = np.zeros(R)
    dlogits, amb, swing, dE = {}, {}, {}, {}
    dz_norm2, swing_sum = np.zeros(R), np.zeros(R)
    dW2 = np.zeros_like(w2) if (has_markov and want_grads) else None
    # tolerance helpers of the head weight gradients (sums over every row the contractions
    # take, so no caller needs every row's dlogits): sum_r dz_r^2 (x) e_r^2 and
    # sum_r swing_r (x) |e_r| for dW2; per row (dz_r^2) . (W2^2) and swing_r . |W2| for dE
    tol_dw2_rss2 = np.zeros_like(w2) if dW2 is not None else None
    tol_dw2_swing = np.zeros_like(w2) if dW2 is not None else None
    tol_de_rss2, tol_de_swing = {}, {}

    for c0 in range(0, len(sup), row_chunk):
        rr = sup[c0:c0 + row_chunk]
        base = draft_r[rr].astype(np.float64)
        if has_markov:
            z_rows = markov_corrected_rows(base, e_all[rr], valid_r[rr], w2, invalid_row_mode)
        else:
            z_rows = base
        if lm_head is not None:
            h_rows = _as_rows(target_hidden, R)[rr]
            if target_norm_weight is not None:
                h_rows = target_final_norm(h_rows, target_norm_weight, target_norm_eps)
            t_rows = _matmul_rows_by_table(h_rows, lm_head)
        elif target_r is not None:
            t_rows = target_r[rr].astype(np.float64)
        else:
            t_rows = None
        dz_live = []
        for i, r in enumerate(rr):
            r = int(r)
            rt = row_terms(z_rows[i], None if t_rows is None else t_rows[i], int(tids[r]))
            ce[r], l1[r], S[r], lse_d[r], lse_t[r] = rt["ce"], rt["l1"], rt["S"], rt["lse_d"], rt["lse_t"]
            if not want_grads:
                continue
            # dCE/dz = p - onehot(tid); dL1/dz = p * (s - S)
            dz = ce_alpha * rt["p"]
            dz[int(tids[r])] -= ce_alpha
            if rt["q"] is not None:
                dz = dz + l1_alpha * rt["p"] * (rt["s"] - rt["S"])
            dz = grad_scale * w_r[r] * dz
            markov_live = has_markov and valid_r[r] != 0
            row_grad = dz
            if has_markov and not markov_live and invalid_row_mode == 0:
                row_grad = np.zeros(V)             # the corrected row is the constant 0
            dz_norm2[r] = float(np.dot(row_grad, row_grad))
            sw_row = np.zeros(V)
            if rt["q"] is not None and row_grad is dz:
                sw_row = np.where(sign_ambiguity(rt["p"], rt["q"]), 2.0 * grad_scale * w_r[r] * l1_alpha * rt["p"], 0.0)
                swing_sum[r] = float(np.sum(sw_row))
            if r in keep:
                dlogits[r] = row_grad
                amb[r] = (sign_ambiguity(rt["p"], rt["q"]) if rt["q"] is not None
                          else np.zeros(V, dtype=bool))
                # where sign(p_j - q_j) is undecided, |p_j - q_j| has every sub-gradient in
                # [-1, 1]: the valid values of dz_j span 2 g w l1_alpha p_j
                swing[r] = (np.where(amb[r], 2.0 * grad_scale * w_r[r] * l1_alpha * rt["p"], 0.0)
                            if row_grad is dz else np.zeros(V))
            if markov_live:
                dz_live.append((r, dz, sw_row))
        if dz_live:
            Dz = np.stack([d for _, d, _ in dz_live])           # [n, V]
            Sw = np.stack([x for _, _, x in dz_live])           # [n, V]
            Er = e_all[[r for r, _, _ in dz_live]]              # [n, rank]
            dW2 += Dz.T @ Er                                     # dW2 = sum_r dz_r (x) e_r
            dEr = Dz @ w2                                        # dE_r = W2^T dz_r
            tol_dw2_rss2 += (Dz ** 2).T @ (Er ** 2)
            tol_dw2_swing += Sw.T @ np.abs(Er)
            de_rss2 = (Dz ** 2) @ (w2 ** 2)
            de_swing = Sw @ np.abs(w2)
            for j, (r, _, _) in enumerate(dz_live):
                dE[r] = dEr[j]
                tol_de_rss2[r], tol_de_swing[r] = de_rss2[j], de_swing[j]

    # confidence / BCE
    y = acceptance_label(l1) if fixed_label is None else np.asarray(fixed_label, dtype=np.float64).reshape(R)
    bce = np.zeros(R)
    if has_conf:
        bce[sup] = bce_with_logits(c_rows[sup], y[sup])
    sel = np.zeros(R, dtype=bool)
    sel[sup] = True
    wsel = np.where(sel, w_r, 0.0)
    ce_num = float(np.sum(wsel * ce))
    l1_num = float(np.sum(wsel * l1))
    conf_num = float(np.sum(wsel * bce))
    loss_num = ce_alpha * ce_num + l1_alpha * l1_num + (conf_alpha * conf_num if has_conf else 0.0)
    n_tok = int(np.sum(m_r))
    acc = acceptance_report(np.where(sel, l1, 0.0), m.reshape(B, N, K), block_keep)
    report = dict(loss=(loss_num, float(n_tok)), ce=(ce_num, float(n_tok)), l1=(l1_num, float(n_tok)),
                  conf=(conf_num, float(n_tok)), accept=acc["accept"], tau=acc["tau"])
    res = dict(loss_num=loss_num, num_tokens=n_tok, report=report, m=m_r, w=w_r, ce=ce, l1=l1, S=S,
               lse_d=lse_d, lse_t=lse_t, conf=c_rows, bce=bce, label=y,
               accept=acc["accept_rows"].reshape(R), tau_blocks=acc["tau_blocks"], rows=sup)
    if not want_grads:
        return res

    dconf = np.zeros(R)
    if has_conf:
        dconf[sup] = grad_scale * w_r[sup] * conf_alpha * (sigmoid(c_rows[sup]) - y[sup])
    res.update(dlogits=dlogits, sign_amb=amb, dlogit_swing=swing, dz_norm2=dz_norm2, swing_sum=swing_sum,
               dconf=dconf)
    if conf_w is not None:
        hv = _as_rows(draft_hidden, R).astype(np.float64)
        H = hv.shape[1]
        live = sel & (valid_r != 0)
        dcl = np.where(live, dconf, 0.0)        # the head's output is constant on invalid slots
        proj = np.asarray(conf_w, dtype=np.float64).reshape(-1)
        d_proj = np.zeros_like(proj)
        d_proj[:H] = dcl @ hv
        if conf_with_markov:
            d_proj[H:] = dcl @ e_all
            for r in np.nonzero(live)[0]:
                r = int(r)
                dE[r] = dE.get(r, 0.0) + dcl[r] * proj[H:]
        res.update(dconf_w=d_proj, dconf_b=float(np.sum(dcl)), dhidden=np.outer(dcl, proj[:H]))
    if has_markov:
        dW1 = {}
        pids = np.asarray(prev_ids, dtype=np.int64).reshape(R)
        for r in sorted(dE):
            dW1[int(pids[r])] = dW1.get(int(pids[r]), 0.0) + dE[r]
        res.update(dW2=dW2, dE=dE, dW1=dW1, tol_dW2_rss2=tol_dw2_rss2, tol_dW2_swing=tol_dw2_swing,
                   tol_dE_rss2=tol_de_rss2, tol_dE_swing=tol_de_swing)
    return res
