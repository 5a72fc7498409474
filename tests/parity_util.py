"""Shared helpers of the GPU parity tests: run the CUDA path through the C ABI, run the
FP64 oracle on the same seeded inputs, and compare with the stated tolerances.

Tolerances (fixed for the whole suite):
  * counts, masks and denominators: bit-exact;
  * summed numerators and report pairs: 1e-4 relative (plus 1e-6 per counted row,
    for numerators whose reference is exactly 0);
  * per-row CE and L1: 1e-3 absolute;
  * dlogits: element-wise |gpu - ref_o| <= max(2e-3 |ref_o|, ulp_o(ref_o)) + 1e-6 max_row |ref|
    where ref_o is the FP64 value rounded to the output dtype (bf16's half-ulp is
    above 2e-3, so a 1-ulp rounding flip is allowed), skipping elements whose
    sign(p - q) is not decided at FP32 precision (either sign is a valid L1
    sub-gradient there); plus a per-row L2 bound against the unrounded FP64 row:
    ||gpu - ref|| <= 2e-3 ||ref|| + ||ulp_o / 2||, the FP32 arithmetic plus the output
    rounding (round to nearest puts each stored value within half an ulp of the FP32
    value it rounds; a value near a rounding boundary may go to the other neighbour than
    the FP64 reference does, a whole ulp from ref_o, which on a row whose mass sits in
    one element exceeds 2e-3 of the rounded row by itself).
Head weight gradients (dW2 = sum_r dz_r (x) e_r, dE_r = W2^T dz_r, hence dW1) are
contracted on the tensor cores from the bf16 dlogits, so they carry the bf16 rounding
of dz (unit roundoff u = 2^-8, one rounding per element, independent across elements):
the error of a sum of rounded products has standard deviation at most
u/sqrt(3) * sqrt(sum_k (dz_k x_k)^2), and check_heads allows 4u times that root-sum-
square (about seven standard deviations) plus 1e-5 of the magnitude for FP32
accumulation.  Where some row's sign(p_j - q_j) is undecided at FP32 precision, every
sub-gradient of |p_j - q_j| is valid: the oracle reports the width of that interval of dz
(``dlogit_swing``), and the bounds add its contraction with |e| (or |W2|).
"""

from __future__ import annotations

import numpy as np
import torch

from oracle import dspark_oracle as O

REL_SUM = 1e-4
ABS_ROW = 1e-3
REL_DLOGIT = 2e-3


def np64(t):
    if t is None:
        return None
    return t.detach().cpu().double().numpy()


def np32(t):
    if t is None:
        return None
    if t.dtype in (torch.bfloat16, torch.float16):
        t = t.float()
    return t.detach().cpu().numpy()


def oracle_run(inp, rows=None, keep_rows=None, invalid_row_mode=0, want_grads=True):
    """The oracle on the inputs of ``inp`` (any device)."""
    return O.dspark_loss(
        np32(inp.draft_logits), np32(inp.target_ids), np32(inp.eval_mask),
        target_logits=np32(inp.target_logits), block_keep=np32(inp.block_keep),
        confidence_logits=np64(inp.confidence_logits), prev_ids=np32(inp.prev_ids),
        valid=np32(inp.valid), markov_w1=np32(inp.markov_w1), markov_w2=np32(inp.markov_w2),
        draft_hidden=np32(inp.draft_hidden), conf_w=np32(inp.conf_w), conf_b=np64(inp.conf_b),
        conf_with_markov=inp.conf_with_markov, target_hidden=np32(inp.target_hidden),
        lm_head=np32(inp.lm_head), target_norm_weight=np32(inp.target_norm_weight),
        target_norm_eps=inp.target_norm_eps, ce_alpha=inp.ce_alpha, l1_alpha=inp.l1_alpha if (
            inp.target_logits is not None or inp.lm_head is not None) else 0.0,
        conf_alpha=inp.conf_alpha, gamma=inp.gamma, grad_scale=inp.grad_scale,
        invalid_row_mode=invalid_row_mode, want_grads=want_grads, rows=rows, keep_rows=keep_rows)


def run_gpu(inp, grads=True, rows=True, invalid_row_mode=0):
    from speculative_decoding_draft_vocab_b200 import torch_api
    call = torch_api.Call(inp, grads=grads, rows=rows, invalid_row_mode=invalid_row_mode)
    call.launch()
    torch.cuda.synchronize()
    return call


def bf16_ulp(x: np.ndarray) -> np.ndarray:
    ax = np.abs(x)
    _, e = np.frexp(np.where(ax > 0, ax, 1.0))
    return np.where(ax > 0, np.ldexp(1.0, e - 8), 0.0)


def round_to(x: np.ndarray, dtype: str) -> np.ndarray:
    if dtype == "bf16":
        return torch.from_numpy(np.asarray(x, dtype=np.float64)).to(torch.bfloat16).double().numpy()
    return np.asarray(x, dtype=np.float32).astype(np.float64)


def check_dlogit_row(gpu_row: np.ndarray, ref_row: np.ndarray, amb: np.ndarray, dtype: str, tag=""):
    ref_o = round_to(ref_row, dtype)
    floor = 1e-6 * float(np.max(np.abs(ref_row))) if ref_row.size else 0.0
    tol = np.maximum(REL_DLOGIT * np.abs(ref_o), bf16_ulp(ref_o) if dtype == "bf16" else 0.0) + floor
    err = np.abs(gpu_row - ref_o)
    bad = (err > tol) & ~amb
    if bad.any():
        j = int(np.argmax(np.where(amb, 0, err - tol)))
        raise AssertionError(f"{tag} dlogits: {int(bad.sum())} elements off; worst j={j} "
                             f"gpu={gpu_row[j]!r} ref={ref_row[j]!r} tol={tol[j]!r}")
    # Row L2, against the unrounded row: the stored value is the output rounding of an
    # FP32 value (at most half an ulp away from it), and that FP32 value is within
    # REL_DLOGIT of the FP64 one; by the triangle inequality the row's error is within
    # the two norms.  (Against the rounded row a single dominant element that rounds to
    # the other neighbour, one whole ulp, 2^-9 to 2^-8 relative, can exceed REL_DLOGIT.)
    keep = ~amb
    nref = np.linalg.norm(ref_row[keep])
    if nref > 0:
        if dtype == "bf16":
            half = 0.5 * np.maximum(bf16_ulp(np.abs(gpu_row)), bf16_ulp(ref_o))
        else:
            half = 0.5 * np.spacing(np.abs(np.asarray(ref_o, dtype=np.float32))).astype(np.float64)
        err = np.linalg.norm((gpu_row - ref_row)[keep])
        bound = REL_DLOGIT * nref + np.linalg.norm(half[keep])
        assert err <= bound, f"{tag} dlogits row L2 error {err:.3e} above {bound:.3e} ({err / nref:.3e} relative)"
    return int(amb.sum())


def compare(inp, call, ref, dlogit_rows=None, check_rows=True):
    """Compare the outputs of a finished GPU call with an oracle result."""
    out = call.out
    R = inp.R
    assert int(out.num_tokens.item()) == ref["num_tokens"]
    rep = out.report.cpu().double().numpy()
    from oracle.dspark_oracle import REPORT_KEYS
    for i, key in enumerate(REPORT_KEYS):
        num, den = ref["report"][key]
        assert rep[i, 1] == den, (key, rep[i, 1], den)
        # 1e-4 relative; a numerator whose reference is 0 gets 1e-6 per counted row
        assert abs(rep[i, 0] - num) <= REL_SUM * abs(num) + 1e-6 * max(den, 1.0), (key, rep[i, 0], num)
    ln = float(out.loss_num.item())
    assert abs(ln - ref["loss_num"]) <= REL_SUM * max(abs(ref["loss_num"]), 1e-6)
    sup = ref["rows"]
    if check_rows and out.ce_rows is not None:
        ce = out.ce_rows.cpu().double().numpy()
        l1 = out.l1_rows.cpu().double().numpy()
        acc = out.accept_rows.cpu().double().numpy()
        np.testing.assert_allclose(ce[sup], ref["ce"][sup], rtol=0, atol=ABS_ROW)
        np.testing.assert_allclose(l1[sup], ref["l1"][sup], rtol=0, atol=ABS_ROW)
        np.testing.assert_allclose(acc[sup], ref["accept"][sup], rtol=0, atol=ABS_ROW)
        unsup = np.setdiff1d(np.arange(R), sup)
        assert np.all(ce[unsup] == 0) and np.all(l1[unsup] == 0)
    if out.dconf is not None and inp.confidence_logits is not None:
        np.testing.assert_allclose(out.dconf.cpu().double().numpy(), ref["dconf"], rtol=1e-4, atol=1e-6)
    n_amb = 0
    if out.dlogits is not None:
        V = inp.V
        g = out.dlogits.view(R, V)
        rows = sorted(ref["dlogits"]) if dlogit_rows is None else dlogit_rows
        for r in rows:
            gr = g[r].float().cpu().double().numpy()
            n_amb += check_dlogit_row(gr, ref["dlogits"][r], ref["sign_amb"][r], inp.dtype, tag=f"row {r}")
        # every unsupervised row is exactly zero
        msk = torch.from_numpy(ref["m"] == 0).to(g.device)
        if bool(msk.any()):
            assert bool((g[msk] == 0).all())
    return n_amb


U_BF16 = 2.0 ** -8


def _live_rows(inp, ref):
    valid = np32(inp.valid).reshape(-1)
    sup = ref["rows"]
    return np.array([int(r) for r in sup if valid[r] != 0], dtype=np.int64)


def check_heads(inp, call, ref, mode, elementwise=True):
    """Confidence logits, dL/dc and the head weight gradients of a finished call.

    dW2 and dW1 are checked element-wise against the bound derived in the module
    docstring (built from the oracle's sums over every contracted row, so no test needs
    every row's dlogits), and in Frobenius norm against the aggregate of that bound (the same sum of independent
    rounding errors: its Frobenius norm is about u/sqrt(3) times that of the
    root-sum-squares; u times it is allowed), plus the width of the valid sub-gradients
    where sign(p - q) is undecided (``dlogit_swing``; changing one s_j also moves S, so
    every other element can move by up to p_k times the same width: a second term of
    the same size)."""
    out = call.out
    R = inp.R
    u = U_BF16
    valid = np32(inp.valid).reshape(-1)
    # confidence logits of every row (0 on invalid slots)
    if inp.conf_w is not None:
        c = out.conf_rows.cpu().double().numpy()
        np.testing.assert_allclose(c, ref["conf"], rtol=1e-4, atol=1e-5)
    np.testing.assert_allclose(out.dconf.cpu().double().numpy(), ref["dconf"], rtol=1e-4, atol=2e-6)
    live = _live_rows(inp, ref)
    stats = {}
    if inp.markov_w2 is not None:
        w2 = np32(inp.markov_w2).astype(np.float64)
        rank = w2.shape[1]
        prev = np32(inp.prev_ids).reshape(-1).astype(np.int64)
        e_live = O.markov_embedding(prev[live], np32(inp.markov_w1)) if len(live) else np.zeros((0, rank))
        e_norm = np.linalg.norm(e_live, axis=1)
        w2_colmax = np.abs(w2).max(0)                  # [rank]
        w2_rowmax = np.linalg.norm(w2, axis=1).max()   # max_j ||W2_j||
        nz2, swt = ref["dz_norm2"][live], ref["swing_sum"][live]
        proj_e = None
        if inp.conf_w is not None and inp.conf_with_markov:
            proj_e = np32(inp.conf_w).reshape(-1).astype(np.float64)[inp.draft_hidden.shape[-1]:]
        # ---- dW2 = sum_r dz_r (x) e_r
        got = out.dW2.cpu().double().numpy()
        want = ref["dW2"]
        agg = u * np.sqrt(np.sum(nz2 * e_norm ** 2)) + 2 * np.sum(swt * e_norm) + 1e-5 * np.linalg.norm(want)
        err_f = np.linalg.norm(got - want)
        assert err_f <= agg, f"dW2 Frobenius error {err_f:.3e} > {agg:.3e}"
        stats["dW2_frob_err"] = err_f / max(agg, 1e-30)
        if elementwise:
            # the oracle's sums over every contracted row: sum_r dz_r^2 e_r^2, sum_r swing_r |e_r|
            bound = (4 * u * np.sqrt(ref["tol_dW2_rss2"]) + ref["tol_dW2_swing"]
                     + (swt[:, None] * np.abs(e_live)).sum(0)[None, :] + 1e-5 * np.abs(want)
                     + 1e-7 * np.abs(want).max())
            bad = np.abs(got - want) > bound
            assert not bad.any(), f"dW2: {int(bad.sum())} entries off; worst {np.max(np.abs(got - want) - bound)}"
        # ---- dW1[id] = sum over rows with that previous id of dE_r = W2^T dz_r + dc_r proj_e
        gotw1 = out.dW1.cpu().double().numpy()
        ids = sorted(ref["dW1"])
        touched = np.zeros(gotw1.shape[0], dtype=bool)
        touched[ids] = True
        assert np.all(gotw1[~touched] == 0.0), "dW1 rows of untouched ids must stay zero"
        if ids:
            want1 = np.stack([ref["dW1"][i] for i in ids])
            conf_part = 0.0
            if proj_e is not None:
                conf_part = 1e-5 * np.sum(np.abs(ref["dconf"][live])) * np.linalg.norm(proj_e)
            agg1 = (u * w2_rowmax * np.sqrt(np.sum(nz2)) + 2 * w2_rowmax * np.sum(swt) + conf_part
                    + 1e-5 * np.linalg.norm(want1))
            err1 = np.linalg.norm(gotw1[ids] - want1)
            assert err1 <= agg1, f"dW1 Frobenius error {err1:.3e} > {agg1:.3e}"
            stats["dW1_frob_err"] = err1 / max(agg1, 1e-30)
        if elementwise and ids:
            var, extra = {}, {}
            for i, r in enumerate(live):
                pid = int(prev[r])
                var[pid] = var.get(pid, 0.0) + ref["tol_dE_rss2"][int(r)]   # (dz_r^2) . (W2^2)
                x = ref["tol_dE_swing"][int(r)] + swt[i] * w2_colmax        # swing_r . |W2| + ...
                if proj_e is not None:
                    x = x + 1e-5 * np.abs(ref["dconf"][r] * proj_e)
                extra[pid] = extra.get(pid, 0.0) + x
            for pid in ids:
                want_row = ref["dW1"][pid]
                err = np.abs(gotw1[pid] - want_row)
                tol = 4 * u * np.sqrt(var[pid]) + extra[pid] + 1e-5 * np.abs(want_row) + 1e-9
                assert np.all(err <= tol), f"dW1[{pid}]: worst {np.max(err - tol)}"
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
