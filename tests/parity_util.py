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
    sub-gradient there); plus a per-row relative L2 error <= 2e-3 against the same
    rounded row ref_o.  (Against the unrounded row, bf16 rounding alone reaches
    2.5e-3 on rows whose mass sits in a few elements: a half-ulp is 2^-9.)
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
        lm_head=np32(inp.lm_head), ce_alpha=inp.ce_alpha, l1_alpha=inp.l1_alpha if (
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
    keep = ~amb
    nref = np.linalg.norm(ref_o[keep])
    if nref > 0:
        rel = np.linalg.norm((gpu_row - ref_o)[keep]) / nref
        assert rel <= REL_DLOGIT, f"{tag} dlogits row relative L2 error {rel:.3e}"
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
