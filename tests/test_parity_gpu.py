"""GPU parity of the fused DSpark loss (C ABI, CUDA kernels) against the FP64 oracle.

Sizes span every sweep build (1, 2, 4 and 8-CTA clusters), ragged vocabulary tails
and ragged masks; the full recipe shape (4 x 16 x 7 x 151936, bf16) is the bench
workload and is checked on every row.
"""

import numpy as np
import pytest
import torch

from speculative_decoding_draft_vocab_b200.synthetic import make_inputs
from tests.parity_util import check_dlogit_row, compare, oracle_run, run_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from speculative_decoding_draft_vocab_b200 import build
    build.build()
    assert torch.cuda.is_available(), "the GPU tests need a CUDA device"


def _run_and_compare(inp, **kw):
    call = run_gpu(inp)
    assert call.check_status() == 0
    ref = oracle_run(inp)
    return call, ref, compare(inp, call, ref, **kw)


def test_tiny_config():
    """1 x 2 x 4 rows of 1024 fp32 logits, given confidence logits."""
    inp = make_inputs("tiny", device="cuda")
    _run_and_compare(inp)


@pytest.mark.parametrize("dtype,V", [("bf16", 1000), ("bf16", 12344), ("bf16", 50008), ("bf16", 151936),
                                     ("f32", 1024), ("f32", 5000), ("f32", 30000), ("f32", 100000)])
def test_recipe_shape_across_vocab_sizes(dtype, V):
    """Every cluster build, ragged tails (V not a multiple of the segment), prefix masks
    with stray ones after the prefix (the cumprod must drop them)."""
    inp = make_inputs("recipe", device="cuda", B=2, N=5, K=7, V=V, dtype=dtype, mask_holes=True, seed=7 + V)
    _run_and_compare(inp)


def test_given_confidence_logits_bf16():
    inp = make_inputs("recipe", device="cuda", B=2, N=4, K=7, V=4096, conf="given", seed=3)
    _run_and_compare(inp)


def test_ce_only_without_teacher():
    inp = make_inputs("recipe", device="cuda", B=2, N=4, K=7, V=8192, no_target=True, seed=4)
    _run_and_compare(inp)


def test_gamma_none_and_grad_scale():
    inp = make_inputs("recipe", device="cuda", B=2, N=4, K=7, V=8192, gamma=None, grad_scale=0.37, seed=5)
    _run_and_compare(inp)


def test_identical_rows_give_zero_l1():
    """draft == teacher: L1 = 0 (the oracle gives exactly 0; the kernel forms the
    draft and teacher exponentials at different program points, which agree to the
    approximation bound of ex2 rather than bit for bit), accept = 1, tau = K + 1."""
    inp = make_inputs("recipe", device="cuda", B=1, N=3, K=7, V=16384, prefix=(7, 7), seed=6)
    inp.target_logits = inp.draft_logits.clone()
    call, ref, _ = _run_and_compare(inp)
    assert np.all(ref["l1"] == 0.0)
    l1 = call.out.l1_rows.cpu().numpy()
    assert np.all(np.abs(l1) <= 1e-6)
    assert np.allclose(call.out.accept_rows.cpu().numpy(), 1.0, atol=1e-6)
    tau = call.out.report[5].tolist()
    assert tau[1] == 3.0 and abs(tau[0] - 3.0 * 8) <= 1e-4 * 24


@pytest.mark.parametrize("separate", [False, True])
def test_identical_rows_dlogits_every_element(separate):
    """draft == teacher puts every |p_j - q_j| at its kink.  The forward's S counts each
    exact tie as +p_j; the fused and the separate backward take that same sign, which
    makes dL/dz = g w ce_alpha (p - onehot), the oracle's value (its sign(0) = 0 gives
    S = 0 and the same dz), on every element, none skipped."""
    from speculative_decoding_draft_vocab_b200 import torch_api
    inp = make_inputs("recipe", device="cuda", B=1, N=3, K=7, V=16384, prefix=(7, 7), seed=6)
    inp.target_logits = inp.draft_logits.clone()
    call = torch_api.Call(inp, grads=True)
    if separate:
        call.out.dlogits.fill_(5.0)
        torch_api.Call(inp, out=call.out, grads=False).launch()
        call.backward()
    else:
        call.launch()
    torch.cuda.synchronize()
    assert call.check_status() == 0
    ref = oracle_run(inp)
    g = call.out.dlogits.view(inp.R, inp.V)
    for r in ref["rows"]:
        check_dlogit_row(g[r].float().cpu().double().numpy(), ref["dlogits"][r],
                         np.zeros(inp.V, dtype=bool), inp.dtype, tag=f"row {r}")


def test_disjoint_rows_l1_two():
    """Disjoint saturated rows: L1 = 2, accept = 0, tau = 1."""
    inp = make_inputs("recipe", device="cuda", B=1, N=2, K=3, V=2048, prefix=(3, 3), seed=8)
    d = torch.full_like(inp.draft_logits, -60.0)
    t = torch.full_like(inp.draft_logits, -60.0)
    for k in range(3):
        d[0, :, k, 10 + k] = 60.0
        t[0, :, k, 1000 + k] = 60.0
    inp.draft_logits, inp.target_logits = d, t
    call, ref, _ = _run_and_compare(inp)
    assert np.allclose(call.out.l1_rows.cpu().numpy(), 2.0, atol=1e-6)
    assert call.out.report[5].tolist() == [2.0, 2.0]


@pytest.mark.parametrize("B,N,K,V", [(8, 40, 7, 4096), (8, 128, 8, 1024), (4, 257, 8, 1024), (2, 9, 3, 2048)])
def test_many_rows_dropped_blocks_and_bad_ids(B, N, K, V):
    """Up to 8224 rows of small vocabularies (many rows per cluster, the row-scalar ring
    refilled several times), masks with holes, blocks dropped at random, then a few
    out-of-range ids on supervised positions: flagged, and their rows dropped from the
    supervised list (zero dlogits)."""
    inp = make_inputs("recipe", device="cuda", B=B, N=N, K=K, V=V, mask_holes=True, seed=31 + B * N * K)
    gen = torch.Generator(device="cpu").manual_seed(B * N)
    drop = (torch.rand(inp.block_keep.shape, generator=gen) < 0.2).to(inp.block_keep.device)
    inp.block_keep[drop] = 0
    call = run_gpu(inp)
    from speculative_decoding_draft_vocab_b200 import abi
    assert call.check_status() == 0
    compare(inp, call, oracle_run(inp))
    # out-of-range ids on supervised positions
    flat = inp.target_ids.view(-1)
    sup = (torch.cumprod(inp.eval_mask.long(), dim=-1) * inp.block_keep.long().unsqueeze(-1)).view(-1)
    cand = torch.nonzero(sup.cpu()).view(-1)
    bad = cand[torch.randperm(cand.numel(), generator=gen)[:3]].to(flat.device)
    flat[bad] = V + 3
    call = run_gpu(inp)
    assert call.check_status() == abi.DSPARK_ERR_ID_OUT_OF_RANGE
    flat[bad] = 0
    for r in bad.tolist():
        b, rest = divmod(r, N * K)
        n, k = divmod(rest, K)
        assert bool((call.out.dlogits[b, n, k] == 0).all())


@pytest.mark.parametrize("heads", [False, True])
def test_fused_call_replays_in_a_cuda_graph(heads):
    """The fused call captured into a CUDA graph (after one eager call, which sets the
    launch attributes up) and replayed: the same outputs bit for bit as the eager call,
    through the programmatic dependent launches of the sweep and the zero-row fill."""
    from speculative_decoding_draft_vocab_b200 import torch_api
    kw = dict(markov=True, conf="head", markov_std=0.2) if heads else {}
    inp = make_inputs("recipe", device="cuda", B=2, N=4, K=7, V=8192, mask_holes=True, seed=61, **kw)
    call = torch_api.Call(inp, grads=True, rows=True)
    call.launch()
    torch.cuda.synchronize()
    assert call.check_status() == 0
    eager = {k: v.clone() for k, v in (("loss", call.out.loss_num), ("report", call.out.report),
                                       ("dlogits", call.out.dlogits), ("l1", call.out.l1_rows))}
    for t in (call.out.loss_num, call.out.report, call.out.dlogits, call.out.l1_rows):
        t.zero_()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call.launch()
    graph.replay()
    torch.cuda.synchronize()
    assert call.check_status() == 0
    assert torch.equal(call.out.loss_num, eager["loss"])
    assert torch.equal(call.out.report, eager["report"])
    assert torch.equal(call.out.l1_rows, eager["l1"])
    assert torch.equal(call.out.dlogits, eager["dlogits"])


def test_all_masked_batch():
    inp = make_inputs("recipe", device="cuda", B=2, N=3, K=7, V=4096, prefix=(0, 0), seed=9)
    call, ref, _ = _run_and_compare(inp)
    assert int(call.out.num_tokens.item()) == 0
    assert float(call.out.loss_num.item()) == 0.0
    assert bool((call.out.dlogits == 0).all())


def test_out_of_range_id_is_flagged_and_skipped():
    inp = make_inputs("recipe", device="cuda", B=1, N=2, K=7, V=4096, prefix=(7, 7), seed=10)
    inp.target_ids[0, 1, 3] = 4096 + 5
    call = run_gpu(inp)
    from speculative_decoding_draft_vocab_b200 import abi
    assert call.check_status() == abi.DSPARK_ERR_ID_OUT_OF_RANGE
    # the offending row is dropped: one token fewer, a zero dlogits row
    assert int(call.out.num_tokens.item()) == 13
    assert bool((call.out.dlogits[0, 1, 3] == 0).all())
    # the next call on the same workspace starts clean
    inp.target_ids[0, 1, 3] = 7
    call2 = run_gpu(inp)
    assert call2.check_status() == 0


def test_separate_backward_matches_oracle():
    """Forward without grads, then dspark_loss_bwd from the saved row statistics."""
    from speculative_decoding_draft_vocab_b200 import torch_api
    inp = make_inputs("recipe", device="cuda", B=2, N=4, K=7, V=30000, conf="given", mask_holes=True, seed=11)
    call = torch_api.Call(inp, grads=True)
    fwd_only = torch_api.Call(inp, out=call.out, grads=False)
    call.out.dlogits.fill_(7.0)
    fwd_only.launch()
    call.backward()
    torch.cuda.synchronize()
    assert call.check_status() == 0
    ref = oracle_run(inp)
    compare(inp, call, ref)


def test_repeat_calls_are_bitwise_identical():
    inp = make_inputs("recipe", device="cuda", B=2, N=4, K=7, V=151936, seed=12)
    a = run_gpu(inp)
    b = run_gpu(inp)
    assert torch.equal(a.out.dlogits, b.out.dlogits)
    assert torch.equal(a.out.report, b.out.report)
    assert torch.equal(a.out.l1_rows, b.out.l1_rows)


def test_acceptance_entry_point_closed_form_and_oracle():
    from oracle import dspark_oracle as O
    from speculative_decoding_draft_vocab_b200 import torch_api
    K = 7
    for a in (0.0, 0.4, 0.9, 1.0):
        l1 = torch.full((2 * 3 * K,), 2 * (1 - a), dtype=torch.float32, device="cuda")
        ev = torch.ones((2, 3, K), dtype=torch.uint8, device="cuda")
        ap, tp, _ = torch_api.acceptance(l1, ev)
        ref = K + 1.0 if a == 1.0 else (1 - a ** (K + 1)) / (1 - a)
        assert tp[1].item() == 6.0
        assert abs(tp[0].item() - 6 * ref) <= 1e-4 * 6 * ref
    g = torch.Generator().manual_seed(0)
    l1 = (torch.rand((4, 9, 16), generator=g) * 2).float()
    L = torch.randint(0, 17, (4, 9), generator=g)
    ev = (torch.arange(16).view(1, 1, 16) < L.view(4, 9, 1)).to(torch.uint8)
    keep = (L >= 1).to(torch.uint8)
    ap, tp, ar = torch_api.acceptance(l1.reshape(-1).cuda(), ev.cuda(), keep.cuda())
    m = O.prefix_supervision_mask(ev.numpy(), keep.numpy())
    rep = O.acceptance_report(l1.double().numpy(), m, keep.numpy())
    assert ap[1].item() == rep["accept"][1] and tp[1].item() == rep["tau"][1]
    assert abs(ap[0].item() - rep["accept"][0]) <= 1e-4 * rep["accept"][0]
    assert abs(tp[0].item() - rep["tau"][0]) <= 1e-4 * rep["tau"][0]
    np.testing.assert_allclose(ar.cpu().numpy(), rep["accept_rows"].reshape(-1), atol=1e-6)


def test_full_recipe_workload_every_row():
    """The bench workload: 4 x 16 x 7 rows of 151936 bf16 logits, every row checked."""
    inp = make_inputs("recipe", device="cuda")
    call, ref, n_amb = _run_and_compare(inp)
    # sign ties are rare: a handful of elements out of ~39M
    assert n_amb < 1000
