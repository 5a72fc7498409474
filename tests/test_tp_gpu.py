"""GPU parity of the vocabulary-parallel path (dspark_tp_partials, dspark_tp_l1,
dspark_tp_finish) against the FP64 oracle of the whole rows.

A tensor-parallel group is emulated on one device: its ranks run one after another over
even shards of the full rows, and the exchange is a stack of their records (what the
all-gather would deliver).  No kernel waits on another.  Every rank must report the
same forward outputs, bit for bit; dlogits are assembled from the ranks' columns.
NeMo RL design doc "DSpark Auxiliary Heads", Tensor Parallelism.
"""

import math
from types import SimpleNamespace

import numpy as np
import pytest
import torch

from oracle import dspark_oracle as O
from speculative_decoding_draft_vocab_b200.synthetic import make_inputs
from tests.parity_util import check_dlogit_row, check_heads, compare, np32, oracle_run

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _built():
    from speculative_decoding_draft_vocab_b200 import build
    build.build()
    assert torch.cuda.is_available(), "the GPU tests need a CUDA device"


def _group(inp, tp_size, grads=True, mode=0):
    from speculative_decoding_draft_vocab_b200 import torch_api
    ranks = torch_api.tp_group_emulated(inp, tp_size, grads=grads, invalid_row_mode=mode)
    torch.cuda.synchronize()
    for r in ranks:
        assert r.check_status() == 0
    return ranks


def _as_call(rank):
    """The fields of one rank that the parity helpers read."""
    return SimpleNamespace(out=SimpleNamespace(
        num_tokens=rank.num_tokens, report=rank.report, loss_num=rank.loss_num, ce_rows=rank.ce_rows,
        l1_rows=rank.l1_rows, accept_rows=rank.accept_rows, conf_rows=rank.conf_rows, dconf=rank.dconf,
        dlogits=rank.dlogits, dW1=rank.dW1, dW2=rank.dW2, dconf_w=rank.dconf_w, dconf_b=rank.dconf_b,
        dhidden=rank.dhidden))


def _check_group(inp, ranks, ref, **kw):
    compare(inp, _as_call(ranks[0]), ref, **kw)
    for r in ranks[1:]:  # every rank holds the same forward outputs
        for name in ("loss_num", "num_tokens", "report", "ce_rows", "l1_rows", "accept_rows", "dconf"):
            assert torch.equal(getattr(r, name), getattr(ranks[0], name)), name


@pytest.mark.parametrize("dtype,V,T", [("bf16", 4096, 1), ("bf16", 4096, 2), ("bf16", 50008, 3),
                                       ("bf16", 151936, 8), ("f32", 5000, 3), ("f32", 30000, 4)])
def test_tp_group_matches_oracle(dtype, V, T):
    """Even shards (uneven where V does not divide), ragged prefix masks with stray ones."""
    inp = make_inputs("recipe", device="cuda", B=2, N=5, K=7, V=V, dtype=dtype, mask_holes=True, seed=40 + V + T)
    ranks = _group(inp, T)
    _check_group(inp, ranks, oracle_run(inp))


def test_tp_dropped_blocks_and_many_rows():
    """Blocks dropped at random (block_keep 0 on blocks whose masks are set) and more rows
    than the step kernels have CTAs: step 1 decides itself which rows are supervised, by
    the prologue's rule, and must agree with the prologue's lists that steps 2 and 3 use."""
    inp = make_inputs("recipe", device="cuda", B=4, N=80, K=7, V=4096, mask_holes=True, seed=48)
    gen = torch.Generator(device="cpu").manual_seed(48)
    drop = (torch.rand(inp.block_keep.shape, generator=gen) < 0.25).to(inp.block_keep.device)
    inp.block_keep[drop] = 0
    ranks = _group(inp, 3)
    _check_group(inp, ranks, oracle_run(inp))


@pytest.mark.parametrize("T,prenorm,heads", [(2, False, False), (3, True, False), (2, False, True)])
def test_tp_teacher_from_hidden_states(T, prenorm, heads):
    """The teacher from the target's hidden states on the vocabulary-parallel path: each
    rank computes its shard's teacher rows from its rows of lm_head (and, pre-norm, the
    final RMS norm of the replicated hidden states); with the heads as well."""
    kw = dict(markov=True, conf="head", markov_std=0.2, valid_p=0.8) if heads else {}
    inp = make_inputs("recipe", device="cuda", B=2, N=5, K=7, V=4096, lm_head=True, target_hidden_size=256,
                      target_prenorm=prenorm, mask_holes=True, seed=50 + T + 2 * int(prenorm), **kw)
    ranks = _group(inp, T)
    _check_group(inp, ranks, oracle_run(inp))


def test_tp_teacher_from_hidden_states_refuses_more_than_one_chunk():
    """All supervised rows' teacher rows stay in the workspace's teacher chunk through the
    three calls: more than 512 rows are refused before anything is enqueued."""
    inp = make_inputs("recipe", device="cuda", B=2, N=37, K=7, V=1024, lm_head=True, target_hidden_size=64,
                      seed=55)
    from speculative_decoding_draft_vocab_b200 import abi, torch_api
    rank = torch_api.TPRank(inp, 2, 0, inp.V, col0=0, width=512)
    with pytest.raises(abi.DSparkError) as e:
        rank.partials()
    assert e.value.status == abi.DSPARK_ERR_UNSUPPORTED


def test_tp_rank_replays_in_a_cuda_graph():
    """One rank's three calls (programmatic dependent launches of steps 1-3) captured into
    a CUDA graph with the group's records fixed, and replayed: rank 0's outputs bit for bit
    as eagerly computed."""
    inp = make_inputs("recipe", device="cuda", B=2, N=5, K=7, V=4096, mask_holes=True, seed=63)
    ranks = _group(inp, 2)
    r0 = ranks[0]
    rec1_all = torch.stack([r.rec1 for r in ranks]).clone()
    rec2_all = torch.stack([r.rec2 for r in ranks]).clone()
    c0, c1 = r0.col0, r0.col0 + r0.width
    eager = (r0.loss_num.clone(), r0.report.clone(), r0.l1_rows.clone(), r0.dlogits[..., c0:c1].clone())
    for t in (r0.loss_num, r0.report, r0.l1_rows):
        t.zero_()
    r0.dlogits[..., c0:c1].zero_()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        r0.partials()
        r0.l1(rec1_all)
        r0.finish(rec2_all)
    graph.replay()
    torch.cuda.synchronize()
    assert r0.check_status() == 0
    assert torch.equal(r0.loss_num, eager[0])
    assert torch.equal(r0.report, eager[1])
    assert torch.equal(r0.l1_rows, eager[2])
    assert torch.equal(r0.dlogits[..., c0:c1], eager[3])


def test_tp_given_confidence_gamma_none_grad_scale():
    inp = make_inputs("recipe", device="cuda", B=2, N=4, K=7, V=8192, conf="given", gamma=None,
                      grad_scale=0.37, seed=41)
    _check_group(inp, _group(inp, 4), oracle_run(inp))


def test_tp_ce_only_without_teacher():
    inp = make_inputs("recipe", device="cuda", B=2, N=4, K=7, V=8192, no_target=True, seed=42)
    _check_group(inp, _group(inp, 2), oracle_run(inp))


def test_tp_forward_only_and_all_masked():
    inp = make_inputs("recipe", device="cuda", B=2, N=3, K=7, V=4096, seed=43)
    ranks = _group(inp, 2, grads=False)
    compare(inp, _as_call(ranks[0]), oracle_run(inp, want_grads=False))
    inp = make_inputs("recipe", device="cuda", B=2, N=3, K=7, V=4096, prefix=(0, 0), seed=44)
    ranks = _group(inp, 4)
    assert int(ranks[0].num_tokens.item()) == 0 and float(ranks[0].loss_num.item()) == 0.0
    assert bool((ranks[0].dlogits == 0).all())


def test_tp_records_follow_the_header():
    """Record 1 holds the shard's base-2 maximum and sum of 2^(x log2 e - m) for draft and
    teacher, and the target logit only on the shard that holds the id."""
    from speculative_decoding_draft_vocab_b200 import torch_api
    inp = make_inputs("recipe", device="cuda", B=1, N=2, K=7, V=8192, prefix=(7, 7), seed=45)
    ranks = _group(inp, 4)
    bounds = torch_api.even_shards(inp.V, 4, 8)
    z = np32(inp.draft_logits).reshape(inp.R, inp.V).astype(np.float64)
    t = np32(inp.target_logits).reshape(inp.R, inp.V).astype(np.float64)
    ids = np32(inp.target_ids).reshape(-1)
    log2e = 1.0 / math.log(2.0)
    for k, rk in enumerate(ranks):
        lo, hi = bounds[k], bounds[k + 1]
        rec = rk.rec1.double().cpu().numpy()
        for r in range(inp.R):
            md, sd = O.lse_partial(z[r, lo:hi])
            mt, st = O.lse_partial(t[r, lo:hi])
            assert abs(rec[r, 0] - md * log2e) <= 1e-6 * abs(md * log2e) + 1e-6
            assert abs(rec[r, 1] - sd) <= 1e-5 * sd
            assert abs(rec[r, 2] - mt * log2e) <= 1e-6 * abs(mt * log2e) + 1e-6
            assert abs(rec[r, 3] - st) <= 1e-5 * st
            assert rec[r, 4] == (z[r, ids[r]] if lo <= ids[r] < hi else 0.0)


def test_tp_out_of_range_id_is_flagged_and_skipped():
    inp = make_inputs("recipe", device="cuda", B=1, N=2, K=7, V=4096, prefix=(7, 7), seed=46)
    inp.target_ids[0, 1, 3] = 4096 + 5
    from speculative_decoding_draft_vocab_b200 import abi, torch_api
    ranks = torch_api.tp_group_emulated(inp, 2)
    assert ranks[0].check_status() == abi.DSPARK_ERR_ID_OUT_OF_RANGE
    assert int(ranks[1].num_tokens.item()) == 13
    assert bool((ranks[0].dlogits[0, 1, 3] == 0).all())


def test_tp_identical_rows():
    """draft == teacher: every |p_j - q_j| is at its kink; the ranks' S counts each tie
    as +p_j and dL/dz takes the same sign, which makes dz = g w ce_alpha (p - onehot),
    the oracle's value, on every element (none skipped)."""
    inp = make_inputs("recipe", device="cuda", B=1, N=3, K=7, V=16384, prefix=(7, 7), seed=6)
    inp.target_logits = inp.draft_logits.clone()
    ranks = _group(inp, 4)
    ref = oracle_run(inp)
    assert np.allclose(ranks[0].l1_rows.cpu().numpy(), 0.0, atol=1e-6)
    g = ranks[0].dlogits.view(inp.R, inp.V)
    for r in ref["rows"]:
        check_dlogit_row(g[r].float().cpu().double().numpy(), ref["dlogits"][r],
                         np.zeros(inp.V, dtype=bool), inp.dtype, tag=f"row {r}")


def test_tp_recipe_workload_every_row():
    """The bench workload (4 x 16 x 7 rows of 151936 bf16 logits) over 8 ranks, every row
    checked, and the group agrees with the single-device fused call."""
    from speculative_decoding_draft_vocab_b200 import torch_api
    inp = make_inputs("recipe", device="cuda")
    ranks = _group(inp, 8)
    ref = oracle_run(inp)
    _check_group(inp, ranks, ref)
    fused = torch_api.Call(inp)
    fused.launch()
    torch.cuda.synchronize()
    assert torch.equal(fused.out.num_tokens, ranks[0].num_tokens)
    rel = (fused.out.report - ranks[0].report).abs() / fused.out.report.abs().clamp_min(1e-6)
    assert float(rel.max()) <= 2e-5


HEADS = dict(B=2, N=4, K=7, V=8192, hidden=512, rank=64, target_vocab=3000, markov_std=0.3,
             conf_bias=0.25, valid_p=0.7, mask_holes=True)


@pytest.mark.parametrize("mode", [0, 1])
@pytest.mark.parametrize("T", [2, 4])
def test_tp_heads_match_oracle(mode, T):
    """Markov head with W2's rows split over the ranks and the confidence head fed the
    Markov embedding: forward, dlogits and every weight gradient against the oracle, for
    both invalid-row readings.  dW2 is assembled from the ranks' rows; dL/de is the sum of
    the ranks' parts, so dW1, dproj, dbias and dh come out the same on every rank."""
    inp = make_inputs("recipe_heads", device="cuda", seed=50 + mode + 2 * T, conf_with_markov=True, **HEADS)
    inp.prev_ids = torch.where(inp.valid != 0, inp.prev_ids, torch.full_like(inp.prev_ids, -1))
    ranks = _group(inp, T, mode=mode)
    ref = oracle_run(inp, invalid_row_mode=mode)
    _check_group(inp, ranks, ref)
    for r in ranks:
        # dW1 is a scatter-add (atomics, in no fixed order): every rank's is checked
        # against the oracle with the derived bound, not bit for bit against rank 0's
        check_heads(inp, _as_call(r), ref, mode)
    for r in ranks[1:]:
        for name in ("dconf_w", "dconf_b", "dhidden", "conf_rows"):
            assert torch.equal(getattr(r, name), getattr(ranks[0], name)), name


def test_tp_markov_without_confidence_and_ragged_rank():
    """rank 72 (a ragged tensor-core tile), three ranks over V = 5000 (uneven shards)."""
    inp = make_inputs("recipe_heads", device="cuda", seed=57, B=3, N=5, K=6, V=5000, hidden=200, rank=72,
                      target_vocab=777, markov_std=0.3, conf=None, valid_p=0.8)
    ranks = _group(inp, 3)
    ref = oracle_run(inp)
    _check_group(inp, ranks, ref)
    check_heads(inp, _as_call(ranks[0]), ref, 0)


def test_tp_recipe_heads_workload_every_row():
    """The recipe shape with both heads (4 x 16 x 7 rows, V = 151936, rank 256, hidden 4096)
    on 8 ranks."""
    inp = make_inputs("recipe_heads", device="cuda")
    ranks = _group(inp, 8)
    ref = oracle_run(inp)
    _check_group(inp, ranks, ref)
    st = check_heads(inp, _as_call(ranks[0]), ref, 0)
    assert st["dW2_frob_err"] <= 1.0 and st["dW1_frob_err"] <= 1.0
