"""The data-parallel path on two CPU ranks (gloo).  Each rank owns whole blocks of the
micro-batch, computes its outputs, and the library's reduction helper
(``torch_api.reduce_report``: one all-reduce of the packed report vector, nothing
divided) sums them.  The sums must equal the full batch's: counts and denominators bit
for bit, numerators to rounding; the per-token mean is formed once, after the sum
([MB-API] Return contract).  The head weight gradients, all-reduced the same way and
divided by the global token count, must equal the full batch's per-token gradient (the
"DP-averaged gradient equals the full-batch gradient" check of Megatron-Bridge pull
request #5241, dp_group commit).  No GPU here: the per-rank outputs come from the oracle;
the reduction is the product helper that bench.py's data-parallel ranks call over NCCL."""

import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import dspark_oracle as O


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _problem(seed=3, B=4, N=5, K=6, V=40, rank=8, H=16):
    rng = np.random.default_rng(seed)
    draft = rng.normal(0, 2, (B, N, K, V))
    target = 0.8 * draft + rng.normal(0, 1, (B, N, K, V))
    ids = rng.integers(0, V, (B, N, K))
    L = rng.integers(0, K + 1, (B, N))
    ev = (np.arange(K)[None, None, :] < L[..., None]).astype(np.uint8)
    keep = (L >= 1).astype(np.uint8)
    heads = dict(prev_ids=rng.integers(0, V, (B, N, K)), valid=(rng.random((B, N, K)) < 0.8).astype(np.uint8),
                 markov_w1=rng.normal(0, 0.3, (V, rank)), markov_w2=rng.normal(0, 0.3, (V, rank)),
                 draft_hidden=rng.normal(0, 1, (B, N, K, H)), conf_w=rng.normal(0, 0.2, (1, H + rank)),
                 conf_b=np.array([0.1]), conf_with_markov=True)
    return draft, target, ids, ev, keep, heads


def _oracle(sl=slice(None)):
    draft, target, ids, ev, keep, h = _problem()
    hs = {k: (v[sl] if k in ("prev_ids", "valid", "draft_hidden") else v) for k, v in h.items()}
    return O.dspark_loss(draft[sl], ids[sl], ev[sl], target_logits=target[sl], block_keep=keep[sl], **hs)


def _as_outputs(res):
    """The library's forward outputs for one rank (FP64 so the check is not limited by
    FP32 storage)."""
    loss = torch.tensor([res["loss_num"]], dtype=torch.float64)
    ntok = torch.tensor([res["num_tokens"]], dtype=torch.int64)
    rep = torch.tensor([res["report"][k] for k in O.REPORT_KEYS], dtype=torch.float64)
    return loss, ntok, rep


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from speculative_decoding_draft_vocab_b200 import torch_api
    res = _oracle(slice(rank * 2, rank * 2 + 2))  # batch entries split over the ranks (whole blocks)
    loss, ntok, rep = torch_api.reduce_report(*_as_outputs(res))
    # head weight gradients: summed over the ranks like any data-parallel gradient
    grads = torch.from_numpy(np.concatenate([res["dW2"].reshape(-1), res["dconf_w"].reshape(-1)]))
    dist.all_reduce(grads, op=dist.ReduceOp.SUM)
    out[rank] = dict(loss=loss.tolist(), ntok=ntok.tolist(), rep=rep.reshape(-1).tolist(),
                     grads=grads.tolist())
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_report_reduction_equals_full_batch():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    full = _oracle()
    f_loss, f_ntok, f_rep = _as_outputs(full)
    f_grads = np.concatenate([full["dW2"].reshape(-1), full["dconf_w"].reshape(-1)])
    for r in range(world):
        got = out[r]
        # counts and denominators exact, numerators to rounding
        assert got["ntok"] == f_ntok.tolist()
        rep = np.array(got["rep"]).reshape(-1, 2)
        assert np.array_equal(rep[:, 1], f_rep.numpy()[:, 1])
        np.testing.assert_allclose(rep[:, 0], f_rep.numpy()[:, 0], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(got["loss"], f_loss.tolist(), rtol=1e-12, atol=1e-12)
        # the per-token mean and the per-token gradient, formed once from the sums
        n = float(got["ntok"][0])
        assert n > 0
        np.testing.assert_allclose(got["loss"][0] / n, full["loss_num"] / full["num_tokens"], rtol=1e-12)
        np.testing.assert_allclose(np.array(got["grads"]) / n, f_grads / full["num_tokens"],
                                   rtol=1e-10, atol=1e-13)


def _bad_worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from speculative_decoding_draft_vocab_b200 import torch_api
    try:
        torch_api.reduce_report(torch.zeros(1), torch.zeros(1, dtype=torch.int64), torch.zeros(5))
        out[rank] = "accepted"
    except ValueError:
        out[rank] = "refused"
    dist.barrier()
    dist.destroy_process_group()


def test_report_reduction_refuses_a_short_report():
    """A report of the wrong length is refused before any collective is issued (so no
    rank is left waiting in an all-reduce the others never join)."""
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_bad_worker, args=(2, port, out), nprocs=2, start_method="spawn", join=True)
    assert dict(out) == {0: "refused", 1: "refused"}
