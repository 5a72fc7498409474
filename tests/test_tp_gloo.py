"""The vocabulary-parallel exchange protocol on CPU ranks (gloo): each rank holds one
vocabulary shard of every row, reduces it to the records include/dspark.h defines
(record 1: base-2 logsumexp partials and the target logit; record 2: L1 and S parts;
with the Markov head, its part of dL/de), and ``torch_api.tp_exchange`` (the binding's
all-gather) hands every rank all ranks' records in rank order.  Merged in that order
they give the full-row CE, L1 and S and the embedding gradient of the oracle,
identically on every rank (NeMo RL design doc "DSpark Auxiliary Heads", Tensor
Parallelism).  The per-shard arithmetic is the oracle's (no GPU here); the record
layout, the exchange and the rank order are the product's."""

import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import dspark_oracle as O

LOG2E = 1.0 / math.log(2.0)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rows(seed=5, R=12, V=64):
    rng = np.random.default_rng(seed)
    z = rng.normal(0, 2, (R, V))
    t = 0.8 * z + rng.normal(0, 1.5, (R, V))
    ids = rng.integers(0, V, R)
    return z, t, ids


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from speculative_decoding_draft_vocab_b200 import abi
    from speculative_decoding_draft_vocab_b200.torch_api import even_shards, tp_exchange
    z, t, ids = _rows()
    R, V = z.shape
    b = even_shards(V, world, 8)
    lo, hi = b[rank], b[rank + 1]
    # record 1 of every row: [m_d, s_d, m_t, s_t, z at the id if held, 0, 0, 0], m in base 2
    rec1 = torch.zeros(R, abi.DSPARK_TP_REC1_FLOATS, dtype=torch.float64)
    for r in range(R):
        md, sd = O.lse_partial(z[r, lo:hi])
        mt, st = O.lse_partial(t[r, lo:hi])
        held = lo <= ids[r] < hi
        rec1[r, :5] = torch.tensor([md * LOG2E, sd, mt * LOG2E, st, z[r, ids[r]] if held else 0.0],
                                  dtype=torch.float64)
    all1 = tp_exchange(rec1)
    assert all1.shape == (world, R, abi.DSPARK_TP_REC1_FLOATS)
    assert torch.equal(all1[rank], rec1)
    rec2 = torch.zeros(R, abi.DSPARK_TP_REC2_FLOATS, dtype=torch.float64)
    lse = []
    for r in range(R):
        lse_d = O.merge_lse_partials([(float(all1[k, r, 0]) / LOG2E, float(all1[k, r, 1])) for k in range(world)])
        lse_t = O.merge_lse_partials([(float(all1[k, r, 2]) / LOG2E, float(all1[k, r, 3])) for k in range(world)])
        zt = sum(float(all1[k, r, 4]) for k in range(world))
        l1, S = O.l1_partial(z[r, lo:hi], t[r, lo:hi], lse_d, lse_t)
        rec2[r, :2] = torch.tensor([l1, S], dtype=torch.float64)
        lse.append((lse_d, lse_t, lse_d - zt))
    all2 = tp_exchange(rec2)
    assert all2.shape == (world, R, abi.DSPARK_TP_REC2_FLOATS)
    res = []
    for r in range(R):
        L1 = sum(float(all2[k, r, 0]) for k in range(world))
        S = sum(float(all2[k, r, 1]) for k in range(world))
        res.append([*lse[r], L1, S])
    out[rank] = res
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_vocab_parallel_records_merge_to_full_rows(world):
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    z, t, ids = _rows()
    for r in range(z.shape[0]):
        full = O.row_terms(z[r], t[r], int(ids[r]))
        for k in range(world):
            lse_d, lse_t, ce, l1, S = out[k][r]
            assert out[k][r] == out[0][r]  # every rank holds the same row statistics
            assert abs(lse_d - full["lse_d"]) <= 1e-12 and abs(lse_t - full["lse_t"]) <= 1e-12
            assert abs(ce - full["ce"]) <= 1e-12
            assert abs(l1 - full["l1"]) <= 1e-12 and abs(S - full["S"]) <= 1e-12


def _heads_problem(seed=9, B=1, N=2, K=4, V=48, rank=8, H=6, Vt=11):
    rng = np.random.default_rng(seed)
    d = rng.normal(0, 1.5, (B, N, K, V))
    t = 0.8 * d + rng.normal(0, 1.0, (B, N, K, V))
    ids = rng.integers(0, V, (B, N, K))
    ev = np.ones((B, N, K), dtype=np.uint8)
    ev[0, 1, 3] = 0
    kw = dict(target_logits=t, prev_ids=rng.integers(0, Vt, (B, N, K)),
              valid=np.array([[[1, 1, 0, 1], [1, 1, 1, 1]]]), markov_w1=rng.normal(0, 0.4, (Vt, rank)),
              markov_w2=rng.normal(0, 0.4, (V, rank)), draft_hidden=rng.normal(size=(B, N, K, H)),
              conf_w=rng.normal(0, 0.3, (1, H + rank)), conf_b=np.array([0.1]), conf_with_markov=True)
    return d, ids, ev, kw


def _heads_worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    from speculative_decoding_draft_vocab_b200.torch_api import even_shards, tp_exchange
    d, ids, ev, kw = _heads_problem()
    res = O.dspark_loss(d, ids, ev, **kw)  # every rank holds the rows' dz (after the three steps)
    R, V = ids.size, d.shape[-1]
    w2 = kw["markov_w2"]
    b = even_shards(V, world, 8)
    lo, hi = b[rank], b[rank + 1]
    # this rank's part of dL/de: its rows of W2 against its columns of dz
    part = torch.zeros(R, w2.shape[1], dtype=torch.float64)
    for r in res["dE"]:
        part[r] = torch.from_numpy(w2[lo:hi].T @ res["dlogits"][r][lo:hi])
    parts = tp_exchange(part)
    proj_e = np.asarray(kw["conf_w"]).reshape(-1)[kw["draft_hidden"].shape[-1]:]  # proj's embedding slice
    merged = {r: sum(parts[k, r].numpy() for k in range(world)) + res["dconf"][r] * proj_e for r in res["dE"]}
    out[rank] = {r: v.tolist() for r, v in merged.items()}
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_vocab_parallel_embedding_gradient_reduced_across_ranks(world):
    """dL/de = sum over ranks of W2_k^T dz_k (the reduce across tensor parallelism), plus
    the replicated confidence head's dc * proj_e once: the oracle's dL/de on every rank."""
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_heads_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    d, ids, ev, kw = _heads_problem()
    ref = O.dspark_loss(d, ids, ev, **kw)
    assert len(ref["dE"]) > 0
    for k in range(world):
        assert out[k] == out[0]
        for r, want in ref["dE"].items():
            np.testing.assert_allclose(out[k][r], want, rtol=0, atol=1e-12)
