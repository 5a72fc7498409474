"""The vocabulary-parallel exchange protocol on CPU ranks (gloo): each rank holds one
vocabulary shard of every row, reduces it to the records include/dspark.h defines
(record 1: base-2 logsumexp partials and the target logit; record 2: L1 and S parts),
and ``torch_api.tp_exchange`` (the binding's all-gather) hands every rank all ranks'
records in rank order.  Merged in that order they give the full-row CE, L1 and S of
the oracle, identically on every rank (NeMo RL design doc "DSpark Auxiliary Heads",
Tensor Parallelism).  The per-shard arithmetic is the oracle's (no GPU here); the
record layout, the exchange and the rank order are the product's."""

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
