"""The data-parallel path on two CPU ranks (gloo): each rank computes its shard of the
blocks, the report vector is summed with all_reduce, and the result equals the
full-batch values; the global ratio is formed once, after the reduction ([MB-API]
Return contract).  The per-rank compute is the oracle (no GPU here); the sharding and
the reduction are the same as bench.py's multi-rank path."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from oracle import dspark_oracle as O


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _problem(seed=3, B=4, N=5, K=6, V=40):
    rng = np.random.default_rng(seed)
    draft = rng.normal(0, 2, (B, N, K, V))
    target = 0.8 * draft + rng.normal(0, 1, (B, N, K, V))
    ids = rng.integers(0, V, (B, N, K))
    L = rng.integers(0, K + 1, (B, N))
    ev = (np.arange(K)[None, None, :] < L[..., None]).astype(np.uint8)
    keep = (L >= 1).astype(np.uint8)
    conf = rng.normal(size=(B, N, K))
    return draft, target, ids, ev, keep, conf


def _report_vector(res):
    v = [res["loss_num"], float(res["num_tokens"])]
    for key in O.REPORT_KEYS:
        v += list(res["report"][key])
    return np.array(v, dtype=np.float64)


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    draft, target, ids, ev, keep, conf = _problem()
    shard = slice(rank * 2, rank * 2 + 2)  # batch rows split over ranks (whole blocks)
    res = O.dspark_loss(draft[shard], ids[shard], ev[shard], target_logits=target[shard],
                        block_keep=keep[shard], confidence_logits=conf[shard])
    t = torch.from_numpy(_report_vector(res))
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    out[rank] = t.numpy().tolist()
    dist.barrier()
    dist.destroy_process_group()


def test_two_rank_report_reduction_equals_full_batch():
    world = 2
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    draft, target, ids, ev, keep, conf = _problem()
    full = _report_vector(O.dspark_loss(draft, ids, ev, target_logits=target, block_keep=keep,
                                        confidence_logits=conf))
    for r in range(world):
        got = np.array(out[r])
        # counts and denominators exact, numerators to rounding
        assert got[1] == full[1]
        assert np.array_equal(got[3::2], full[3::2])
        np.testing.assert_allclose(got, full, rtol=1e-12, atol=1e-12)
    # the global mean is formed once, after the reduction
    loss_mean = full[0] / full[1]
    assert np.isfinite(loss_mean)
