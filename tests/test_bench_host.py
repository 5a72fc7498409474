"""The roofline arithmetic of bench.py, pinned to sums written out by hand: the
algorithmic bytes and tensor-core FLOPs of each workload's call and of one
vocabulary-parallel rank.  Shapes only (meta tensors); no GPU."""

from types import SimpleNamespace

import torch

import bench

V = 151936


def _inp(R=448, dtype="bf16", target=True, markov_rank=None, hidden=None, lm_hidden=None, Vt=V):
    meta = dict(device="meta")
    return SimpleNamespace(
        dtype=dtype, V=V, R=R,
        target_logits=torch.empty(R, V, **meta) if target else None,
        markov_w2=torch.empty(V, markov_rank, **meta) if markov_rank else None,
        markov_w1=torch.empty(Vt, markov_rank, **meta) if markov_rank else None,
        conf_w=torch.empty(1, hidden, **meta) if hidden else None,
        draft_hidden=torch.empty(R, hidden, **meta) if hidden else None,
        lm_head=torch.empty(V, lm_hidden, **meta) if lm_hidden else None)


def test_recipe_bytes():
    """251 supervised rows of 448: draft and teacher read once (2 B each per logit),
    dlogits written for every row."""
    assert bench.algorithmic_bytes(_inp(), 251) == 251 * V * 2 * 2 + 448 * V * 2 == 288_678_400
    assert bench.algorithmic_flops(_inp(), 251) == 0


def test_heads_bytes_and_flops():
    """Markov rank 256 (W2 read in bf16, dW2 written in fp32; the supervised rows'
    embeddings and their dW1 rows) and the confidence head's hidden rows (read and
    gradient written, bf16); three rank-256 contractions against the vocabulary."""
    inp = _inp(markov_rank=256, hidden=4096)
    want = (252 * V * 2 * 2 + 448 * V * 2) + V * 256 * (2 + 4) + 252 * 256 * (2 + 4) + 448 * 4096 * 2 * 2
    assert bench.algorithmic_bytes(inp, 252) == want
    assert bench.algorithmic_flops(inp, 252) == 3 * 2 * 252 * V * 256


def test_teacher_from_hidden_bytes_and_flops():
    """lm_head [V, 4096] and the supervised rows' hidden states read instead of teacher
    logits; the teacher product is 2 * rows * V * 4096 FLOPs."""
    inp = _inp(target=False, lm_hidden=4096)
    assert bench.algorithmic_bytes(inp, 245) == 245 * V * 2 + 448 * V * 2 + V * 4096 * 2 + 245 * 4096 * 2
    assert bench.algorithmic_flops(inp, 245) == 2 * 245 * V * 4096


def test_tp_rank_bytes():
    """One rank of eight: 18992 columns of the 251 supervised rows' draft and teacher,
    and of all 448 rows' dlogits."""
    assert bench.tp_algorithmic_bytes(_inp(), 251, 18992) == 251 * 18992 * 4 + 448 * 18992 * 2 == 36_084_800
    assert bench.tp_algorithmic_bytes(_inp(target=False), 251, 18992) == 251 * 18992 * 2 + 448 * 18992 * 2


def test_tp_rank_heads_bytes_flops_and_launches():
    """A rank's W2 rows (read bf16, gradient written fp32), the supervised embeddings and
    dW1 rows, the hidden states; three rank-256 contractions against its columns."""
    inp = _inp(markov_rank=256, hidden=4096)
    want = 252 * 18992 * 4 + 448 * 18992 * 2 + 18992 * 256 * 6 + 252 * 256 * 6 + 448 * 4096 * 4
    assert bench.tp_algorithmic_bytes(inp, 252, 18992) == want
    assert bench.tp_algorithmic_flops(inp, 252, 18992) == 6 * 252 * 18992 * 256
    assert bench.tp_launches_per_step(_inp()) == 4
    assert bench.tp_launches_per_step(inp) == 4 + 1 + 5 + 3


def test_roofline_entry_bound_and_fractions():
    """The recipe call (4 x 16 x 7 x 151936 bf16, 251 supervised rows): 288,678,400 B in
    0.0974 ms is 2963.8 GB/s, 0.459 of the measured 6458.1 GB/s and 0.370 of the nominal
    8 TB/s; the dense figure counts every row's draft, teacher and dlogits (448 x 151936
    x 6 B)."""
    hbm, tc = (6458.1, "measured"), (1590.0, "measured")
    r = bench.roofline_entry(288_678_400, 0, 0.0974, hbm, tc, "t", traffic=1, dense=bench.dense_bytes(_inp()))
    assert r["bound"] == "hbm" and r["unit"] == "GB/s" and r["traffic"] == 1
    assert r["achieved"] == round(288_678_400 / 0.0974e-3 / 1e9, 1)
    assert r["frac"] == round(288_678_400 / 0.0974e-3 / 1e9 / 6458.1, 4) == 0.4589
    assert r["frac_of_nominal"] == round(288_678_400 / 0.0974e-3 / 1e9 / 8000.0, 4)
    assert r["dense_bytes"] == 448 * V * 6 == 408_403_968
    # the teacher product's FLOPs outweigh its bytes at these peaks: a tensor bound
    t = bench.roofline_entry(1_000_000, 10**12, 1.0, hbm, tc, "t")  # 1 TFLOP in 1 ms: 1000 TFLOP/s
    assert t["bound"] == "tensor" and t["unit"] == "TFLOP/s" and t["achieved"] == 1000.0
    assert t["frac"] == round(1000.0 / 1590.0, 4)
    assert "frac_of_nominal" not in t


def test_oracle_pool_baseline_on_the_tiny_workload():
    """The CPU baseline: whole blocks of the workload drawn on the CPU, the oracle run in
    worker processes forked before any CUDA call, on one core and on every core."""
    inp = bench.cpu_inputs("tiny")
    pool = bench.OraclePool({"tiny": bench.oracle_view(inp)}, procs=2)
    try:
        res = bench.cpu_baseline(pool, "tiny", 0.05)
        # one task over both blocks reproduces the whole micro-batch's supervised rows
        rows, _ = pool.run([("tiny", 0, 2)])[0]
    finally:
        pool.close()
    assert rows == int(inp.eval_mask.sum())
    assert res["one_core"]["cores"] == 1 and res["all_cores"]["cores"] == 2
    assert res["one_core"]["value"] > 0 and res["all_cores"]["value"] > 0


def test_block_ranges_wrap_and_stay_in_bounds():
    r = bench._block_ranges(5, 8, 3, 4)
    assert r == [(5, 8), (0, 3), (3, 6), (6, 8)]
    assert all(0 <= a < b <= 8 for a, b in r)


def test_gpus_flag_starts_one_process_per_gpu(monkeypatch):
    """Without a launcher, --gpus N re-runs the script under torch.distributed.run with N
    processes on 127.0.0.1; under a launcher the world size must match --gpus."""
    seen = {}

    class FakeProc:
        pid = 0

        def __init__(self, cmd, env=None, start_new_session=False):
            seen["cmd"], seen["env"] = cmd, env

        def wait(self, timeout=None):
            return 0

    monkeypatch.delenv("WORLD_SIZE", raising=False)
    monkeypatch.setattr(bench.subprocess, "Popen", FakeProc)
    assert bench.main(["--gpus", "4", "--steps", "5", "--warmup", "3"]) == 0
    cmd = seen["cmd"]
    assert cmd[1:4] == ["-m", "torch.distributed.run", "--nnodes=1"]
    assert "--nproc-per-node=4" in cmd and cmd[cmd.index("--master-addr") + 1] == "127.0.0.1"
    assert cmd[-6:] == ["--gpus", "4", "--steps", "5", "--warmup", "3"]
    assert seen["env"]["NCCL_DEBUG"]
    monkeypatch.setenv("WORLD_SIZE", "2")
    import pytest
    with pytest.raises(SystemExit):
        bench.main(["--gpus", "4"])
