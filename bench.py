"""Benchmark of the fused DSpark loss forward+backward (one step = one call of
dspark_loss_fwd with the fused backward over one synthetic micro-batch).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload recipe] [--impl reference]

With --gpus N > 1 and no launcher around it, the script starts N ranks itself under
torch.distributed.run (one process per GPU, NCCL); under a launcher it reads RANK,
LOCAL_RANK and WORLD_SIZE.  Every rank draws its own micro-batch (seed offset by rank)
and processes it alone: rows are independent, so there is no collective on the data
path ("scaling": "weak").  The step time is the maximum over ranks.

Prints one JSON line.  `value` is supervised rows per second over all ranks: the rows of
one micro-batch per rank over the maximum across ranks of the median per-call device
time (CUDA events around each call; the L2 cache is flushed by a 512 MiB write before
every timed call, untimed).  `e2e` is the same metric through the same call with the
inputs in pinned host memory: every step copies the micro-batch to the device, runs the
call, sums the report over the data-parallel ranks (one all-reduce, the library's
reduce_report) and reads it back.  At one GPU the line also carries `workloads` (the
recipe micro-batch with the heads, with the teacher from hidden states, and the
8192-row shape, each timed in the same run) and `cpu_baselines` (the FP64 oracle on one
core and on every core, for the recipe and the 8192-row workloads).  Every workload is
drawn once on the CPU and copied to the device, so the oracle and the GPU see the same
inputs.

Other modes:
  --impl reference   times the FP64 CPU oracle (all host cores) on a bounded sample of
                     rows per step, on the same workload draw;
  --tp T             times one rank of a T-way vocabulary-parallel group on one GPU;
  --profile-calls C  runs C fused calls of the workload and exits with the device status
                     (the command the profiles' ncu captures run).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import socket
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from speculative_decoding_draft_vocab_b200.synthetic import CONFIG_ORDER, CONFIGS, make_inputs  # noqa: E402

METRIC = "supervised rows/s, DSpark loss fwd+bwd @V=151936; achieved HBM GB/s vs peak"
PEAKS = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
NOMINAL_HBM_GBS = 8000.0  # the B200 data-sheet HBM3e bandwidth the loss target is quoted against
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "sweep_recipe_traffic.md")
KERNEL_SOURCES = ["speculative_decoding_draft_vocab_b200/csrc/sweep.cu",
                  "speculative_decoding_draft_vocab_b200/csrc/prologue.cu",
                  "speculative_decoding_draft_vocab_b200/csrc/finalize.cuh",
                  "speculative_decoding_draft_vocab_b200/csrc/ptx.cuh",
                  "speculative_decoding_draft_vocab_b200/csrc/internal.cuh"]
EXTRA_WORKLOADS = ("recipe_heads", "lm_head_teacher", "large")
CPU_BASELINE_WORKLOADS = ("recipe", "large")
WEIGHTS = ("markov_w1", "markov_w2", "conf_w", "conf_b", "lm_head", "target_norm_weight")  # resident
HOST_SLACK_CYCLES = 200_000  # device spin before each timed call: about 100 us at 1965 MHz


def workload_desc(name: str, inp) -> str:
    c = CONFIGS[name]
    parts = [f"{name}: B={inp.B} N={inp.N} K={inp.K} V={inp.V} {inp.dtype}",
             f"prefix length U{{{c['prefix'][0]}..{c['prefix'][1]}}}", "gamma=4.0",
             "alphas 0.1/0.9/1.0", "fused fwd+bwd"]
    if inp.markov_w2 is not None:
        parts.append("Markov rank 256")
    if inp.conf_w is not None:
        parts.append("confidence head")
    if inp.lm_head is not None:
        parts.append("teacher from lm_head")
    return ", ".join(parts)


def seed_of(name: str, rank: int = 0) -> int:
    """The workload's seed: 1234 + its index, plus 1000 per data-parallel rank."""
    return 1234 + CONFIG_ORDER.index(name) + 1000 * rank


def cpu_inputs(name: str, rank: int = 0):
    """The workload drawn with the CPU generator (the same tensors for every arm)."""
    return make_inputs(name, device="cpu", seed=seed_of(name, rank))


def algorithmic_bytes(inp, n_sup: int) -> int:
    """The bytes a perfect single-pass implementation must move: the base draft and the
    teacher logits of every supervised row read once, dlogits written for every row;
    with the heads, the Markov tables read and their gradients written once, the
    hidden states read once and their gradient written once; with the teacher from
    hidden states, lm_head and the target hidden states read once instead of teacher
    logits.  Corrected rows, teacher chunks and re-reads of dlogits by the weight
    gradients are not counted: they are this implementation's overhead."""
    es = 2 if inp.dtype == "bf16" else 4
    b = n_sup * inp.V * es + inp.R * inp.V * es
    if inp.target_logits is not None:
        b += n_sup * inp.V * es
    if inp.lm_head is not None:
        b += inp.lm_head.numel() * 2 + n_sup * inp.lm_head.shape[1] * 2
    if inp.markov_w2 is not None:
        r = inp.markov_w2.shape[1]
        b += inp.V * r * (2 + 4) + n_sup * r * (2 + 4)
    if inp.conf_w is not None:
        b += inp.draft_hidden.numel() * 2 * 2
    return b


def dense_bytes(inp) -> int:
    """Every row's draft (and teacher) logits read and dlogits written, masked or not: the
    dense "logits read plus dlogits written" figure."""
    es = 2 if inp.dtype == "bf16" else 4
    return inp.R * inp.V * es * (3 if inp.target_logits is not None else 2)


def roofline_entry(alg: int, flops: int, ms: float, hbm, tensor, timed: str, traffic=None,
                   dense=None) -> dict:
    """The roofline object of a JSON line: the bound is whichever of the algorithmic bytes
    (at the measured HBM peak) and FLOPs (at the measured bf16 peak) takes longer; an HBM
    bound also reports the fraction of the nominal bandwidth and, given ``dense``, the
    dense figure's rate.  ``ms`` is the device time of one launch."""
    (peak, peak_kind), (tpeak, tpeak_kind) = hbm, tensor
    sec = ms / 1e3
    common = {"traffic": traffic, "algorithmic_bytes": alg, "algorithmic_flops": flops, "timed": timed}
    if alg / (peak * 1e9) >= flops / (tpeak * 1e12):
        achieved = alg / sec / 1e9
        r = {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
             "frac": round(achieved / peak, 4), "peak_kind": peak_kind, **common,
             "nominal_peak": NOMINAL_HBM_GBS, "frac_of_nominal": round(achieved / NOMINAL_HBM_GBS, 4)}
        if dense is not None:
            r["dense_bytes"] = dense
            r["dense_achieved"] = round(dense / sec / 1e9, 1)
        return r
    achieved = flops / sec / 1e12
    return {"bound": "tensor", "achieved": round(achieved, 1), "peak": tpeak, "unit": "TFLOP/s",
            "frac": round(achieved / tpeak, 4), "peak_kind": tpeak_kind, **common}


def tp_algorithmic_bytes(inp, n_sup: int, width: int) -> int:
    """One vocabulary-parallel rank's share of the single-pass bytes: its columns of the
    supervised rows' draft and teacher logits read once, its columns of every row's
    dlogits written once; with the heads, its rows of W2 read and of dW2 written, the
    supervised rows' embeddings and dW1 rows, and the hidden states read and their
    gradient written (the replicated heads' work is every rank's)."""
    es = 2 if inp.dtype == "bf16" else 4
    b = n_sup * width * es * (2 if inp.target_logits is not None else 1) + inp.R * width * es
    if inp.lm_head is not None:  # the teacher from hidden states: lm_head's shard rows, the hidden rows
        ht = inp.lm_head.shape[1]
        b += width * ht * 2 + n_sup * ht * 2
    if inp.markov_w2 is not None:
        r = inp.markov_w2.shape[1]
        b += width * r * (2 + 4) + n_sup * r * (2 + 4)
    if inp.conf_w is not None:
        b += inp.draft_hidden.numel() * 2 * 2
    return b


def tp_algorithmic_flops(inp, n_sup: int, width: int) -> int:
    """One rank's tensor-core work: the Markov bias, dE and dW2 contractions against its
    columns (2 * rows * width * rank each), and the teacher's against its lm_head rows."""
    f = 3 * 2 * n_sup * width * inp.markov_w2.shape[1] if inp.markov_w2 is not None else 0
    if inp.lm_head is not None:
        f += 2 * n_sup * width * inp.lm_head.shape[1]
    return f


def tp_launches_per_step(inp) -> int:
    """Kernels one rank's calls launch per micro-batch."""
    n = 4  # mask prologue, the three steps
    markov, conf = inp.markov_w2 is not None, inp.conf_w is not None
    if markov or conf:
        n += 1  # embeddings and confidence logits
    if markov:
        n += 1 + 3 + 1  # bias GEMM; dE GEMM, dW2 GEMM, split sum; the merge of the ranks' parts
    if conf:
        n += 3  # dproj partials, dproj final, dhidden
    if inp.lm_head is not None:
        n += 2  # hidden-state gather, the shard's teacher GEMM
    return n


def algorithmic_flops(inp, n_sup: int) -> int:
    """Tensor-core work a perfect implementation must do: the Markov bias, dE and dW2
    contractions (2 * rows * V * rank each) and the teacher product (2 * rows * V * Ht)."""
    f = 0
    if inp.markov_w2 is not None:
        f += 3 * 2 * n_sup * inp.V * inp.markov_w2.shape[1]
    if inp.lm_head is not None:
        f += 2 * n_sup * inp.V * inp.lm_head.shape[1]
    return f


def launches_per_call(inp) -> int:
    """Kernels one fused call launches (the launch sequence of dspark_loss_fwd)."""
    markov, conf_head, lm = inp.markov_w2 is not None, inp.conf_w is not None, inp.lm_head is not None
    n = 2 if lm else 3  # mask prologue, sweep (and, without lm_head, the zero-row fill behind it)
    if markov or conf_head:
        n += 1  # gather of embeddings and confidence logits
    if markov:
        n += 1 + 3  # bias GEMM; dE GEMM, dW2 GEMM, dE reduction and dW1 scatter
    if conf_head:
        n += 3  # dproj partials, dproj final, dhidden
    if lm:
        chunks = (inp.R + 511) // 512
        n += 1 + chunks + (chunks - 1)  # hidden gather, teacher GEMM per chunk, sweep per chunk
    return n


def sources_sha() -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic():
    """Per-launch DRAM bytes from the committed ncu summary, if it matches the sources."""
    try:
        with open(TRAFFIC_FILE) as f:
            text = f.read()
    except OSError:
        return None
    vals = {}
    for line in text.splitlines():
        if ":" in line and line.strip().startswith("- "):
            k, v = line.strip()[2:].split(":", 1)
            vals[k.strip()] = v.strip().strip("`")
    if vals.get("source_sha256_16") != sources_sha():
        return None
    try:
        return int(vals["dram_bytes_per_launch"])
    except (KeyError, ValueError):
        return None


def hbm_peak():
    try:
        with open(PEAKS) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def tensor_peak():
    """Dense bf16 TFLOP/s, burst figure (the GEMMs of one call are timed inside it)."""
    try:
        with open(PEAKS) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_BF16_TFLOPS, "fallback"


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while the timed loop runs."""

    def __init__(self, device_index: int, period_s: float = 0.005):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period = period_s
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:  # noqa: BLE001 - NVML missing: report no clocks
            self.nv = None
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        names = {}
        if self.nv is not None:
            for nm in ("HwSlowdown", "HwThermalSlowdown", "SwThermalSlowdown", "SwPowerCap",
                       "HwPowerBrakeSlowdown", "SyncBoost", "ApplicationsClocksSetting", "GpuIdle"):
                v = getattr(self.nv, "nvmlClocksEventReason" + nm, None)
                if v is None:
                    v = getattr(self.nv, "nvmlClocksThrottleReason" + nm, None)
                if v is not None:
                    names[nm] = v
        while True:
            if self.nv is not None:
                try:
                    self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                    r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                    for nm, bit in names.items():
                        if r & bit and nm != "GpuIdle":
                            self.reasons.add(nm)
                except Exception:  # noqa: BLE001
                    pass
            if self._stop.wait(self.period):
                break

    def __enter__(self):
        self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        self._t.join()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ------------------------------------------------------------ the oracle on host cores
# The oracle runs in worker processes forked BEFORE the first CUDA call (a process forked
# after CUDA is initialised can hang).  The workers inherit, copy-on-write, the workloads
# drawn on the CPU; each task is a set of whole blocks of one workload, run as a
# sub-batch of those blocks (rows and blocks are independent, so every row's work is the
# same as in the whole micro-batch).
_ORACLE_DATA = {}


def _bf16_rows_f32(t):
    """bf16 tensor -> float32 numpy, bit-exactly, with numpy alone (no torch threads in a
    forked worker)."""
    import numpy as np
    u = t.contiguous().view(torch.int16).numpy().view(np.uint16)
    return (u.astype(np.uint32) << 16).view(np.float32)


def oracle_view(inp) -> dict:
    """What a worker needs to run the oracle on blocks of ``inp``: the per-row tensors as
    they are (sliced per task) and the head weights converted once, in the parent."""
    import numpy as np

    def f64(t):
        if t is None:
            return None
        return (_bf16_rows_f32(t) if t.dtype == torch.bfloat16 else t.numpy()).astype(np.float64)
    return dict(inp=inp, w1=f64(inp.markov_w1), w2=f64(inp.markov_w2), conf_w=f64(inp.conf_w),
                conf_b=f64(inp.conf_b), lm_head=f64(inp.lm_head))


def _oracle_task(args):
    """Worker: the oracle on the blocks [b0, b1) (flattened b*N + n) of a workload; returns
    (supervised rows computed, seconds)."""
    import numpy as np
    from threadpoolctl import threadpool_limits
    from oracle import dspark_oracle as O
    name, b0, b1 = args
    d = _ORACLE_DATA[name]
    inp = d["inp"]
    K = inp.K
    nb = b1 - b0

    def rows(t):
        if t is None:
            return None
        x = t.reshape(inp.B * inp.N, K, -1)[b0:b1]
        x = _bf16_rows_f32(x) if x.dtype == torch.bfloat16 else x.contiguous().numpy()
        return x.reshape(1, nb, K, -1)

    def per_row(t):
        return None if t is None else t.reshape(inp.B * inp.N, K)[b0:b1].contiguous().numpy().reshape(1, nb, K)
    keep = None if inp.block_keep is None else inp.block_keep.reshape(-1)[b0:b1].numpy().reshape(1, nb)
    ev = per_row(inp.eval_mask)
    with threadpool_limits(limits=1):
        t0 = time.perf_counter()
        res = O.dspark_loss(rows(inp.draft_logits), per_row(inp.target_ids), ev,
                            target_logits=rows(inp.target_logits), block_keep=keep,
                            confidence_logits=None if inp.confidence_logits is None else
                            per_row(inp.confidence_logits).astype(np.float64),
                            prev_ids=per_row(inp.prev_ids), valid=per_row(inp.valid),
                            markov_w1=d["w1"], markov_w2=d["w2"], draft_hidden=rows(inp.draft_hidden),
                            conf_w=d["conf_w"], conf_b=d["conf_b"], conf_with_markov=inp.conf_with_markov,
                            target_hidden=rows(inp.target_hidden), lm_head=d["lm_head"],
                            target_norm_weight=None if inp.target_norm_weight is None else
                            _bf16_rows_f32(inp.target_norm_weight), target_norm_eps=inp.target_norm_eps,
                            gamma=inp.gamma)
        dt = time.perf_counter() - t0
    return int(res["num_tokens"]), dt


class OraclePool:
    """Worker processes for the oracle, forked before any CUDA call; ``views`` maps a
    workload name to oracle_view(inputs)."""

    def __init__(self, views: dict, procs: int = 0):
        import multiprocessing as mpc
        if torch.cuda.is_initialized():
            raise RuntimeError("the oracle pool must be forked before the first CUDA call")
        _ORACLE_DATA.clear()
        _ORACLE_DATA.update(views)
        self.procs = procs or len(os.sched_getaffinity(0))
        self.pool = mpc.get_context("fork").Pool(self.procs)

    def blocks(self, name):
        inp = _ORACLE_DATA[name]["inp"]
        return inp.B * inp.N

    def run(self, tasks):
        return self.pool.map(_oracle_task, tasks, chunksize=1)

    def close(self):
        self.pool.close()
        self.pool.join()


def _block_ranges(start: int, nblocks: int, per_task: int, ntasks: int):
    """ntasks consecutive ranges of per_task blocks from `start`, wrapping around."""
    out = []
    for i in range(ntasks):
        b0 = (start + i * per_task) % nblocks
        out.append((b0, min(nblocks, b0 + per_task)))
    return out


def cpu_baseline(pool: OraclePool, name: str, budget_s: float) -> dict:
    """The oracle on one core and on every core, each on a bounded sample of whole blocks
    of the workload (about budget_s seconds of work each), in supervised rows/s."""
    nblk = pool.blocks(name)
    pool.run([(name, 0, 1)] * pool.procs)  # every worker imports and touches the data once
    rows, dt = pool.run([(name, 0, 2)])[0]  # calibration: two blocks
    per_blk = max(dt / 2, 1e-3)
    one_n = int(max(1, min(nblk, budget_s / per_blk)))
    rows1, dt1 = pool.run([(name, 0, one_n)])[0]
    per_task = int(max(1, min(nblk, budget_s / per_blk)))
    t0 = time.perf_counter()
    res = pool.run([(name, a, b) for a, b in _block_ranges(0, nblk, per_task, pool.procs)])
    wall = time.perf_counter() - t0
    rows_all = sum(r for r, _ in res)
    return {
        "one_core": {"value": round(rows1 / dt1, 2), "unit": "rows/s", "cores": 1, "kind": "oracle",
                     "sample": f"{rows1} supervised rows ({one_n} whole blocks) of one {name} micro-batch, "
                               f"FP64 numpy, one thread", "seconds": round(dt1, 3)},
        "all_cores": {"value": round(rows_all / wall, 2), "unit": "rows/s", "cores": pool.procs,
                      "kind": "oracle",
                      "sample": f"{rows_all} supervised rows: {pool.procs} processes, each {per_task} whole "
                                f"blocks of one {name} micro-batch (wrapping around), FP64 numpy, one "
                                f"thread each, wall clock", "seconds": round(wall, 3)}}


# ------------------------------------------------------------------- GPU timing
def time_calls(call, steps: int, warmup: int, flush, clk_device: int):
    """Per-call device times (ms) of `steps` calls after `warmup`, the L2 flushed before
    each (untimed), and the clock record of the timed loop."""
    for _ in range(warmup):
        call.launch()
    torch.cuda.synchronize()
    status = call.check_status()
    if status != 0:
        raise SystemExit(f"device status {status} after warm-up")
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    torch.cuda.synchronize()
    with ClockSampler(clk_device) as clk:
        wall0 = time.perf_counter()
        for i in range(steps):
            flush.zero_()
            # a spin of about 100 us on the device after the flush: the host enqueues the
            # start event and the call meanwhile, so the device never waits for the host
            # between the two events (host launch latency is not device time)
            torch.cuda._sleep(HOST_SLACK_CYCLES)
            starts[i].record()
            call.launch()
            ends[i].record()
        torch.cuda.synchronize()
        wall = time.perf_counter() - wall0
    status = call.check_status()
    if status != 0:
        raise SystemExit(f"device status {status} after the timed calls")
    return [s.elapsed_time(e) for s, e in zip(starts, ends)], clk.summary(), wall


def timed_label(inp) -> str:
    n = launches_per_call(inp)
    return (f"dspark_loss_fwd with fused backward ({n} kernels: "
            + ("mask prologue, sweep, zero-row fill" if n == 3 else "prologue, heads, sweep, head gradients")
            + "), median CUDA-event duration per call")


def measure_workload(name: str, inp_cpu, torch_api, steps: int, warmup: int, flush, local: int) -> dict:
    """One workload timed on this GPU: median ms per call, rows/s and its roofline."""
    inp = inp_cpu.to("cuda")
    call = torch_api.Call(inp, grads=True, rows=False)
    per, clk, _ = time_calls(call, steps, warmup, flush, local)
    n_sup = int(call.out.num_tokens.item())
    med = statistics.median(per)
    rl = roofline_entry(algorithmic_bytes(inp, n_sup), algorithmic_flops(inp, n_sup), med, hbm_peak(),
                        tensor_peak(), timed_label(inp))
    del call, inp
    torch.cuda.empty_cache()
    return {"workload": workload_desc(name, inp_cpu), "supervised_rows": n_sup, "rows": inp_cpu.R,
            "steps": steps, "ms_per_call": round(med, 5), "ms_mean": round(statistics.mean(per), 5),
            "rows_per_s": round(n_sup / (med / 1e3), 1), "gpu_launches_per_call": launches_per_call(inp_cpu),
            "roofline": rl, "clocks": clk}


def run_e2e(inp_cpu, inp, steps: int, torch_api, dist) -> dict:
    """Per step: pinned host -> device copy of the micro-batch (logits, ids, masks, hidden
    states; the head weights stay resident like model parameters), the call, the report
    summed over the data-parallel ranks (one all-reduce), and a device -> host read of the
    loss, token count and report.  Median CUDA-event time per step."""
    dev_tensors = {k: v for k, v in inp.tensors().items() if k not in WEIGHTS}
    host = {k: inp_cpu.tensors()[k].pin_memory() for k in dev_tensors}
    call = torch_api.Call(inp, grads=True, rows=False)
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    out_host = torch.empty(torch_api.REPORT_VECTOR_LEN, dtype=torch.float64).pin_memory()
    d2h = out_host.numel() * out_host.element_size()
    s = torch.cuda.current_stream()
    times = []
    for i in range(steps + 3):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        for k, t in host.items():
            dev_tensors[k].copy_(t, non_blocking=True)
        call.launch()
        o = call.out
        if dist is not None:
            loss, ntok, rep = torch_api.reduce_report(o.loss_num, o.num_tokens, o.report)
        else:
            loss, ntok, rep = o.loss_num, o.num_tokens, o.report
        vec = torch.cat([loss.double().reshape(1), ntok.double().reshape(1), rep.double().reshape(-1)])
        out_host.copy_(vec, non_blocking=True)
        e1.record()
        s.synchronize()
        if i >= 3:
            times.append(e0.elapsed_time(e1))
    return {"ms": statistics.median(times), "h2d": h2d, "d2h": d2h, "tokens": float(out_host[1])}


# ------------------------------------------------------------------- entry points
def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def relaunch(args, argv) -> int:
    """Start args.gpus ranks of this script under torch.distributed.run (one process per
    GPU) and return the launcher's exit status; rank 0 prints the JSON line."""
    env = dict(os.environ)
    env.setdefault("NCCL_DEBUG", "INFO")  # the communicator log shows every rank joining
    env.setdefault("NCCL_DEBUG_SUBSYS", "INIT")
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={args.gpus}",
           "--master-addr", "127.0.0.1", "--master-port", str(_free_port()), os.path.abspath(__file__), *argv]
    p = subprocess.Popen(cmd, env=env, start_new_session=True)
    try:
        return p.wait(timeout=args.launch_timeout)
    except subprocess.TimeoutExpired:
        os.killpg(p.pid, 15)
        try:
            p.wait(timeout=60)
        except subprocess.TimeoutExpired:
            os.killpg(p.pid, 9)
        return 124


def main(argv=None):
    argv = sys.argv[1:] if argv is None else argv
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="recipe", choices=sorted(CONFIGS))
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-budget", type=float, default=5.0, help="seconds of oracle work per baseline sample")
    ap.add_argument("--extra-steps", type=int, default=20, help="timed calls of each extra workload")
    ap.add_argument("--no-extra", action="store_true", help="skip the extra workloads and CPU baselines")
    ap.add_argument("--tp", type=int, default=1, help="time one rank of a vocabulary-parallel group of this size")
    ap.add_argument("--profile-calls", type=int, default=0, help="run this many calls and exit with the status")
    ap.add_argument("--launch-timeout", type=float, default=1800.0, help="seconds before the ranks are stopped")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        raise SystemExit("--warmup must be at least 3")

    world = int(os.environ.get("WORLD_SIZE", "0"))
    if world == 0:  # no launcher around this process
        if args.gpus > 1 and args.impl == "native":
            return relaunch(args, argv)
        world = 1
    elif args.gpus != world:
        raise SystemExit(f"--gpus {args.gpus} but the launcher started {world} ranks")
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        return run_reference(args, world, rank)
    if args.profile_calls:
        return run_profile_calls(args)

    if world > 1:  # the ranks draw their inputs side by side
        torch.set_num_threads(max(1, len(os.sched_getaffinity(0)) // world))
    inp_cpu = cpu_inputs(args.workload, rank)
    extras, pool = {}, None
    if world == 1 and args.tp == 1 and not args.no_extra:
        for name in EXTRA_WORKLOADS:
            if name != args.workload:
                extras[name] = cpu_inputs(name)
        views = {}
        for name in CPU_BASELINE_WORKLOADS:
            src = inp_cpu if name == args.workload else extras.get(name)
            if src is None:
                src = extras[name] = cpu_inputs(name)
            views[name] = oracle_view(src)
        if args.workload not in views:
            views[args.workload] = oracle_view(inp_cpu)
        pool = OraclePool(views)  # forked before the first CUDA call

    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    from speculative_decoding_draft_vocab_b200 import torch_api

    inp = inp_cpu.to("cuda")
    if args.tp > 1:
        if world > 1:
            raise SystemExit("--tp times one rank on one GPU")
        return run_tp(args, inp, torch_api)
    call = torch_api.Call(inp, grads=True, rows=False)
    flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device="cuda")

    # ---- timed region: K calls, L2 flushed before each, device time per call
    if dist is not None:
        dist.barrier()
    per_step, clocks, wall = time_calls(call, args.steps, args.warmup, flush, local)
    if dist is not None:
        dist.barrier()
    n_sup = int(call.out.num_tokens.item())
    med = statistics.median(per_step)
    t_all = torch.tensor([med, float(n_sup)], dtype=torch.float64, device="cuda")
    if dist is not None:
        tmax = t_all[:1].clone()
        dist.all_reduce(tmax, op=dist.ReduceOp.MAX)
        rows = t_all[1:].clone()
        dist.all_reduce(rows, op=dist.ReduceOp.SUM)
        ms_step, rows_all = float(tmax.item()), float(rows.item())
    else:
        ms_step, rows_all = med, float(n_sup)
    value = rows_all / (ms_step / 1e3)

    # ---- roofline of the call: HBM bytes and tensor FLOPs a perfect implementation
    # needs; the bound is whichever takes longer at its measured peak
    plain = inp.markov_w2 is None and inp.conf_w is None and inp.lm_head is None
    traffic = recorded_traffic() if plain else None
    roofline = roofline_entry(algorithmic_bytes(inp, n_sup), algorithmic_flops(inp, n_sup), med, hbm_peak(),
                              tensor_peak(), timed_label(inp), traffic=traffic,
                              dense=dense_bytes(inp) if plain else None)
    roofline["traffic_source"] = ("recorded: the ncu DRAM bytes of the sweep kernel in "
                                  "profiles/sweep_recipe_traffic.md, taken on the same kernel sources (the "
                                  "zero-row fill beside it writes the unsupervised rows)" if traffic is not None
                                  else None)

    # ---- end to end from pinned host buffers, the report summed over the ranks
    e2e = run_e2e(inp_cpu, inp, args.e2e_steps, torch_api, dist)
    if dist is not None:
        ee = torch.tensor([e2e["ms"]], dtype=torch.float64, device="cuda")
        dist.all_reduce(ee, op=dist.ReduceOp.MAX)
        e2e["ms"] = float(ee.item())
    e2e_value = rows_all / (e2e["ms"] / 1e3)
    del call

    workloads = {}
    if rank == 0 and world == 1 and extras:
        for name in EXTRA_WORKLOADS:
            if name in extras:
                workloads[name] = measure_workload(name, extras[name], torch_api, args.extra_steps, 3, flush, local)
    del flush
    cpu, cpu_all = None, {}
    if pool is not None:
        for name in CPU_BASELINE_WORKLOADS + (() if args.workload in CPU_BASELINE_WORKLOADS else (args.workload,)):
            cpu_all[name] = cpu_baseline(pool, name, args.cpu_budget)
        pool.close()
        cpu = cpu_all[args.workload]["one_core"]

    if rank == 0:
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": "rows/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "bf16" if inp.dtype == "bf16" else "f32",
            "data": "synthetic (seeded on the CPU, copied to the device; shapes and distributions of the "
                    "Qwen3-8B DSpark recipe)",
            "config": {"workload": workload_desc(args.workload, inp), "supervised_rows_per_rank": n_sup,
                       "supervised_rows_all_ranks": int(rows_all), "rows_per_rank": inp.R,
                       "global_batch": inp.B * world, "parallelism": f"dp{world}",
                       "l2": "flushed before every timed call (512 MiB write, untimed)",
                       "timing": "median per-call CUDA-event time, maximum over ranks; a ~100 us device "
                                 "spin after each flush keeps host launch latency out of the events",
                       "ms_mean": round(statistics.mean(per_step), 5)},
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": {"value": round(e2e_value, 1), "unit": "rows/s", "h2d_bytes_per_step": e2e["h2d"],
                    "d2h_bytes_per_step": e2e["d2h"], "ms_per_step": round(e2e["ms"], 4),
                    "reduced_num_tokens": int(e2e["tokens"])},
            "gpu_launches": launches_per_call(inp) * args.steps,
            "clocks": clocks,
            "wall_s_timed_region": round(wall, 3),
        }
        if workloads:
            line["workloads"] = workloads
        if cpu_all:
            line["cpu_baselines"] = cpu_all
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_profile_calls(args) -> int:
    """args.profile_calls fused calls of the workload (the CPU draw, copied to the device);
    exits with the device status of the last call."""
    from speculative_decoding_draft_vocab_b200 import torch_api
    inp = cpu_inputs(args.workload).to("cuda")
    call = torch_api.Call(inp, rows=False)
    for _ in range(args.profile_calls):
        call.launch()
    torch.cuda.synchronize()
    status = call.check_status()
    print(args.workload, "status", status, "supervised rows", int(call.out.num_tokens.item()), flush=True)
    return status


def run_tp(args, inp, torch_api):
    """One rank (rank 0) of a vocabulary-parallel group of args.tp ranks: its calls per step
    on its shard (three, four with a head), L2 flushed before each step, CUDA events
    around them; the other ranks' records come from one emulated group run before."""
    ranks = torch_api.tp_group_emulated(inp, args.tp, rows=False)
    torch.cuda.synchronize()
    for r in ranks:
        if r.check_status() != 0:
            raise SystemExit("device status after the emulated group")
    rec1_all = torch.stack([r.rec1 for r in ranks])
    rec2_all = torch.stack([r.rec2 for r in ranks])
    de_all = torch.stack([r.de_part for r in ranks]) if ranks[0].de_part is not None else None
    r0 = ranks[0]
    del ranks[1:]
    n_sup = int(r0.num_tokens.item())
    flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device="cuda")

    def step():
        r0.partials()
        r0.l1(rec1_all)
        r0.finish(rec2_all)
        if r0.has_heads:
            r0.heads_bwd(de_all)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    with ClockSampler(0) as clk:
        for i in range(args.steps):
            flush.zero_()
            torch.cuda._sleep(HOST_SLACK_CYCLES)  # the host enqueues the step meanwhile
            starts[i].record()
            step()
            ends[i].record()
        torch.cuda.synchronize()
    if r0.check_status() != 0:
        raise SystemExit("device status after the timed steps")
    per_step = [s_.elapsed_time(e) for s_, e in zip(starts, ends)]
    med = statistics.median(per_step)
    width = r0.width
    alg = tp_algorithmic_bytes(inp, n_sup, width)
    flops = tp_algorithmic_flops(inp, n_sup, width)
    timed = ("one rank's dspark_tp_partials + dspark_tp_l1 + dspark_tp_finish"
             + (" + dspark_tp_heads_bwd" if r0.has_heads else "")
             + f" ({tp_launches_per_step(inp)} kernels), median CUDA-event time")
    roofline = roofline_entry(alg, flops, med, hbm_peak(), tensor_peak(), timed)
    line = {
        "metric": METRIC, "value": round(n_sup / (med / 1e3), 1), "unit": "rows/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(med, 5),
        "higher_is_better": True, "scaling": None, "vs_baseline": None,
        "dtype": "bf16" if inp.dtype == "bf16" else "f32", "data": "synthetic",
        "config": {"workload": workload_desc(args.workload, inp), "parallelism": f"tp{args.tp} (one rank timed)",
                   "shard_columns": width, "supervised_rows": n_sup,
                   "l2": "flushed before every timed step (512 MiB write, untimed)",
                   "not_timed": "the all-gathers of per-row records between the calls"},
        "roofline": roofline,
        "cpu_baseline": None, "e2e": None,
        "gpu_launches": tp_launches_per_step(inp) * args.steps,
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)
    return 0


def run_reference(args, world, rank):
    """The oracle arm: rank 0 times the FP64 CPU oracle on every host core (one process per
    core, each on whole blocks of the same workload draw), a bounded sample per step; the
    other ranks exit without work."""
    if rank != 0:
        return 0
    inp = cpu_inputs(args.workload)
    pool = OraclePool({args.workload: oracle_view(inp)})
    try:
        nblk = pool.blocks(args.workload)
        pool.run([(args.workload, 0, 1)] * pool.procs)  # every worker imports and touches the data once
        rows, dt = pool.run([(args.workload, 0, 1)])[0]
        budget = 120.0  # seconds for the whole run
        per_task = int(max(1, min(nblk, budget / (args.steps + args.warmup) / max(dt, 1e-3))))
        times, rows_done = [], []
        start = 0
        for i in range(args.warmup + args.steps):
            tasks = [(args.workload, a, b) for a, b in _block_ranges(start, nblk, per_task, pool.procs)]
            start = (start + per_task * pool.procs) % nblk
            t0 = time.perf_counter()
            res = pool.run(tasks)
            if i >= args.warmup:
                times.append(time.perf_counter() - t0)
                rows_done.append(sum(r for r, _ in res))
    finally:
        pool.close()
    rates = [r / t for r, t in zip(rows_done, times)]
    value = statistics.median(rates)
    sample = (f"{pool.procs} processes per step, each {per_task} whole block(s) of one {args.workload} "
              f"micro-batch (the same draw as the GPU arm), FP64 numpy oracle, one thread each; median "
              f"over steps of supervised rows / wall seconds")
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 2), "unit": "rows/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(statistics.median(times) * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_desc(args.workload, inp), "parallelism": "cpu"},
            "cpu_baseline": {"value": round(value, 2), "unit": "rows/s", "cores": pool.procs, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 2), "unit": "rows/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
