"""Benchmark of the fused DSpark loss forward+backward (one step = one call of
dspark_loss_fwd with the fused backward over one synthetic micro-batch).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload recipe] [--impl reference]

For N > 1 run it under torch.distributed.run; every rank draws its own micro-batch
(seed offset by rank) and processes it alone (rows are independent: weak scaling, no
collective on the data path); the step time is the maximum over ranks.

Prints one JSON line.  `value` is supervised rows per second over all ranks, timed on
the device with CUDA events around each call; the L2 cache is flushed (a 512 MiB
write) before every timed call and the flush is not timed.  `e2e` is the same metric
through the same call with the inputs in pinned host memory: every step copies the
micro-batch to the device, runs the call and reads the loss and report back.
`--impl reference` times the FP64 CPU oracle instead, on a bounded sample of rows.
`--tp T` (one GPU) times instead one rank of a T-way vocabulary-parallel group: the three
calls dspark_tp_partials, dspark_tp_l1 and dspark_tp_finish on that rank's 1/T shard of
the micro-batch, the other ranks' records computed beforehand (the two all-gathers
between the calls are not timed).
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from speculative_decoding_draft_vocab_b200.synthetic import CONFIGS, make_inputs  # noqa: E402

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


WEIGHTS = ("markov_w1", "markov_w2", "conf_w", "conf_b", "lm_head", "target_norm_weight")  # resident


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


def roofline_entry(alg: int, flops: int, mean_ms: float, hbm, tensor, timed: str, traffic=None,
                   dense=None) -> dict:
    """The roofline object of a JSON line: the bound is whichever of the algorithmic bytes
    (at the measured HBM peak) and FLOPs (at the measured bf16 peak) takes longer; an HBM
    bound also reports the fraction of the nominal bandwidth and, given ``dense``, the
    dense figure's rate."""
    (peak, peak_kind), (tpeak, tpeak_kind) = hbm, tensor
    sec = mean_ms / 1e3
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
    if inp.markov_w2 is not None:
        r = inp.markov_w2.shape[1]
        b += width * r * (2 + 4) + n_sup * r * (2 + 4)
    if inp.conf_w is not None:
        b += inp.draft_hidden.numel() * 2 * 2
    return b


def tp_algorithmic_flops(inp, n_sup: int, width: int) -> int:
    """One rank's tensor-core work: the Markov bias, dE and dW2 contractions against its
    columns (2 * rows * width * rank each)."""
    return 3 * 2 * n_sup * width * inp.markov_w2.shape[1] if inp.markov_w2 is not None else 0


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
    n = 2  # mask prologue, sweep
    markov, conf_head, lm = inp.markov_w2 is not None, inp.conf_w is not None, inp.lm_head is not None
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


def oracle_kwargs(inp):
    """The oracle's keyword arguments for a CPU copy of the inputs."""
    def a(t):
        return None if t is None else t.float().numpy()
    return dict(target_logits=a(inp.target_logits), block_keep=a(inp.block_keep),
                confidence_logits=a(inp.confidence_logits), prev_ids=a(inp.prev_ids), valid=a(inp.valid),
                markov_w1=a(inp.markov_w1), markov_w2=a(inp.markov_w2), draft_hidden=a(inp.draft_hidden),
                conf_w=a(inp.conf_w), conf_b=a(inp.conf_b), conf_with_markov=inp.conf_with_markov,
                target_hidden=a(inp.target_hidden), lm_head=a(inp.lm_head),
                target_norm_weight=a(inp.target_norm_weight), target_norm_eps=inp.target_norm_eps,
                gamma=inp.gamma)


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

    def __init__(self, device_index: int, period_s: float = 0.02):
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
        while not self._stop.is_set():
            if self.nv is not None:
                try:
                    self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                    r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                    for nm, bit in names.items():
                        if r & bit and nm != "GpuIdle":
                            self.reasons.add(nm)
                except Exception:  # noqa: BLE001
                    pass
            time.sleep(self.period)

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


def run_cpu_baseline(name: str, budget_s: float, seed: int = None):
    """Time the FP64 oracle on a bounded sample of supervised rows of the workload, with
    numpy's BLAS held to one thread (so `cores` is exactly 1)."""
    from threadpoolctl import threadpool_limits
    with threadpool_limits(limits=1):
        return _cpu_baseline(name, budget_s, seed)


def _cpu_baseline(name: str, budget_s: float, seed: int = None):
    import numpy as np
    from oracle import dspark_oracle as O
    inp = make_inputs(name, device="cpu", seed=seed)
    m = O.prefix_supervision_mask(inp.eval_mask.numpy(), inp.block_keep.numpy()).reshape(-1)
    sup = np.nonzero(m)[0]
    draft = inp.draft_logits.float().numpy()
    kw = oracle_kwargs(inp)
    # calibrate on 2 rows, then take as many rows as the budget allows
    t0 = time.perf_counter()
    O.dspark_loss(draft, inp.target_ids.numpy(), inp.eval_mask.numpy(), rows=sup[:2], **kw)
    per_row = (time.perf_counter() - t0) / 2
    n = int(max(2, min(len(sup), budget_s / max(per_row, 1e-6))))
    t0 = time.perf_counter()
    O.dspark_loss(draft, inp.target_ids.numpy(), inp.eval_mask.numpy(), rows=sup[:n], **kw)
    dt = time.perf_counter() - t0
    return {"value": n / dt, "unit": "rows/s", "cores": 1, "kind": "oracle",
            "sample": f"{n} of the {len(sup)} supervised rows of one {name} micro-batch, "
                      f"FP64 numpy, one thread (elementwise numpy ops)", "seconds": dt}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="recipe", choices=sorted(CONFIGS))
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-budget", type=float, default=12.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--tp", type=int, default=1, help="time one rank of a vocabulary-parallel group of this size")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be at least 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        return run_reference(args, world, rank)

    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    from speculative_decoding_draft_vocab_b200 import torch_api

    seed = 1234 + ["tiny", "recipe", "recipe_heads", "lm_head_teacher", "large"].index(args.workload) + 1000 * rank
    inp = make_inputs(args.workload, device="cuda", seed=seed)
    if args.tp > 1:
        if world > 1:
            raise SystemExit("--tp times one rank on one GPU")
        return run_tp(args, inp, torch_api)
    call = torch_api.Call(inp, grads=True, rows=False)
    flush = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device="cuda")
    for _ in range(args.warmup):
        call.launch()
    torch.cuda.synchronize()
    status = call.check_status()
    if status != 0:
        raise SystemExit(f"device status {status} after warm-up")
    n_sup = int(call.out.num_tokens.item())

    # ---- timed region: K calls, L2 flushed before each, device time per call
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        wall0 = time.perf_counter()
        for i in range(args.steps):
            flush.zero_()
            starts[i].record()
            call.launch()
            ends[i].record()
        torch.cuda.synchronize()
        wall = time.perf_counter() - wall0
    if dist is not None:
        dist.barrier()
    per_step = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = sum(per_step)
    t_all = torch.tensor([total_ms, float(n_sup)], dtype=torch.float64, device="cuda")
    if dist is not None:
        tmax = t_all[:1].clone()
        dist.all_reduce(tmax, op=dist.ReduceOp.MAX)
        rows = t_all[1:].clone()
        dist.all_reduce(rows, op=dist.ReduceOp.SUM)
        total_ms, rows_all = float(tmax.item()), float(rows.item())
    else:
        rows_all = float(n_sup)
    ms_per_step = total_ms / args.steps
    value = rows_all * args.steps / (total_ms / 1e3)

    # ---- roofline of the call: HBM bytes and tensor FLOPs a perfect implementation
    # needs; the bound is whichever takes longer at its measured peak
    alg = algorithmic_bytes(inp, n_sup)
    flops = algorithmic_flops(inp, n_sup)
    mean_ms = statistics.mean(per_step)
    n_launch = launches_per_call(inp)
    timed = (f"dspark_loss_fwd with fused backward ({n_launch} kernels: "
             + ("mask prologue + sweep" if n_launch == 2 else "prologue, heads, sweep, head gradients")
             + "), mean CUDA-event duration per call")
    roofline = roofline_entry(alg, flops, mean_ms, hbm_peak(), tensor_peak(), timed,
                              traffic=recorded_traffic() if n_launch == 2 else None,
                              dense=dense_bytes(inp) if n_launch == 2 else None)

    # ---- end to end from pinned host buffers
    e2e = run_e2e(inp, args.e2e_steps, torch_api)
    if dist is not None:
        ee = torch.tensor([e2e["ms"]], dtype=torch.float64, device="cuda")
        dist.all_reduce(ee, op=dist.ReduceOp.MAX)
        e2e["ms"] = float(ee.item())
    e2e_value = rows_all / (e2e["ms"] / 1e3)

    if rank == 0:
        cpu = run_cpu_baseline(args.workload, args.cpu_budget) if world == 1 else None
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": "rows/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16" if inp.dtype == "bf16" else "f32",
            "data": "synthetic (seeded; shapes and distributions of the Qwen3-8B DSpark recipe)",
            "config": {"workload": workload_desc(args.workload, inp), "supervised_rows_per_rank": n_sup,
                       "rows_per_rank": inp.R, "global_batch": inp.B * world, "parallelism": f"dp{world}",
                       "l2": "flushed before every timed call (512 MiB write, untimed)"},
            "roofline": roofline,
            "cpu_baseline": cpu,
            "e2e": {"value": round(e2e_value, 1), "unit": "rows/s", "h2d_bytes_per_step": e2e["h2d"],
                    "d2h_bytes_per_step": e2e["d2h"], "ms_per_step": round(e2e["ms"], 4)},
            "gpu_launches": n_launch * args.steps,
            "clocks": clk.summary(),
            "wall_s_timed_region": round(wall, 3),
        }
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


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
            starts[i].record()
            step()
            ends[i].record()
        torch.cuda.synchronize()
    if r0.check_status() != 0:
        raise SystemExit("device status after the timed steps")
    per_step = [s_.elapsed_time(e) for s_, e in zip(starts, ends)]
    mean_ms = statistics.mean(per_step)
    width = r0.width
    alg = tp_algorithmic_bytes(inp, n_sup, width)
    flops = tp_algorithmic_flops(inp, n_sup, width)
    timed = ("one rank's dspark_tp_partials + dspark_tp_l1 + dspark_tp_finish"
             + (" + dspark_tp_heads_bwd" if r0.has_heads else "")
             + f" ({tp_launches_per_step(inp)} kernels), mean CUDA-event time")
    roofline = roofline_entry(alg, flops, mean_ms, hbm_peak(), tensor_peak(), timed)
    line = {
        "metric": METRIC, "value": round(n_sup / (mean_ms / 1e3), 1), "unit": "rows/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(mean_ms, 5),
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


def run_e2e(inp, steps: int, torch_api):
    """Per step: pinned host -> device copy of the micro-batch (logits, ids, masks, hidden
    states; the head weights stay resident like model parameters), the call, and a
    device -> host read of the loss, token count and report."""
    dev_tensors = {k: v for k, v in inp.tensors().items() if k not in WEIGHTS}
    host = {k: v.cpu().pin_memory() for k, v in dev_tensors.items()}
    call = torch_api.Call(inp, grads=True, rows=False)
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    out_host = torch.empty(1 + 2 * 6 + 2, dtype=torch.float32).pin_memory()
    d2h = (1 + 2 * 6) * 4 + 8
    s = torch.cuda.current_stream()
    times = []
    for i in range(steps + 3):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        for k, t in host.items():
            dev_tensors[k].copy_(t, non_blocking=True)
        call.launch()
        out_host[:1].copy_(call.out.loss_num, non_blocking=True)
        out_host[1:13].copy_(call.out.report.view(-1), non_blocking=True)
        out_host[13:15].copy_(call.out.num_tokens.view(torch.float32), non_blocking=True)
        e1.record()
        s.synchronize()
        if i >= 3:
            times.append(e0.elapsed_time(e1))
    return {"ms": statistics.mean(times), "h2d": h2d, "d2h": d2h}


def run_reference(args, world, rank):
    """The oracle arm: rank 0 times the FP64 CPU oracle on a bounded sample per step
    (numpy's BLAS held to one thread)."""
    if rank != 0:
        return
    from threadpoolctl import threadpool_limits
    with threadpool_limits(limits=1):
        _run_reference(args, world)


def _run_reference(args, world):
    import numpy as np
    from oracle import dspark_oracle as O
    inp = make_inputs(args.workload, device="cpu")
    m = O.prefix_supervision_mask(inp.eval_mask.numpy(), inp.block_keep.numpy()).reshape(-1)
    sup = np.nonzero(m)[0]
    draft = inp.draft_logits.float().numpy()
    kw = oracle_kwargs(inp)
    t0 = time.perf_counter()
    O.dspark_loss(draft, inp.target_ids.numpy(), inp.eval_mask.numpy(), rows=sup[:1], **kw)
    per_row = time.perf_counter() - t0
    budget = 120.0  # seconds for the whole run
    rows_per_step = int(max(1, min(len(sup), budget / (args.steps + args.warmup) / max(per_row, 1e-6))))
    times = []
    for i in range(args.warmup + args.steps):
        sel = sup[(i * rows_per_step) % len(sup):][:rows_per_step]
        if len(sel) < rows_per_step:
            sel = np.concatenate([sel, sup[:rows_per_step - len(sel)]])
        t0 = time.perf_counter()
        O.dspark_loss(draft, inp.target_ids.numpy(), inp.eval_mask.numpy(), rows=sel, **kw)
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    total = sum(times)
    value = rows_per_step * args.steps / total
    sample = (f"{rows_per_step} supervised row(s) per step of one {args.workload} micro-batch, "
              f"FP64 numpy oracle, one thread")
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 2), "unit": "rows/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(total / args.steps * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": workload_desc(args.workload, inp), "parallelism": "cpu"},
            "cpu_baseline": {"value": round(value, 2), "unit": "rows/s", "cores": 1, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(value, 2), "unit": "rows/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
