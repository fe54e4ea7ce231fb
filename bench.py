#!/usr/bin/env python
"""Throughput of the fused LM-head + cross-entropy forward+backward on B200.

One step = one call of lmh_loss_fwd with dH and dW requested on the large-vocabulary
workload (N = 8192 rows, d = 4096, V = 128256, Zipf(1.1) labels, 3 % ignored rows): the
logits GEMM with its online-LSE epilogue, the row finalize, the softmax-gradient rescale, and
the dH and dW GEMMs, over one chunk of all rows. TFLOP/s counts 6 N V d per step.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

With --gpus N > 1 (under torch.distributed.run, one process per GPU) every rank runs its
own replica on its own seeded batch (weak scaling, no collective on the data path); the
time is the maximum over ranks. --impl reference times the fp64 CPU oracle instead, on a
bounded sample of the same workload, on the host cores. Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "LM-head+CE fwd+bwd TFLOP/s (6·N·V·d) and % of bf16 tensor peak, 1×B200"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# the sources of the GEMM kernels whose DRAM traffic profiles/traffic.json records
KERNEL_SOURCES = ["lm_head_cross_tcgen05_b200/csrc/gemm.cuh",
                  "lm_head_cross_tcgen05_b200/csrc/epilogues.cuh",
                  "lm_head_cross_tcgen05_b200/csrc/sm100.cuh"]


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=40)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="large_vocab")
    ap.add_argument("--entry", choices=["fused_ce", "ce_separate", "support_kl",
                                        "support_kl_separate", "vocab_parallel",
                                        "data_parallel"],
                    default="fused_ce",
                    help="fused_ce: lmh_loss_fwd with dH/dW (the headline step); ce_separate: "
                         "lmh_loss_fwd then lmh_loss_bwd (recomputed logits); support_kl: "
                         "lmh_support_kl_fwd_bwd (the mean KL's forward and backward in one "
                         "pass); support_kl_separate: lmh_support_kl then lmh_loss_bwd; "
                         "vocab_parallel: one "
                         "CE problem with W split over the GPUs (strong scaling); "
                         "data_parallel: each GPU's own rows, the global mean and the dW sum "
                         "over the GPUs in rank order (weak scaling)")
    ap.add_argument("--chunk-rows", type=int, default=0,
                    help="rows per chunk (the memory budget); 0: the workload's own plan")
    ap.add_argument("--vocab", type=int, default=0,
                    help="override the workload's V (a smaller case for profiler captures; the "
                         "line's config then names the changed shape)")
    ap.add_argument("--rows", type=int, default=0, help="override the workload's N (as --vocab)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--ref-seconds", type=float, default=150.0,
                    help="--impl reference: total oracle time the timed and warm-up steps share")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    return ap.parse_args()


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as fh:
            d = json.load(fh)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def source_hash() -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


ENTRY_TEXT = {"fused_ce": "fused CE forward+backward",
              "ce_separate": "CE forward, then backward with recomputed logits",
              "support_kl": "support-set KL forward (K candidates) and its backward, fused",
              "support_kl_separate": "support-set KL forward (K candidates), then its backward "
                                     "with recomputed logits",
              "vocab_parallel": "vocabulary-parallel fused CE forward+backward (W split over "
                                "the GPUs)",
              "data_parallel": "row data-parallel fused CE forward+backward (global mean, dW "
                               "summed over the GPUs in rank order)"}


def workload_config(wl, chunk_rows, n_gpus, entry="fused_ce"):
    vp = entry == "vocab_parallel"
    return {"workload": f"{wl.name}: {ENTRY_TEXT[entry]}, N={wl.N} d={wl.d} V={wl.V}, "
                        f"{wl.labels} labels, {wl.num_ignored} ignored rows, bf16 H/W",
            "entry": entry,
            "N": wl.N, "d": wl.d, "V": wl.V, "chunk_rows": chunk_rows,
            "parallelism": (f"vocab-parallel over {n_gpus}" if vp else
                            f"data-parallel over {n_gpus}" if entry == "data_parallel" else
                            f"replicas x{n_gpus}"),
            "rows_per_gpu": wl.N, "total_rows": wl.N if vp else wl.N * n_gpus,
            "l2": "inputs larger than L2 (W alone is %.2f GB)" % (wl.V * wl.d * 2 / 1e9)}


# ----------------------------------------------------------------------------- ranks

def replica_seed(wl, rank: int) -> int:
    """Each rank's replica draws its own batch (weak scaling: rows per GPU are fixed)."""
    return wl.seed + 1000 * rank


def reduce_max(value: float, world: int, device=None) -> float:
    """Maximum of a per-rank value over all ranks (the job time is the slowest rank's)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(flops_per_rank_step: float, world: int, ms_per_step: float) -> float:
    """Whole-job throughput: the work of all ranks over the slowest rank's step time."""
    return flops_per_rank_step * world / (ms_per_step / 1e3) / 1e12


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """SM clock, power and clock-event reasons of one GPU during the timed region: NVML read
    every 10 ms on a thread (nvidia-smi's 100 ms floor gives too few samples for a region of
    about a second), else nvidia-smi -lms 100. Reads only; no setting is changed."""
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
             "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
             "clocks_event_reasons.sw_power_cap")
    NAMES = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    # NVML clock-event reason bits of the four names above
    NVML_BITS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
                 "sw_power_cap": 0x4}

    def __init__(self, gpu_id: str, period_s: float = 0.01):
        self.gpu_id = gpu_id
        self.period_s = period_s
        self.proc = None
        self.thread = None
        self.samples = []

    def _nvml_handle(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            if self.gpu_id.startswith("GPU-"):
                return pynvml, pynvml.nvmlDeviceGetHandleByUUID(self.gpu_id)
            return pynvml, pynvml.nvmlDeviceGetHandleByIndex(int(self.gpu_id))
        except Exception:
            return None, None

    def start(self):
        import threading
        nv, h = self._nvml_handle()
        if h is not None:
            reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or getattr(
                nv, "nvmlDeviceGetCurrentClocksThrottleReasons")
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            self.stop_flag = threading.Event()

            def loop():
                while not self.stop_flag.is_set():
                    try:
                        self.samples.append((float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)),
                                             nv.nvmlDeviceGetPowerUsage(h) / 1e3, int(reasons(h))))
                    except Exception:
                        pass
                    self.stop_flag.wait(self.period_s)
            self.thread = threading.Thread(target=loop, daemon=True)
            self.thread.start()
            return
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_id}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.thread is not None:
            self.stop_flag.set()
            self.thread.join(timeout=5)
            if not self.samples:
                return None
            sm = [c for c, _, _ in self.samples]
            bits = 0
            for _, _, b in self.samples:
                bits |= b
            reasons = sorted(n for n, b in self.NVML_BITS.items() if bits & b)
            return {"sm_mhz": statistics.median(sm), "sm_max_mhz": self.max_mhz,
                    "reasons": reasons, "samples": len(sm), "source": "nvml, every 10 ms",
                    "sm_mhz_p10_p90": [sorted(sm)[len(sm) // 10], sorted(sm)[(9 * len(sm)) // 10]],
                    "power_w_median": statistics.median(p for _, p, _ in self.samples)}
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], None, set()
        for line in out.strip().splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 8:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for name, val in zip(self.NAMES, f[4:8]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "source": "nvidia-smi, every 100 ms"}


# bf16 dense tensor throughput of one SM per clock (4096 multiply-adds)
BF16_FLOP_PER_SM_CLK = 8192


def tensor_peak_at(sm_mhz: float, sms: int) -> float:
    """TFLOP/s the tensor pipes can do at this SM clock: SMs x 8192 flop/clk x clock."""
    return sms * BF16_FLOP_PER_SM_CLK * sm_mhz * 1e6 / 1e12


def pick_peak(peaks: dict, timed_s: float) -> tuple:
    """The bf16 peak a kernel timed in this region is held to: the burst figure for a region
    of a few seconds at most (the power cap has not pulled the clock down to its sustained
    level), the sustained one for longer regions."""
    if timed_s <= 3.0:
        return peaks["bf16_tflops"], "burst"
    return peaks["bf16_tflops_sustained"], "sustained"


def gpu_id_for_smi(torch, dev) -> str:
    try:
        u = str(torch.cuda.get_device_properties(dev).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
        return vis.split(",")[dev] if vis else str(dev)


# ----------------------------------------------------------------------------- oracle timing

def oracle_runner(wl, entry):
    """The oracle's work for one step of `entry` on the first n rows of the workload (full V
    and d): run(n) does it, `what` names it. Both CE entries compute forward, dH and dW; the
    support entry computes the candidate log-probs, the KL and its backward."""
    from oracle import lmh_oracle as O
    from workloads import make_inputs
    x = make_inputs(wl.scaled(N=min(wl.N, 4096)), device="cpu")
    if entry.startswith("support_kl"):
        def run(n):
            O.support_kl(x["H"][:n], x["W"], x["ids"][:n], x["ref_logp"][:n])
            g = [1.0 / wl.N] * n
            O.backward(O.BWD_SUPPORT_KL, x["H"][:n], x["W"], x["ids"][:n], g,
                       x["ref_logp"][:n])
        return run, "fp64 numpy oracle support_kl + backward (dH, dW)"

    def run(n):
        O.ce_fused(x["H"][:n], x["W"], x["labels"][:n])
    return run, "fp64 numpy oracle ce_fused (forward, dH, dW)"


def _timed(fn, n):
    t = time.perf_counter()
    fn(n)
    return time.perf_counter() - t


def _rows_for(fn, target_s, n0, n1, cap=2048):
    """Rows that take about target_s seconds, from t(n) = a + b n at two calibration sizes
    (a is the per-call fp64 widening of W, b the per-row work)."""
    t0, t1 = _timed(fn, n0), _timed(fn, n1)
    b = max((t1 - t0) / float(n1 - n0), 1e-6)
    a = max(t0 - n0 * b, 0.0)
    return int(max(n0, min(cap, (target_s - a) / b)))


def _cores():
    import threadpoolctl
    return max([i.get("num_threads", 1) for i in threadpoolctl.threadpool_info()] + [1])


def oracle_sample(wl, target_s: float, entry="fused_ce"):
    """Times the fp64 oracle's step on the first n rows of the workload (full V and d), with
    n chosen so that the run takes about target_s seconds."""
    run, what = oracle_runner(wl, entry)
    n = _rows_for(run, target_s, 8, 40)
    return n, _timed(run, n), _cores(), what


def run_reference(args, wl, n_gpus):
    """The oracle as it stands, on the host cores, steps of a bounded sample."""
    run, what = oracle_runner(wl, args.entry)
    budget = args.ref_seconds / max(1, args.steps + args.warmup)       # seconds per step
    n = _rows_for(run, budget, 4, 20)
    for _ in range(args.warmup):
        run(n)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run(n)
    dt = (time.perf_counter() - t0) / max(1, args.steps)
    value = 6.0 * n * wl.V * wl.d / dt / 1e12
    sample = f"first {n} rows of {wl.name} (full V={wl.V}, d={wl.d}) per step, {what}"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
            "n_gpus": n_gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(wl, wl.chunk_rows or wl.N, 1, args.entry),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": _cores(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- main

def main():
    args = parse_args()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    from workloads import WORKLOADS, make_inputs
    wl = WORKLOADS[args.workload]
    if args.vocab or args.rows:
        wl = wl.scaled(V=args.vocab or wl.V, N=args.rows or wl.N,
                       name=f"{wl.name}[N={args.rows or wl.N},V={args.vocab or wl.V}]")

    if args.impl == "reference":
        if rank == 0:
            run_reference(args, wl, world)
        return

    import datetime

    import torch
    import torch.distributed as dist

    import lm_head_cross_tcgen05_b200 as L
    from lm_head_cross_tcgen05_b200._abi import lib

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    if world > 1:
        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=120))

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    def max_over_ranks(v: float) -> float:
        return reduce_max(v, world, dev)

    vp_entry = args.entry == "vocab_parallel"
    # replicas draw one batch per rank; the vocabulary-parallel ranks share one problem
    x = make_inputs(wl, device=dev, seed=wl.seed if vp_entry else replica_seed(wl, rank))
    H, W, y = x["H"], x["W"], x["labels"]
    N, d, V = wl.N, wl.d, wl.V
    chunk = args.chunk_rows or wl.chunk_rows or N
    f32, i32, bf = torch.float32, torch.int32, torch.bfloat16
    # several chunks: the fp32 dW accumulator is the caller's (the workspace holds one chunk's
    # softmax buffer, within the memory budget); the first chunk stores into it, so no step
    # needs a zeroing pass
    dW_acc = (torch.empty(V, d, dtype=f32, device=dev) if chunk < N else None)
    acc_flags = L.F_DW_ACC_GIVEN | L.F_DW_ACC_STORE if dW_acc is not None else 0
    shape = L.make_shape(N, d, V, 0, chunk, L.F_MEAN | L.F_FUSED_BWD | acc_flags)
    ws = L.workspace(shape, L.ENTRY_LOSS_FWD, dev)
    out = dict(loss_rows=torch.empty(N, dtype=f32, device=dev),
               lse=torch.empty(N, dtype=f32, device=dev),
               logprob=torch.empty(N, dtype=f32, device=dev),
               argmax=torch.empty(N, dtype=i32, device=dev),
               loss_mean=torch.empty(1, dtype=f32, device=dev),
               n_valid=torch.empty(1, dtype=i32, device=dev),
               dH=torch.empty(N, d, dtype=bf, device=dev),
               dW=torch.empty(V, d, dtype=bf, device=dev))
    stream = torch.cuda.current_stream()

    # the step's per-batch inputs (W is model state and stays resident)
    batch = {"H": H, "labels": y}
    if args.entry == "fused_ce":
        def step(b=batch):
            L.lmh_loss_fwd(shape, b["H"], W, b["labels"], out["loss_rows"], out["lse"], out["logprob"],
                           out["argmax"], out["loss_mean"], out["n_valid"], None, out["dH"],
                           out["dW"], dW_acc, workspace=ws, stream=stream)
    elif args.entry == "ce_separate":
        fshape = L.make_shape(N, d, V, 0, chunk, L.F_MEAN)
        fws = L.workspace(fshape, L.ENTRY_LOSS_FWD, dev)
        bshape = L.make_shape(N, d, V, 1, chunk, L.F_MEAN)
        bws = L.workspace(bshape, L.ENTRY_LOSS_BWD, dev)

        def step(b=batch):
            L.lmh_loss_fwd(fshape, b["H"], W, b["labels"], out["loss_rows"], out["lse"],
                           out["logprob"],
                           out["argmax"], out["loss_mean"], out["n_valid"], workspace=fws,
                           stream=stream)
            # backward of the mean loss: no grad given, 1 / n_valid taken on the device
            L.lmh_loss_bwd(bshape, L.BWD_CE, b["H"], W, b["labels"], out["lse"], None, None,
                           out["dH"], out["dW"], None, workspace=bws, stream=stream)
    elif vp_entry:
        from lm_head_cross_tcgen05_b200.vocab_parallel import VocabParallelCE
        chunk = N                                   # the fused step runs all rows as one chunk
        vp = VocabParallelCE(V, chunk_rows=chunk)      # the default group when world > 1
        W_shard = W[vp.v0:vp.v1].contiguous()

        def step(b=batch):
            f = vp.forward_backward(b["H"], W_shard, b["labels"])   # fused: 3 GEMMs per shard
            out["loss_mean"].copy_(f["loss_mean"])
            out["n_valid"].copy_(f["n_valid"])
    elif args.entry == "data_parallel":
        from lm_head_cross_tcgen05_b200.data_parallel import DataParallelCE
        dp = DataParallelCE(chunk_rows=chunk)          # the default group when world > 1

        def step(b=batch):
            # fused step on this rank's rows with the global count, then the rank-ordered
            # sums of the mean's shares and of the fp32 dW
            f = dp.forward_backward(b["H"], W, b["labels"])
            out["loss_mean"].copy_(f["loss_mean"])
            out["n_valid"].copy_(f["n_valid"])
    else:
        batch = {"H": H, "ids": x["ids"], "ref_logp": x["ref_logp"]}
        K = batch["ids"].shape[1]
        sshape = L.make_shape(N, d, V, K, chunk, L.F_MEAN)
        kl_rows = torch.empty(N, dtype=f32, device=dev)
        lp = torch.empty(N, K, dtype=f32, device=dev)
        if args.entry == "support_kl":
            fshape = L.make_shape(N, d, V, K, chunk, L.F_MEAN | L.F_FUSED_BWD)
            fws = L.workspace(fshape, L.ENTRY_SUPPORT_KL, dev)

            def step(b=batch):
                # forward and the mean KL's backward in one pass (3 GEMMs per chunk)
                L.lmh_support_kl_fwd_bwd(fshape, b["H"], W, b["ids"], b["ref_logp"], kl_rows,
                                         out["loss_mean"], lp, out["lse"], out["dH"],
                                         out["dW"], None, workspace=fws, stream=stream)
        else:
            sws = L.workspace(sshape, L.ENTRY_SUPPORT_KL, dev)
            bws = L.workspace(sshape, L.ENTRY_LOSS_BWD, dev)

            def step(b=batch):
                L.lmh_support_kl(sshape, b["H"], W, b["ids"], b["ref_logp"], kl_rows,
                                 out["loss_mean"], lp, out["lse"], workspace=sws, stream=stream)
                # backward of the mean KL: no grad given, 1 / N on the device
                L.lmh_loss_bwd(sshape, L.BWD_SUPPORT_KL, b["H"], W, b["ids"], out["lse"], None,
                               b["ref_logp"], out["dH"], out["dW"], None, workspace=bws,
                               stream=stream)

    for _ in range(max(3, args.warmup)):
        step()
    barrier()

    sampler = ClockSampler(gpu_id_for_smi(torch, local))
    sampler.start()
    if sampler.thread is None:
        time.sleep(0.3)          # nvidia-smi needs a moment before its first sample
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    lib().lmh_profile_enable(1)
    barrier()
    e0.record(stream)
    for _ in range(args.steps):
        step()
    e1.record(stream)
    barrier()
    lib().lmh_profile_enable(0)
    clocks = sampler.stop()
    ms_total = max_over_ranks(e0.elapsed_time(e1))
    ms_step = ms_total / args.steps
    flops_step = 6.0 * N * V * d
    jobs = 1 if vp_entry else world          # problems solved per step by the whole job
    value = job_tflops(flops_step, jobs, ms_step)

    # per-kernel device times of the timed region (event pairs on the launching stream)
    import ctypes
    cap = 64 * args.steps + 64
    kid_buf = (ctypes.c_int32 * cap)()
    ms_buf = (ctypes.c_float * cap)()
    n_rec = lib().lmh_profile_read(cap, kid_buf, ms_buf)
    per = {}
    for i in range(n_rec):
        name = lib().lmh_kernel_name(kid_buf[i]).decode()
        c, t = per.get(name, (0, 0.0))
        per[name] = (c + 1, t + ms_buf[i])
    kernels = {k: {"launches": c, "total_ms": t, "avg_ms": t / c,
                   "share": t / max(1e-9, sum(v[1] for v in per.values()))}
               for k, (c, t) in sorted(per.items(), key=lambda kv: -kv[1][1])}
    dom = next(iter(kernels)) if kernels else None
    peaks, peak_src = load_peaks()
    roofline = None
    if dom:
        V_gemm = (vp.v1 - vp.v0) if vp_entry else V     # the vocabulary one GEMM spans
        gemm_flops = 2.0 * chunk * V_gemm * d           # one GEMM launch over one chunk
        hbm_bytes = {"gbuild": 4.0 * chunk * ((V + 7) // 8 * 8)}
        if dom.startswith("gemm"):
            ach = gemm_flops / (kernels[dom]["avg_ms"] / 1e3) / 1e12
            pk, kind = pick_peak(peaks, ms_total / 1e3)
            roofline = {"bound": "tensor", "kernel": dom, "achieved": ach, "peak": pk,
                        "unit": "TFLOP/s", "frac": ach / pk,
                        "peak_kind": f"bf16 dense, {kind} (timed region {ms_total / 1e3:.2f} s), "
                                     f"of {peak_src}",
                        "frac_of_sustained": ach / peaks["bf16_tflops_sustained"],
                        "algorithmic_per_launch": gemm_flops}
            if clocks:
                at = tensor_peak_at(clocks["sm_mhz"], sms)
                roofline["at_sampled_clock"] = {
                    "sm_mhz": clocks["sm_mhz"], "sms": sms, "tensor_peak": at,
                    "frac": ach / at,
                    "how": "achieved / (SMs x 8192 bf16 flop/clk x median sampled SM clock)"}
        else:
            b = hbm_bytes.get(dom, 0.0)
            ach = b / (kernels[dom]["avg_ms"] / 1e3) / 1e9
            pk = peaks["hbm_gbs"]
            roofline = {"bound": "hbm", "kernel": dom, "achieved": ach, "peak": pk,
                        "unit": "GB/s", "frac": ach / pk, "peak_kind": f"copy, of {peak_src}",
                        "algorithmic_per_launch": b}
        roofline["traffic"] = None
        tpath = os.path.join(ROOT, "profiles", "traffic.json")
        if os.path.exists(tpath):
            with open(tpath) as fh:
                tr = json.load(fh)
            ent = tr.get(dom)
            if (ent and ent.get("source_hash") == source_hash()
                    and ent.get("workload") == wl.name and ent.get("entry") == args.entry
                    and chunk == (wl.chunk_rows or N)):
                roofline["traffic"] = ent["bytes_per_launch"]

    # end to end through the public API: pinned host batch in, loss out, every step
    e2e = None
    if not args.no_e2e:
        # every step uploads its batch (H and labels, or H, candidate ids and reference
        # log-probs) from pinned host memory and reads back its mean loss (and valid count);
        # the upload of step i+1 runs on a copy stream while step i computes (two device
        # buffers), as a training loop would overlap it
        host = {k: v.cpu().pin_memory() for k, v in batch.items()}
        dbuf = [{k: torch.empty_like(v) for k, v in batch.items()} for _ in range(2)]
        reads = [out["loss_mean"]] + ([out["n_valid"]] if not args.entry.startswith("support")
                                      else [])
        reads_h = [torch.empty_like(t, device="cpu").pin_memory() for t in reads]
        ready = [torch.cuda.Event() for _ in range(2)]
        free = [torch.cuda.Event() for _ in range(2)]
        copy_stream = torch.cuda.Stream(device=dev)

        def upload(i):
            b = i % 2
            with torch.cuda.stream(copy_stream):
                copy_stream.wait_event(free[b])
                for k, v in host.items():
                    dbuf[b][k].copy_(v, non_blocking=True)
                ready[b].record(copy_stream)

        def compute(i):
            b = i % 2
            stream.wait_event(ready[b])
            step(dbuf[b])
            free[b].record(stream)
            for th, td in zip(reads_h, reads):
                th.copy_(td, non_blocking=True)

        def run(n):
            copy_stream.wait_stream(stream)
            upload(0)
            for i in range(n):
                if i + 1 < n:
                    upload(i + 1)
                compute(i)

        run(2)
        barrier()
        e0.record(stream)
        run(args.steps)
        e1.record(stream)
        barrier()
        ms_e2e = max_over_ranks(e0.elapsed_time(e1)) / args.steps
        e2e = {"value": job_tflops(flops_step, jobs, ms_e2e), "unit": "TFLOP/s",
               "h2d_bytes_per_step": sum(v.numel() * v.element_size() for v in host.values()),
               "d2h_bytes_per_step": sum(t.numel() * t.element_size() for t in reads_h),
               "ms_per_step": ms_e2e,
               "note": f"every step copies its {', '.join(host)} in from pinned host memory (on "
                       "a copy stream, overlapped with the previous step) and reads its mean "
                       "back; W stays resident as model state"}

    cpu_baseline = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        n, t, cores, what = oracle_sample(wl, args.cpu_seconds, args.entry)
        cpu_baseline = {"value": 6.0 * n * V * d / t / 1e12, "unit": "TFLOP/s", "cores": cores,
                        "kind": "oracle",
                        "sample": f"first {n} rows of {wl.name} (full V={V}, d={d}): {what}, "
                                  f"{t:.1f} s"}

    if rank == 0:
        cfg = workload_config(wl, chunk, world, args.entry)
        if args.entry == "fused_ce":
            cfg["workspace_bytes"] = int(ws.numel())
            cfg["dW_accumulator"] = ("caller-owned fp32 [V, d], stored by the first chunk"
                                     if dW_acc is not None else "none (one chunk: bf16 dW)")
        if not vp_entry:  # the first chunk's dH tiling, which decides dH's summation order
            wide, splits = L.lmh_dh_plan(min(chunk, wl.N), d, V)
            cfg["dH_tiles"] = (f"{'256x512' if wide else '256x256'} CTA-pair tiles, "
                               f"{splits} vocabulary range{'s' if splits > 1 else ''}")
        line = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
                "higher_is_better": True, "scaling": "strong" if vp_entry else "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
                "config": cfg,
                "peak_frac": {"of_burst": value / world / peaks["bf16_tflops"],
                              "of_sustained": value / world / peaks["bf16_tflops_sustained"],
                              "of_sampled_clock": (value / world / tensor_peak_at(
                                  clocks["sm_mhz"], sms) if clocks else None),
                              "peaks": peak_src},
                "roofline": roofline, "cpu_baseline": cpu_baseline, "e2e": e2e,
                "gpu_launches": n_rec, "kernels": kernels, "clocks": clocks}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
