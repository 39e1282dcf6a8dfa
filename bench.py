"""Benchmark of the single-GPU MoE-layer forward (tokens/s, device-timed).

python bench.py --gpus N --steps K --warmup W [--workload NAME] [--impl reference]

One step = one whole forward of the layer (router, dispatch scan, dispatch
scatter, persistent expert GEMM, finalize) over one batch of T synthetic
tokens whose inputs are already resident in HBM. Between timed steps the L2
cache is flushed by writing a 256 MB buffer (outside the per-step events).
With N > 1 (torchrun, one process per GPU) every rank runs an independent
replica on its own T tokens (the same weights, tokens drawn from a seed offset
by the rank; weak scaling, no collective in the data path); the step time is
the max over ranks.

The JSON line also carries:
* roofline: the expert-GEMM kernel's achieved TFLOP/s (6*T*k*H*I algorithmic
  FLOP per launch / its mean CUDA-event duration on the launching stream)
  against the measured dense bf16 peak, and the whole layer's fraction of
  max(FLOP / TC peak, bytes / HBM peak);
* e2e: the same metric through the host-buffer entry point (x copied in from
  pinned memory, y copied back, every step);
* cpu_baseline: the fp64 CPU oracle timed on a bounded sample on rank 0;
* clocks: SM clock samples and throttle reasons taken during the timed steps.

The tensor peak is the measured burst bf16 figure, or the sustained one when
the power cap shows among the clocks sampled during the timed steps
(choose_tc_peak); the line reports the fraction against both.

--fp8 runs the same layer with FP8 E4M3 expert GEMMs (weights quantized once before timing);
its roofline peak is twice the chosen bf16 figure (the nominal dense fp8/bf16 ratio) and its
byte count takes 1-byte weights plus their fp32 column scales.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

BASELINE_METRIC = "MoE-layer fwd tokens/s on 1 B200 (device-timed); % of max(TC, HBM) roofline"
# the largest single-GPU workload is the headline; the others run under --workload
DEFAULT_WORKLOAD = "fine_grained_prefill"
FLUSH_BYTES = 256 << 20
# tokens of the fp64 oracle per reference-arm step (about a second each on 16 host cores, so that a
# --steps 100 run ends in minutes) and for the cpu_baseline of the native arm (about 10 s of work)
ORACLE_SAMPLE = {"tiny": 64, "mixtral": 128, "fine_grained_prefill": 4, "decode": 4, "skewed": 512}
CPU_BASELINE_SAMPLE = {"tiny": 64, "mixtral": 1024, "fine_grained_prefill": 32, "decode": 32, "skewed": 4096}


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm_gbs=d["hbm_gbs"], bf16_tflops=d["bf16_tflops"],
                    bf16_tflops_sustained=d.get("bf16_tflops_sustained", d["bf16_tflops"]), source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


def choose_tc_peak(peaks: dict, clocks: dict):
    """The dense bf16 peak that applies to a run, from the clocks sampled during its timed steps.

    The burst figure (cuBLAS timed alone, at full clock) applies when no sample of the timed
    region shows the power cap; the sustained one (cuBLAS in a seconds-long loop, settled
    under the power cap) applies when at least one does. Unsampled clocks count as capped
    only if the run is long enough to reach the cap, which nothing here can tell, so they
    take the burst figure (the stricter one). Returns (peak TFLOP/s, name of the figure).
    """
    reasons = clocks.get("reasons") or []
    if "sw_power_cap" in reasons:
        return peaks["bf16_tflops_sustained"], "bf16_tflops_sustained"
    return peaks["bf16_tflops"], "bf16_tflops"


GEMM_SOURCES = ("common.cuh", "ptx.cuh", "expert_gemm.cuh", "expert_gemm2.cuh")   # what the expert GEMMs are built from


def code_text(src: str) -> str:
    """C++ source without comments and blank lines (what the compiler sees, for the hash below)."""
    import re
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    return "\n".join(line.rstrip() for line in src.splitlines() if line.strip())


def kernel_source_hash(read=None) -> str:
    """sha256 (16 hex) of the expert-GEMM sources' code, comments excluded."""
    import hashlib
    if read is None:
        read = lambda f: open(os.path.join(ROOT, "moe_megakernel_b200", "csrc", f)).read()
    h = hashlib.sha256()
    for f in GEMM_SOURCES:
        h.update(code_text(read(f)).encode())
    return h.hexdigest()[:16]


def measured_traffic(workload: str, table=None, source_hash=None):
    """ncu DRAM bytes per expert-GEMM launch, if captured on the current kernel sources.

    `workload` is the table's key (the workload name, + "+fp8" / "+shared<S>" for those forwards);
    a row counts only if its source hash is the current one (the counters of a changed kernel are
    not reported)."""
    p = table if table is not None else os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(p):
        return None
    cur = source_hash if source_hash is not None else kernel_source_hash()
    for line in open(p):
        f = line.split()
        if len(f) >= 3 and not f[0].startswith("#") and f[0] == workload and f[1] == cur:
            return int(f[2])
    return None


def reduce_max_over_ranks(value: float, dist, device) -> float:
    """Max of a per-rank number over all ranks (identity on one process)."""
    if dist is None:
        return value
    import torch
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(tokens_per_rank: int, world: int, max_ms: float) -> float:
    """Whole-job throughput: every rank's tokens over the slowest rank's step time."""
    return tokens_per_rank * world / (max_ms * 1e-3)


def workload_label(s, n_shared=0, fp8=False):
    return (f"{s.name}: T={s.T} H={s.H} I={s.I} E={s.E} k={s.k}" + (" zipf-bias" if s.zipf_bias else "")
            + (f" +{n_shared} shared" if n_shared else "") + (" fp8-e4m3 expert GEMMs" if fp8 else ""))


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """SM clock, power and throttle reasons polled through NVML every 2 ms in a
    thread (read-only queries); stats cover the samples taken between
    begin() and end(), i.e. during the timed steps. Falls back to one
    nvidia-smi query per sample if NVML cannot be loaded."""

    REASON_BITS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40, "sw_thermal_slowdown": 0x20,
                   "sw_power_cap": 0x4}

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.samples = []          # (t, sm_mhz, power_w, reasons_mask)
        self.t0 = self.t1 = None
        self.max_mhz = None
        self._stop = threading.Event()
        self._thread = None
        self._nvml = None

    def _poll_nvml(self, nv, h):
        while not self._stop.is_set():
            try:
                self.samples.append((time.perf_counter(), nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM),
                                     nv.nvmlDeviceGetPowerUsage(h) / 1000.0,
                                     nv.nvmlDeviceGetCurrentClocksEventReasons(h)))
            except Exception:
                return
            time.sleep(0.002)

    def _poll_smi(self):
        q = "clocks.sm,power.draw,clocks_event_reasons.active"
        while not self._stop.is_set():
            try:
                out = subprocess.run(["nvidia-smi", "-i", str(self.idx), f"--query-gpu={q}",
                                      "--format=csv,noheader,nounits"], capture_output=True, text=True,
                                     timeout=5).stdout.strip().split(",")
                self.samples.append((time.perf_counter(), float(out[0]), float(out[1]), int(out[2].strip(), 16)))
            except Exception:
                return

    def start(self):
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = nv.nvmlDeviceGetHandleByIndex(self.idx)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            self._nvml = nv
            self._thread = threading.Thread(target=self._poll_nvml, args=(nv, h), daemon=True)
        except Exception:
            self._thread = threading.Thread(target=self._poll_smi, daemon=True)
        self._thread.start()

    def begin(self):
        self.t0 = time.perf_counter()

    def end(self):
        self.t1 = time.perf_counter()

    def stop(self):
        self._stop.set()
        if self._thread is not None:
            self._thread.join(timeout=10)
        rows = [r for r in self.samples if self.t0 is not None and self.t1 is not None and self.t0 <= r[0] <= self.t1]
        if not rows and self.samples and self.t1 is not None:
            rows = [min(self.samples, key=lambda r: abs(r[0] - self.t1))]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unsampled"], "samples": 0}
        reasons = sorted({n for r in rows for n, b in self.REASON_BITS.items() if r[3] & b})
        return {"sm_mhz": statistics.median(r[1] for r in rows), "sm_min_mhz": min(r[1] for r in rows),
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(rows),
                "power_w_max": max(r[2] for r in rows),
                "source": "nvml" if self._nvml is not None else "nvidia-smi"}


# ------------------------------------------------------------------ oracle timing
def time_oracle(inp, n_tokens: int, fp8: bool = False):
    """The fp64 CPU oracle as it stands, on the first n_tokens tokens (host copies of the inputs)."""
    import numpy as np
    import torch

    import oracle.moe_oracle as O
    x = inp["x"][:n_tokens].double().cpu().numpy()
    Wg = inp["Wg"].double().cpu().numpy()
    bias = None if inp["bias"] is None else inp["bias"].double().cpu().numpy()
    W1c, W3c, W2c = inp["W1"].cpu(), inp["W3"].cpu(), inp["W2"].cpu()
    S = inp.get("n_shared", 0)
    Wsc = [inp[n].cpu() for n in ("Ws1", "Ws3", "Ws2")] if S else None

    def load(e):
        return (W1c[e].double().numpy(), W3c[e].double().numpy(), W2c[e].double().numpy())

    def load_shared(s):
        return tuple(w[s].double().numpy() for w in Wsc)

    t0 = time.perf_counter()
    O.moe_forward(x, Wg, bias, load, inp["k"], shared_weights=load_shared if S else None, n_shared=S, fp8=fp8)
    dt = time.perf_counter() - t0
    cores = None
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        cores = max([i.get("num_threads", 0) for i in info] + [torch.get_num_threads()])
    except Exception:
        cores = torch.get_num_threads()
    del np
    return n_tokens / dt, dt, cores


# ------------------------------------------------------------------ main GPU arm
def run_gpu(args, rank, world, local_rank):
    import torch

    from moe_megakernel_b200 import MoEPlan, quantize_weights_fp8
    from synth.moe_inputs import WORKLOADS, make_inputs

    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    shape = WORKLOADS[args.workload]
    S = args.shared
    # replicated weights, each rank its own tokens (rank 0 draws the single-GPU tokens)
    inp = make_inputs(shape, device=dev, seed=args.seed, n_shared=S, x_seed=args.seed + rank)
    T, H, I, E, k = shape.T, shape.H, shape.I, shape.E, shape.k
    plan = MoEPlan(T, H, I, E, k, device=dev, n_shared=S, fp8=args.fp8, task_log=args.task_log)
    shared_kw = dict(Ws1=inp["Ws1"], Ws3=inp["Ws3"], Ws2=inp["Ws2"]) if S else {}
    if args.cta_pairs is not None:
        plan.set_cta_pairs(bool(args.cta_pairs))
    if args.task_order is not None:
        plan.set_task_order(args.task_order)
    if args.half_tails is not None:
        plan.set_half_tails(bool(args.half_tails))
    if args.wide_l1 is not None:
        plan.set_wide_l1(bool(args.wide_l1))
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    y = torch.empty((T, H), dtype=torch.bfloat16, device=dev)
    args_fwd = (inp["x"], inp["Wg"], inp["bias"], inp["W1"], inp["W3"], inp["W2"])
    if args.fp8:
        # weights are quantized once, like loading a checkpoint (outside every timed region)
        W1q, s1 = quantize_weights_fp8(inp["W1"])
        W3q, s3 = quantize_weights_fp8(inp["W3"])
        W2q, s2 = quantize_weights_fp8(inp["W2"])
        fp8_w = (W1q, s1, W3q, s3, W2q, s2)

    def fwd():
        if args.fp8:
            plan.forward_fp8(inp["x"], inp["Wg"], inp["bias"], *fp8_w, y=y)
        else:
            plan.forward(*args_fwd, y=y, **shared_kw)

    # host-buffer steps: the pipelined entry (copies on the plan's own streams overlap the
    # neighbouring steps' kernels); the plain one for shared experts
    pipelined = S == 0

    def fwd_host(x_host, y_host):
        if pipelined and args.fp8:
            plan.forward_host_pipelined_fp8(x_host, inp["Wg"], inp["bias"], *fp8_w, y_host)
        elif pipelined:
            plan.forward_host_pipelined(x_host, inp["Wg"], inp["bias"], inp["W1"], inp["W3"], inp["W2"], y_host)
        else:
            plan.forward_host(x_host, inp["Wg"], inp["bias"], inp["W1"], inp["W3"], inp["W2"], y_host, **shared_kw)

    def barrier():
        if dist is not None:
            dist.barrier(device_ids=[local_rank])

    for _ in range(args.warmup):
        fwd()
    plan.check()

    # timed device steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    clocks = ClockSampler(local_rank)
    plan.set_profiling(True)
    barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    clocks.begin()
    for i in range(args.steps):
        flush.zero_()
        ev[i][0].record(stream)
        fwd()
        ev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    clocks.end()
    barrier()
    clk = clocks.stop()
    plan.check()
    kernel_ms, nprof = plan.profile_read()
    plan.set_profiling(False)
    step_ms = [a.elapsed_time(b) for a, b in ev]
    mean_ms = reduce_max_over_ranks(sum(step_ms) / len(step_ms), dist, dev)

    # end to end through the host-buffer entry point
    x_host = inp["x"].cpu().pin_memory()
    y_hosts = [torch.empty((T, H), dtype=torch.bfloat16).pin_memory() for _ in range(2)]
    for i in range(max(1, args.warmup)):
        fwd_host(x_host, y_hosts[i % 2])
    if pipelined:
        plan.host_pipeline_join(stream)
    plan.check()
    e2e_steps = max(3, args.steps)
    barrier()
    torch.cuda.synchronize(dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    if pipelined:
        plan.host_pipeline_after(stream)   # the first copy-in starts after e0
    for i in range(e2e_steps):
        fwd_host(x_host, y_hosts[i % 2])
    if pipelined:
        plan.host_pipeline_join(stream)    # e1 after the last copy-out
    e1.record(stream)
    torch.cuda.synchronize(dev)
    plan.check()
    e2e_ms = reduce_max_over_ranks(e0.elapsed_time(e1) / e2e_steps, dist, dev)

    # task log of the last forward: how busy each SM's MMA issue was over the expert GEMM
    tlog = None
    if args.task_log:
        lg = plan.task_log()
        span = float(lg["t_done"].max() - lg["t_first_mma"].min())
        busy = torch.zeros(int(lg["cta"].max()) + 1, dtype=torch.float64)
        busy.scatter_add_(0, lg["cta"], (lg["t_last_mma"] - lg["t_first_mma"]).double())
        issuing = busy[busy > 0] / span
        tlog = {"tasks": int(lg["task"].numel()), "ctas_issuing_mma": int(issuing.numel()), "span_us": span / 1e3,
                "mma_issue_occupancy": {"mean": float(issuing.mean()), "min": float(issuing.min()),
                                        "max": float(issuing.max())},
                "note": "per MMA-issuing CTA (the leader of a pair): sum over its tasks of first-to-last MMA "
                        "issue time, over the launch's span (first MMA to last epilogue)"}

    # routing statistics for the roofline's byte count
    r = plan.routing(T)
    counts = r["expert_count"].cpu()
    active = int((counts > 0).sum())
    num_padded = int(r["num_padded"].item())

    cpu = None
    if rank == 0 and not args.no_cpu_baseline:
        n = min(T, CPU_BASELINE_SAMPLE.get(args.workload, 64))
        v, dt, cores = time_oracle(inp, n, fp8=args.fp8)
        cpu = {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
               "sample": f"fp64 oracle (gate, dispatch, expert FFN, combine{', FP8 expert GEMMs' if args.fp8 else ''}) "
                         f"on the first {n} of {T} tokens of the same inputs, {dt:.1f} s wall"}

    if rank == 0:
        peaks = measured_peaks()
        flop = 6.0 * T * (k + S) * H * I                     # routed pairs and shared-expert rows
        alg_bytes = 2.0 * 3 * H * I * (active + S) + 2.0 * H * E + 2.0 * T * H * 2
        if args.fp8:   # W1/W3/W2 as 1-byte codes plus fp32 column scales
            alg_bytes += (-3.0 * H * I + 4.0 * (2 * I + H)) * active
        gemm_ms = kernel_ms["expert_gemm"] / max(nprof, 1)
        achieved_tflops = flop / (gemm_ms * 1e-3) / 1e12
        # burst peak unless the sampled clocks show the power cap during the timed steps
        tc_peak, tc_peak_name = choose_tc_peak(peaks, clk)
        fp8_ratio = 2.0 if args.fp8 else 1.0
        if args.fp8:
            # both expert GEMMs at the FP8 rate, taken as 2x the measured bf16 rate
            # (the nominal dense ratio, 4.5 vs 2.25 PFLOP/s)
            tc_peak = 2.0 * tc_peak
        t_tc = flop / (tc_peak * 1e12)
        t_hbm = alg_bytes / (peaks["hbm_gbs"] * 1e9)
        bound = "tensor" if t_tc >= t_hbm else "hbm"
        if bound == "tensor":
            roof = {"bound": "tensor", "achieved": achieved_tflops, "peak": tc_peak, "unit": "TFLOP/s",
                    "frac": achieved_tflops / tc_peak}
        else:
            gbs = alg_bytes / (gemm_ms * 1e-3) / 1e9
            roof = {"bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": gbs / peaks["hbm_gbs"]}
        roof.update({"kernel": "moe_expert_gemm2_kernel" if plan.cta_pairs else "moe_expert_gemm_kernel",
                     "traffic": measured_traffic(args.workload + ("+fp8" if args.fp8 else "")
                                                 + (f"+shared{S}" if S else "")),
                     "traffic_unit": "bytes per launch (ncu dram read+write)",
                     "peak_source": f"{peaks['source']} ({tc_peak_name if bound == 'tensor' else 'hbm_gbs'})"
                                    + (" x 2: FP8 at the nominal fp8/bf16 ratio" if args.fp8 and bound == "tensor"
                                       else "")
                                    + ("; burst unless sw_power_cap was sampled in the timed steps"
                                       if bound == "tensor" else ""),
                     "kernel_ms": gemm_ms,
                     # the same kernel time in SM cycles at the median sampled clock, and the fraction
                     # against both measured tensor peaks, so that the clock dependence is visible
                     "kernel_mcycles": gemm_ms * 1e-3 * clk["sm_mhz"] * 1e6 / 1e6 if clk.get("sm_mhz") else None,
                     "frac_vs_burst": achieved_tflops / (fp8_ratio * peaks["bf16_tflops"]),
                     "frac_vs_sustained": achieved_tflops / (fp8_ratio * peaks["bf16_tflops_sustained"]),
                     "flop_per_launch": flop,
                     "layer_t_roof_ms": max(t_tc, t_hbm) * 1e3,
                     "layer_frac": max(t_tc, t_hbm) * 1e3 / mean_ms,
                     "kernel_ms_per_step": {kk: v / max(nprof, 1) for kk, v in kernel_ms.items()}})
        line = {
            "metric": BASELINE_METRIC,
            "value": job_tokens_per_s(T, world, mean_ms),
            "unit": "tokens/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": mean_ms,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "e4m3 (expert GEMMs) + bf16" if args.fp8 else "bf16",
            "data": "synthetic (seeded N(0,1) x, N(0,1/H) Wg/W1/W3, N(0,1/I) W2, bf16; random-init weights)",
            "config": {"workload": workload_label(shape, S, args.fp8), "T_per_gpu": T, "H": H, "I": I, "E": E, "k": k,
                       "block_m": plan.block_m, "cta_pairs": plan.cta_pairs, "task_order": plan.task_order,
                       "half_tails": plan.half_tails, "wide_l1": plan.wide_l1, "active_experts": active,
                       "padded_slots": num_padded,
                       "l2": "flushed between steps (256 MB write, outside per-step events)",
                       "parallelism": "replicas" if world > 1 else "single"},
            "roofline": roof,
            "cpu_baseline": cpu,
            "e2e": {"value": job_tokens_per_s(T, world, e2e_ms), "unit": "tokens/s",
                    "h2d_bytes_per_step": T * H * 2, "d2h_bytes_per_step": T * H * 2,
                    "ms_per_step": e2e_ms,
                    "api": (f"moe_forward_host_pipelined{'_fp8' if args.fp8 else ''} (pinned host x and y; the "
                            "copies of each step overlap the neighbouring steps' kernels)") if pipelined
                    else "moe_forward_host_shared (pinned host x and y)"},
            # FP8: + the x quantizer and, per block group, a first-GEMM launch, the activation
            # quantizer and a second-GEMM launch (the library counts them)
            "gpu_launches": args.steps * plan.forward_launches(args.fp8),
            "clocks": clk,
        }
        if tlog is not None:
            line["task_log"] = tlog
        print(json.dumps(line), flush=True)
    if dist is not None:
        dist.barrier(device_ids=[local_rank])
        dist.destroy_process_group()


# ------------------------------------------------------------------ backward (--backward)
BACKWARD_METRIC = "MoE-layer bwd tokens/s on 1 B200 (device-timed); % of TC roofline"


def run_backward(args):
    """Device-timed moe_backward steps (routing, dgrad, gate, weight gradients) on one GPU.

    FLOP per step: 16*T*k*H*I (dgrad: g, u and dy W2^T 6, dx 4; weight gradients 6) plus the
    gate's 2*T*H*E for dWg; roofline against the dense bf16 peak chosen from the sampled clocks.
    """
    import torch

    from moe_megakernel_b200 import MoEPlan
    from synth.moe_inputs import WORKLOADS, make_dy, make_inputs
    torch.cuda.set_device(0)
    dev = torch.device("cuda", 0)
    shape = WORKLOADS[args.workload]
    inp = make_inputs(shape, device=dev, seed=args.seed)
    dy = make_dy(shape, device=dev, seed=args.seed)
    T, H, I, E, k = shape.T, shape.H, shape.I, shape.E, shape.k
    plan = MoEPlan(T, H, I, E, k, device=dev, backward=True)
    out = plan.backward(inp["x"], inp["Wg"], inp["bias"], inp["W1"], inp["W3"], inp["W2"], dy)
    for _ in range(args.warmup):
        plan.backward(inp["x"], inp["Wg"], inp["bias"], inp["W1"], inp["W3"], inp["W2"], dy, out=out)
    plan.check()
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    clocks = ClockSampler(0)
    torch.cuda.synchronize(dev)
    clocks.start()
    clocks.begin()
    for i in range(args.steps):
        flush.zero_()
        ev[i][0].record(stream)
        plan.backward(inp["x"], inp["Wg"], inp["bias"], inp["W1"], inp["W3"], inp["W2"], dy, out=out)
        ev[i][1].record(stream)
    torch.cuda.synchronize(dev)
    clocks.end()
    clk = clocks.stop()
    plan.check()
    ms = sum(a.elapsed_time(b) for a, b in ev) / args.steps
    flop = 16.0 * T * k * H * I + 2.0 * T * H * E
    peaks = measured_peaks()
    peak, peak_name = choose_tc_peak(peaks, clk)
    achieved = flop / (ms * 1e-3) / 1e12
    print(json.dumps({
        "metric": BACKWARD_METRIC, "value": T / (ms * 1e-3), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic (seeded x, weights and dy ~ N(0,1) dy; random-init weights)",
        "config": {"workload": workload_label(shape) + " backward", "T": T, "H": H, "I": I, "E": E, "k": k,
                   "block_m": plan.block_m, "l2": "flushed between steps (256 MB write, outside per-step events)"},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "peak_source": f"{peaks['source']} ({peak_name})", "flop_per_step": flop,
                     "frac_vs_burst": achieved / peaks["bf16_tflops"],
                     "frac_vs_sustained": achieved / peaks["bf16_tflops_sustained"]},
        # router, scan, scatter, dgrad-1, dgrad-2, Wg transpose, gate, dW1/dW3, dW2, dWg, and with
        # BLOCK_M >= 64 the permutation of x and dy rows into slot order
        "gpu_launches": args.steps * (10 + (1 if plan.block_m >= 64 else 0)),
        "clocks": clk,
    }), flush=True)


# ------------------------------------------------------------------ reference arm (the oracle)
def run_reference(args, rank, world):
    if rank != 0:
        return
    import torch

    from synth.moe_inputs import WORKLOADS, make_inputs
    shape = WORKLOADS[args.workload]
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    inp = make_inputs(shape, device=dev, seed=args.seed, n_shared=args.shared)
    n = min(shape.T, ORACLE_SAMPLE.get(args.workload, 64))
    for _ in range(args.warmup):
        time_oracle(inp, max(1, n // 8), fp8=args.fp8)
    times, cores = [], None
    for _ in range(args.steps):
        v, dt, cores = time_oracle(inp, n, fp8=args.fp8)
        times.append(dt)
    value = n * len(times) / sum(times)
    sample = f"fp64 CPU oracle on the first {n} of {shape.T} tokens per step"
    print(json.dumps({
        "impl": "reference", "metric": BASELINE_METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sum(times) / len(times) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": workload_label(shape, args.shared, args.fp8)},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD,
                    help="named workload, or 'custom' with --shape")
    ap.add_argument("--shape", default=None,
                    help="T,H,I,E,k[,zipf] for --workload custom (e.g. a scaled-down case for profiling)")
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--shared", type=int, default=0,
                    help="shared experts (weight 1, every token) on top of the workload's routed experts")
    ap.add_argument("--fp8", action="store_true",
                    help="FP8 E4M3 expert GEMMs with power-of-two per-token / per-column scales")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cta-pairs", type=int, default=None, choices=[0, 1],
                    help="expert GEMM on CTA pairs (1) or one CTA per block (0); default: the plan's")
    ap.add_argument("--task-order", type=int, default=None, choices=[-1, 0, 1],
                    help="expert-GEMM task order: -1 automatic, 0 staggered, 1 interleaved; default: the plan's")
    ap.add_argument("--half-tails", type=int, default=None, choices=[0, 1],
                    help="an expert's lone last block as M = 128 pair MMAs (1) or a full pair (0); default: the plan's")
    ap.add_argument("--wide-l1", type=int, default=None, choices=[0, 1],
                    help="256-column (1) or 128-column (0) first-GEMM tasks on CTA pairs; default: the plan's")
    ap.add_argument("--task-log", action="store_true",
                    help="record the expert GEMM's task log and report each SM's MMA-issue occupancy")
    ap.add_argument("--backward", action="store_true",
                    help="time moe_backward (routing, dgrad, gate, weight gradients) instead of the forward")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.fp8 and args.shared:
        ap.error("--fp8 runs without shared experts")
    if args.workload == "custom":
        if not args.shape:
            ap.error("--workload custom needs --shape T,H,I,E,k[,zipf]")
        from synth.moe_inputs import WORKLOADS, custom_shape
        f = args.shape.split(",")
        WORKLOADS["custom"] = custom_shape(*[int(v) for v in f[:5]], zipf=len(f) > 5 and f[5] == "zipf",
                                           name="custom")
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if world != args.gpus:
        world = max(world, 1)
    if args.impl == "reference":
        run_reference(args, rank, world)
    elif args.backward:
        if world > 1:
            ap.error("--backward runs on one GPU")
        run_backward(args)
    else:
        run_gpu(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
