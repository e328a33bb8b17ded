#!/usr/bin/env python
"""Benchmark of the MoE routing hot path on B200 (one JSON line on rank 0).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--M M]
    python bench.py --impl reference ...        # the CPU oracle on host cores

A *step* is one pass of the whole routing path (load logits, score, bias,
group scores, group mask, top-k, gather, renormalise, scale, store) over one
batch of M synthetic tokens, i.e. one call of the library's C entry point.
The default workload is the sigmoid + correction_bias top-k with one group
(E=256, k=8, renormalise, bf16 logits N(0, 2^2), fp32 bias N(0, 0.05^2),
M=16384 tokens) - the aiter biased_grouped_topk(num_expert_group=1,
topk_group=1) call of the SGLang routing pages.

Timing: inputs are resident in HBM before the timed region; every step reads a
different buffer of a rotating pool larger than L2, so reads come from DRAM.
The K steps are replayed from CUDA graphs (exactly K launches of the routing
kernel) and timed with CUDA events on the launching stream, bracketed by a
barrier and a device synchronise; the job time is the max over ranks.  A
short GPU sleep is queued before the start event so that the host's graph
launch is not inside the timed region.  Under torchrun each rank routes its
own batches (no data-path collective: rows are independent), so scaling is
weak.

On one GPU the line also carries ``per_config``: every workload size the
routing spec names, timed cold (rotating pool) and hot (one buffer), with a
parity sample against the oracle taken in the CPU-baseline leg.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "routed tokens/s & µs/call (E=256,k=8 biased grouped top-k); % of HBM roofline"
# The other workloads report the same quantities under their own description.
WORKLOAD_METRICS = {
    "grouped": "routed tokens/s & µs/call (E=160,k=6 softmax grouped top-k); % of HBM roofline",
    "softmax": "routed tokens/s & µs/call (E=8,k=2 softmax top-k); % of HBM roofline",
    "fused": ("routed tokens/s & µs/call (router GEMM K=7168,E=256 + biased grouped top-k); "
              "% of the dense bf16 tensor roofline"),
    "top1": "routed tokens/s & µs/call (E=8 router projection + softcap + top-1); % of HBM roofline",
}


def metric_for(name: str) -> str:
    return WORKLOAD_METRICS.get(name, METRIC)


L2_BYTES = 126 * 1024 * 1024
ROUTING = ("sigmoid", "biased", "grouped", "softmax")
# Every size the routing spec quotes (the workload, M): the per-config table.
PER_CONFIG = [("softmax", 64), ("sigmoid", 1), ("sigmoid", 16), ("sigmoid", 64), ("sigmoid", 256),
              ("sigmoid", 4096), ("sigmoid", 16384), ("biased", 4096), ("biased", 32), ("grouped", 16384),
              ("fused", 8192), ("fused", 64), ("top1", 8192), ("top1", 64)]
# GPU sleep queued before the start event: about 100 us at the B200's clocks,
# longer than the host needs to submit the first graph of the timed region.
SLEEP_CYCLES = 200_000


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=48000)
    ap.add_argument("--warmup", type=int, default=480)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="sigmoid",
                    choices=["sigmoid", "biased", "grouped", "softmax", "fused", "top1", "permute"])
    ap.add_argument("--M", type=int, default=None, help="tokens per step (default: workload's)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true")
    ap.add_argument("--per-config-steps", type=int, default=1000)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-soak", action="store_true", help="skip the 1 s clock-sampling soak")
    return ap.parse_args(argv)


DEFAULT_M = {"sigmoid": 16384, "biased": 4096, "grouped": 16384, "softmax": 64, "fused": 8192, "top1": 8192,
             "permute": 16384}
PERM_K, PERM_E = 8, 256  # the permutation step after the sigmoid workload's routing


def workload_desc(name: str, M: int) -> dict:
    from moe_expert_routing_token_b200 import inputs
    sp = inputs.SPECS[name]
    d = {"M": M, "E": sp.E, "topk": sp.topk, "renormalize": sp.renormalize,
         "num_expert_group": sp.num_expert_group, "topk_group": sp.topk_group,
         "routed_scaling_factor": sp.routed_scaling_factor,
         "logits_dtype": str(sp.dtype).replace("torch.", "")}
    if name == "sigmoid":
        d["workload"] = (f"sigmoid+correction_bias top-k, one group (biased grouped top-k "
                         f"G=1 TG=1), E=256, k=8, M={M}, bf16 logits N(0,2^2), fp32 bias")
    elif name == "biased":
        d["workload"] = (f"biased grouped top-k DeepSeek-V3 shape, E=256 G=8 TG=4 k=8 "
                         f"RSF=2.5, M={M}, bf16 logits")
    elif name == "grouped":
        d["workload"] = f"softmax grouped top-k DeepSeek-V2 shape, E=160 G=8 TG=3 k=6, M={M}, fp32"
    elif name == "softmax":
        d["workload"] = f"softmax top-k E=8 k=2 renormalise, M={M}, fp32 logits"
    elif name == "top1":
        d["workload"] = (f"fused top-1 router (tcgen05 projection): (M,{sp.K}) bf16 x ({sp.E},{sp.K}) bf16 "
                         f"weight, softcap {sp.softcap:g}, top-1 with weight 1/sum exp, M={M}")
        d["K"] = sp.K
        d["softcap"] = sp.softcap
    else:
        d["workload"] = (f"fused router (M,{sp.K})x({sp.K},{sp.E}) bf16 + biased grouped top-k "
                         f"G=8 TG=4 k=8, M={M}")
        d["K"] = sp.K
    return d


def algorithmic_bytes(name: str, M: int) -> int:
    """Bytes a launch must move at minimum: logits in, (weights, ids) out, bias."""
    from moe_expert_routing_token_b200 import inputs
    sp = inputs.SPECS[name]
    esz = 2 if str(sp.dtype).endswith("bfloat16") else 4
    out = M * sp.topk * 8
    bias = sp.E * 4 if sp.bias_std is not None else 0
    if name in ("fused", "top1"):
        return M * sp.K * 2 + sp.K * sp.E * 2 + out + bias
    return M * sp.E * esz + out + bias


def measured_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def kernel_source_hash(files=None) -> str:
    """sha256 prefix of the kernel sources (all csrc/*.cu{,h}, or the listed
    files, in sorted order)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "moe_expert_routing_token_b200", "csrc")
    names = sorted(files) if files else sorted(os.listdir(csrc))
    for f in names:
        if f.endswith((".cu", ".cuh")):
            h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def profiled_traffic(name: str, M: int):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel sources (else None).  The summary names the source files
    its kernel is built from (``kernel_sources:``) and their hash."""
    path = os.path.join(ROOT, "profiles", f"traffic_{name}_M{M}.txt")
    if not os.path.exists(path):
        return None
    text = open(path).read()
    src = re.search(r"kernel_source_sha:\s*(\w+)", text)
    val = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
    files = re.search(r"kernel_sources:\s*(.+)", text)
    files = files.group(1).split() if files else None
    if not src or not val or src.group(1) != kernel_source_hash(files):
        return None
    return float(val.group(1))


def host_cpu() -> dict:
    """The host the CPU baseline runs on: core count and model name."""
    model = None
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                model = line.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    return {"nproc": os.cpu_count(), "cpu_model": model}


# ---------------------------------------------------------------------------
# clocks
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.proc = None
        self.gpu_index = gpu_index
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={gpu_index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (FileNotFoundError, OSError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sms, maxs, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sms.append(float(parts[1]))
                maxs.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sms:
            return None
        return {"sm_mhz": statistics.median(sms), "sm_max_mhz": max(maxs),
                "reasons": sorted(reasons), "samples": len(sms)}


# ---------------------------------------------------------------------------
# CPU oracle timing (reference arm and cpu_baseline)
# ---------------------------------------------------------------------------
def oracle_call(name: str, d: dict, rows):
    """The oracle on the rows ``rows`` (a slice or an index array) of workload
    input ``d``."""
    import oracle
    sp = d["spec"]
    if name == "top1":
        return oracle.fused_router_top1(d["hidden"][rows], d["weight"], sp.softcap, weight_layout=1)
    if name == "fused":
        return oracle.fused_router_topk(d["hidden"][rows], d["weight"], d["bias"], sp.topk,
                                        sp.renormalize, sp.num_expert_group, sp.topk_group,
                                        sp.routed_scaling_factor)
    x = d["logits"][rows]
    if name in ("softmax", "grouped"):
        return oracle.grouped_topk(x, sp.topk, sp.renormalize, sp.num_expert_group,
                                   sp.topk_group, sp.routed_scaling_factor)
    return oracle.biased_grouped_topk(x, d["bias"], sp.topk, sp.renormalize, sp.num_expert_group,
                                      sp.topk_group, sp.routed_scaling_factor)


def time_oracle(name: str, M: int, seconds: float) -> dict:
    """Oracle throughput on a bounded sample: whole batches (or a row slice for
    the fused workload) repeated until `seconds` of single-thread CPU work."""
    from moe_expert_routing_token_b200 import inputs
    d = inputs.make(name, M)
    rows = M if name not in ("fused", "top1") else min(M, 4 if name == "fused" else 256)
    oracle_call(name, d, slice(0, min(rows, 8)))  # compile / warm
    n = 0
    t0 = time.perf_counter()
    while True:
        oracle_call(name, d, slice(0, rows))
        n += rows
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    return dict({"value": n / el, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                 "sample": f"{n} tokens ({n // rows} x {rows}-token batches of the {name} workload, "
                           f"M={M} draw), single-threaded C oracle in double, {el:.1f} s"}, **host_cpu())


# ---------------------------------------------------------------------------
# Multi-rank host logic (no data-path collective: each rank routes its own rows)
def rank_seed(name: str, M: int, rank: int) -> int:
    """Each rank draws its own batch of the workload (rows sharded by rank)."""
    from moe_expert_routing_token_b200 import inputs
    return inputs.default_seed(name, M) + 7919 * rank


def job_elapsed_ms(local_ms: float, world: int, device) -> float:
    """The job's time: the maximum of the ranks' device-timed elapsed times."""
    if world == 1:
        return float(local_ms)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(local_ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tokens_per_s(M: int, steps: int, world: int, ms: float) -> float:
    """Whole-job throughput: the tokens every rank routed over the job time."""
    return M * steps * world / (ms / 1e3)


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    name = args.workload
    M = args.M or DEFAULT_M[name]
    from moe_expert_routing_token_b200 import inputs
    d = inputs.make(name, M)
    # bounded sample per step so that warmup + steps finish in about a minute
    t_row = _oracle_row_time(name, d)
    budget = 60.0
    rows = int(max(1, min(M, budget / max(1, args.steps + args.warmup) / t_row)))
    for _ in range(args.warmup):
        oracle_call(name, d, slice(0, rows))
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle_call(name, d, slice(0, rows))
    el = time.perf_counter() - t0
    value = rows * args.steps / el
    cfg = workload_desc(name, M)
    cfg["sample_tokens_per_step"] = rows
    line = {"impl": "reference", "metric": metric_for(name), "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": el * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": cfg,
            "cpu_baseline": dict({"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                                  "sample": f"{rows} of {M} tokens per step"}, **host_cpu()),
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def _oracle_row_time(name, d):
    rows = 4 if name == "fused" else 512
    oracle_call(name, d, slice(0, 2))
    t0 = time.perf_counter()
    oracle_call(name, d, slice(0, rows))
    return (time.perf_counter() - t0) / rows


# ---------------------------------------------------------------------------
# the GPU arm
# ---------------------------------------------------------------------------
class Workload:
    """Device buffers and the C-ABI call of one workload at one size: a pool
    of input/output sets whose total exceeds 4x L2 (``rotate``), or one set."""

    def __init__(self, name: str, M: int, dev, seed: int, rotate: bool = True, d=None):
        import torch

        from moe_expert_routing_token_b200 import inputs, routing
        self.name, self.M, self.dev = name, M, dev
        self.lib = routing.lib()
        self.sp = sp = inputs.SPECS[name]
        self.d = d = inputs.make(name, M, seed=seed) if d is None else d
        self.per_set = algorithmic_bytes(name, M)
        self.pool = max(2, min(256, -(-4 * L2_BYTES // self.per_set))) if rotate else 1
        if name in ("fused", "top1"):
            src = d["hidden"].to(dev)
            self.wgt = d["weight"].to(dev)
        else:
            src = d["logits"].to(dev)
        self.xs = [src] + [src.clone() for _ in range(self.pool - 1)]
        self.bias = d["bias"].to(dev) if d["bias"] is not None else None
        self.ws = [torch.empty(M, sp.topk, dtype=torch.float32, device=dev) for _ in range(self.pool)]
        self.ids = [torch.empty(M, sp.topk, dtype=torch.int32, device=dev) for _ in range(self.pool)]
        self.wsp_bytes = routing.fused_router_workspace_size(M, sp.K, sp.E) if name == "fused" else 0
        self.wsp = [torch.zeros(max(1, self.wsp_bytes), dtype=torch.uint8, device=dev) for _ in range(self.pool)]
        self.dcode = routing.MOE_DTYPE_BF16 if sp.dtype == torch.bfloat16 else routing.MOE_DTYPE_F32
        # the fused router's decode path (one tile, long K: a workspace) is two launches
        self.launches_per_call = 2 if (name == "fused" and self.wsp_bytes > 0) else 1

    def call(self, i: int, stream_ptr: int, logits_out=None):
        from moe_expert_routing_token_b200 import routing
        lib, sp, M, name = self.lib, self.sp, self.M, self.name
        j = i % self.pool
        bptr = self.bias.data_ptr() if self.bias is not None else None
        lptr = logits_out.data_ptr() if logits_out is not None else None
        if name == "fused":
            st = lib.moe_fused_router_topk(self.xs[j].data_ptr(), self.wgt.data_ptr(), routing.MOE_WEIGHT_K_BY_E,
                                           bptr, M, sp.K, sp.E, sp.topk, int(sp.renormalize),
                                           sp.num_expert_group, sp.topk_group, sp.routed_scaling_factor,
                                           self.ws[j].data_ptr(), self.ids[j].data_ptr(), lptr,
                                           self.wsp[j].data_ptr() if self.wsp_bytes else None, self.wsp_bytes,
                                           stream_ptr)
        elif name == "top1":
            st = lib.moe_fused_router_top1(self.xs[j].data_ptr(), self.wgt.data_ptr(), routing.MOE_WEIGHT_E_BY_K,
                                           M, sp.K, sp.E, sp.softcap, self.ws[j].data_ptr(), self.ids[j].data_ptr(),
                                           lptr, stream_ptr)
        elif name in ("softmax", "grouped"):
            st = lib.moe_grouped_topk(self.xs[j].data_ptr(), self.dcode, M, sp.E, sp.topk, int(sp.renormalize),
                                      sp.num_expert_group, sp.topk_group, sp.routed_scaling_factor,
                                      self.ws[j].data_ptr(), self.ids[j].data_ptr(), stream_ptr)
        else:
            st = lib.moe_biased_grouped_topk(self.xs[j].data_ptr(), self.dcode, bptr, M, sp.E, sp.topk,
                                             int(sp.renormalize), sp.num_expert_group, sp.topk_group,
                                             sp.routed_scaling_factor, self.ws[j].data_ptr(),
                                             self.ids[j].data_ptr(), stream_ptr)
        if st != 0:
            raise RuntimeError(lib.moe_last_error().decode())


class GraphTimer:
    """CUDA graphs of consecutive calls of one workload - a whole number of
    passes over its buffer pool, at least 64 calls - and of the remainders,
    replayed for exactly n steps and timed with CUDA events on the launching
    stream."""

    def __init__(self, call, pool: int, steps: int, warmup: int, stream):
        import torch
        self.stream = stream
        self.pool = pool = pool * max(1, -(-64 // pool))  # calls per graph
        sptr = stream.cuda_stream

        def capture(nsteps: int):
            if nsteps == 0:
                return None
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for i in range(nsteps):
                    call(i, sptr)
            return g

        for i in range(3):  # eager warm-up of the C ABI (first-call set-up happens here)
            call(i, sptr)
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            self.g_pool = capture(pool)
            self.g_rem = {steps % pool: capture(steps % pool), warmup % pool: capture(warmup % pool)}

    def run(self, n: int):
        for _ in range(n // self.pool):
            self.g_pool.replay()
        g = self.g_rem.get(n % self.pool)
        if g is not None:
            g.replay()

    def time_ms(self, n: int, barrier=None) -> float:
        """Device time of exactly n steps: synchronise (and barrier), queue a
        GPU sleep that covers the host's graph submission, then events around
        the n steps."""
        import torch
        if barrier is not None:
            barrier()
        torch.cuda.synchronize()
        start = torch.cuda.Event(enable_timing=True)
        stop = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(self.stream):
            torch.cuda._sleep(SLEEP_CYCLES)
            start.record(self.stream)
            self.run(n)
            stop.record(self.stream)
        torch.cuda.synchronize()
        if barrier is not None:
            barrier()
        return start.elapsed_time(stop)

    def release(self):
        self.g_pool = None
        self.g_rem = {}


def roofline(name: str, M: int, us_per_call: float, clocks, peaks) -> dict:
    from moe_expert_routing_token_b200 import inputs
    sp = inputs.SPECS[name]
    if name == "fused":
        flops = 2.0 * M * sp.K * sp.E
        achieved = flops / (us_per_call * 1e-6) / 1e12
        # A long loop of GEMMs runs under the power cap: then the sustained
        # cuBLAS figure is the comparable peak, else the burst one.
        capped = bool(clocks) and ("sw_power_cap" in clocks.get("reasons", []) or
                                   clocks.get("sm_mhz", 0) < 0.9 * clocks.get("sm_max_mhz", 1))
        if capped and peaks.get("bf16_tflops_sustained"):
            peak, kind = peaks["bf16_tflops_sustained"], "bf16 sustained (run under the power cap)"
        else:
            peak, kind = peaks["bf16_tflops"], "bf16 burst"
        return {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": profiled_traffic(name, M),
                "algorithmic_flops_per_launch": flops, "peak_source": f"{peaks['source']} {kind}"}
    per_set = algorithmic_bytes(name, M)
    achieved = per_set / (us_per_call * 1e-6) / 1e9
    return {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": achieved / peaks["hbm_gbs"], "traffic": profiled_traffic(name, M),
            "algorithmic_bytes_per_launch": per_set, "peak_source": f"{peaks['source']} HBM copy"}


def sample_rows(M: int, n: int):
    """Rows for a parity sample: all rows when M <= n, else the first and the
    last n / 2 rows (the last covers the ragged tail of the grid)."""
    import numpy as np
    if M <= n:
        return np.arange(M)
    h = n // 2
    return np.concatenate([np.arange(h), np.arange(M - (n - h), M)])


def parity_sample(wl: Workload, stream) -> dict:
    """CPU-baseline leg: the oracle on a sample of the workload's rows against
    the GPU's outputs for them (the inputs of every pool slot are the same
    draw).  Fused and top-1 routers: one extra untimed call returns the fp32
    logits, the oracle routes those (the routing step, bit-exact rules) and the
    logits are checked against the oracle's double-precision projection."""
    import numpy as np
    import torch

    import oracle
    from oracle import parity
    name, M, sp, d = wl.name, wl.M, wl.sp, wl.d
    n = {"fused": 64, "top1": 512}.get(name, 2048)
    rows = sample_rows(M, n)
    out = {"rows": int(len(rows))}
    logits = None
    if name in ("fused", "top1"):
        logits = torch.empty(M, sp.E, dtype=torch.float32, device=wl.dev)
        wl.call(0, stream.cuda_stream, logits_out=logits)
    torch.cuda.synchronize()
    w = wl.ws[0].cpu().numpy()[rows]
    ids = wl.ids[0].cpu().numpy()[rows]
    if name in ROUTING:
        orc = oracle_call(name, d, rows)
        rep = parity.compare(w, ids, orc, E=sp.E, G=sp.num_expert_group, TG=sp.topk_group, k=sp.topk,
                             renorm=sp.renormalize, rsf=sp.routed_scaling_factor,
                             fp32_logits=(sp.dtype == torch.float32))
    elif name == "fused":
        lg = logits.cpu().double().numpy()[rows]
        ref = oracle.router_logits(d["hidden"][rows], d["weight"], weight_layout=0)
        out["max_logit_err"] = float(np.abs(lg - ref).max())
        orc = oracle.biased_grouped_topk(lg, d["bias"], sp.topk, sp.renormalize, sp.num_expert_group,
                                         sp.topk_group, sp.routed_scaling_factor)
        rep = parity.compare(w, ids, orc, E=sp.E, G=sp.num_expert_group, TG=sp.topk_group, k=sp.topk,
                             renorm=sp.renormalize, rsf=sp.routed_scaling_factor, fp32_logits=False)
    else:
        lg = logits.cpu().double().numpy()[rows]
        ref = oracle.router_logits(d["hidden"][rows], d["weight"], weight_layout=1)
        out["max_logit_err"] = float(np.abs(lg - ref).max())
        orc = oracle.topk_softmax(oracle.softcap_logits(lg, sp.softcap), 1, False)
        rep = parity.compare(w, ids, orc, E=sp.E, G=1, TG=1, k=1, renorm=False, rsf=1.0, fp32_logits=True,
                             w_rtol=2e-5)
    out.update({"near_tie": rep.near_tie, "max_weight_err": rep.max_weight_err, "ok": rep.ok(),
                "checked_by": "oracle on the sampled rows (CPU-baseline leg)"})
    if not rep.ok():
        out["failures"] = rep.failures[:4]
    return out


def run_per_config(dev, stream, steps: int, peaks, with_parity: bool) -> list:
    """Every size the routing spec names: cold (rotating pool > 4x L2) and hot
    (one buffer) device time per call, roofline fraction, parity sample."""
    import torch
    rows = []
    for name, M in PER_CONFIG:
        from moe_expert_routing_token_b200 import inputs
        seed = inputs.default_seed(name, M)
        entry = {"workload": name, "M": M}
        d = inputs.make(name, M, seed=seed)
        for kind, rotate in (("cold", True), ("hot", False)):
            wl = Workload(name, M, dev, seed, rotate=rotate, d=d)
            gt = GraphTimer(wl.call, wl.pool, steps, 3, stream)
            gt.run(3)
            ms = gt.time_ms(steps)
            entry[f"us_per_call_{kind}"] = ms * 1e3 / steps
            if kind == "cold":
                entry["pool_sets"] = wl.pool
                entry["tokens_per_s"] = M * steps / (ms / 1e3)
                rf = roofline(name, M, entry["us_per_call_cold"], None, peaks)
                entry["roofline"] = {k: rf[k] for k in ("bound", "achieved", "peak", "unit", "frac")}
                if with_parity:
                    entry["parity"] = parity_sample(wl, stream)
            gt.release()
            del wl
            torch.cuda.synchronize()
        rows.append(entry)
    return rows


def run_ours(args):
    import torch
    import torch.distributed as dist

    from moe_expert_routing_token_b200 import build, routing

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py: no CUDA device; the routing library has no CPU path")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    if rank == 0:
        build.build()
    if world > 1:
        dist.barrier()
    routing.lib()

    name = args.workload
    M = args.M or DEFAULT_M[name]
    # a dedicated stream: graphs cannot be captured on the legacy default stream
    stream = torch.cuda.Stream(dev)
    torch.cuda.set_stream(stream)

    wl = Workload(name, M, dev, rank_seed(name, M, rank))
    gt = GraphTimer(wl.call, wl.pool, args.steps, args.warmup, stream)
    sampler = ClockSampler(local_rank) if rank == 0 else None
    gt.run(args.warmup)
    # untimed soak so that the clock sampler sees the GPU under this load
    t_soak = time.time()
    while not args.no_soak and time.time() - t_soak < 1.0:
        gt.g_pool.replay()
        torch.cuda.synchronize()
    ms = gt.time_ms(args.steps, barrier=dist.barrier if world > 1 else None)
    clocks = sampler.stop() if sampler else None
    ms = job_elapsed_ms(ms, world, dev)
    value = job_tokens_per_s(M, args.steps, world, ms)
    us_per_call = ms * 1e3 / args.steps

    # ---- end to end through the public API with host buffers ----------------
    e2e = None
    if not args.no_e2e:
        e2e = e2e_measure(name, M, wl.sp, wl.d, dev, stream, world, args)

    peaks = measured_peaks()
    line = {"metric": metric_for(name), "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
            "us_per_call": us_per_call, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": dict(workload_desc(name, M), parallelism=f"dp{world} (rows sharded, no collective)",
                           l2=(f"rotating pool of {wl.pool} input/output sets, "
                               f"{wl.pool * wl.per_set / 2**20:.0f} MiB > 126 MiB L2"),
                           timing=("CUDA graphs of the C-ABI calls, CUDA events on the launch stream; "
                                   "a GPU sleep before the start event covers the host's graph launch")),
            "gpu_launches": args.steps * wl.launches_per_call,
            "clocks": clocks,
            "roofline": roofline(name, M, us_per_call, clocks, peaks)}
    line["e2e"] = e2e
    with_cpu = rank == 0 and world == 1 and not args.no_cpu_baseline
    if with_cpu:
        line["cpu_baseline"] = time_oracle(name, M, args.cpu_seconds)
        p = parity_sample(wl, stream)
        line["near_tie"] = p["near_tie"]
        line["max_weight_err"] = p["max_weight_err"]
        line["parity_sample"] = p
    gt.release()
    del wl
    if world == 1 and not args.no_per_config:
        line["per_config"] = run_per_config(dev, stream, args.per_config_steps, peaks, with_cpu)
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def e2e_measure(name, M, sp, d, dev, stream, world, args):
    """Host-resident inputs: per step H2D of the logits (or hidden states) from
    pinned memory (in row-chunks on parallel copy streams), the C-ABI call,
    D2H of weights and ids into pinned memory.  Consecutive steps overlap as
    a serving loop would: step i + 1's input crosses PCIe into the second of
    two device buffers while step i is routed and its outputs are read back."""
    import torch
    import torch.distributed as dist

    from moe_expert_routing_token_b200 import routing
    steps = max(1, min(args.steps, 200))
    src = (d["hidden"] if name in ("fused", "top1") else d["logits"]).pin_memory()
    xs = [torch.empty_like(src, device=dev) for _ in range(2)]
    wgt = d["weight"].to(dev) if name in ("fused", "top1") else None
    bias = d["bias"].to(dev) if d["bias"] is not None else None
    w = torch.empty(M, sp.topk, dtype=torch.float32, device=dev)
    ids = torch.empty(M, sp.topk, dtype=torch.int32, device=dev)
    hw = torch.empty(M, sp.topk, dtype=torch.float32).pin_memory()
    hi = torch.empty(M, sp.topk, dtype=torch.int32).pin_memory()
    need = routing.fused_router_workspace_size(M, sp.K, sp.E) if name == "fused" else 0
    wsp = torch.zeros(max(1, need), dtype=torch.uint8, device=dev)

    # The step's input crosses PCIe as n_chunks row-chunks on their own
    # streams: one 8 MiB pinned copy moved 12 GB/s on some B200 boxes, four
    # concurrent ones 47 GB/s.
    n_chunks = 4
    rows = src.shape[0]
    bounds = [rows * c // n_chunks for c in range(n_chunks + 1)]
    copy_streams = [torch.cuda.Stream(device=dev) for _ in range(n_chunks)]
    copied = [[torch.cuda.Event() for _ in range(n_chunks)] for _ in range(2)]
    read = [torch.cuda.Event() for _ in range(2)]  # the last call that read buffer b is done
    count = [0]

    def step():
        b = count[0] % 2
        count[0] += 1
        x = xs[b]
        cur = torch.cuda.current_stream()
        for c in range(n_chunks):
            cs = copy_streams[c]
            cs.wait_event(read[b])  # the call two steps back has finished reading this buffer
            with torch.cuda.stream(cs):
                x[bounds[c]:bounds[c + 1]].copy_(src[bounds[c]:bounds[c + 1]], non_blocking=True)
                copied[b][c].record(cs)
        for c in range(n_chunks):
            cur.wait_event(copied[b][c])
        if name == "fused":
            routing.fused_router_topk(x, wgt, bias, sp.topk, sp.renormalize, sp.num_expert_group,
                                      sp.topk_group, sp.routed_scaling_factor, workspace=wsp,
                                      out=(w, ids))
        elif name == "top1":
            routing.fused_router_top1(x, wgt, sp.softcap, weight_layout="ek", out=(w, ids))
        elif name in ("softmax", "grouped"):
            routing.grouped_topk(x, sp.topk, sp.renormalize, sp.num_expert_group, sp.topk_group,
                                 sp.routed_scaling_factor, out=(w, ids))
        else:
            routing.biased_grouped_topk(x, bias, sp.topk, sp.renormalize, sp.num_expert_group,
                                        sp.topk_group, sp.routed_scaling_factor, out=(w, ids))
        read[b].record(cur)
        hw.copy_(w, non_blocking=True)
        hi.copy_(ids, non_blocking=True)

    with torch.cuda.stream(stream):
        for _ in range(3):
            step()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(steps):
            step()
        b.record(stream)
        torch.cuda.synchronize()
    ms = job_elapsed_ms(a.elapsed_time(b), world, dev)
    return {"value": job_tokens_per_s(M, steps, world, ms), "unit": "tokens/s",
            "h2d_bytes_per_step": src.numel() * src.element_size(),
            "d2h_bytes_per_step": hw.numel() * 4 + hi.numel() * 4, "steps": steps}


# ---------------------------------------------------------------------------
# The expert permutation after routing (moe_expert_permutation)
PERM_METRIC = "permuted tokens/s & us/call (expert-sorted permutation of (M, k=8) ids, E=256); % of HBM roofline"


def perm_bytes(M: int) -> int:
    """Bytes a permutation call must move: ids and weights in; gather, scatter
    and gate out; counts and offsets."""
    n = M * PERM_K
    return n * 4 * 5 + (2 * PERM_E + 1) * 4


def perm_desc(M: int) -> dict:
    return {"M": M, "k": PERM_K, "E": PERM_E,
            "workload": (f"expert-sorted permutation of a routing result: topk_ids (M={M}, k={PERM_K}) int32 "
                         f"(k distinct uniform experts of E={PERM_E} per token), fp32 weights -> counts, "
                         f"offsets, gather, scatter, gate")}


def time_perm_oracle(M: int, seconds: float) -> dict:
    import oracle
    from moe_expert_routing_token_b200 import inputs
    ids, w = inputs.routed_ids(M, PERM_K, PERM_E, seed=4242)
    ids_np, w_np = ids.numpy(), w.numpy()
    oracle.expert_permutation(ids_np[:8], PERM_E, w_np[:8])
    n, t0 = 0, time.perf_counter()
    while True:
        oracle.expert_permutation(ids_np, PERM_E, w_np)
        n += M
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    return dict({"value": n / el, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                 "sample": f"{n} tokens ({n // M} x {M}-token batches), single-threaded C oracle, {el:.1f} s"},
                **host_cpu())


class PermWorkload:
    """Device buffers and the C-ABI call of the expert permutation."""

    def __init__(self, M: int, dev, seed: int):
        import torch

        from moe_expert_routing_token_b200 import inputs, routing
        self.M, self.n = M, M * PERM_K
        self.lib = routing.lib()
        self.ids_h, self.w_h = inputs.routed_ids(M, PERM_K, PERM_E, seed=seed)
        self.per_set = perm_bytes(M)
        self.pool = max(2, min(256, -(-4 * L2_BYTES // self.per_set)))
        self.ids = [self.ids_h.to(dev) for _ in range(self.pool)]
        self.wts = [self.w_h.to(dev) for _ in range(self.pool)]
        n = self.n
        self.outs = [[torch.empty(PERM_E, dtype=torch.int32, device=dev),
                      torch.empty(PERM_E + 1, dtype=torch.int32, device=dev),
                      torch.empty(n, dtype=torch.int32, device=dev), torch.empty(n, dtype=torch.int32, device=dev),
                      torch.empty(n, dtype=torch.float32, device=dev)] for _ in range(self.pool)]
        self.wsb = routing.expert_permutation_workspace_size(M, PERM_K, PERM_E)
        self.wsp = [torch.empty(max(1, self.wsb), dtype=torch.uint8, device=dev) for _ in range(self.pool)]

    def call(self, i: int, stream_ptr: int, src_ids=None, src_w=None, out=None, ws=None):
        j = i % self.pool
        o = out if out is not None else self.outs[j]
        st = self.lib.moe_expert_permutation((src_ids if src_ids is not None else self.ids[j]).data_ptr(),
                                             (src_w if src_w is not None else self.wts[j]).data_ptr(), self.M,
                                             PERM_K, PERM_E, o[0].data_ptr(), o[1].data_ptr(), o[2].data_ptr(),
                                             o[3].data_ptr(), o[4].data_ptr(),
                                             (ws if ws is not None else self.wsp[j]).data_ptr(), self.wsb,
                                             stream_ptr)
        if st != 0:
            raise RuntimeError(self.lib.moe_last_error().decode())


def run_permute(args):
    import torch
    import torch.distributed as dist

    from moe_expert_routing_token_b200 import build, routing

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank != 0:
            return 0
        M = args.M or DEFAULT_M["permute"]
        base = time_perm_oracle(M, min(args.cpu_seconds, 10.0))
        line = {"impl": "reference", "metric": PERM_METRIC, "value": base["value"], "unit": "tokens/s",
                "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": M / base["value"] * 1e3, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "int32", "data": "synthetic", "config": perm_desc(M),
                "cpu_baseline": base,
                "e2e": {"value": base["value"], "unit": "tokens/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
        print(json.dumps(line), flush=True)
        return 0
    if not torch.cuda.is_available():
        raise SystemExit("bench.py: no CUDA device; the routing library has no CPU path")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    if rank == 0:
        build.build()
    if world > 1:
        dist.barrier()
    routing.lib()
    M = args.M or DEFAULT_M["permute"]
    stream = torch.cuda.Stream(dev)
    torch.cuda.set_stream(stream)
    pw = PermWorkload(M, dev, rank_seed("sigmoid", M, rank))
    gt = GraphTimer(pw.call, pw.pool, args.steps, args.warmup, stream)
    sampler = ClockSampler(local_rank) if rank == 0 else None
    gt.run(args.warmup)
    t_soak = time.time()
    while not args.no_soak and time.time() - t_soak < 1.0:
        gt.g_pool.replay()
        torch.cuda.synchronize()
    ms = job_elapsed_ms(gt.time_ms(args.steps, barrier=dist.barrier if world > 1 else None), world, dev)
    clocks = sampler.stop() if sampler else None
    value = job_tokens_per_s(M, args.steps, world, ms)
    us_per_call = ms * 1e3 / args.steps

    e2e = None
    if not args.no_e2e:
        # host buffers in, permutation out, every step
        h_ids = pw.ids_h.pin_memory()
        h_w = pw.w_h.pin_memory()
        h_out = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in pw.outs[0]]
        d_ids, d_w = pw.ids[0], pw.wts[0]
        steps = 200

        def step():
            d_ids.copy_(h_ids, non_blocking=True)
            d_w.copy_(h_w, non_blocking=True)
            pw.call(0, stream.cuda_stream, d_ids, d_w, pw.outs[0], pw.wsp[0])
            for h, d in zip(h_out, pw.outs[0]):
                h.copy_(d, non_blocking=True)

        with torch.cuda.stream(stream):
            for _ in range(3):
                step()
            torch.cuda.synchronize()
            if world > 1:
                dist.barrier()
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            for _ in range(steps):
                step()
            b.record(stream)
            torch.cuda.synchronize()
        ems = job_elapsed_ms(a.elapsed_time(b), world, dev)
        e2e = {"value": job_tokens_per_s(M, steps, world, ems), "unit": "tokens/s",
               "h2d_bytes_per_step": pw.n * 8, "d2h_bytes_per_step": sum(t.numel() * 4 for t in h_out),
               "steps": steps}

    peaks = measured_peaks()
    achieved = pw.per_set / (us_per_call * 1e-6) / 1e9
    line = {"metric": PERM_METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
            "us_per_call": us_per_call, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int32", "data": "synthetic",
            "config": dict(perm_desc(M), parallelism=f"dp{world} (rows sharded, no collective)",
                           l2=f"rotating pool of {pw.pool} sets, {pw.pool * pw.per_set / 2**20:.0f} MiB > 126 MiB L2",
                           timing=("CUDA graphs of the C-ABI calls, CUDA events on the launch stream; "
                                   "a GPU sleep before the start event covers the host's graph launch")),
            "gpu_launches": 2 * args.steps, "clocks": clocks,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / peaks["hbm_gbs"], "traffic": None,
                         "algorithmic_bytes_per_launch": pw.per_set,
                         "peak_source": f"{peaks['source']} HBM copy"},
            "e2e": e2e}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = time_perm_oracle(M, args.cpu_seconds)
    gt.release()
    if world > 1:
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def main():
    args = parse_args()
    if args.workload == "permute":
        return run_permute(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
