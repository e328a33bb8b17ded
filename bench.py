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
barrier and a device synchronise; the job time is the max over ranks.  Under
torchrun each rank routes its own batches (no data-path collective: rows are
independent), so scaling is weak.
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


def parse_args():
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
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-soak", action="store_true", help="skip the 1 s clock-sampling soak")
    return ap.parse_args()


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
        d["workload"] = (f"small-E fused router on the CUDA cores: (M,{sp.K}) bf16 x ({sp.E},{sp.K}) bf16 "
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
def oracle_call(name: str, d: dict, rows: slice):
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
    return {"value": n / el, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{n} tokens ({n // rows} x {rows}-token batches of the {name} workload, "
                      f"M={M} draw), single-threaded C oracle in double, {el:.1f} s"}


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
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                             "sample": f"{rows} of {M} tokens per step"},
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
def run_ours(args):
    import torch
    import torch.distributed as dist

    from moe_expert_routing_token_b200 import build, inputs, routing

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
    lib = routing.lib()

    name = args.workload
    M = args.M or DEFAULT_M[name]
    sp = inputs.SPECS[name]
    d = inputs.make(name, M, seed=rank_seed(name, M, rank))
    # a dedicated stream: graphs cannot be captured on the legacy default stream
    stream = torch.cuda.Stream(dev)
    torch.cuda.set_stream(stream)
    sptr = stream.cuda_stream

    # ---- rotating device pool larger than L2 --------------------------------
    per_set = algorithmic_bytes(name, M)
    pool = max(2, min(256, -(-4 * L2_BYTES // per_set)))
    if name in ("fused", "top1"):
        src_x = d["hidden"].to(dev)
        wgt = d["weight"].to(dev)
    else:
        src_x = d["logits"].to(dev)
    xs = [src_x.clone() for _ in range(pool)]
    bias = d["bias"].to(dev) if d["bias"] is not None else None
    bptr = bias.data_ptr() if bias is not None else None
    ws = [torch.empty(M, sp.topk, dtype=torch.float32, device=dev) for _ in range(pool)]
    ids = [torch.empty(M, sp.topk, dtype=torch.int32, device=dev) for _ in range(pool)]
    wsp_bytes = routing.fused_router_workspace_size(M, sp.K, sp.E) if name == "fused" else 0
    wsp = [torch.zeros(max(1, wsp_bytes), dtype=torch.uint8, device=dev) for _ in range(pool)]

    dcode = routing.MOE_DTYPE_BF16 if sp.dtype == torch.bfloat16 else routing.MOE_DTYPE_F32

    def call(i: int):
        j = i % pool
        if name == "fused":
            st = lib.moe_fused_router_topk(xs[j].data_ptr(), wgt.data_ptr(), routing.MOE_WEIGHT_K_BY_E,
                                           bptr, M, sp.K, sp.E, sp.topk, int(sp.renormalize),
                                           sp.num_expert_group, sp.topk_group,
                                           sp.routed_scaling_factor, ws[j].data_ptr(),
                                           ids[j].data_ptr(), None,
                                           wsp[j].data_ptr() if wsp_bytes else None, wsp_bytes, sptr)
        elif name == "top1":
            st = lib.moe_fused_router_top1(xs[j].data_ptr(), wgt.data_ptr(), routing.MOE_WEIGHT_E_BY_K, M, sp.K,
                                           sp.E, sp.softcap, ws[j].data_ptr(), ids[j].data_ptr(), None, sptr)
        elif name in ("softmax", "grouped"):
            st = lib.moe_grouped_topk(xs[j].data_ptr(), dcode, M, sp.E, sp.topk, int(sp.renormalize),
                                      sp.num_expert_group, sp.topk_group, sp.routed_scaling_factor,
                                      ws[j].data_ptr(), ids[j].data_ptr(), sptr)
        else:
            st = lib.moe_biased_grouped_topk(xs[j].data_ptr(), dcode, bptr, M, sp.E, sp.topk,
                                             int(sp.renormalize), sp.num_expert_group,
                                             sp.topk_group, sp.routed_scaling_factor,
                                             ws[j].data_ptr(), ids[j].data_ptr(), sptr)
        if st != 0:
            raise RuntimeError(lib.moe_last_error().decode())

    # ---- graphs: one of `pool` steps and one of the remainder -----------------
    for i in range(3):  # eager warm-up of the C ABI (first-call set-up happens here)
        call(i)
    torch.cuda.synchronize()

    def capture(nsteps: int):
        if nsteps == 0:
            return None
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(nsteps):
                call(i)
        return g

    with torch.cuda.stream(stream):
        g_pool = capture(pool)
        g_rem = capture(args.steps % pool)
        g_warm_rem = capture(args.warmup % pool)

    def run_steps(n: int, rem_graph):
        for _ in range(n // pool):
            g_pool.replay()
        if rem_graph is not None:
            rem_graph.replay()

    sampler = ClockSampler(local_rank) if rank == 0 else None
    run_steps(args.warmup, g_warm_rem)
    # untimed soak so that the clock sampler sees the GPU under this load
    t_soak = time.time()
    while not args.no_soak and time.time() - t_soak < 1.0:
        g_pool.replay()
        torch.cuda.synchronize()

    start = torch.cuda.Event(enable_timing=True)
    stop = torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    start.record(stream)
    run_steps(args.steps, g_rem)
    stop.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = start.elapsed_time(stop)
    clocks = sampler.stop() if sampler else None
    ms = job_elapsed_ms(ms, world, dev)
    value = job_tokens_per_s(M, args.steps, world, ms)
    us_per_call = ms * 1e3 / args.steps

    # ---- end to end through the public API with host buffers ----------------
    e2e = None
    if not args.no_e2e:
        e2e = e2e_measure(name, M, sp, d, dev, stream, world, args)

    peaks = measured_peaks()
    line = {"metric": metric_for(name), "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
            "us_per_call": us_per_call, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": dict(workload_desc(name, M), parallelism=f"dp{world} (rows sharded, no collective)",
                           l2=(f"rotating pool of {pool} input/output sets, "
                               f"{pool * per_set / 2**20:.0f} MiB > 126 MiB L2"),
                           timing="CUDA graphs of the C-ABI calls, CUDA events on the launch stream"),
            "gpu_launches": args.steps,
            "clocks": clocks}
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
        line["roofline"] = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                            "frac": achieved / peak, "traffic": profiled_traffic(name, M),
                            "peak_source": f"{peaks['source']} {kind}"}
    else:
        achieved = per_set / (us_per_call * 1e-6) / 1e9
        peak = peaks["hbm_gbs"]
        line["roofline"] = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                            "frac": achieved / peak, "traffic": profiled_traffic(name, M),
                            "algorithmic_bytes_per_launch": per_set,
                            "peak_source": f"{peaks['source']} HBM copy"}
    line["e2e"] = e2e
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = time_oracle(name, M, args.cpu_seconds)
    if world > 1:
        del g_pool, g_rem, g_warm_rem
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def e2e_measure(name, M, sp, d, dev, stream, world, args):
    """Host-resident inputs: per step H2D of the logits (or hidden states) from
    pinned memory, the C-ABI call, D2H of weights and ids into pinned memory."""
    import torch
    import torch.distributed as dist

    from moe_expert_routing_token_b200 import routing
    lib = routing.lib()
    steps = max(1, min(args.steps, 200))
    src = (d["hidden"] if name in ("fused", "top1") else d["logits"]).pin_memory()
    x = torch.empty_like(src, device=dev)
    wgt = d["weight"].to(dev) if name in ("fused", "top1") else None
    bias = d["bias"].to(dev) if d["bias"] is not None else None
    w = torch.empty(M, sp.topk, dtype=torch.float32, device=dev)
    ids = torch.empty(M, sp.topk, dtype=torch.int32, device=dev)
    hw = torch.empty(M, sp.topk, dtype=torch.float32).pin_memory()
    hi = torch.empty(M, sp.topk, dtype=torch.int32).pin_memory()
    need = routing.fused_router_workspace_size(M, sp.K, sp.E) if name == "fused" else 0
    wsp = torch.zeros(max(1, need), dtype=torch.uint8, device=dev)

    def step():
        x.copy_(src, non_blocking=True)
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
    return {"value": n / el, "unit": "tokens/s", "cores": 1, "kind": "oracle",
            "sample": f"{n} tokens ({n // M} x {M}-token batches), single-threaded C oracle, {el:.1f} s"}


def run_permute(args):
    import torch
    import torch.distributed as dist

    from moe_expert_routing_token_b200 import build, inputs, routing

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
    lib = routing.lib()
    M = args.M or DEFAULT_M["permute"]
    n = M * PERM_K
    ids_h, w_h = inputs.routed_ids(M, PERM_K, PERM_E, seed=rank_seed("sigmoid", M, rank))
    stream = torch.cuda.Stream(dev)
    torch.cuda.set_stream(stream)
    sptr = stream.cuda_stream
    per_set = perm_bytes(M)
    pool = max(2, min(256, -(-4 * L2_BYTES // per_set)))
    ids = [ids_h.to(dev) for _ in range(pool)]
    wts = [w_h.to(dev) for _ in range(pool)]
    outs = [[torch.empty(PERM_E, dtype=torch.int32, device=dev), torch.empty(PERM_E + 1, dtype=torch.int32, device=dev),
             torch.empty(n, dtype=torch.int32, device=dev), torch.empty(n, dtype=torch.int32, device=dev),
             torch.empty(n, dtype=torch.float32, device=dev)] for _ in range(pool)]
    wsb = routing.expert_permutation_workspace_size(M, PERM_K, PERM_E)
    wsp = [torch.empty(max(1, wsb), dtype=torch.uint8, device=dev) for _ in range(pool)]

    def call(i: int, src_ids=None, src_w=None, out=None, ws=None):
        j = i % pool
        o = out if out is not None else outs[j]
        st = lib.moe_expert_permutation((src_ids if src_ids is not None else ids[j]).data_ptr(),
                                        (src_w if src_w is not None else wts[j]).data_ptr(), M, PERM_K, PERM_E,
                                        o[0].data_ptr(), o[1].data_ptr(), o[2].data_ptr(), o[3].data_ptr(),
                                        o[4].data_ptr(), (ws if ws is not None else wsp[j]).data_ptr(), wsb, sptr)
        if st != 0:
            raise RuntimeError(lib.moe_last_error().decode())

    for i in range(3):
        call(i)
    torch.cuda.synchronize()

    def capture(nsteps: int):
        if nsteps == 0:
            return None
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            for i in range(nsteps):
                call(i)
        return g

    with torch.cuda.stream(stream):
        g_pool = capture(pool)
        g_rem = capture(args.steps % pool)
        g_warm_rem = capture(args.warmup % pool)

    def run_steps(nst: int, rem_graph):
        for _ in range(nst // pool):
            g_pool.replay()
        if rem_graph is not None:
            rem_graph.replay()

    sampler = ClockSampler(local_rank) if rank == 0 else None
    run_steps(args.warmup, g_warm_rem)
    t_soak = time.time()
    while not args.no_soak and time.time() - t_soak < 1.0:
        g_pool.replay()
        torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    stop = torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    start.record(stream)
    run_steps(args.steps, g_rem)
    stop.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    ms = job_elapsed_ms(start.elapsed_time(stop), world, dev)
    clocks = sampler.stop() if sampler else None
    value = job_tokens_per_s(M, args.steps, world, ms)
    us_per_call = ms * 1e3 / args.steps

    e2e = None
    if not args.no_e2e:
        # host buffers in, permutation out, every step
        h_ids = ids_h.pin_memory()
        h_w = w_h.pin_memory()
        h_out = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in outs[0]]
        d_ids, d_w = ids[0], wts[0]
        steps = 200

        def step():
            d_ids.copy_(h_ids, non_blocking=True)
            d_w.copy_(h_w, non_blocking=True)
            call(0, d_ids, d_w, outs[0], wsp[0])
            for h, d in zip(h_out, outs[0]):
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
               "h2d_bytes_per_step": n * 8, "d2h_bytes_per_step": sum(t.numel() * 4 for t in h_out),
               "steps": steps}

    peaks = measured_peaks()
    achieved = per_set / (us_per_call * 1e-6) / 1e9
    line = {"metric": PERM_METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms / args.steps,
            "us_per_call": us_per_call, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "int32", "data": "synthetic",
            "config": dict(perm_desc(M), parallelism=f"dp{world} (rows sharded, no collective)",
                           l2=f"rotating pool of {pool} sets, {pool * per_set / 2**20:.0f} MiB > 126 MiB L2",
                           timing="CUDA graphs of the C-ABI calls, CUDA events on the launch stream"),
            "gpu_launches": 3 * args.steps, "clocks": clocks,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / peaks["hbm_gbs"], "traffic": None,
                         "algorithmic_bytes_per_launch": per_set,
                         "peak_source": f"{peaks['source']} HBM copy"},
            "e2e": e2e}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = time_perm_oracle(M, args.cpu_seconds)
    if world > 1:
        del g_pool, g_rem, g_warm_rem
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
