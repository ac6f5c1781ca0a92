#!/usr/bin/env python
"""Benchmark of the routed MoE FFN layer (DeepSeek-V4-Flash, MXFP4 experts,
int8 shared expert) on B200: prints ONE JSON line.

A step is one pass of the whole layer -- route, permute, forward -- over one
synthetic batch of the chosen workload (default: the full-size layer at decode
batch 1). Inputs are resident in HBM when timing starts; between timed steps
L2 is flushed (512 MiB write, then a 256 MiB read so that no dirty lines are
left for the next step to write back); every step is timed with CUDA events on
the launch stream and the sum over steps is taken, max over ranks.

Multi-GPU: replicas only (one process per GPU, each runs its own batch; no
collective on the data path), launched with torch.distributed.run.

`--impl reference` times the CPU oracle (the plain fp64 definition) on a
bounded sample of the same workload and prints the same line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MoE-layer tokens/s"
LINEAR_METRIC = "W8A16 linear tokens/s"

# W8A16 linear workloads: the linears_w8a16 targets of the config's attention
# at prefill size, name -> (T tokens, G groups, N outputs per group, K inputs
# per group). Shapes read from the config: fused_wqa_wkv q_lora_rank +
# head_dim from hidden_size; wq_b num_attention_heads * head_dim from
# q_lora_rank; wo_a o_groups groups of o_lora_rank from the group's heads *
# head_dim; wo_b hidden_size from o_groups * o_lora_rank; the indexer's wq_b
# index_n_heads * index_head_dim from q_lora_rank; the indexer compressor's wkv
# index_head_dim from hidden_size (its width is not printed: the plainest
# reading).
LINEAR_WORKLOADS = {
    "linear_fused_wqa_wkv_4096": (4096, 1, 1024 + 512, 4096),
    "linear_wq_b_4096": (4096, 1, 64 * 512, 1024),
    "linear_wo_a_4096": (4096, 8, 1024, 64 * 512 // 8),
    "linear_wo_b_4096": (4096, 1, 4096, 8 * 1024),
    "linear_indexer_wq_b_4096": (4096, 1, 64 * 128, 1024),
    "linear_indexer_wkv_4096": (4096, 1, 128, 4096),
}
HEADLINE = "decode_b1"   # the full-size layer at decode batch 1
L2_FLUSH_BYTES = 512 << 20
L2_CLEAN_BYTES = 256 << 20


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=None,
                    help="one workload only (default: the headline decode_b1 line with every "
                         "workload of the layer in its 'workloads' block)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--check-ranks", action="store_true",
                    help="start the ranks and check their plumbing on the CPU (gloo); measures nothing")
    return ap.parse_args()


# ----------------------------------------------------------------------------- accounting

def expert_bytes(wl):
    w13 = 2 * wl.I * wl.H // 2 + 2 * wl.I * wl.H // 32
    w2 = wl.H * wl.I // 2 + wl.H * wl.I // 32
    return w13, w2


def shared_bytes(wl):
    if wl.Is == 0:
        return 0, 0
    return 2 * wl.Is * wl.H + 2 * wl.Is * 4, wl.H * wl.Is + wl.H * 4


def algorithmic(wl, ids, token_ids=None):
    """Algorithmic bytes/FLOPs of one step and of each kernel kind."""
    T, H, I, Is, E, k = wl.T, wl.H, wl.I, wl.Is, wl.E, wl.k
    S = T * k
    n_hit = int(len(np.unique(ids))) if ids.size else 0
    e13, e2 = expert_bytes(wl)
    s13, s2 = shared_bytes(wl)
    route_b = E * H * 2 + E * 4                     # gate + bias
    if wl.routing == "hash":
        n_tok = int(len(np.unique(token_ids))) if token_ids is not None else T
        route_b = E * H * 2 + T * 4 + n_tok * k * 4  # gate + token ids + touched table rows
    step_b = n_hit * (e13 + e2) + s13 + s2 + route_b + 4 * T * H + 48 * T
    flops = S * 6 * H * I + T * 6 * H * Is + 2 * T * E * H
    # per kernel kind: routed experts only, shared expert only, or both in one kernel
    r13_b = n_hit * e13 + T * H * 2 + S * I * 2
    r2_b = n_hit * e2 + S * I * 2 + S * H * 4
    sh13_b = s13 + T * H * 2 + T * Is * 2
    sh2_b = s2 + T * Is * 2 + S * H * 4 + T * H * 2
    r13_f, r2_f = S * 2 * (2 * I) * H, S * 2 * H * I
    sh13_f, sh2_f = T * 2 * (2 * Is) * H, T * 2 * H * Is
    per_kernel_bytes = {
        "routed_w13": r13_b, "routed_w2": r2_b, "shared_w13": sh13_b, "shared_w2": sh2_b,
        "w13": n_hit * e13 + s13 + T * H * 2 + S * I * 2 + T * Is * 2,
        "w2": n_hit * e2 + s2 + S * I * 2 + T * Is * 2 + T * H * 2,
    }
    per_kernel_flops = {
        "routed_w13": r13_f, "routed_w2": r2_f, "shared_w13": sh13_f, "shared_w2": sh2_f,
        "w13": r13_f + sh13_f, "w2": r2_f + sh2_f,
    }
    return dict(n_hit=n_hit, step_bytes=step_b, step_flops=flops, kernel_bytes=per_kernel_bytes,
                kernel_flops=per_kernel_flops)


def kernel_kind(name):
    """Which part of the layer a kernel computes: the decode kernels take the
    routed experts and the shared expert together; on the tensor-core path the
    block-scaled kernels (mx*, mxt*) take the routed experts and the f16 ones
    (sh*, tc*) the shared expert."""
    part = "w13" if "w13" in name else "w2" if "w2" in name else None
    if part is None:
        return None
    if name.startswith("dec_"):
        return part
    if name.startswith("mx"):
        return "routed_" + part
    if name.startswith(("sh_", "tc_")):
        return "shared_" + part
    return part


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm=d["hbm_gbs"], bf16=d["bf16_tflops"], bf16_sus=d["bf16_tflops_sustained"],
                    src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


def source_hash(fname):
    """Hash of one kernel source file under csrc/ (the file the kernel lives in)."""
    path = os.path.join(ROOT, "mxfp4_routed_expert_v4moe_b200", "csrc", fname)
    if not os.path.exists(path):
        return None
    return hashlib.sha256(open(path, "rb").read()).hexdigest()[:16]


def recorded_traffic(kernel, workload):
    """DRAM bytes per launch from a committed ncu summary, if the kernel's
    source file is unchanged since the capture."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    try:
        e = json.load(open(p)).get(f"{kernel}@{workload}")
        if e and e.get("hash") == source_hash(e.get("file", "")):
            return e.get("bytes_per_launch")
    except Exception:
        return None
    return None


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid):
        self.uuid = uuid
        self.lines = []
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            if self.uuid and self.uuid not in parts[0]:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "samples": len(sm),
                "reasons": sorted(reasons)}


# ----------------------------------------------------------------------------- ranks

def rank_env():
    """(world, rank, local_rank) from the launcher's environment (1, 0, 0 alone)."""
    return (int(os.environ.get("WORLD_SIZE", "1")), int(os.environ.get("RANK", "0")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init_ranks(world, dev, backend="nccl"):
    """One process per GPU: the process group (short timeout) when world > 1."""
    if world > 1:
        import datetime

        import torch.distributed as dist
        kw = {"device_id": dev} if backend == "nccl" else {}
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300), **kw)


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(values, world, dev):
    """Element-wise maximum over ranks of a list of floats (device times)."""
    import torch
    t = torch.tensor(list(values), dtype=torch.float64, device=dev)
    if world > 1:
        import torch.distributed as dist
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def close_ranks(world):
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ----------------------------------------------------------------------------- CPU oracle

def oracle_sample(wl, li, n_tok, seconds, threads=1):
    """Time the oracle (route + layer) on n_tok tokens of the workload, repeated
    until about `seconds` of wall time; the layer part splits the tokens over
    `threads` host threads (each runs the single-threaded oracle on its share).
    Returns (tokens/s, tokens, reps, secs). When n_tok exceeds the batch, the
    batch's tokens are taken again (independent copies of the same work)."""
    import inputs as IN
    import oracle as O
    toks = np.arange(n_tok, dtype=np.int32) % wl.T
    sub = IN.LayerInputs(wl=wl.with_T(len(toks)), x=np.ascontiguousarray(li.x[toks]), gate=li.gate,
                         bias=li.bias,
                         token_ids=None if li.token_ids is None else np.ascontiguousarray(li.token_ids[toks]),
                         tid2eid=li.tid2eid, w13_codes=li.w13_codes, w13_scales=li.w13_scales,
                         w2_codes=li.w2_codes, w2_scales=li.w2_scales, sh13=li.sh13,
                         sh13_scale=li.sh13_scale, sh2=li.sh2, sh2_scale=li.sh2_scale)
    lay = O.Layer(sub)
    reps, t0 = 0, time.perf_counter()
    while True:
        ids, w, _, _ = lay.route()
        lay.moe_tokens(np.arange(len(toks)), ids, w, threads=threads)
        reps += 1
        el = time.perf_counter() - t0
        if el >= seconds:
            break
    return reps * len(toks) / el, len(toks), reps, el


def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


def cpu_baseline(wl, li, seconds):
    """The oracle on all host cores (one token per thread, the batch's tokens
    taken again when it has fewer), with the single-core figure beside it."""
    C = host_cores()
    tps, ntk, reps, el = oracle_sample(wl, li, C, seconds, threads=C)
    tps1, ntk1, reps1, el1 = oracle_sample(wl, li, 1, seconds / 2, threads=1)
    return {"value": tps, "unit": "tokens/s", "cores": C, "kind": "oracle",
            "sample": f"{reps} x {ntk} token(s) of {wl.name} (route over all {wl.E} experts + layer) "
                      f"on {C} host threads, {el:.1f} s, fp64",
            "single_core": {"value": tps1, "unit": "tokens/s", "cores": 1,
                            "sample": f"{reps1} x {ntk1} token(s), {el1:.1f} s"}}


# ----------------------------------------------------------------------------- main

def run_reference_linear(args):
    import inputs as IN
    import oracle as O
    if int(os.environ.get("RANK", "0")) != 0:
        return
    T, G, N, K = LINEAR_WORKLOADS[args.workload]
    x_bits = IN.normal_bf16(0, 1, T * G * K).reshape(T, G * K)
    q, sc = IN.int8_normal(0, 2, G * N, K, 0.02)
    times = []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        O.linear_w8a16_grouped(x_bits, q, sc, G, rows=[0])
        if i >= args.warmup:
            times.append(time.perf_counter() - t0)
    ms = 1e3 * float(np.mean(times))
    value = 1 / (ms / 1e3)
    print(json.dumps({"impl": "reference", "metric": LINEAR_METRIC, "value": value, "unit": "tokens/s",
                      "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
                      "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                      "data": "synthetic", "config": {"workload": args.workload, "T": T, "G": G, "N": N, "K": K},
                      "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                                       "sample": f"1 token row of {args.workload} per step"},
                      "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                              "d2h_bytes_per_step": 0}}), flush=True)


def run_reference(args):
    """The oracle as it stands on the host cores (one token of the workload per
    thread per step), same metric and workload as the GPU arm; rank 0 only."""
    import inputs as IN
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    wl = IN.WORKLOADS[args.workload or HEADLINE]
    li = IN.make_layer_inputs(wl)
    C = host_cores()
    step_times = []
    for i in range(args.warmup + args.steps):
        tps, ntk, reps, el = oracle_sample(wl, li, C, 0.0, threads=C)
        if i >= args.warmup:
            step_times.append(el / reps)
    ms = 1e3 * float(np.mean(step_times))
    value = C / (ms / 1e3)
    import oracle as O
    cfg = workload_config(wl, 1)
    cfg["experts_hit"] = int(len(np.unique(O.Layer(li).route()[0]))) if wl.T <= 64 else wl.E
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": cfg,
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": C, "kind": "oracle",
                             "sample": f"{C} token(s) of {wl.name} per step, one per host thread (route "
                                       f"over all {wl.E} experts + {wl.k} routed experts + shared expert)"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_linear(args):
    """One W8A16 linear call per step (v4moe_linear_w8a16_grouped), same timing rules."""
    import torch

    import inputs as IN
    import mxfp4_routed_expert_v4moe_b200 as V
    T, G, N, K = LINEAR_WORKLOADS[args.workload]
    world, rank, local = rank_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_ranks(world, dev)
    x_bits = IN.normal_bf16(0, 1, T * G * K).reshape(T, G * K)
    q, sc = IN.int8_normal(0, 2, G * N, K, 0.02)
    x = torch.from_numpy(x_bits.view(np.int16)).to(dev).view(torch.bfloat16)
    qd, sd = torch.from_numpy(q).to(dev), torch.from_numpy(sc).to(dev)
    out = torch.empty((T, G * N), dtype=torch.bfloat16, device=dev)
    nb = V.v4moe_linear_w8a16_grouped_workspace_bytes(T, G, N, K)
    ws = torch.zeros(nb, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    clean = torch.ones(L2_CLEAN_BYTES // 4, dtype=torch.float32, device=dev)

    def flush_l2(i):
        flush.fill_(i & 0xFF)
        clean.sum()

    def step(xx=x, oo=out):
        V.check(V.v4moe_linear_w8a16_grouped(T, G, N, K, xx, qd, sd, oo, ws, nb), "v4moe_linear_w8a16_grouped")

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    clocks = ClockSampler(str(torch.cuda.get_device_properties(dev).uuid))
    clocks.start()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize(dev)
    launches0 = V.v4moe_launch_count()
    for i in range(args.steps):
        flush_l2(i)
        evs[i][0].record(stream)
        step()
        evs[i][1].record(stream)
    torch.cuda.synchronize(dev)
    launches = V.v4moe_launch_count() - launches0
    barrier(world)
    ms_total = sum(a.elapsed_time(b) for a, b in evs)
    x_host = torch.from_numpy(x_bits.view(np.int16)).view(torch.bfloat16).pin_memory()
    out_host = torch.empty((T, G * N), dtype=torch.bfloat16).pin_memory()
    x_dev = torch.empty_like(x)
    e2e_evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    for i in range(args.steps):
        flush_l2(i)
        e2e_evs[i][0].record(stream)
        x_dev.copy_(x_host, non_blocking=True)
        step(x_dev)
        out_host.copy_(out, non_blocking=True)
        e2e_evs[i][1].record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = sum(a.elapsed_time(b) for a, b in e2e_evs)
    clk = clocks.stop()
    ms_total, e2e_ms = max_over_ranks([ms_total, e2e_ms], world, dev)
    ms_step = ms_total / args.steps
    e2e_ms /= args.steps
    V.v4moe_profile_reset()
    V.v4moe_profile_enable(True)
    for i in range(args.steps):
        flush_l2(i)
        step()
    torch.cuda.synchronize(dev)
    prof = V.v4moe_profile_read()
    V.v4moe_profile_enable(False)
    pk = peaks()
    flops = 2.0 * T * G * N * K
    gemm_ms = prof.get("lin_gemm", (0.0, 1))[0] / max(prof.get("lin_gemm", (0.0, 1))[1], 1)
    achieved = flops / (gemm_ms / 1e3) / 1e12 if gemm_ms > 0 else 0.0
    lin_bytes = G * (N * K + 4 * N + 2 * T * K + 2 * T * N)
    line = {"metric": LINEAR_METRIC, "value": T * world / (ms_step / 1e3), "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": args.workload, "T": T, "G": G, "N": N, "K": K,
                       "weights": "int8 per output channel + fp32 scales", "parallelism": f"replicas{world}",
                       "l2": "flushed between timed steps (512 MiB write, then 256 MiB read)"},
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": pk["bf16"], "unit": "TFLOP/s",
                         "frac": achieved / pk["bf16"], "peak_src": pk["src"], "kernel": "lin_gemm",
                         "kernel_ms": gemm_ms, "algorithmic_per_launch": flops,
                         "traffic": recorded_traffic("lin_gemm", args.workload)},
            "layer_roofline": {"algorithmic_flops": flops, "algorithmic_bytes": lin_bytes,
                               "roofline_ms": max(flops / (pk["bf16"] * 1e12), lin_bytes / (pk["hbm"] * 1e9)) * 1e3},
            "kernels": {k: {"ms_per_launch": v[0] / max(v[1], 1), "launches_per_step": v[1] / args.steps}
                        for k, v in sorted(prof.items(), key=lambda kv: -kv[1][0])},
            "e2e": {"value": T * world / (e2e_ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": int(T * G * K * 2),
                    "d2h_bytes_per_step": int(T * G * N * 2)},
            "gpu_launches": int(launches), "clocks": clk}
    line["layer_roofline"]["frac"] = line["layer_roofline"]["roofline_ms"] / ms_step
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle as O
        rows, reps, t0 = [0, 1], 0, time.perf_counter()
        while time.perf_counter() - t0 < args.cpu_seconds:
            O.linear_w8a16_grouped(x_bits, q, sc, G, rows=rows)
            reps += 1
        el = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": reps * len(rows) / el, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                                "sample": f"{reps} x {len(rows)} token rows of {args.workload}, {el:.1f} s single-threaded fp64"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    close_ranks(world)


def workload_config(wl, world):
    return {"workload": wl.name, "T": wl.T, "H": wl.H, "I": wl.I, "E": wl.E, "k": wl.k,
            "shared_inter": wl.Is, "routing": wl.routing, "global_batch": wl.T * world,
            "parallelism": f"replicas{world}",
            "l2": "flushed between timed steps (512 MiB write, then 256 MiB read)",
            "weights": "MXFP4 routed (E2M1 + E8M0/32), int8 shared, bf16 gate"}


class Bench:
    """Device state shared by the workloads: the L2 flush buffers, the stream,
    one layer object per weight set (the full-size workloads share theirs)."""

    def __init__(self, dev, world, args):
        import torch
        self.torch, self.dev, self.world, self.args = torch, dev, world, args
        self.stream = torch.cuda.current_stream(dev)
        self.flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        self.clean = torch.ones(L2_CLEAN_BYTES // 4, dtype=torch.float32, device=dev)
        self.layers = {}
        self.weights = {}

    def flush_l2(self, i):
        # Write a buffer larger than L2, then read another one: the timed step
        # starts with no useful data in L2 and no dirty lines left to write back.
        self.flush.fill_(i & 0xFF)
        self.clean.sum()

    def inputs(self, wl):
        import inputs as IN
        from mxfp4_routed_expert_v4moe_b200 import MoELayer
        key = (wl.H, wl.I, wl.E, wl.k, wl.Is, wl.w_std, wl.gate_std, wl.seed)
        if key not in self.weights:
            self.weights[key] = IN.make_weights(wl)
        li = IN.make_layer_inputs(wl, weights=self.weights[key])
        if key not in self.layers:
            self.layers[key] = MoELayer.from_host(li, device=self.dev)
        return li, self.layers[key]

    def measure(self, wl, li, layer):
        """Timed steps (inputs resident), the end-to-end pass (pinned host x in,
        out back) and the per-kernel pass of one workload -> result dict."""
        import mxfp4_routed_expert_v4moe_b200 as V
        torch, dev, args, stream = self.torch, self.dev, self.args, self.stream
        x = torch.from_numpy(li.x).view(torch.bfloat16).to(dev)
        bias = None if li.bias is None else torch.from_numpy(li.bias).to(dev)
        tok = None if li.token_ids is None else torch.from_numpy(li.token_ids).to(dev)
        tab = None if li.tid2eid is None else torch.from_numpy(li.tid2eid).to(dev)

        def step():
            return layer(x, bias, tok, tab)

        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize(dev)
        acc = algorithmic(wl, layer.buffers(wl.T)["topk_ids"].cpu().numpy(), li.token_ids)

        # ---- timed region: K steps, L2 flushed between steps ----------------
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        barrier(self.world)
        torch.cuda.synchronize(dev)
        launches0 = V.v4moe_launch_count()
        for i in range(args.steps):
            self.flush_l2(i)
            evs[i][0].record(stream)
            step()
            evs[i][1].record(stream)
        torch.cuda.synchronize(dev)
        launches = V.v4moe_launch_count() - launches0
        barrier(self.world)
        ms_total = sum(a.elapsed_time(b) for a, b in evs)

        # ---- end to end through the public API: pinned host in, host out ----
        x_host = torch.from_numpy(li.x).view(torch.bfloat16).pin_memory()
        tok_host = None if li.token_ids is None else torch.from_numpy(li.token_ids).pin_memory()
        out_host = torch.empty((wl.T, wl.H), dtype=torch.bfloat16).pin_memory()
        x_dev = torch.empty_like(x)
        tok_dev = None if tok is None else torch.empty_like(tok)
        e2e_evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(args.steps)]
        for i in range(args.steps):
            self.flush_l2(i)
            e2e_evs[i][0].record(stream)
            x_dev.copy_(x_host, non_blocking=True)
            if tok_dev is not None:
                tok_dev.copy_(tok_host, non_blocking=True)
            out = layer(x_dev, bias, tok_dev, tab)
            out_host.copy_(out, non_blocking=True)
            e2e_evs[i][1].record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = sum(a.elapsed_time(b) for a, b in e2e_evs)

        # ---- per-kernel timing pass (events around every kernel) ------------
        V.v4moe_profile_reset()
        V.v4moe_profile_enable(True)
        for i in range(args.steps):
            self.flush_l2(i)
            step()
        torch.cuda.synchronize(dev)
        prof = V.v4moe_profile_read()
        V.v4moe_profile_enable(False)

        ms_total, e2e_ms = max_over_ranks([ms_total, e2e_ms], self.world, dev)
        ms_step = ms_total / args.steps
        tokens_total = wl.T * self.world
        pk = peaks()
        decode = wl.T <= 64
        # dominant kernel = most device time in the profiled pass
        dom_name, (dom_ms, dom_n) = max(prof.items(), key=lambda kv: kv[1][0]) if prof else ("none", (0.0, 1))
        kind = kernel_kind(dom_name)
        per_launch_s = dom_ms / max(dom_n, 1) / 1e3
        steps_per_launch = max(dom_n, 1) / args.steps
        if decode or kind is None:
            alg = acc["kernel_bytes"].get(kind, acc["step_bytes"]) / steps_per_launch
            achieved = alg / per_launch_s / 1e9 if per_launch_s > 0 else 0.0
            roof = {"bound": "hbm", "achieved": achieved, "peak": pk["hbm"], "unit": "GB/s",
                    "frac": achieved / pk["hbm"], "peak_src": pk["src"]}
        else:
            alg = acc["kernel_flops"][kind] / steps_per_launch
            achieved = alg / per_launch_s / 1e12 if per_launch_s > 0 else 0.0
            roof = {"bound": "tensor", "achieved": achieved, "peak": pk["bf16"], "unit": "TFLOP/s",
                    "frac": achieved / pk["bf16"], "peak_src": pk["src"]}
        roof.update(kernel=dom_name, kernel_ms=dom_ms / max(dom_n, 1), algorithmic_per_launch=alg,
                    traffic=recorded_traffic(dom_name, wl.name))
        step_s = ms_step / 1e3
        t_hbm = acc["step_bytes"] / (pk["hbm"] * 1e9)
        t_tc = acc["step_flops"] / (pk["bf16"] * 1e12)
        layer_roof_s = max(t_hbm, t_tc)
        cfg = workload_config(wl, self.world)
        cfg["experts_hit"] = acc["n_hit"]
        return {"ms_per_step": ms_step, "value": tokens_total / step_s, "config": cfg,
                "layer_roofline": {"algorithmic_bytes": acc["step_bytes"],
                                   "algorithmic_flops": acc["step_flops"],
                                   "bound": "hbm" if t_hbm >= t_tc else "tensor",
                                   "roofline_ms": layer_roof_s * 1e3,
                                   "frac": layer_roof_s / step_s,
                                   "achieved_GBps": acc["step_bytes"] / step_s / 1e9,
                                   "achieved_TFLOPs": acc["step_flops"] / step_s / 1e12},
                "roofline": roof,
                "kernels": {k: {"ms_per_launch": v[0] / max(v[1], 1), "launches_per_step": v[1] / args.steps}
                            for k, v in sorted(prof.items(), key=lambda kv: -kv[1][0])},
                "e2e": {"value": tokens_total / (e2e_ms / args.steps / 1e3), "unit": "tokens/s",
                        "h2d_bytes_per_step": int(x_host.numel() * 2 +
                                                  (0 if tok_host is None else tok_host.numel() * 4)),
                        "d2h_bytes_per_step": int(out_host.numel() * 2)},
                "gpu_launches": int(launches)}


def free_port():
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        return sk.getsockname()[1]


def spawn_command(n, argv):
    """The torch.distributed.run command that starts n ranks of this script
    (one process per GPU) with the same arguments."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
            "--master-addr", "127.0.0.1", "--master-port", str(free_port()),
            os.path.abspath(__file__), *argv]


def check_ranks(args):
    """The rank plumbing alone, on the CPU over gloo: every rank joins, the
    per-rank numbers reduce to their maximum, rank 0 prints the count. No
    measurement (nothing of the layer runs)."""
    import torch
    world, rank, _ = rank_env()
    dev = torch.device("cpu")
    init_ranks(world, dev, backend="gloo")
    barrier(world)
    got = max_over_ranks([float(rank + 1)], world, dev)
    if rank == 0:
        print(json.dumps({"check_ranks": True, "n_gpus": world, "ranks_joined": int(got[0])}), flush=True)
    close_ranks(world)


def main():
    args = parse()
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ and args.impl == "ours":
        # one process per GPU: start the ranks under torch.distributed.run
        return subprocess.call(spawn_command(args.gpus, sys.argv[1:]))
    if args.check_ranks:
        return check_ranks(args)
    if args.workload in LINEAR_WORKLOADS:
        if args.impl == "reference":
            return run_reference_linear(args)
        return run_linear(args)
    if args.impl == "reference":
        return run_reference(args)
    import torch

    import inputs as IN

    world, rank, local = rank_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    init_ranks(world, dev)
    B = Bench(dev, world, args)
    head_name = args.workload or HEADLINE
    # the headline workload; with no --workload, every workload of the layer
    # beside it (same weights for the full-size ones)
    others = [] if args.workload else [w for w in IN.WORKLOAD_ORDER if w != head_name]

    uuid = None
    try:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    wl = IN.WORKLOADS[head_name]
    li, layer = B.inputs(wl)
    clocks = ClockSampler(uuid)
    clocks.start()
    r = B.measure(wl, li, layer)
    clk = clocks.stop()

    line = {"metric": METRIC, "value": r["value"], "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": r["config"], "layer_roofline": r["layer_roofline"],
            "roofline": r["roofline"], "kernels": r["kernels"], "e2e": r["e2e"],
            "gpu_launches": r["gpu_launches"], "clocks": clk}
    if others:
        block = {}
        for name in others:
            wlo = IN.WORKLOADS[name]
            lio, layo = B.inputs(wlo)
            ck = ClockSampler(uuid)
            ck.start()
            ro = B.measure(wlo, lio, layo)
            ro["clocks"] = ck.stop()
            block[name] = ro
        block[head_name] = {k: r[k] for k in ("ms_per_step", "value", "config", "layer_roofline", "roofline",
                                               "kernels", "e2e", "gpu_launches")}
        block[head_name]["clocks"] = clk
        line["workloads"] = {n: block[n] for n in IN.WORKLOAD_ORDER if n in block}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wl, li, args.cpu_seconds)
    if rank == 0:
        print(json.dumps(line), flush=True)
    close_ranks(world)


if __name__ == "__main__":
    sys.exit(main() or 0)
