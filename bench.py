"""Benchmark of the FP8 MoE layer forward on B200: one JSON line on rank 0.

A step is one pass of the whole layer (router, top-k, quantisation, permutation, grouped FP8
FFN, combine) over one batch of synthetic tokens of the Mixtral-8x7B-shaped workload
(d=4096, E=8, F=14336, top-2, T=512 tokens per GPU) through the C ABI entry point moe_forward.

* value: tokens/s over all ranks, device time (CUDA events on the launching stream around each
  step) with every input resident in HBM; L2 flushed (256 MiB write + 256 MiB read) between
  steps, outside the timed events.
* e2e: the same metric with the step's hidden states copied from pinned host memory and the
  output copied back inside the timed region.
* roofline: the dominant kernel (the gate/up GEMM + SwiGLU) timed by events around its launch,
  in a second pass over the same steps with an event before every kernel of the layer.
* cpu_baseline (rank 0, N=1): the CPU oracle timed on a bounded token sample.
* --impl reference: the CPU oracle as the reference arm (no GPU work).
Multi-GPU: independent replicas (one batch per rank, seed = rank), no collective on the path.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "mixtral_T512"
METRIC = "MoE-layer µs and tokens/s at 1 B200; % of HBM (decode) / FP8 TC (prefill) roofline"
FLUSH_BYTES = 256 << 20
# A ~0.2 ms GPU sleep (cycles at ~2 GHz) before each timed step: the host enqueues the step's
# kernels (tens of microseconds of launches) while the GPU sleeps, so the events measure device
# time and not the host's launch rate. The host cost is in the e2e number.
HOST_AHEAD_CYCLES = 400_000
ACTIVE_REASONS = {  # nvidia-smi clocks_event_reasons bitmask
    0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
    0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
    0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clocks_setting"}


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-sample", type=int, default=8, help="tokens in the CPU oracle sample")
    return ap.parse_args()


def dist_env():
    from fp8_moe_layer_b200.replicas import rank_env
    return rank_env()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return dict(hbm_gbs=p["hbm_gbs"], source="of measured")
    return dict(hbm_gbs=6650.0, source="of fallback")


# ------------------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi sampled every 200 ms while the timed region runs."""

    def __init__(self, index: int):
        self.index, self.rows, self.proc = index, [], None

    def __enter__(self):
        q = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={q}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append([c.strip() for c in line.split(",")])

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            self.proc.wait(timeout=5)

    def summary(self):
        if not self.rows:
            return None
        sm, smax, reasons = [], [], set()
        for r in self.rows:
            try:
                sm.append(float(r[0]))
                smax.append(float(r[1]))
                mask = int(r[3], 16)
            except (ValueError, IndexError):
                continue
            for bit, name in ACTIVE_REASONS.items():
                if mask & bit:
                    reasons.add(name)
        if not sm:
            return None
        return dict(sm_mhz=float(np.median(sm)), sm_max_mhz=max(smax), samples=len(sm),
                    reasons=sorted(reasons - {"gpu_idle"}))


# ------------------------------------------------------------------------------ work model
def algorithmic(shape, offsets: np.ndarray):
    """Bytes and flops the method itself must move / compute for one step (counts from the
    step's own routing): every distinct active expert's FP8 weights and scales once, the router
    weights, the bf16 hidden in and y out; flops 6 d F per routed row (+ shared) + 2 T E d."""
    counts = np.diff(offsets[: shape.E + 1])
    active = int((counts > 0).sum()) + (1 if shape.F_shared else 0)
    R = int(offsets[shape.E])
    d, F = shape.d, shape.F
    expert_bytes = 3 * d * F + (2 * F + d) * 4
    B = active * expert_bytes + shape.E * d * 4 + 2 * shape.T * d * 2
    flops = 6 * d * F * (R + (shape.T if shape.F_shared else 0)) + 2 * shape.T * shape.E * d
    # the gate/up kernel alone: its weight bytes, the FP8 rows it reads, the fp32 rows it writes
    rows = R + (shape.T if shape.F_shared else 0)
    g1_bytes = active * (2 * F * d + 2 * F * 4) + rows * (d + 4 + 4 * F + 4)
    return dict(active_experts=active, routed_rows=R, bytes=B, flops=flops, gemm1_bytes=g1_bytes)


def kernel_src_digest() -> str:
    """sha256 (first 16 hex digits) over the sources the grouped GEMM kernels are compiled from."""
    h = hashlib.sha256()
    for name in ("gemm.cu", "common.cuh", "kernels.cuh"):
        with open(os.path.join(ROOT, "fp8_moe_layer_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_tag: str):
    """DRAM bytes per launch from the committed ncu summary, if the kernel source is unchanged
    since it was captured (else None)."""
    path = os.path.join(ROOT, "profiles", f"{kernel_tag}.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    if rec.get("kernel_src_sha256_16") != kernel_src_digest():
        return None
    return rec.get("dram_bytes_per_launch")


# ------------------------------------------------------------------------------ CPU oracle
def cpu_oracle_time(inp, n_tokens: int, seed: int = 0):
    """Time the oracle (as it stands) on a sample of n tokens of this workload on the host."""
    import torch
    from oracle import moe_oracle as O
    s = inp.shape
    rng = np.random.default_rng(seed)
    tokens = np.sort(rng.choice(s.T, size=min(n_tokens, s.T), replace=False))
    hb = inp.hidden.view(torch.int16).numpy().view(np.uint16)
    shared = None
    if s.F_shared:
        shared = (inp.w13_shared.numpy(), inp.w13s_scale.numpy(), inp.w2_shared.numpy(),
                  inp.w2s_scale.numpy())
    t0 = time.perf_counter()
    O.moe_forward(hb, inp.router_w.numpy(),
                  None if inp.router_bias is None else inp.router_bias.numpy(), s.k,
                  None if inp.k_per_token is None else inp.k_per_token.numpy(), inp.w13.numpy(),
                  inp.w13_scale.numpy(), inp.w2.numpy(), inp.w2_scale.numpy(), shared=shared,
                  tokens=tokens, k_max=s.k_max)
    dt = time.perf_counter() - t0
    return len(tokens), dt


def launches_per_step(shape) -> int:
    """Kernels one moe_forward launches for this shape (the library's router and grouping paths:
    fused router for E <= 32, tensor-core router (split + GEMM + top-k) for E > 32 and T >= 64,
    else CUDA-core logits + top-k; one grouping kernel for T*k_max <= 8192, else three)."""
    if shape.E <= 32 and shape.d <= 8192:
        router = 1
    elif shape.T >= 64:
        router = 3
    else:
        router = 2
    permute = 1 if shape.T * shape.k_max <= 8192 else 3
    return router + permute + 5      # gather, gate/up GEMM, requant, down GEMM, combine


def host_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


# ------------------------------------------------------------------------------ arms
def run_reference(args):
    """CPU oracle arm: each step routes the whole batch and runs the FFN of one token."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    from fp8_moe_layer_b200 import inputs as I
    shape = I.WORKLOADS[args.workload]
    inp = I.make_inputs(shape, seed=0)
    times = []
    for i in range(args.warmup + args.steps):
        n, dt = cpu_oracle_time(inp, 1, seed=i)
        if i >= args.warmup:
            times.append(dt / n)
    per_token = float(np.mean(times))
    value = 1.0 / per_token
    sample = (f"per step: routing and grouping of all {shape.T} tokens + the expert FFN and "
              f"combine of 1 token")
    line = dict(metric=METRIC, value=value, unit="tokens/s", n_gpus=args.gpus, steps=args.steps,
                warmup=args.warmup, ms_per_step=per_token * 1e3, higher_is_better=True,
                scaling="weak", vs_baseline=None, dtype="f64", data="synthetic",
                impl="reference",
                config=dict(workload=args.workload, T=shape.T, d=shape.d, E=shape.E, F=shape.F,
                            k=shape.k),
                cpu_baseline=dict(value=value, unit="tokens/s", cores=host_threads(),
                                  kind="oracle", sample=sample),
                e2e=dict(value=value, unit="tokens/s", h2d_bytes_per_step=0,
                         d2h_bytes_per_step=0))
    print(json.dumps(line), flush=True)


def run_ours(args):
    import torch
    import torch.distributed as dist

    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    from fp8_moe_layer_b200 import inputs as I
    from fp8_moe_layer_b200 import ops

    shape = I.WORKLOADS[args.workload]
    from fp8_moe_layer_b200 import replicas
    inp = I.make_inputs(shape, seed=replicas.replica_seed(0, rank), quant_device=f"cuda:{local}")
    layer = ops.MoELayerFP8(inp, device=f"cuda:{local}")
    dev = torch.device(f"cuda:{local}")
    hidden = inp.hidden.to(dev)
    kpt = None if inp.k_per_token is None else inp.k_per_token.to(dev)
    y = torch.empty(shape.T, shape.d, dtype=torch.bfloat16, device=dev)
    # L2 flush between timed steps: write one buffer larger than L2, then read another, so the
    # next step starts with a cold L2 that holds no dirty lines
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_rd = torch.ones(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    for _ in range(args.warmup):
        layer(hidden, kpt, y=y)
    torch.cuda.synchronize(dev)
    if ops.device_status(layer.ws) != ops.MOE_OK:
        raise RuntimeError("device status not ok after warm-up")
    _, dbg = layer(hidden, kpt, debug=True)
    work = algorithmic(shape, dbg["expert_offsets"].cpu().numpy())

    # (a) the step time: events around each moe_forward only (no events between its kernels,
    #     which would serialise the programmatic launches)
    s_start = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    s_end = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clocks:
        for i in range(args.steps):
            flush.fill_(i & 0xFF)                       # evict L2 (outside the timed events)
            flush_rd.sum()
            torch.cuda._sleep(HOST_AHEAD_CYCLES)        # the host enqueues the step meanwhile
            s_start[i].record(stream)
            layer(hidden, kpt, y=y)
            s_end[i].record(stream)
        torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    step_ms = np.array([s_start[i].elapsed_time(s_end[i]) for i in range(args.steps)])
    ms = float(step_ms.mean())

    # (b) per-kernel times: the same steps with an event before every kernel of the layer
    n_ev = ops.NUM_STAGES + 1
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
              for _ in range(args.steps)]
    torch.cuda.synchronize(dev)
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        flush_rd.sum()
        torch.cuda._sleep(HOST_AHEAD_CYCLES)
        layer(hidden, kpt, y=y, stage_events=events[i])
    torch.cuda.synchronize(dev)
    stage_ms = np.array([[events[i][j].elapsed_time(events[i][j + 1]) for j in range(n_ev - 1)]
                         for i in range(args.steps)])

    # e2e: pinned host hidden -> device, layer, y -> pinned host, all inside the events
    h_host = inp.hidden.pin_memory()
    y_host = torch.empty(shape.T, shape.d, dtype=torch.bfloat16).pin_memory()
    e_start = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    e_end = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    h_dev = torch.empty_like(hidden)
    for i in range(args.warmup):
        h_dev.copy_(h_host, non_blocking=True)
        layer(h_dev, kpt, y=y)
        y_host.copy_(y, non_blocking=True)
    torch.cuda.synchronize(dev)
    for i in range(args.steps):
        flush.fill_(i & 0xFF)
        flush_rd.sum()
        e_start[i].record(stream)
        h_dev.copy_(h_host, non_blocking=True)
        layer(h_dev, kpt, y=y)
        y_host.copy_(y, non_blocking=True)
        e_end[i].record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = float(np.mean([e_start[i].elapsed_time(e_end[i]) for i in range(args.steps)]))

    ms, e2e_ms = replicas.max_over_ranks([ms, e2e_ms], device=dev)
    total_tokens = shape.T * world
    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return

    pk = peaks()
    g1_ms = float(stage_ms[:, 4].mean())
    g1_gbs = work["gemm1_bytes"] / (g1_ms * 1e-3) / 1e9
    layer_gbs = work["bytes"] / (ms * 1e-3) / 1e9
    stages = {name: round(float(stage_ms[:, j].mean()) * 1e3, 2)
              for j, name in enumerate(ops.STAGE_NAMES)}
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        n, dt = cpu_oracle_time(inp, args.cpu_sample)
        cpu = dict(value=n / dt, unit="tokens/s", cores=host_threads(), kind="oracle",
                   sample=f"{n} of {shape.T} tokens through the FFN and combine; routing and "
                          f"grouping of all {shape.T} tokens ({dt:.1f} s)")
    line = dict(
        metric=METRIC, value=replicas.aggregate_tokens_per_s(shape.T, world, ms), unit="tokens/s", n_gpus=world,
        steps=args.steps, warmup=args.warmup, ms_per_step=ms, us_per_layer=ms * 1e3,
        higher_is_better=True, scaling="weak", vs_baseline=None, dtype="fp8_e4m3",
        data="synthetic (seeded, random-init weights of the layer shape)",
        config=dict(workload=args.workload, T=shape.T, d=shape.d, E=shape.E, F=shape.F,
                    k=shape.k, F_shared=shape.F_shared, parallelism=f"replicas x{world}",
                    l2="flushed between timed steps (256 MiB write + 256 MiB read, outside the events)"),
        roofline=dict(bound="hbm", kernel="gemm_gateup_swiglu", achieved=g1_gbs,
                      peak=pk["hbm_gbs"], unit="GB/s", frac=g1_gbs / pk["hbm_gbs"],
                      traffic=ncu_traffic(f"gemm_gateup_{args.workload}"),
                      algorithmic_bytes=work["gemm1_bytes"], launch_us=g1_ms * 1e3,
                      peak_source=pk["source"]),
        layer_roofline=dict(bound="hbm", achieved=layer_gbs, peak=pk["hbm_gbs"], unit="GB/s",
                            frac=layer_gbs / pk["hbm_gbs"], algorithmic_bytes=work["bytes"],
                            active_experts=work["active_experts"],
                            routed_rows=work["routed_rows"], flops=work["flops"]),
        stage_us=stages,
        e2e=dict(value=replicas.aggregate_tokens_per_s(shape.T, world, e2e_ms), unit="tokens/s",
                 h2d_bytes_per_step=shape.T * shape.d * 2, d2h_bytes_per_step=shape.T * shape.d * 2),
        gpu_launches=launches_per_step(shape) * args.steps,
        clocks=clocks.summary(),
        cpu_baseline=cpu,
    )
    print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
