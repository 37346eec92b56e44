"""Benchmark of the FP8 MoE layer forward on B200: one JSON line on rank 0.

A step is one pass of the whole layer (router, top-k, quantisation, permutation, grouped FP8
FFN, combine) over one batch of synthetic tokens through the C ABI entry point moe_forward. The
default workload is the largest configuration that fits one GPU: the DeepSeek-V3-shaped layer
(d=7168, 256 routed experts + 1 shared expert, F=2048, top-8, Zipf(1.2) router skew, T=8192
tokens per GPU, 11.6 GB of FP8 expert weights).

* value: tokens/s over all ranks, device time (CUDA events on the launching stream around each
  step) with every input resident in HBM; L2 flushed (256 MiB write + 256 MiB read) between
  steps, outside the timed events. p10 / p50 / p90 of the step times beside the mean.
* e2e: the same metric with the step's hidden states copied from pinned host memory and the
  output copied back inside the timed region.
* roofline: the dominant kernel (the gate/up GEMM + SwiGLU) timed by events around its launch, in
  a second pass over the same steps with an event before every kernel of the layer, against the
  FP8 tensor-core peak (tensor-bound workloads) or the HBM copy bandwidth (bytes-bound ones).
* layer_roofline: t_roof = max(B_alg / BW, F_alg / P_fp8) over the measured step time, against
  the measured and the nominal (8 TB/s, 4.5 PFLOP/s) denominators.
* l2_cold_check: the same layer timed with 2 to 8 copies of its weights used in turn and no L2
  flush (median), beside the flushed median: a cross-check that the flush gives cold-L2 times.
* other_configs: every other workload of the layer timed the same way (shorter), each with the
  same rotated-copies cross-check.
* cpu_baseline (rank 0, N=1): the CPU oracle's whole-layer time, estimated from a bounded sample.
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

WORKLOAD = "deepseek_T8192"
METRIC = "MoE-layer µs and tokens/s at 1 B200; % of HBM (decode) / FP8 TC (prefill) roofline"
FLUSH_BYTES = 256 << 20
# A ~1 ms GPU sleep (cycles at ~2 GHz) before each timed step: the host enqueues the step's
# kernels (tens to hundreds of microseconds of launches and argument set-up) while the GPU
# sleeps, so the events measure device time and not the host's launch rate. The host cost is in
# the e2e number.
HOST_AHEAD_CYCLES = 2_000_000
# nominal B200 figures: HBM3e bandwidth, dense FP8 tensor-core throughput; FP8 / bf16 ratio
NOMINAL_HBM_GBS = 8000.0
NOMINAL_FP8_TFLOPS = 4500.0
FP8_PER_BF16 = 2.0
ACTIVE_REASONS = {  # nvidia-smi clocks_event_reasons bitmask
    0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
    0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
    0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clocks_setting"}
GATEUP_STAGE = 4      # stage index of the gate/up GEMM + SwiGLU in moe_forward's stage events


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-other-configs", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=15.0,
                    help="seconds of oracle work in the CPU baseline's sample")
    return ap.parse_args()


def dist_env():
    from fp8_moe_layer_b200.replicas import rank_env
    return rank_env()


def peaks():
    """Roofline denominators: MEASURED_PEAKS.json (copy bandwidth; cuBLAS bf16 burst and
    sustained, times the nominal FP8 / bf16 ratio of 2), else fallback figures measured earlier on
    B200s (6650 GB/s copy; 1590 / 1400 TFLOP/s bf16 burst / sustained)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        burst = float(p.get("bf16_tflops", 1590.0))
        sust = float(p.get("bf16_tflops_sustained", burst))
        return dict(hbm_gbs=float(p["hbm_gbs"]), fp8_tflops=FP8_PER_BF16 * sust,
                    fp8_tflops_burst=FP8_PER_BF16 * burst, source="of measured")
    return dict(hbm_gbs=6650.0, fp8_tflops=FP8_PER_BF16 * 1400.0,
                fp8_tflops_burst=FP8_PER_BF16 * 1590.0, source="of fallback")


def fp8_cublas_tflops(n: int = 8192, seconds: float = 1.0) -> float:
    """cuBLAS e4m3 GEMM (torch._scaled_mm, n^3) looped for about `seconds`: context for the FP8
    peak under the same power and clock state as the layer."""
    import torch
    a = torch.randn(n, n, device="cuda").to(torch.float8_e4m3fn)
    b = torch.randn(n, n, device="cuda").to(torch.float8_e4m3fn)
    one = torch.tensor(1.0, device="cuda")
    mm = lambda: torch._scaled_mm(a, b.t(), scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
    for _ in range(3):
        mm()
    torch.cuda.synchronize()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    reps = 20
    s.record()
    for _ in range(reps):
        mm()
    e.record()
    torch.cuda.synchronize()
    reps = max(reps, int(reps * seconds / max(s.elapsed_time(e) * 1e-3, 1e-6)))
    s.record()
    for _ in range(reps):
        mm()
    e.record()
    torch.cuda.synchronize()
    return 2.0 * n ** 3 * reps / (s.elapsed_time(e) * 1e-3) / 1e12


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
        sm, smax, power, reasons = [], [], [], set()
        for r in self.rows:
            try:
                sm.append(float(r[0]))
                smax.append(float(r[1]))
                power.append(float(r[2]))
                mask = int(r[3], 16)
            except (ValueError, IndexError):
                continue
            for bit, name in ACTIVE_REASONS.items():
                if mask & bit:
                    reasons.add(name)
        if not sm:
            return None
        return dict(sm_mhz=float(np.median(sm)), sm_max_mhz=max(smax), samples=len(sm),
                    power_w_median=float(np.median(power)) if power else None,
                    reasons=sorted(reasons - {"gpu_idle"}))


# ------------------------------------------------------------------------------ work model
def algorithmic(shape, offsets: np.ndarray):
    """Bytes and flops the method itself must move / compute for one step (counts from the
    step's own routing): every distinct active expert's FP8 weights and scales once, the router
    weights, the bf16 hidden in and y out; flops 6 d F per routed row (+ shared) + 2 T E d.
    Intermediates are not counted (a fused design keeps them on chip or in L2)."""
    counts = np.diff(offsets[: shape.E + 1])
    active = int((counts > 0).sum()) + (1 if shape.F_shared else 0)
    R = int(offsets[shape.E])
    d, F = shape.d, shape.F
    expert_bytes = 3 * d * F + (2 * F + d) * 4
    B = active * expert_bytes + shape.E * d * 4 + 2 * shape.T * d * 2
    rows = R + (shape.T if shape.F_shared else 0)
    flops = 6 * d * F * rows + 2 * shape.T * shape.E * d
    # the gate/up kernel alone: 4 d F flops per row, the active experts' W13 and its scales
    g1_flops = 4 * d * F * rows
    g1_bytes = active * (2 * F * d + 2 * F * 4)
    return dict(active_experts=active, routed_rows=R, bytes=B, flops=flops, gemm1_flops=g1_flops,
                gemm1_bytes=g1_bytes)


def layer_roofline(work, us, pk):
    """t_roof = max(B / BW, F / P_fp8) over the measured time, for both denominators."""
    def one(bw_gbs, fp8_tflops):
        t_hbm = work["bytes"] / (bw_gbs * 1e9) * 1e6
        t_fp8 = work["flops"] / (fp8_tflops * 1e12) * 1e6
        t_roof = max(t_hbm, t_fp8)
        return dict(t_hbm_us=round(t_hbm, 2), t_fp8_us=round(t_fp8, 2),
                    binds="hbm" if t_hbm >= t_fp8 else "fp8", frac=round(t_roof / us, 4))
    return dict(measured=dict(hbm_gbs=pk["hbm_gbs"], fp8_tflops=pk["fp8_tflops"],
                              **one(pk["hbm_gbs"], pk["fp8_tflops"])),
                nominal=dict(hbm_gbs=NOMINAL_HBM_GBS, fp8_tflops=NOMINAL_FP8_TFLOPS,
                             **one(NOMINAL_HBM_GBS, NOMINAL_FP8_TFLOPS)))


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
def host_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def oracle_layer_seconds(inp, budget_s: float, seed: int = 0, min_experts: int = 1):
    """The CPU oracle's whole-layer wall time on this workload, estimated from a bounded sample.

    Timed as the oracle stands: (a) its routing, top-k, weights, activation quantisation and
    grouping of all T tokens (moe_forward with an empty output-token list); (b) its expert FFN
    of randomly chosen active experts over ALL of their routed rows, until about ``budget_s``
    seconds have been spent, scaled by (active experts / experts timed); (c) the shared expert
    (if any) over a row sample, scaled by rows; (d) its combine of a token sample, scaled by
    tokens. Returns (seconds, description)."""
    import torch
    from oracle import moe_oracle as O
    s = inp.shape
    np_ = lambda t: None if t is None else t.numpy()
    hb = inp.hidden.view(torch.int16).numpy().view(np.uint16)
    w13, s13, w2, s2 = np_(inp.w13), np_(inp.w13_scale), np_(inp.w2), np_(inp.w2_scale)
    t0 = time.perf_counter()
    ref = O.moe_forward(hb, np_(inp.router_w), np_(inp.router_bias), s.k, np_(inp.k_per_token),
                        w13, s13, w2, s2, shared=None, tokens=np.zeros(0, np.int64),
                        k_max=s.k_max)
    t_route = time.perf_counter() - t0
    offsets, perm, xq, xs = ref["offsets"], ref["perm_token"], ref["xq"], ref["x_scale"]
    active = [e for e in range(s.E) if offsets[e + 1] > offsets[e]]
    rng = np.random.default_rng(seed)
    order = rng.permutation(active)
    t_sample, timed = 0.0, 0
    for e in order:
        tok = perm[offsets[e]:offsets[e + 1]]
        t0 = time.perf_counter()
        O.expert_ffn(xq[tok], xs[tok], w13[e], s13[e], w2[e], s2[e])
        t_sample += time.perf_counter() - t0
        timed += 1
        if timed >= min_experts and t_sample >= budget_s:
            break
    t_ffn = t_sample * len(active) / timed
    t_shared, n_sh = 0.0, 0
    if s.F_shared:
        n_sh = min(s.T, 512)
        tok = np.sort(rng.choice(s.T, size=n_sh, replace=False))
        t0 = time.perf_counter()
        O.expert_ffn(xq[tok], xs[tok], np_(inp.w13_shared), np_(inp.w13s_scale),
                     np_(inp.w2_shared), np_(inp.w2s_scale))
        t_shared = (time.perf_counter() - t0) * s.T / n_sh
    n_c = min(s.T, 1024)
    tok = np.sort(rng.choice(s.T, size=n_c, replace=False))
    rows = {int(r): np.zeros(s.d) for t in tok for r in ref["inv_row"][t] if r >= 0}
    t0 = time.perf_counter()
    O.combine(rows, ref["topk_w"], ref["inv_row"], ref["k_t"], tok)
    t_comb = (time.perf_counter() - t0) * s.T / n_c
    total = t_route + t_ffn + t_shared + t_comb
    desc = (f"extrapolated: routing/top-k/quantisation/grouping of all {s.T} tokens timed "
            f"({t_route:.1f} s); expert FFN of {timed} of {len(active)} active experts over all "
            f"their rows timed ({t_sample:.1f} s) and scaled by {len(active)}/{timed}"
            + (f"; shared expert on {n_sh} of {s.T} rows scaled by rows" if s.F_shared else "")
            + f"; combine of {n_c} tokens scaled by tokens")
    return total, desc


# ------------------------------------------------------------------------------ arms
def run_reference(args):
    """CPU oracle arm: each step estimates the oracle's whole-layer time from a bounded sample
    (routing of all tokens + one expert's FFN over all its rows, scaled)."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    from fp8_moe_layer_b200 import inputs as I
    shape = I.WORKLOADS[args.workload]
    inp = I.make_inputs(shape, seed=0)
    times, desc = [], ""
    for i in range(args.warmup + args.steps):
        sec, desc = oracle_layer_seconds(inp, budget_s=0.0, seed=i, min_experts=1)
        if i >= args.warmup:
            times.append(sec)
    per_layer = float(np.mean(times))
    value = shape.T / per_layer
    line = dict(metric=METRIC, value=value, unit="tokens/s", n_gpus=args.gpus, steps=args.steps,
                warmup=args.warmup, ms_per_step=per_layer * 1e3, higher_is_better=True,
                scaling="weak", vs_baseline=None, dtype="f64", data="synthetic",
                impl="reference",
                config=dict(workload=args.workload, T=shape.T, d=shape.d, E=shape.E, F=shape.F,
                            k=shape.k, F_shared=shape.F_shared),
                cpu_baseline=dict(value=value, unit="tokens/s", cores=host_threads(),
                                  kind="oracle", sample="per step: " + desc),
                e2e=dict(value=value, unit="tokens/s", h2d_bytes_per_step=0,
                         d2h_bytes_per_step=0))
    print(json.dumps(line), flush=True)


def _timed_steps(layer, hidden, kpt, y, steps, flush, flush_rd, stream, stage_events=None):
    """Device time (ms) of each step: CUDA events around moe_forward only, L2 flushed and the
    host ahead of the GPU before each step."""
    import torch
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
    for i in range(steps):
        flush.fill_(i & 0xFF)                       # evict L2 (outside the timed events)
        flush_rd.sum()
        torch.cuda._sleep(HOST_AHEAD_CYCLES)        # the host enqueues the step meanwhile
        starts[i].record(stream)
        layer(hidden, kpt, y=y, stage_events=None if stage_events is None else stage_events[i])
        ends[i].record(stream)
    torch.cuda.synchronize()
    return np.array([starts[i].elapsed_time(ends[i]) for i in range(steps)])


L2_BYTES = 126 << 20


def rotated_us(layer, hidden, kpt, y, touched_bytes, steps, stream):
    """Cross-check of the L2-flush timing: µs / layer (median) with R copies of the layer's weights
    used in turn and no flush, R chosen so that the weights the other copies touch between two
    uses of one copy exceed twice the L2 (at most 8 copies). Returns (us, R)."""
    import torch
    from fp8_moe_layer_b200 import ops
    R = int(min(8, max(2, np.ceil(2 * L2_BYTES / max(touched_bytes, 1)) + 1)))
    cp = lambda t: None if t is None else t.clone()
    reps = [(layer.router_w, layer.w13, layer.w13_scale, layer.w2, layer.w2_scale, layer.shared)]
    for _ in range(R - 1):
        reps.append((cp(layer.router_w), cp(layer.w13), cp(layer.w13_scale), cp(layer.w2),
                     cp(layer.w2_scale),
                     None if layer.shared is None else tuple(cp(t) for t in layer.shared)))
    s = layer.shape
    run = lambda r: ops.moe_forward(hidden, r[0], layer.router_bias, s.k, kpt, r[1], r[2], r[3],
                                    r[4], s.k_max, shared=r[5], ws=layer.ws, y=y)
    for i in range(2 * R):
        run(reps[i % R])
    n = max(steps, 2 * R)
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(n)]
    for i in range(n):
        torch.cuda._sleep(HOST_AHEAD_CYCLES)
        starts[i].record(stream)
        run(reps[i % R])
        ends[i].record(stream)
    torch.cuda.synchronize()
    us = float(np.median([starts[i].elapsed_time(ends[i]) for i in range(n)])) * 1e3
    del reps
    torch.cuda.empty_cache()
    return us, R


def other_configs(main_name, main_layer, args, flush, flush_rd, stream, pk):
    """Every other workload of the layer: µs / layer (median of the steps) and its roofline
    fractions. Workloads of one layer shape share its weights (they differ in T only)."""
    import torch
    from fp8_moe_layer_b200 import inputs as I
    from fp8_moe_layer_b200 import ops
    fams = {}
    for name, s in I.WORKLOADS.items():
        if name != "tiny_T16":
            fams.setdefault(name.rsplit("_T", 1)[0], []).append(s)
    out = []
    for fam, shapes in fams.items():
        big = max(shapes, key=lambda s: s.T)
        if big.name == main_name:
            layer = main_layer
        else:
            inp = I.make_inputs(big, seed=0, quant_device="cuda")
            layer = ops.MoELayerFP8(inp, device="cuda")
            del inp
        for s in sorted(shapes, key=lambda s: s.T):
            if s.name == main_name:
                continue
            h = I.make_hidden(s, 0).cuda()
            kpt = I.make_k_per_token(s, 0)
            kpt = None if kpt is None else kpt.cuda()
            y = torch.empty(s.T, s.d, dtype=torch.bfloat16, device="cuda")
            for _ in range(3):
                layer(h, kpt, y=y)
            _, dbg = layer(h, kpt, debug=True)
            work = algorithmic(s, dbg["expert_offsets"].cpu().numpy())
            ms = _timed_steps(layer, h, kpt, y, 10, flush, flush_rd, stream)
            us = float(np.median(ms)) * 1e3
            lr = layer_roofline(work, us, pk)
            us_rot, reps = rotated_us(layer, h, kpt, y, work["bytes"], 10, stream)
            out.append(dict(workload=s.name, T=s.T, us_per_layer=round(us, 2),
                            tokens_per_s=round(s.T / (us * 1e-6)),
                            active_experts=work["active_experts"],
                            frac_measured=lr["measured"]["frac"],
                            binds=lr["measured"]["binds"], frac_nominal=lr["nominal"]["frac"],
                            us_weights_rotated=round(us_rot, 2), weight_copies=reps))
            if ops.device_status(layer.ws) != ops.MOE_OK:
                raise RuntimeError(f"device status not ok on {s.name}")
        if layer is not main_layer:
            del layer
            torch.cuda.empty_cache()
    return out


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
    from fp8_moe_layer_b200 import replicas

    shape = I.WORKLOADS[args.workload]
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
    #     which would serialise the programmatic launches); the library's own launch counter
    #     counts its kernels in the timed region
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    n0 = ops.kernel_launch_count()
    with ClockSampler(local) as clocks:
        step_ms = _timed_steps(layer, hidden, kpt, y, args.steps, flush, flush_rd, stream)
    launches = ops.kernel_launch_count() - n0
    if world > 1:
        dist.barrier()
    ms = float(step_ms.mean())

    # (b) per-kernel times: the same steps with an event before every kernel of the layer
    n_ev = ops.NUM_STAGES + 1
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(n_ev)]
              for _ in range(args.steps)]
    _timed_steps(layer, hidden, kpt, y, args.steps, flush, flush_rd, stream, stage_events=events)
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
    if ops.device_status(layer.ws) != ops.MOE_OK:
        raise RuntimeError("device status not ok after the timed steps")

    ms, e2e_ms = replicas.max_over_ranks([ms, e2e_ms], device=dev)
    if rank != 0:
        if world > 1:
            dist.destroy_process_group()
        return

    pk = peaks()
    us = ms * 1e3
    g1_ms = float(stage_ms[:, GATEUP_STAGE].mean())
    g1_tflops = work["gemm1_flops"] / (g1_ms * 1e-3) / 1e12
    g1_gbs = work["gemm1_bytes"] / (g1_ms * 1e-3) / 1e9
    lr = layer_roofline(work, us, pk)
    tensor_bound = work["gemm1_flops"] / (pk["fp8_tflops"] * 1e12) >= \
        work["gemm1_bytes"] / (pk["hbm_gbs"] * 1e9)
    if tensor_bound:
        roof = dict(bound="tensor", achieved=g1_tflops, peak=pk["fp8_tflops"], unit="TFLOP/s",
                    frac=g1_tflops / pk["fp8_tflops"])
    else:
        roof = dict(bound="hbm", achieved=g1_gbs, peak=pk["hbm_gbs"], unit="GB/s",
                    frac=g1_gbs / pk["hbm_gbs"])
    roof.update(traffic=ncu_traffic(f"gemm_gateup_{args.workload}"), kernel="gemm_gateup_swiglu",
                launch_us=round(g1_ms * 1e3, 2), algorithmic_flops=work["gemm1_flops"],
                algorithmic_bytes=work["gemm1_bytes"],
                peak_source=pk["source"] + (" (cuBLAS bf16 sustained x 2, the nominal FP8/bf16 "
                                            "ratio)" if tensor_bound else " (copy bandwidth)"),
                hbm_frac=round(g1_gbs / pk["hbm_gbs"], 4),
                tensor_frac=round(g1_tflops / pk["fp8_tflops"], 4),
                tensor_frac_of_burst=round(g1_tflops / pk["fp8_tflops_burst"], 4),
                tensor_frac_nominal=round(g1_tflops / NOMINAL_FP8_TFLOPS, 4))
    stages = {name: round(float(stage_ms[:, j].mean()) * 1e3, 2)
              for j, name in enumerate(ops.STAGE_NAMES)}
    # the L2-flush timing cross-checked by rotating copies of the weights instead (one GPU)
    l2_check = None
    if world == 1:
        us_rot, copies = rotated_us(layer, hidden, kpt, y, work["bytes"], args.steps, stream)
        l2_check = dict(weight_copies=copies, us_per_layer_median=round(us_rot, 2),
                        us_per_layer_median_flushed=round(float(np.median(step_ms)) * 1e3, 2))
    others = None
    if world == 1 and not args.no_other_configs:
        others = other_configs(args.workload, layer, args, flush, flush_rd, stream, pk)
    fp8_cublas = fp8_cublas_tflops() if world == 1 else None
    cpu = None
    if world == 1 and not args.no_cpu_baseline:
        sec, desc = oracle_layer_seconds(inp, budget_s=args.cpu_budget)
        cpu = dict(value=shape.T / sec, unit="tokens/s", cores=host_threads(), kind="oracle",
                   sample=desc, seconds_per_layer=round(sec, 1))
    line = dict(
        metric=METRIC, value=replicas.aggregate_tokens_per_s(shape.T, world, ms), unit="tokens/s",
        n_gpus=world, steps=args.steps, warmup=args.warmup, ms_per_step=ms, us_per_layer=us,
        us_p10_p50_p90=[round(float(np.percentile(step_ms, q)) * 1e3, 2) for q in (10, 50, 90)],
        higher_is_better=True, scaling="weak", vs_baseline=None, dtype="fp8_e4m3",
        data="synthetic (seeded, random-init weights of the layer shape)",
        config=dict(workload=args.workload, T=shape.T, d=shape.d, E=shape.E, F=shape.F,
                    k=shape.k, F_shared=shape.F_shared, parallelism=f"replicas x{world}",
                    l2="flushed between timed steps (256 MiB write + 256 MiB read, outside the events)"),
        roofline=roof,
        layer_roofline=dict(lr, algorithmic_bytes=work["bytes"], flops=work["flops"],
                            active_experts=work["active_experts"],
                            routed_rows=work["routed_rows"]),
        fp8_cublas_tflops_same_run=None if fp8_cublas is None else round(fp8_cublas, 1),
        stage_us=stages,
        l2_cold_check=l2_check,
        e2e=dict(value=replicas.aggregate_tokens_per_s(shape.T, world, e2e_ms), unit="tokens/s",
                 h2d_bytes_per_step=shape.T * shape.d * 2, d2h_bytes_per_step=shape.T * shape.d * 2),
        gpu_launches=int(launches),
        clocks=clocks.summary(),
        other_configs=others,
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
