"""Grouped GEMM kernel times with uniform groups against ragged ones, and cuBLAS FP8 beside them.

Runs the split FFN entry point (moe_grouped_ffn_fp8) on a DeepSeek-V3-sized expert (d = 7168,
F = 2048) with 32 experts and caller-made groups: every group exactly 256, 512 or 1024 rows (all
tiles full), and multinomial counts around 256 (ragged, like a routed batch). Kernel times come
from the CUDA profiler (torch.profiler, median of 5 calls). For scale, cuBLAS's FP8 GEMM
(torch._scaled_mm) of the same FLOPs as the 256-row case, once as one dense GEMM and once per
expert. Synthetic random weights; the outputs are not checked here (the tests do that).

    python -m fp8_moe_layer_b200.gemm_uniform_probe
"""
import statistics

import torch
from torch.profiler import profile, ProfilerActivity
from fp8_moe_layer_b200 import ops

D, F, E = 7168, 2048, 32


def _weights(dev):
    g = torch.Generator(device=dev)
    g.manual_seed(0)
    w13 = (torch.randn(E, 2 * F, D, device=dev, generator=g) * 20).clamp(-448, 448)
    w2 = (torch.randn(E, D, F, device=dev, generator=g) * 20).clamp(-448, 448)
    return (w13.to(torch.float8_e4m3fn), torch.full((E, 2 * F), 1e-3, device=dev),
            w2.to(torch.float8_e4m3fn), torch.full((E, D), 1e-3, device=dev), g)


def case(name, counts, T, k_max, wts, dev="cuda"):
    """Kernel medians of moe_grouped_ffn_fp8 with group sizes `counts` (one per expert)."""
    w13, w13s, w2, w2s, g = wts
    counts = torch.tensor(counts, dtype=torch.int64)
    offs = torch.zeros(E + 1, dtype=torch.int32)
    offs[1:] = torch.cumsum(counts, 0).to(torch.int32)
    R = int(offs[-1])
    assert R <= T * k_max
    perm = (torch.arange(R, dtype=torch.int32) % T).to(dev)
    offs = offs.to(dev)
    h = torch.randn(T, D, device=dev, generator=g).to(torch.bfloat16)
    ws = ops.alloc_workspace(ops.dims(T, D, E, F, k_max), dev)
    run = lambda: ops.moe_grouped_ffn_fp8(h, w13, w13s, w2, w2s, offs, perm, k_max, ws=ws)
    for _ in range(3):
        run()
    torch.cuda.synchronize()
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        for _ in range(5):
            run()
        torch.cuda.synchronize()
    times = {}
    for ev in prof.events():
        if ev.device_type == torch.autograd.DeviceType.CUDA:
            times.setdefault(ev.name[:60], []).append(ev.device_time_total)
    fl_gu, fl_dn = 2.0 * R * 2 * F * D, 2.0 * R * D * F
    for k, v in sorted(times.items()):
        med = statistics.median(v)
        extra = ""
        if "grouped_gemm_kernel" in k and ", 0," in k:
            extra = f"  gate/up {fl_gu / med / 1e6:.0f} TFLOP/s"
        elif "grouped_gemm_kernel" in k and ", 1," in k:
            extra = f"  down {fl_dn / med / 1e6:.0f} TFLOP/s"
        print(f"{name:6s} {k:60s} n={len(v):3d} median {med:9.1f} us{extra}", flush=True)


def cublas(dev="cuda", w13=None):
    one = torch.ones((), device=dev)
    a = torch.randn(8192, D, device=dev).to(torch.float8_e4m3fn)
    b = torch.randn(2 * F, D, device=dev).to(torch.float8_e4m3fn)
    for _ in range(3):
        torch._scaled_mm(a, b.t(), scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    st, en = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    st.record()
    for _ in range(10):
        torch._scaled_mm(a, b.t(), scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
    en.record()
    torch.cuda.synchronize()
    t = st.elapsed_time(en) / 10 * 1e3
    print(f"cuBLAS dense 8192 x {2 * F} x {D} e4m3: {t:.1f} us, {2.0 * 8192 * 2 * F * D / t / 1e6:.0f} TFLOP/s")
    a2 = torch.randn(256, D, device=dev).to(torch.float8_e4m3fn)
    st.record()
    for _ in range(3):
        for e in range(E):
            torch._scaled_mm(a2, w13[e].t(), scale_a=one, scale_b=one, out_dtype=torch.bfloat16)
    en.record()
    torch.cuda.synchronize()
    t = st.elapsed_time(en) / 3 * 1e3
    print(f"cuBLAS one GEMM per expert, {E} x (256 x {2 * F} x {D}): {t:.1f} us, "
          f"{2.0 * E * 256 * 2 * F * D / t / 1e6:.0f} TFLOP/s")


def main():
    torch.manual_seed(1)
    wts = _weights("cuda")
    case("U256", [256] * E, 1024, 8, wts)
    case("U512", [512] * E, 2048, 8, wts)
    case("U1024", [1024] * E, 4096, 8, wts)
    rag = torch.multinomial(torch.ones(E), 8192, replacement=True).bincount(minlength=E).tolist()
    print("ragged counts", rag)
    case("R256", rag, 1024, 8, wts)
    cublas(w13=wts[0])


if __name__ == "__main__":
    main()
