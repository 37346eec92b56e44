"""Where the grouped GEMMs' time goes: per-role wait cycles of the library's role-counter build.

    python -m fp8_moe_layer_b200.role_counters --workloads deepseek_T8192 qwen3_T4096

Builds (if needed) and loads libfp8moe_roles.so (-DMOE_ROLE_COUNTERS, include/moe_testing.h),
runs one layer forward per workload after two warm-up forwards, and prints, per GEMM, the
averages over its CTAs of: cycles from set-up to the end, tiles, cycles the TMA producer waited
for a free stage, cycles the MMA issuer waited for a stage's data and for a free accumulator,
K blocks, and cycles the epilogue waited for an accumulator. clock64 counts SM cycles, so the
fractions do not depend on the clock; the counting itself slows the kernels a little.
"""
from __future__ import annotations

import argparse
import ctypes
import json

import numpy as np
import torch

from . import build as B
from . import inputs as I
from . import ops

MODES = {0: "gate_up_swiglu", 1: "down", 2: "gate_up_ksplit_partials"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--workloads", nargs="+", default=["deepseek_T8192"])
    args = ap.parse_args()
    lib = ops.load_library(B.build(lib=B.LIB_ROLES))
    lib.moe_role_counters_read.argtypes = [ctypes.c_void_p]
    lib.moe_role_counters_read.restype = ctypes.c_int
    lib.moe_role_counters_reset.argtypes = []
    lib.moe_role_counters_reset.restype = ctypes.c_int
    buf = np.zeros((3, 256, 8), dtype=np.uint64)
    for name in args.workloads:
        s = I.WORKLOADS[name]
        inp = I.make_inputs(s, seed=0, quant_device="cuda")
        layer = ops.MoELayerFP8(inp)
        h = inp.hidden.cuda()
        kpt = None if inp.k_per_token is None else inp.k_per_token.cuda()
        run = lambda: ops.moe_forward(h, layer.router_w, layer.router_bias, s.k, kpt, layer.w13,
                                      layer.w13_scale, layer.w2, layer.w2_scale, s.k_max,
                                      shared=layer.shared, ws=layer.ws, lib=lib)
        run()
        run()
        torch.cuda.synchronize()
        if lib.moe_role_counters_reset() != 0:
            raise RuntimeError("moe_role_counters_reset failed")
        run()
        torch.cuda.synchronize()
        if ops.device_status(layer.ws) != ops.MOE_OK:
            raise RuntimeError("device status not ok")
        if lib.moe_role_counters_read(buf.ctypes.data) != 0:
            raise RuntimeError("moe_role_counters_read failed")
        out = {}
        for mode, mname in MODES.items():
            b = buf[mode].astype(np.float64)
            ran = b[:, 5] > 0
            if not ran.any():
                continue
            m = b[ran].mean(axis=0)
            issuers = b[:, 3] > 0                 # CTAs whose MMA thread issued (pair leaders)
            mi = b[issuers].mean(axis=0) if issuers.any() else m
            total = max(m[5], 1.0)
            out[mname] = dict(
                ctas=int(ran.sum()), cycles=round(m[5]), tiles=round(m[6], 1),
                producer_wait_stage=round(m[0] / total, 3),
                mma_wait_data=round(mi[2] / max(mi[5], 1.0), 3),
                mma_wait_accumulator=round(mi[1] / max(mi[5], 1.0), 3),
                mma_cycles_per_kblock=round((mi[5] - mi[2] - mi[1]) / max(mi[3], 1.0)),
                epilogue_wait_accumulator=round(m[4] / total, 3))
        print(json.dumps(dict(workload=name, **out)), flush=True)
        del layer, inp
        torch.cuda.empty_cache()


if __name__ == "__main__":
    main()
