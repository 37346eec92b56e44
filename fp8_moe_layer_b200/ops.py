"""Python binding of the FP8 MoE layer's C ABI (``include/moe.h``), through ctypes.

Argument marshalling only: every step of the layer runs in the CUDA library ``libfp8moe.so``.
Importing this module loads that library and raises if it has not been built; there is no other
implementation to fall back to. Tensors are torch CUDA tensors (torch provides device memory and
streams); bf16 tensors are passed as their bit patterns and e4m3 tensors as uint8 codes.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfp8moe.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = -1
MOE_ERR_UNSUPPORTED = -2
MOE_ERR_WORKSPACE = -3
MOE_ERR_CUDA = -4
MOE_ERR_DEVICE_TIMEOUT = -5
MOE_ERR_DEVICE_CHECK = -6
NUM_STAGES = 8
STAGE_NAMES = ("router_logits", "topk_quant", "permute", "gather", "gemm_gateup_swiglu",
               "requant", "gemm_down", "combine")


class MoEDims(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d", ctypes.c_int32), ("E", ctypes.c_int32),
                ("F", ctypes.c_int32), ("k_max", ctypes.c_int32), ("F_shared", ctypes.c_int32)]


class MoEDebugOut(ctypes.Structure):
    _fields_ = [("topk_ids", ctypes.c_void_p), ("topk_w", ctypes.c_void_p),
                ("expert_offsets", ctypes.c_void_p), ("perm_token", ctypes.c_void_p),
                ("inv_row", ctypes.c_void_p), ("y_f32", ctypes.c_void_p),
                ("stage_events", ctypes.POINTER(ctypes.c_void_p))]


class MoEError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {status_string(status)} (status {status})")


def _load(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(
            f"{path} is missing: build it with `python -m fp8_moe_layer_b200.build` "
            "(nvcc, sm_100a). The FP8 MoE layer has no other implementation.")
    lib = ctypes.CDLL(path)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
    dims_p = ctypes.POINTER(MoEDims)
    sig = {
        "moe_workspace_bytes": (sz, [dims_p]),
        "moe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "moe_clear_status": (ctypes.c_int, [vp, vp]),
        "moe_device_status": (ctypes.c_int, [vp, vp, ctypes.POINTER(i32)]),
        "moe_route_topk": (ctypes.c_int, [dims_p, vp, vp, vp, i32, vp, vp, vp, vp, sz, vp]),
        "moe_permute": (ctypes.c_int, [dims_p, vp, i32, vp, vp, vp, vp, vp, sz, vp]),
        "moe_grouped_ffn_fp8": (ctypes.c_int, [dims_p, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp,
                                               sz, vp]),
        "moe_combine": (ctypes.c_int, [dims_p, vp, vp, vp, vp, vp, vp, vp]),
        "moe_forward": (ctypes.c_int, [dims_p, vp, vp, vp, i32, vp, vp, vp, vp, vp, vp, vp, vp,
                                       vp, vp, vp, sz, vp, ctypes.POINTER(MoEDebugOut)]),
        "moe_route_topk_noalloc": (ctypes.c_int, [dims_p, vp, vp, vp, i32, vp, vp, vp, vp]),
        "moe_kernel_launch_count": (ctypes.c_uint64, []),
        "moe_ep_dispatch": (ctypes.c_int, [dims_p, i32, vp, vp, vp, i32, vp, vp, vp, vp, vp, vp,
                                           vp, vp, sz, vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


LIB = _load()


def load_library(path: str) -> ctypes.CDLL:
    """Another build of the same C ABI (e.g. the wait-test build), with the argument types set."""
    return _load(path)


def kernel_launch_count() -> int:
    """Kernels the library has launched in this process so far (a host-side counter)."""
    return int(LIB.moe_kernel_launch_count())


def status_string(status: int) -> str:
    return LIB.moe_status_string(int(status)).decode()


def _check(status: int, where: str):
    if status != MOE_OK:
        raise MoEError(status, where)


def dims(T: int, d: int, E: int, F: int, k_max: int, F_shared: int = 0) -> MoEDims:
    return MoEDims(int(T), int(d), int(E), int(F), int(k_max), int(F_shared))


def workspace_bytes(dm: MoEDims) -> int:
    return int(LIB.moe_workspace_bytes(ctypes.byref(dm)))


def alloc_workspace(dm: MoEDims, device=None) -> torch.Tensor:
    """Workspace for every entry point with these dims, its status word cleared."""
    n = workspace_bytes(dm)
    if n == 0:
        raise MoEError(MOE_ERR_INVALID_ARG, "workspace_bytes")
    ws = torch.empty(n, dtype=torch.uint8, device=device or "cuda")
    _check(LIB.moe_clear_status(ws.data_ptr(), _stream(ws.device)), "moe_clear_status")
    return ws


def _stream(device=None) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must be on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


def _bits(t: torch.Tensor) -> torch.Tensor:
    """bf16 tensor -> its int16 view (bit patterns) without a copy."""
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16)
    if t.dtype in (torch.int16, torch.uint16):
        return t
    raise TypeError("expected a bf16 tensor")


def _u8(t: Optional[torch.Tensor]) -> Optional[torch.Tensor]:
    if t is None:
        return None
    if t.dtype == torch.float8_e4m3fn:
        return t.view(torch.uint8)
    if t.dtype != torch.uint8:
        raise TypeError("expected e4m3 codes (uint8 or float8_e4m3fn)")
    return t


def device_status(ws: torch.Tensor) -> int:
    out = ctypes.c_int32(0)
    _check(LIB.moe_device_status(ws.data_ptr(), _stream(ws.device), ctypes.byref(out)),
           "moe_device_status")
    return int(out.value)


def clear_status(ws: torch.Tensor) -> None:
    _check(LIB.moe_clear_status(ws.data_ptr(), _stream(ws.device)), "moe_clear_status")


# ------------------------------------------------------------------------------ entry points
def moe_route_topk(hidden, router_w, router_bias, k, k_per_token, k_max, F=16, ws=None):
    """Router + softmax + top-k: returns (topk_ids int32 [T, k_max], topk_w fp32 [T, k_max])."""
    T, d = hidden.shape
    E = router_w.shape[0]
    dm = dims(T, d, E, F, k_max)
    ws = alloc_workspace(dm, hidden.device) if ws is None else ws
    ids = torch.empty(T, k_max, dtype=torch.int32, device=hidden.device)
    w = torch.empty(T, k_max, dtype=torch.float32, device=hidden.device)
    _check(LIB.moe_route_topk(ctypes.byref(dm), _p(_bits(hidden)), _p(router_w), _p(router_bias),
                              int(k), _p(k_per_token), _p(ids), _p(w), _p(ws), ws.numel(),
                              _stream(hidden.device)), "moe_route_topk")
    return ids, w


def moe_permute(topk_ids, k, k_per_token, E, d=16, F=16, ws=None):
    """Stable grouping by expert: returns (expert_offsets [E+1], perm_token [T*k_max],
    inv_row [T, k_max]), all int32."""
    T, k_max = topk_ids.shape
    dm = dims(T, d, E, F, k_max)
    ws = alloc_workspace(dm, topk_ids.device) if ws is None else ws
    dev = topk_ids.device
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm = torch.full((max(T * k_max, 1),), -1, dtype=torch.int32, device=dev)
    inv = torch.empty(T, k_max, dtype=torch.int32, device=dev)
    _check(LIB.moe_permute(ctypes.byref(dm), _p(topk_ids), int(k), _p(k_per_token), _p(offsets),
                           _p(perm), _p(inv), _p(ws), ws.numel(), _stream(dev)), "moe_permute")
    return offsets, perm, inv


def moe_grouped_ffn_fp8(hidden, w13, w13_scale, w2, w2_scale, expert_offsets, perm_token, k_max,
                        ws=None, want_act_scale=False):
    """Grouped W8A8 FP8 SwiGLU experts over routed rows: returns expert_out fp32 [T*k_max, d]
    (and the per-token activation scales when asked)."""
    T, d = hidden.shape
    E, twoF, _ = w13.shape
    dm = dims(T, d, E, twoF // 2, k_max)
    dev = hidden.device
    ws = alloc_workspace(dm, dev) if ws is None else ws
    out = torch.zeros(max(T * k_max, 1), d, dtype=torch.float32, device=dev)
    xs = torch.empty(T, dtype=torch.float32, device=dev) if want_act_scale else None
    _check(LIB.moe_grouped_ffn_fp8(ctypes.byref(dm), _p(_bits(hidden)), _p(_u8(w13)),
                                   _p(w13_scale), _p(_u8(w2)), _p(w2_scale), _p(expert_offsets),
                                   _p(perm_token), _p(out), _p(xs), _p(ws), ws.numel(),
                                   _stream(dev)), "moe_grouped_ffn_fp8")
    return (out, xs) if want_act_scale else out


def moe_combine(expert_out, topk_w, inv_row, shared_out=None, want_f32=False):
    """Weighted combine in token order: returns y bf16 [T, d] (and the fp32 sum when asked)."""
    T, k_max = topk_w.shape
    d = expert_out.shape[1]
    dm = dims(T, d, 1, 16, k_max)
    dev = expert_out.device
    y = torch.empty(T, d, dtype=torch.bfloat16, device=dev)
    yf = torch.empty(T, d, dtype=torch.float32, device=dev) if want_f32 else None
    _check(LIB.moe_combine(ctypes.byref(dm), _p(expert_out), _p(topk_w), _p(inv_row),
                           _p(shared_out), _p(y.view(torch.int16)), _p(yf), _stream(dev)),
           "moe_combine")
    return (y, yf) if want_f32 else y


def ep_local_k(E: int, k_max: int, n_ranks: int) -> int:
    """Expert slots per dispatched row: a token has at most min(k_max, E / n_ranks) experts on
    one rank."""
    return min(k_max, E // n_ranks)


def moe_ep_dispatch(hidden, topk_ids, topk_w, k, k_per_token, E, n_ranks, ws=None):
    """Expert-parallel dispatch plan and row gather. Returns a dict: send_hidden bf16
    [T*min(n_ranks, k_max), d], send_ids int32 / send_w fp32 [same rows, kl], send_counts int32
    [n_ranks] (device), slot_of int32 / slot_w fp32 [T, n_ranks]."""
    T, d = hidden.shape
    k_max = topk_ids.shape[1]
    dev = hidden.device
    dm = dims(T, d, E, 16, k_max)
    kl = ep_local_k(E, k_max, n_ranks)
    cap = max(T * min(n_ranks, k_max), 1)
    out = dict(send_hidden=torch.empty(cap, d, dtype=torch.bfloat16, device=dev),
               send_ids=torch.empty(cap, kl, dtype=torch.int32, device=dev),
               send_w=torch.empty(cap, kl, dtype=torch.float32, device=dev),
               send_counts=torch.empty(n_ranks, dtype=torch.int32, device=dev),
               slot_of=torch.empty(max(T, 1), n_ranks, dtype=torch.int32, device=dev),
               slot_w=torch.empty(max(T, 1), n_ranks, dtype=torch.float32, device=dev))
    ws = alloc_workspace(dims(max(T, 1), d, E, 16, k_max), dev) if ws is None else ws
    _check(LIB.moe_ep_dispatch(ctypes.byref(dm), int(n_ranks), _p(_bits(hidden)), _p(topk_ids),
                               _p(topk_w), int(k), _p(k_per_token),
                               _p(out["send_hidden"].view(torch.int16)), _p(out["send_ids"]),
                               _p(out["send_w"]), _p(out["send_counts"]), _p(out["slot_of"]),
                               _p(out["slot_w"]), _p(ws), ws.numel(), _stream(dev)),
           "moe_ep_dispatch")
    return out


def moe_forward(hidden, router_w, router_bias, k, k_per_token, w13, w13_scale, w2, w2_scale,
                k_max, shared: Optional[Sequence[torch.Tensor]] = None, ws=None, y=None,
                debug: bool = False, stage_events: Optional[Sequence] = None, lib=None):
    """The whole layer. Returns y bf16 [T, d], or (y, dict of debug outputs) when debug=True.
    ``lib``: another build of the library loaded with ``load_library`` (default: this one)."""
    T, d = hidden.shape
    E, twoF, _ = w13.shape
    F = twoF // 2
    Fs = shared[0].shape[0] // 2 if shared is not None else 0
    dm = dims(T, d, E, F, k_max, Fs)
    dev = hidden.device
    ws = alloc_workspace(dm, dev) if ws is None else ws
    y = torch.empty(T, d, dtype=torch.bfloat16, device=dev) if y is None else y
    w13s, s13s, w2s, s2s = shared if shared is not None else (None, None, None, None)
    dbg_struct, dbg = None, None
    ev_arr = None
    if debug or stage_events is not None:
        dbg = {}
        if debug:
            dbg = dict(topk_ids=torch.empty(T, k_max, dtype=torch.int32, device=dev),
                       topk_w=torch.empty(T, k_max, dtype=torch.float32, device=dev),
                       expert_offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
                       perm_token=torch.empty(max(T * k_max, 1), dtype=torch.int32, device=dev),
                       inv_row=torch.empty(T, k_max, dtype=torch.int32, device=dev),
                       y_f32=torch.empty(T, d, dtype=torch.float32, device=dev))
        if stage_events is not None:
            for e in stage_events:            # torch creates its events lazily, on first record
                if e is not None and not e.cuda_event:
                    e.record()
            ev_arr = (ctypes.c_void_p * (NUM_STAGES + 1))(
                *[ctypes.c_void_p(e.cuda_event if e is not None else 0) for e in stage_events])
        dbg_struct = MoEDebugOut(*(dbg[n].data_ptr() if n in dbg else None for n in
                                   ("topk_ids", "topk_w", "expert_offsets", "perm_token",
                                    "inv_row", "y_f32")),
                                 ctypes.cast(ev_arr, ctypes.POINTER(ctypes.c_void_p))
                                 if ev_arr is not None else None)
    status = (lib or LIB).moe_forward(
        ctypes.byref(dm), _p(_bits(hidden)), _p(router_w), _p(router_bias), int(k),
        _p(k_per_token), _p(_u8(w13)), _p(w13_scale), _p(_u8(w2)), _p(w2_scale), _p(_u8(w13s)),
        _p(s13s), _p(_u8(w2s)), _p(s2s), _p(y.view(torch.int16)), _p(ws), ws.numel(),
        _stream(dev), ctypes.byref(dbg_struct) if dbg_struct is not None else None)
    _check(status, "moe_forward")
    return (y, dbg) if debug else y


class MoELayerFP8:
    """Device-resident FP8 MoE layer: owns the weights and a workspace sized for ``max_T``."""

    def __init__(self, inputs, device="cuda", max_T: Optional[int] = None):
        s = inputs.shape
        self.shape = s
        self.device = torch.device(device)
        dev = self.device
        self.router_w = inputs.router_w.to(dev)
        self.router_bias = None if inputs.router_bias is None else inputs.router_bias.to(dev)
        self.w13, self.w13_scale = inputs.w13.to(dev), inputs.w13_scale.to(dev)
        self.w2, self.w2_scale = inputs.w2.to(dev), inputs.w2_scale.to(dev)
        self.shared = None
        if s.F_shared:
            self.shared = (inputs.w13_shared.to(dev), inputs.w13s_scale.to(dev),
                           inputs.w2_shared.to(dev), inputs.w2s_scale.to(dev))
        self.max_T = max_T or s.T
        self.dims = dims(self.max_T, s.d, s.E, s.F, s.k_max, s.F_shared)
        # split counts depend on T, so size the workspace for the largest need over 1..max_T
        need = max(workspace_bytes(dims(t, s.d, s.E, s.F, s.k_max, s.F_shared))
                   for t in range(1, self.max_T + 1))
        self.ws = torch.empty(need, dtype=torch.uint8, device=dev)
        clear_status(self.ws)

    def __call__(self, hidden, k_per_token=None, y=None, debug=False, stage_events=None,
                 k: Optional[int] = None):
        """y = layer(hidden); per-token k from ``k_per_token`` if given, else the fixed ``k``
        (default: the layer's k)."""
        if hidden.shape[0] > self.max_T:
            raise ValueError("more tokens than the workspace was sized for")
        k = self.shape.k if k is None else int(k)
        return moe_forward(hidden, self.router_w, self.router_bias, k, k_per_token,
                           self.w13, self.w13_scale, self.w2, self.w2_scale, self.shape.k_max,
                           shared=self.shared, ws=self.ws, y=y, debug=debug,
                           stage_events=stage_events)
