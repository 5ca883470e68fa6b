"""Thin ctypes binding of the C ABI in include/routed_nvfp4.h.

Argument marshalling only: every step of the site runs in the CUDA kernels of
librouted_nvfp4.so. PyTorch supplies device memory (``data_ptr``) and the
current CUDA stream. Importing this module fails loudly when the library has
not been built; there is no fallback.
"""
from __future__ import annotations

import ctypes as C
import dataclasses
import math
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "librouted_nvfp4.so")

MOE_OK = 0
STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED", 3: "MOE_ERR_WORKSPACE",
                4: "MOE_ERR_CUDA", 5: "MOE_ERR_DEVICE_TIMEOUT", 6: "MOE_ERR_DEVICE_BOUNDS"}
PATH_DECODE, PATH_PREFILL, PATH_PREFILL_W4A16 = 0, 1, 2
PROJ_GATE_UP, PROJ_DOWN = 0, 1

# every symbol include/routed_nvfp4.h declares
EXPORTED = (
    "moe_workspace_size", "moe_plan_size", "moe_plan_carve", "moe_router_topk", "moe_permute",
    "nvfp4_expert_gemv", "clamped_swiglu", "moe_combine", "dense_ffn_workspace_size", "dense_ffn_bf16",
    "nvfp4_dequant", "moe_forward", "moe_workspace_views", "moe_read_device_status", "moe_last_error",
    "moe_set_stage_events", "moe_forward_decode_noalloc", "moe_padded_rows", "moe_prepared_size",
    "moe_prepare_weights", "nvfp4_quantize_rows", "nvfp4_grouped_gemm", "moe_unpermute", "moe_unpermute_combine",
    "moe_combine_f32", "moe_noalloc_read_device_status", "moe_set_wait_limit", "nvfp4_grouped_gemm_w4a16",
)
STAGES = ("router_logits", "topk", "permute", "act_quant", "expert_gate_up", "h_quant", "expert_down", "shared",
          "combine")


class MoEError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


class MoeConfig(C.Structure):
    _fields_ = [("hidden", C.c_int32), ("intermediate", C.c_int32), ("shared_intermediate", C.c_int32),
                ("num_experts", C.c_int32), ("local_begin", C.c_int32), ("local_end", C.c_int32),
                ("top_k", C.c_int32), ("routed_scaling_factor", C.c_float), ("swiglu_limit", C.c_float)]


class Nvfp4Bank(C.Structure):
    _fields_ = [("codes", C.c_void_p), ("scales", C.c_void_p), ("tensor_scale", C.c_void_p)]


class MoeWeights(C.Structure):
    _fields_ = [("router_w", C.c_void_p), ("router_bias", C.c_void_p), ("gate", Nvfp4Bank), ("up", Nvfp4Bank),
                ("down", Nvfp4Bank), ("shared_gate", C.c_void_p), ("shared_up", C.c_void_p),
                ("shared_down", C.c_void_p), ("prepared", C.c_void_p)]


class MoePlan(C.Structure):
    _fields_ = [("counts", C.c_void_p), ("offsets", C.c_void_p), ("sorted", C.c_void_p), ("inv", C.c_void_p),
                ("tile_offsets", C.c_void_p), ("active", C.c_void_p), ("first", C.c_void_p),
                ("tile_rows", C.c_void_p)]


class MoeViews(C.Structure):
    _fields_ = [("logits", C.c_void_p), ("ids", C.c_void_p), ("weights", C.c_void_p), ("plan", MoePlan),
                ("h", C.c_void_p), ("r", C.c_void_p), ("shared", C.c_void_p), ("xq_codes", C.c_void_p),
                ("xq_sf", C.c_void_p), ("xq_scale", C.c_void_p), ("hq_codes", C.c_void_p), ("hq_sf", C.c_void_p),
                ("hq_scale", C.c_void_p)]


def load_library(path: str = _LIB_PATH) -> C.CDLL:
    if not os.path.exists(path):
        raise RuntimeError(f"CUDA library {path} is missing: build it with "
                           f"`python -m routed_nvfp4_expert_b200.build` (there is no CPU fallback)")
    lib = C.CDLL(path)
    i32, sz, vp, st = C.c_int32, C.c_size_t, C.c_void_p, C.c_int
    cfgp = C.POINTER(MoeConfig)
    sig = {
        "moe_workspace_size": (sz, [cfgp, i32, i32]),
        "moe_plan_size": (sz, [cfgp, i32]),
        "moe_plan_carve": (st, [cfgp, i32, vp, sz, C.POINTER(MoePlan)]),
        "moe_router_topk": (st, [cfgp, vp, i32, vp, vp, vp, vp, vp, vp]),
        "moe_permute": (st, [cfgp, vp, i32, C.POINTER(MoePlan), vp, sz, vp]),
        "nvfp4_expert_gemv": (st, [cfgp, i32, vp, i32, C.POINTER(MoePlan), vp, C.POINTER(MoeWeights), vp, vp, sz, vp]),
        "clamped_swiglu": (st, [vp, i32, i32, C.c_float, vp, vp]),
        "moe_combine": (st, [i32, i32, i32, vp, vp, vp, vp]),
        "moe_combine_f32": (st, [i32, i32, i32, vp, vp, vp, vp]),
        "dense_ffn_workspace_size": (sz, [i32, i32, i32]),
        "dense_ffn_bf16": (st, [i32, i32, C.c_float, vp, i32, vp, vp, vp, vp, vp, sz, vp]),
        "nvfp4_dequant": (st, [vp, vp, vp, i32, i32, vp, vp]),
        "moe_forward": (st, [cfgp, C.POINTER(MoeWeights), vp, i32, i32, vp, vp, sz, vp]),
        "moe_workspace_views": (st, [cfgp, i32, i32, vp, sz, C.POINTER(MoeViews)]),
        "moe_read_device_status": (st, [vp, vp]),
        "moe_last_error": (C.c_char_p, []),
        "moe_set_stage_events": (st, [C.POINTER(C.c_void_p), i32]),
        "moe_forward_decode_noalloc": (st, [cfgp, C.POINTER(MoeWeights), vp, i32, vp, vp]),
        "moe_noalloc_read_device_status": (st, [vp]),
        "moe_set_wait_limit": (st, [C.c_int64]),
        "nvfp4_grouped_gemm_w4a16": (st, [cfgp, i32, vp, vp, i32, C.POINTER(MoePlan), vp, C.POINTER(MoeWeights), vp,
                                          vp, sz, vp]),
        "moe_padded_rows": (C.c_int64, [cfgp, i32]),
        "moe_prepared_size": (sz, [cfgp]),
        "moe_prepare_weights": (st, [cfgp, C.POINTER(MoeWeights), vp, sz, vp]),
        "nvfp4_quantize_rows": (st, [vp, i32, i32, vp, vp, vp, vp]),
        "nvfp4_grouped_gemm": (st, [cfgp, i32, vp, vp, vp, i32, C.POINTER(MoePlan), vp, C.POINTER(MoeWeights), vp,
                                    vp, sz, vp]),
        "moe_unpermute": (st, [cfgp, vp, i32, C.POINTER(MoePlan), vp, vp, vp]),
        "moe_unpermute_combine": (st, [cfgp, vp, i32, C.POINTER(MoePlan), vp, vp, vp, vp]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype, f.argtypes = res, args
    return lib


_lib: C.CDLL | None = None


def lib() -> C.CDLL:
    global _lib
    if _lib is None:
        _lib = load_library()
    return _lib


def _check(status: int):
    if status != MOE_OK:
        raise MoEError(status, lib().moe_last_error().decode())


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return getattr(stream, "cuda_stream", stream)


def _p(t) -> int | None:
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return t.data_ptr()


# ------------------------------------------------------------------ config / weights

@dataclasses.dataclass
class SiteConfig:
    hidden: int
    intermediate: int
    shared_intermediate: int
    num_experts: int
    local_begin: int
    local_end: int
    top_k: int
    routed_scaling_factor: float
    swiglu_limit: float

    def c(self) -> MoeConfig:
        return MoeConfig(self.hidden, self.intermediate, self.shared_intermediate, self.num_experts,
                         self.local_begin, self.local_end, self.top_k, self.routed_scaling_factor,
                         self.swiglu_limit)


@dataclasses.dataclass
class DeviceSite:
    """Device copies of one site's weights (torch owns the memory)."""
    router_w: torch.Tensor
    router_bias: torch.Tensor
    banks: dict            # proj -> (codes, scales, ts)
    shared: tuple | None   # (gate, up, down) bf16 or None
    prepared: torch.Tensor | None = None   # block-scale atoms of moe_prepare_weights (prefill)

    def c(self) -> MoeWeights:
        b = {p: Nvfp4Bank(_p(c), _p(s), _p(t)) for p, (c, s, t) in self.banks.items()}
        sh = self.shared or (None, None, None)
        return MoeWeights(_p(self.router_w), _p(self.router_bias), b["gate"], b["up"], b["down"],
                          _p(sh[0]), _p(sh[1]), _p(sh[2]), _p(self.prepared))


def bf16_tensor(bits, device="cuda") -> torch.Tensor:
    """uint16 bf16 bit patterns (numpy) -> torch.bfloat16 tensor on device."""
    import numpy as np
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.view(torch.bfloat16).to(device)


def site_to_device(inp: dict, device="cuda") -> DeviceSite:
    banks = {}
    for p in ("gate", "up", "down"):
        banks[p] = (torch.from_numpy(inp[f"{p}_codes"]).to(device), torch.from_numpy(inp[f"{p}_scales"]).to(device),
                    torch.from_numpy(inp[f"{p}_ts"]).to(device))
    shared = None
    if "shared_gate" in inp:
        shared = tuple(bf16_tensor(inp[f"shared_{p}"], device) for p in ("gate", "up", "down"))
    return DeviceSite(torch.from_numpy(inp["router_w"]).to(device), torch.from_numpy(inp["router_bias"]).to(device),
                      banks, shared)


def config_for(wl, local=None) -> SiteConfig:
    lb, le = local if local is not None else (0, wl.E)
    return SiteConfig(wl.H, wl.I, wl.Is, wl.E, lb, le, wl.k, float(wl.rsf), float(wl.limit))


# ------------------------------------------------------------------ entry points

def moe_workspace_size(cfg: SiteConfig, T: int, path: int) -> int:
    n = lib().moe_workspace_size(C.byref(cfg.c()), T, path)
    if n == 0:
        raise MoEError(1, lib().moe_last_error().decode())
    return n


def alloc_workspace(cfg: SiteConfig, T: int, path: int, device="cuda") -> torch.Tensor:
    return torch.empty(moe_workspace_size(cfg, T, path), dtype=torch.uint8, device=device)


def moe_plan_size(cfg: SiteConfig, T: int) -> int:
    return lib().moe_plan_size(C.byref(cfg.c()), T)


def moe_plan_carve(cfg: SiteConfig, T: int, buf: torch.Tensor) -> MoePlan:
    plan = MoePlan()
    _check(lib().moe_plan_carve(C.byref(cfg.c()), T, _p(buf), buf.numel() * buf.element_size(), C.byref(plan)))
    return plan


def moe_router_topk(cfg: SiteConfig, x, router_w, router_bias, logits, ids, weights, stream=None):
    _check(lib().moe_router_topk(C.byref(cfg.c()), _p(x), x.shape[0], _p(router_w), _p(router_bias), _p(logits),
                                 _p(ids), _p(weights), _stream(stream)))


def moe_permute(cfg: SiteConfig, ids, plan: MoePlan, ws, stream=None):
    _check(lib().moe_permute(C.byref(cfg.c()), _p(ids), ids.shape[0], C.byref(plan), _p(ws), ws.numel(),
                             _stream(stream)))


def nvfp4_expert_gemv(cfg: SiteConfig, proj: int, act, T: int, plan: MoePlan, weights, site: DeviceSite, out,
                      ws, stream=None):
    w = site.c()
    _check(lib().nvfp4_expert_gemv(C.byref(cfg.c()), proj, _p(act), T, C.byref(plan), _p(weights), C.byref(w),
                                   _p(out), _p(ws), ws.numel(), _stream(stream)))


def clamped_swiglu(gu, limit: float, h, stream=None):
    M, I2 = gu.shape
    _check(lib().clamped_swiglu(_p(gu), M, I2 // 2, C.c_float(limit), _p(h), _stream(stream)))


def moe_combine(r, shared, y, stream=None):
    """bf16 rows r [T, k, H] (+ bf16 shared [T, H] or None) -> y bf16; fp32
    rows (and an fp32 shared row) go through moe_combine_f32."""
    T, k, H = r.shape
    fn = lib().moe_combine_f32 if r.dtype == torch.float32 else lib().moe_combine
    _check(fn(T, k, H, _p(r), _p(shared), _p(y), _stream(stream)))


def dense_ffn_workspace_size(H: int, I: int, T: int) -> int:
    return lib().dense_ffn_workspace_size(H, I, T)


def dense_ffn_bf16(limit: float, x, wg, wu, wd, y, ws, stream=None):
    T, H = x.shape
    I = wg.shape[0]
    _check(lib().dense_ffn_bf16(H, I, C.c_float(limit), _p(x), T, _p(wg), _p(wu), _p(wd), _p(y), _p(ws),
                                ws.numel(), _stream(stream)))


def nvfp4_dequant(codes, scales, tensor_scale, out, stream=None):
    rows, K = out.shape
    _check(lib().nvfp4_dequant(_p(codes), _p(scales), _p(tensor_scale), rows, K, _p(out), _stream(stream)))


def moe_forward(cfg: SiteConfig, site: DeviceSite, x, path: int, y, ws, stream=None, w_c: MoeWeights | None = None):
    w = w_c if w_c is not None else site.c()
    _check(lib().moe_forward(C.byref(cfg.c()), C.byref(w), _p(x), x.shape[0], path, _p(y), _p(ws), ws.numel(),
                             _stream(stream)))


def moe_forward_decode_noalloc(cfg: SiteConfig, site: DeviceSite, x, y, stream=None):
    """Decode forward on the library's own 8 MiB device scratch buffer (for
    callers that cannot allocate a workspace); see the C header."""
    w = site.c()
    _check(lib().moe_forward_decode_noalloc(C.byref(cfg.c()), C.byref(w), _p(x), x.shape[0], _p(y),
                                            _stream(stream)))


def moe_noalloc_read_device_status(stream=None):
    """Device-side errors of the last moe_forward_decode_noalloc call on the
    current device (reads and clears the status word of the library's scratch)."""
    _check(lib().moe_noalloc_read_device_status(_stream(stream)))


def moe_padded_rows(cfg: SiteConfig, T: int) -> int:
    return lib().moe_padded_rows(C.byref(cfg.c()), T)


def moe_prepared_size(cfg: SiteConfig) -> int:
    return lib().moe_prepared_size(C.byref(cfg.c()))


def moe_prepare_weights(cfg: SiteConfig, site: DeviceSite, stream=None) -> torch.Tensor:
    """Allocate and fill the prefill block-scale atoms; also attaches them to
    ``site.prepared``."""
    n = moe_prepared_size(cfg)
    dst = torch.empty(n, dtype=torch.uint8, device=site.router_w.device)
    w = site.c()
    _check(lib().moe_prepare_weights(C.byref(cfg.c()), C.byref(w), _p(dst), n, _stream(stream)))
    site.prepared = dst
    return dst


def nvfp4_quantize_rows(src, codes, sf_atoms, row_scale, stream=None):
    rows, K = src.shape
    _check(lib().nvfp4_quantize_rows(_p(src), rows, K, _p(codes), _p(sf_atoms), _p(row_scale), _stream(stream)))


def nvfp4_grouped_gemm(cfg: SiteConfig, proj: int, act_codes, act_sf, act_scale, T: int, plan: MoePlan, weights,
                       site: DeviceSite, out, ws, stream=None):
    w = site.c()
    _check(lib().nvfp4_grouped_gemm(C.byref(cfg.c()), proj, _p(act_codes), _p(act_sf), _p(act_scale), T,
                                    C.byref(plan), _p(weights), C.byref(w), _p(out), _p(ws), ws.numel(),
                                    _stream(stream)))


def nvfp4_grouped_gemm_w4a16(cfg: SiteConfig, proj: int, act, act_scale, T: int, plan: MoePlan, weights,
                             site: DeviceSite, out, ws, stream=None):
    w = site.c()
    _check(lib().nvfp4_grouped_gemm_w4a16(C.byref(cfg.c()), proj, _p(act), _p(act_scale), T, C.byref(plan),
                                          _p(weights), C.byref(w), _p(out), _p(ws), ws.numel(), _stream(stream)))


def moe_unpermute(cfg: SiteConfig, rows, T: int, plan: MoePlan, ids, out, stream=None):
    _check(lib().moe_unpermute(C.byref(cfg.c()), _p(rows), T, C.byref(plan), _p(ids), _p(out), _stream(stream)))


def moe_unpermute_combine(cfg: SiteConfig, rows, T: int, plan: MoePlan, ids, shared, y, stream=None):
    _check(lib().moe_unpermute_combine(C.byref(cfg.c()), _p(rows), T, C.byref(plan), _p(ids), _p(shared), _p(y),
                                       _stream(stream)))


def moe_workspace_views(cfg: SiteConfig, T: int, path: int, ws) -> MoeViews:
    v = MoeViews()
    _check(lib().moe_workspace_views(C.byref(cfg.c()), T, path, _p(ws), ws.numel(), C.byref(v)))
    return v


def moe_set_stage_events(events):
    """events: list of len(STAGES)+1 entries, each a torch.cuda.Event (already
    recorded once so the CUDA event exists) or None (not recorded); or None to
    turn stage timing off."""
    if not events:
        _check(lib().moe_set_stage_events(None, 0))
        return
    arr = (C.c_void_p * len(events))(*[(e.cuda_event if e is not None else None) for e in events])
    _check(lib().moe_set_stage_events(arr, len(events)))


def moe_set_wait_limit(ns: int):
    """Test hook: limit of the BF16 tensor-core GEMM's main-loop waits (ns < 0
    restores the default)."""
    _check(lib().moe_set_wait_limit(int(ns)))


def moe_read_device_status(ws, stream=None):
    _check(lib().moe_read_device_status(_p(ws), _stream(stream)))


def view_tensor(ptr: int, shape, dtype, device="cuda") -> torch.Tensor:
    """Wrap a device pointer inside a torch-owned workspace as a tensor view
    (the workspace tensor must outlive the view)."""
    n = math.prod(shape)
    nbytes = n * torch.empty((), dtype=dtype).element_size()
    buf = _ptr_holder(ptr, nbytes, device)
    return buf.view(dtype)[:n].view(*shape)


def _ptr_holder(ptr: int, nbytes: int, device):
    class _Holder:
        __cuda_array_interface__ = {"shape": (nbytes,), "typestr": "|u1", "data": (ptr, False), "version": 3}
    return torch.as_tensor(_Holder(), device=device)
