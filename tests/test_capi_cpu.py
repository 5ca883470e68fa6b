"""The C-ABI library without a GPU: it loads, exports every function the
header declares, and rejects bad arguments before touching the device."""
import ctypes as C
import math
import os
import re

import pytest

from conftest import ROOT
from routed_nvfp4_expert_b200 import capi


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s+\*?([a-z_][a-z0-9_]*)\s*\(", src, re.M):
                names.add(m.group(1))
    return names


def test_library_exports_every_declared_symbol():
    lib = C.CDLL(capi._LIB_PATH)
    declared = _declared()
    assert len(declared) >= 15
    for name in declared:
        assert hasattr(lib, name), name
    assert declared == set(capi.EXPORTED)


def _cfg(**kw):
    base = dict(hidden=256, intermediate=128, shared_intermediate=128, num_experts=16, local_begin=0, local_end=16,
                top_k=4, routed_scaling_factor=2.5, swiglu_limit=7.0)
    base.update(kw)
    return capi.SiteConfig(**base)


@pytest.mark.parametrize("kw,frag", [
    (dict(top_k=17), "top_k"), (dict(top_k=0), "top_k"), (dict(num_experts=3, local_end=3), "top_k"),
    (dict(hidden=100), "hidden"), (dict(intermediate=0), "intermediate"), (dict(shared_intermediate=32), "shared"),
    (dict(swiglu_limit=math.nan), "swiglu_limit"), (dict(swiglu_limit=-1.0), "swiglu_limit"),
    (dict(routed_scaling_factor=math.inf), "routed_scaling_factor"), (dict(local_end=17), "local range"),
    (dict(local_begin=5, local_end=4), "local range"), (dict(num_experts=2000, local_end=2000), "num_experts"),
])
def test_config_validation(kw, frag):
    cfg = _cfg(**kw)
    lib = capi.lib()
    assert lib.moe_workspace_size(C.byref(cfg.c()), 4, 0) == 0
    assert frag in lib.moe_last_error().decode()
    w = capi.MoeWeights()
    st = lib.moe_forward(C.byref(cfg.c()), C.byref(w), 16, 4, 0, 16, 256, 1 << 20, None)
    assert st in (1, 2)


def test_swiglu_limit_inf_is_valid():
    assert capi.lib().moe_workspace_size(C.byref(_cfg(swiglu_limit=math.inf).c()), 4, 0) > 0


def test_t_zero_is_a_noop_and_bad_pointers_are_rejected():
    lib = capi.lib()
    cfg = _cfg().c()
    w = capi.MoeWeights()
    assert lib.moe_forward(C.byref(cfg), C.byref(w), None, 0, 0, None, None, 0, None) == 0
    # misaligned x
    st = lib.moe_forward(C.byref(cfg), C.byref(w), 0x1001, 4, 0, 0x2000, 0x3000, 1 << 30, None)
    assert st == 1 and "x" in lib.moe_last_error().decode()
    # unknown path
    assert lib.moe_forward(C.byref(cfg), C.byref(w), 0x1000, 4, 7, 0x2000, 0x3000, 1 << 30, None) == 1
    # combine: k > 16
    assert lib.moe_combine(4, 17, 256, 0x1000, None, 0x2000, None) == 1
    assert lib.moe_combine(0, 4, 256, None, None, None, None) == 0


def test_workspace_too_small_is_rejected_before_launch():
    lib = capi.lib()
    cfg = _cfg().c()
    need = lib.moe_workspace_size(C.byref(cfg), 4, 0)
    assert need > 0
    ids = 0x10000
    plan = capi.MoePlan(0x20000, 0x30000, 0x40000, 0x50000, 0x60000, 0x70000, 0x80000, 0x90000)
    # moe_permute needs the status word and the sort scratch only
    st = lib.moe_permute(C.byref(cfg), ids, 4, C.byref(plan), 0x100000, 256, None)
    assert st == 3 and "workspace" in lib.moe_last_error().decode()
    w = capi.MoeWeights()
    st = lib.moe_forward(C.byref(cfg), C.byref(w), 0x10000, 4, 0, 0x20000, 0x100000, need - 256, None)
    assert st != 0


def test_plan_carve_is_host_arithmetic():
    lib = capi.lib()
    cfg = _cfg().c()
    n = lib.moe_plan_size(C.byref(cfg), 10)
    plan = capi.MoePlan()
    assert lib.moe_plan_carve(C.byref(cfg), 10, 0x100000, n, C.byref(plan)) == 0
    ptrs = [plan.counts, plan.offsets, plan.sorted, plan.inv, plan.tile_offsets, plan.active, plan.first,
            plan.tile_rows]
    assert ptrs == sorted(ptrs) and all(p % 256 == 0 for p in ptrs) and ptrs[0] == 0x100000
    assert lib.moe_plan_carve(C.byref(cfg), 10, 0x100000, n - 1, C.byref(plan)) == 3


def test_noalloc_rejects_oversized_requests_before_touching_the_device():
    lib = capi.lib()
    cfg = _cfg(hidden=4096, intermediate=1024, shared_intermediate=1024, num_experts=288, local_end=288, top_k=8).c()
    need = lib.moe_workspace_size(C.byref(cfg), 4096, 0)
    assert need > 8 << 20
    w = capi.MoeWeights()
    st = lib.moe_forward_decode_noalloc(C.byref(cfg), C.byref(w), 0x1000, 4096, 0x2000, None)
    assert st == 3 and "built-in buffer" in lib.moe_last_error().decode()


def _fake_weights(prepared=None):
    w = capi.MoeWeights()
    w.router_w, w.router_bias = 0x10000, 0x11000
    for i, b in enumerate((w.gate, w.up, w.down)):
        b.codes, b.scales, b.tensor_scale = 0x100000 * (i + 1), 0x100000 * (i + 1) + 0x80000, 0x12000 + 0x100 * i
    w.prepared = prepared
    return w


def test_padded_rows_and_prepared_size_are_host_arithmetic():
    lib = capi.lib()
    cfg = _cfg()                                   # E = 16, k = 4, H = 256, I = 128
    for T in (0, 1, 10, 300, 4096):
        A = T * 4
        n = min(A, 16)
        assert lib.moe_padded_rows(C.byref(cfg.c()), T) == (A + 255 * n) // 256 * 256
    # EP range: only the local experts get tiles
    assert lib.moe_padded_rows(C.byref(_cfg(local_begin=4, local_end=6).c()), 100) == (400 + 255 * 2) // 256 * 256
    up = lambda v: (v + 255) // 256 * 256
    per = 16 * 128 * 256 // 16
    # gate / up / down scale atoms, then the router weight as three bf16 terms
    assert lib.moe_prepared_size(C.byref(cfg.c())) == up(3 * per) + up(16 * 3 * 256 * 2)


def test_prefill_entry_points_validate_before_launch():
    lib = capi.lib()
    cfg = _cfg().c()
    w = _fake_weights(prepared=0x800000)
    plan = capi.MoePlan(*[0x900000 + 0x1000 * i for i in range(8)])
    # shapes the tensor-core prefill does not cover
    bad = _cfg(hidden=192).c()
    assert lib.nvfp4_grouped_gemm(C.byref(bad), 0, 0x1000, 0x2000, 0x3000, 4, C.byref(plan), 0x4000, C.byref(w),
                                  0x5000, 0x6000, 1 << 30, None) == 2
    assert "hidden" in lib.moe_last_error().decode()
    assert lib.moe_prepare_weights(C.byref(bad), C.byref(w), 0x700000, 1 << 30, None) == 2
    # unknown projection, T = 0, missing prepared weights, short workspace
    assert lib.nvfp4_grouped_gemm(C.byref(cfg), 5, 0x1000, 0x2000, 0x3000, 4, C.byref(plan), 0x4000, C.byref(w),
                                  0x5000, 0x6000, 1 << 30, None) == 1
    assert lib.nvfp4_grouped_gemm(C.byref(cfg), 0, None, None, None, 0, None, None, C.byref(w), None, None, 0,
                                  None) == 0
    w0 = _fake_weights(prepared=None)
    assert lib.nvfp4_grouped_gemm(C.byref(cfg), 0, 0x1000, 0x2000, 0x3000, 4, C.byref(plan), 0x4000, C.byref(w0),
                                  0x5000, 0x6000, 1 << 30, None) == 1
    assert "prepared" in lib.moe_last_error().decode()
    assert lib.nvfp4_grouped_gemm(C.byref(cfg), 1, 0x1000, 0x2000, 0x3000, 4, C.byref(plan), 0x4000, C.byref(w),
                                  0x5000, 0x6000, 256, None) == 3
    # weight preparation: misaligned or short destination
    need = lib.moe_prepared_size(C.byref(cfg))
    assert lib.moe_prepare_weights(C.byref(cfg), C.byref(w), 0x700010, need, None) == 1
    assert lib.moe_prepare_weights(C.byref(cfg), C.byref(w), 0x700000, need - 1, None) == 3
    assert lib.moe_prepare_weights(C.byref(cfg), C.byref(capi.MoeWeights()), 0x700000, need, None) == 1
    # row encoding: K must be a multiple of 64; no rows is a no-op
    assert lib.nvfp4_quantize_rows(0x1000, 4, 100, 0x2000, 0x3000, 0x4000, None) == 1
    assert lib.nvfp4_quantize_rows(0x1000, 0, 256, 0x2000, 0x3000, 0x4000, None) == 0


def test_unpermute_entry_points_validate_before_launch():
    lib = capi.lib()
    cfg = _cfg().c()
    plan = capi.MoePlan(*[0x900000 + 0x1000 * i for i in range(8)])
    assert lib.moe_unpermute(C.byref(cfg), None, 0, None, None, None, None) == 0
    assert lib.moe_unpermute(C.byref(cfg), 0x1000, 4, None, 0x2000, 0x3000, None) == 1
    assert "plan" in lib.moe_last_error().decode()
    assert lib.moe_unpermute(C.byref(cfg), 0x1008, 4, C.byref(plan), 0x2000, 0x3000, None) == 1
    assert "rows" in lib.moe_last_error().decode()
    assert lib.moe_unpermute_combine(C.byref(cfg), 0x1000, 4, C.byref(plan), 0x2000, 0x3008, 0x4000, None) == 1
    assert "shared" in lib.moe_last_error().decode()
    assert lib.moe_unpermute_combine(C.byref(cfg), None, 0, None, None, None, None, None) == 0


def test_decode_workspace_holds_the_grouped_gemm_buffers_from_nine_tokens():
    """Decode batches of 9 or more tokens run on the grouped W4A16 GEMM when
    the workspace holds its buffers: moe_workspace_size sizes them (x as f16
    rows of the padded tile layout, h as f16 padded rows), and a workspace of
    that size lays them out behind the decode's own (host arithmetic only)."""
    lib = capi.lib()
    cfg = _cfg()                                   # E = 16, k = 4, H = 256, I = 128
    c = cfg.c()
    w8 = lib.moe_workspace_size(C.byref(c), 8, 0)
    w9 = lib.moe_workspace_size(C.byref(c), 9, 0)
    P9 = lib.moe_padded_rows(C.byref(c), 9)
    assert P9 % 256 == 0 and P9 >= 9 * 4
    # the gathered f16 x rows alone take P * H * 2 bytes
    assert w9 > w8 + P9 * 256 * 2
    # a shape the grouped GEMM does not take keeps the plain layout
    odd = _cfg(intermediate=96, shared_intermediate=96).c()
    assert lib.moe_workspace_size(C.byref(odd), 9, 0) < lib.moe_workspace_size(C.byref(c), 9, 0)
    base = 0x1000000
    v = capi.MoeViews()
    assert lib.moe_workspace_views(C.byref(c), 9, 0, base, w9, C.byref(v)) == 0
    # h (f16 padded rows, at least 4 bytes per assignment element) ends before r
    assert v.r - v.h >= max(2 * P9, 4 * 36) * 128
    # r stays [T*k, H] fp32 in assignment order on both forms
    assert v.shared - v.r >= 4 * 36 * 256
