"""GPU parity of the decode path (W4A16 GEMV) against the CPU oracle, called
through the C ABI: NVFP4 dequant (bit-exact), router logits / ids / weights,
the routing plan (bit-exact), the expert GEMVs, the shared expert, combine, and
the whole site on the tiny site and the H=4096, E=288 decode shapes."""
import math

import numpy as np
import pytest
import torch

from helpers import (LOGIT_REL, WEIGHT_REL, assert_bf16_close, bf16_np, device_site, oracle_cfg, rel_l2,
                     site_inputs, workload)
from oracle import formats as OF
from oracle import site as OS

pytestmark = pytest.mark.gpu

capi = pytest.importorskip("routed_nvfp4_expert_b200.capi")


def _x(inp):
    return capi.bf16_tensor(inp["x"])


# ------------------------------------------------------------------ dequant

def test_dequant_bit_exact_every_code_and_scale():
    # every (code, scale) pair: 256 scale bytes x 16 codes, each block holds all 16 codes
    codes = np.tile(np.array([0x10, 0x32, 0x54, 0x76, 0x98, 0xBA, 0xDC, 0xFE], np.uint8), (256, 1))
    scales = np.arange(256, dtype=np.uint8).reshape(256, 1)
    for ts in (np.float32(1.0), np.float32(0.0123), np.float32(3.1e-5)):
        out = torch.empty((256, 16), dtype=torch.float32, device="cuda")
        capi.nvfp4_dequant(torch.from_numpy(codes).cuda(), torch.from_numpy(scales).cuda(),
                           torch.tensor([ts], device="cuda"), out)
        got = out.cpu().numpy()
        ref = OF.nvfp4_dequant(codes, scales, ts).astype(np.float32)   # exact fp64 product, one rounding
        nan = np.isnan(ref)
        assert np.array_equal(np.isnan(got), nan)
        assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def test_dequant_bit_exact_random_bank():
    wl = workload("tiny_t4")
    inp = site_inputs(wl)
    for p, rows, K in (("gate", wl.I, wl.H), ("down", wl.H, wl.I)):
        for e in (0, 7, wl.E - 1):
            out = torch.empty((rows, K), dtype=torch.float32, device="cuda")
            capi.nvfp4_dequant(torch.from_numpy(inp[f"{p}_codes"][e]).cuda(),
                               torch.from_numpy(inp[f"{p}_scales"][e]).cuda(),
                               torch.from_numpy(inp[f"{p}_ts"][e:e + 1]).cuda(), out)
            ref = OF.nvfp4_dequant(inp[f"{p}_codes"][e], inp[f"{p}_scales"][e], inp[f"{p}_ts"][e]).astype(np.float32)
            assert np.array_equal(out.cpu().numpy().view(np.uint32), ref.view(np.uint32))


# ------------------------------------------------------------------ router

def _run_router(wl, inp):
    cfg = capi.config_for(wl)
    T = wl.T
    logits = torch.empty((T, wl.E), dtype=torch.float32, device="cuda")
    ids = torch.empty((T, wl.k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, wl.k), dtype=torch.float32, device="cuda")
    site = device_site(wl, inp)
    capi.moe_router_topk(cfg, _x(inp), site.router_w, site.router_bias, logits, ids, w)
    return logits.cpu().numpy(), ids.cpu().numpy(), w.cpu().numpy()


@pytest.mark.parametrize("name,T", [("tiny_t4", None), ("decode_t1", None), ("decode_t8", None),
                                    ("decode_t64", None), ("decode_t1", 300)])
def test_router_logits_ids_weights(name, T):
    wl = workload(name, T)
    inp = site_inputs(wl)
    lg, ids, w = _run_router(wl, inp)
    ref = OS.router_logits(inp["x"], inp["router_w"])
    scale = np.maximum(np.abs(ref), np.abs(ref).max(axis=1, keepdims=True))
    assert np.all(np.abs(lg - ref) <= LOGIT_REL * scale), np.abs(lg - ref).max()
    # ids: bit-exact against the oracle's selection on the GPU's own fp32 logits
    assert np.array_equal(ids, OS.select_experts(lg, inp["router_bias"], wl.k))
    wref = OS.routing_weights(ref, ids, wl.rsf)
    assert np.all(np.abs(w - wref) <= WEIGHT_REL * np.abs(wref)), np.abs(w - wref).max()


def test_router_exact_ties_and_k1():
    wl = workload("tiny_t4", T=40)
    inp = site_inputs(wl)
    inp["router_bias"][:] = np.float32(0.25)
    inp["x"][5:] = 0          # zero tokens: all keys equal -> lowest indices, weights exactly rsf/k
    lg, ids, w = _run_router(wl, inp)
    assert np.array_equal(ids[5:], np.tile(np.arange(wl.k, dtype=np.int32), (35, 1)))
    assert np.all(w[5:] == np.float32(wl.rsf / wl.k))
    assert np.array_equal(ids, OS.select_experts(lg, inp["router_bias"], wl.k))
    wl1 = workload("tiny_t4", k=1)
    _, _, w1 = _run_router(wl1, site_inputs(wl1))
    assert np.all(w1 == np.float32(wl1.rsf))


# ------------------------------------------------------------------ plan

def _plan_tensors(cfg, T):
    buf = torch.empty(capi.moe_plan_size(cfg, T), dtype=torch.uint8, device="cuda")
    return buf, capi.moe_plan_carve(cfg, T, buf)


def _read_plan(plan, E, A):
    def arr(ptr, n):
        return capi.view_tensor(ptr, (n,), torch.int32).cpu().numpy().copy()
    return dict(counts=arr(plan.counts, E), offsets=arr(plan.offsets, E + 1), sorted=arr(plan.sorted, A),
                inv=arr(plan.inv, A), tile_offsets=arr(plan.tile_offsets, E + 1), active=arr(plan.active, E + 1),
                first=arr(plan.first, E))


def _check_plan(got, ids, E, local=(0, None)):
    lb, le = local[0], local[1] if local[1] is not None else E
    ref = OS.permute(ids, E)
    A = ids.size
    for key in ("counts", "offsets", "sorted", "inv"):
        assert np.array_equal(got[key], ref[key]), key
    tiles = np.where((np.arange(E) >= lb) & (np.arange(E) < le), (ref["counts"] + 255) // 256, 0)   # 256-row tiles
    assert np.array_equal(got["tile_offsets"], np.concatenate([[0], np.cumsum(tiles)]))
    act = [e for e in range(lb, le) if ref["counts"][e] > 0]
    assert got["active"][0] == len(act) and np.array_equal(got["active"][1:1 + len(act)], act)
    assert np.array_equal(got["first"][:len(act)], [ref["sorted"][ref["offsets"][e]] for e in act])
    assert A == ref["offsets"][-1]


@pytest.mark.parametrize("T,E,k,local", [(1, 288, 8, (0, 288)), (64, 288, 8, (0, 288)), (100, 32, 4, (8, 20)),
                                          (4096, 288, 8, (0, 288)), (3000, 100, 6, (10, 90)),
                                          (16384, 288, 8, (0, 288))])
def test_permute_bit_exact(T, E, k, local):
    rng = np.random.default_rng(T + E)
    # skewed ids: 60% of picks from 10 experts, distinct per token
    hot = rng.choice(E, 10, replace=False)
    ids = np.empty((T, k), np.int32)
    for t in range(T):
        pool = np.concatenate([hot, rng.choice(E, 3 * k)]) if rng.random() < 0.6 else rng.permutation(E)
        _, first = np.unique(pool, return_index=True)
        ids[t] = pool[np.sort(first)][:k] if len(first) >= k else rng.choice(E, k, replace=False)
    cfg = capi.SiteConfig(256, 128, 0, E, local[0], local[1], k, 2.5, 7.0)
    buf, plan = _plan_tensors(cfg, T)
    ws = capi.alloc_workspace(cfg, T, capi.PATH_PREFILL)
    capi.moe_permute(cfg, torch.from_numpy(ids).cuda(), plan, ws)
    capi.moe_read_device_status(ws)
    _check_plan(_read_plan(plan, E, T * k), ids, E, local)


def test_permute_out_of_range_id_sets_bounds_status():
    E, k, T = 16, 2, 8
    ids = np.tile(np.array([[0, 1]], np.int32), (T, 1))
    ids[3, 1] = 99
    cfg = capi.SiteConfig(256, 128, 0, E, 0, E, k, 2.5, 7.0)
    buf, plan = _plan_tensors(cfg, T)
    ws = capi.alloc_workspace(cfg, T, capi.PATH_PREFILL)
    capi.moe_permute(cfg, torch.from_numpy(ids).cuda(), plan, ws)
    with pytest.raises(capi.MoEError) as ei:
        capi.moe_read_device_status(ws)
    assert ei.value.status == 6
    got = _read_plan(plan, E, T * k)
    assert got["offsets"][E] == T * k - 1 and got["inv"][7] == -1
    capi.moe_read_device_status(ws)          # cleared by the read


# ------------------------------------------------------------------ site

def _forward(wl, inp, local=None, rsf=None, limit=None, prepared=True):
    """One decode forward. With the prepared scale atoms, batches of 9 or more
    tokens run on the grouped W4A16 GEMM; without them, on the GEMV kernels."""
    cfg = capi.config_for(wl, local)
    if rsf is not None:
        cfg.routed_scaling_factor = rsf
    if limit is not None:
        cfg.swiglu_limit = limit
    site = device_site(wl, inp)
    if prepared:
        capi.moe_prepare_weights(cfg, site)
    x = _x(inp)
    y = torch.empty_like(x)
    ws = capi.alloc_workspace(cfg, wl.T, capi.PATH_DECODE)
    capi.moe_forward(cfg, site, x, capi.PATH_DECODE, y, ws)
    capi.moe_read_device_status(ws)
    v = capi.moe_workspace_views(cfg, wl.T, capi.PATH_DECODE, ws)
    logits = capi.view_tensor(v.logits, (wl.T, wl.E), torch.float32).cpu().numpy().copy()
    return y, logits, ws, v


@pytest.mark.parametrize("name,T,prepared", [("tiny_t4", None, True), ("tiny_t4", 33, True), ("tiny_t4", 33, False),
                                             ("decode_t1", None, True), ("decode_t8", None, True),
                                             ("decode_t32", None, True), ("decode_t32", None, False),
                                             ("decode_t64", None, True)])
def test_moe_forward_decode_matches_oracle(name, T, prepared):
    wl = workload(name, T)
    inp = site_inputs(wl)
    y, lg, ws, v = _forward(wl, inp, prepared=prepared)
    tokens = np.arange(wl.T) if wl.T <= 16 else np.random.default_rng(1).choice(wl.T, 16, replace=False)
    ref = OS.site_forward(inp, oracle_cfg(wl), "decode", tokens=tokens, gpu_logits=lg[tokens], want_parts=True)
    got = bf16_np(y)[tokens]
    assert_bf16_close(got, ref["y"], what=f"{wl.name} y")
    assert rel_l2(got, ref["y"]) < 5e-3
    # intermediates: per-assignment rows r[t, j] and the shared row (fp32 on
    # the decode path)
    r = capi.view_tensor(v.r, (wl.T, wl.k, wl.H), torch.float32)
    assert_bf16_close(bf16_np(r)[tokens], ref["r"], what="r")
    sh = capi.view_tensor(v.shared, (wl.T, wl.H), torch.float32)
    assert_bf16_close(bf16_np(sh)[tokens], ref["shared"], what="shared")


@pytest.mark.parametrize("name,T,local", [("decode_t1", None, None), ("decode_t8", None, None), ("tiny_t4", 1, None),
                                          ("tiny_t4", None, (3, 11)), ("tiny_t4", 8, (0, 8)), ("decode_t32", None, None)])
def test_forward_plan_matches_permute(name, T, local):
    """The decode forward builds the routing plan in the top-k launch when the
    tokens fit one top-k CTA (else with the permute kernels): either way the
    plan equals the oracle's permutation of the forward's own ids."""
    wl = workload(name, T)
    inp = site_inputs(wl)
    y, lg, ws, v = _forward(wl, inp, local=local)
    ids = capi.view_tensor(v.ids, (wl.T, wl.k), torch.int32).cpu().numpy().copy()
    _check_plan(_read_plan(v.plan, wl.E, wl.T * wl.k), ids, wl.E, local or (0, None))
    assert np.array_equal(ids, OS.select_experts(lg, inp["router_bias"], wl.k))


def test_moe_forward_is_deterministic():
    wl = workload("decode_t64")
    inp = site_inputs(wl)
    y1, _, _, _ = _forward(wl, inp)
    y2, _, _, _ = _forward(wl, inp)
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))


def test_shared_expert_never_scaled_on_gpu():
    wl = workload("tiny_t4")
    inp = site_inputs(wl)
    y0, _, _, v = _forward(wl, inp, rsf=0.0)
    sh = capi.view_tensor(v.shared, (wl.T, wl.H), torch.float32).to(torch.bfloat16)
    assert torch.equal(y0.view(torch.int16), sh.view(torch.int16))
    ya, _, _, _ = _forward(wl, inp, rsf=2.5)
    yb, _, _, _ = _forward(wl, inp, rsf=5.0)
    d1, d0 = bf16_np(yb) - bf16_np(ya), bf16_np(ya) - bf16_np(y0)
    assert rel_l2(d1, d0) < 2e-2


@pytest.mark.parametrize("name", ["tiny_t4", "decode_t8"])
def test_clamp_invisible_off_the_tails(name):
    wl = workload(name)
    inp = site_inputs(wl)
    y7, _, _, _ = _forward(wl, inp, limit=7.0)
    yinf, _, _, _ = _forward(wl, inp, limit=math.inf)
    assert torch.equal(y7.view(torch.int16), yinf.view(torch.int16))


@pytest.mark.parametrize("T", [16, 1])
def test_clamp_fires_on_tails_and_matches_oracle(T):
    """Activations x 64: the clamp fires on a large share of elements and the
    output still holds the elementwise gate (h, the routed rows and the shared
    row stay fp32 up to the one rounding of y)."""
    wl = workload("tiny_t4", T=T, x_scale=64.0)
    inp = site_inputs(wl)
    y, lg, ws, v = _forward(wl, inp)
    ref = OS.site_forward(inp, oracle_cfg(wl), "decode", gpu_logits=lg, want_parts=True)
    assert 0.05 * ref["clamp_total"] < ref["clamp_fired"] < ref["clamp_total"]
    got = bf16_np(y)
    assert_bf16_close(got, ref["y"], what="clamped y")


@pytest.mark.parametrize("T", [1, 12])
def test_local_range_masks_remote_experts(T):
    wl = workload("tiny_t4", T=T)
    inp = site_inputs(wl)
    for local in ((0, 8), (8, 16), (3, 3), (5, 11)):
        y, lg, _, _ = _forward(wl, inp, local=local)
        ref = OS.site_forward(inp, oracle_cfg(wl, local), "decode", gpu_logits=lg)
        assert_bf16_close(bf16_np(y), ref["y"], what=f"local {local}")


@pytest.mark.parametrize("name,T", [("tiny_t4", 9), ("tiny_t4", 1), ("decode_t1", 1)])
def test_expert_gemv_standalone_and_combine(name, T):
    wl = workload(name, T=T)
    inp = site_inputs(wl)
    cfg = capi.config_for(wl)
    site = device_site(wl, inp)
    T, k = wl.T, wl.k
    logits = torch.empty((T, wl.E), dtype=torch.float32, device="cuda")
    ids = torch.empty((T, k), dtype=torch.int32, device="cuda")
    w = torch.empty((T, k), dtype=torch.float32, device="cuda")
    capi.moe_router_topk(cfg, _x(inp), site.router_w, site.router_bias, logits, ids, w)
    buf, plan = _plan_tensors(cfg, T)
    ws = capi.alloc_workspace(cfg, T, capi.PATH_PREFILL)
    capi.moe_permute(cfg, ids, plan, ws)
    h = torch.empty((T * k, wl.I), dtype=torch.float32, device="cuda")
    r = torch.full((T, k, wl.H), 5.0, dtype=torch.float32, device="cuda")
    wsd = capi.alloc_workspace(cfg, T, capi.PATH_DECODE)
    capi.nvfp4_expert_gemv(cfg, capi.PROJ_GATE_UP, _x(inp), T, plan, None, site, h, wsd)
    capi.nvfp4_expert_gemv(cfg, capi.PROJ_DOWN, h, T, plan, w, site, r, wsd)
    capi.moe_read_device_status(wsd)
    y = torch.empty((T, wl.H), dtype=torch.bfloat16, device="cuda")
    capi.moe_combine(r, None, y)
    ref = OS.site_forward(inp, oracle_cfg(wl), "decode", gpu_logits=logits.cpu().numpy(), want_parts=True)
    assert_bf16_close(bf16_np(y), ref["y"] - ref["shared"], what="routed-only y")
    assert_bf16_close(bf16_np(r), ref["r"], what="r rows")
    # combine itself: fp32 sum of the fp32 rows in rank order, one rounding
    # (checked against torch)
    acc = r[:, 0].clone()
    for j in range(1, k):
        acc = acc + r[:, j]
    assert torch.equal(y.view(torch.int16), acc.to(torch.bfloat16).view(torch.int16))
    # and the bf16-row form
    rb = r.to(torch.bfloat16)
    yb = torch.empty_like(y)
    capi.moe_combine(rb, None, yb)
    accb = rb[:, 0].float()
    for j in range(1, k):
        accb = accb + rb[:, j].float()
    assert torch.equal(yb.view(torch.int16), accb.to(torch.bfloat16).view(torch.int16))


def test_clamped_swiglu_standalone():
    rng = np.random.default_rng(0)
    M, I = 37, 192
    gu = (rng.standard_normal((M, 2 * I)) * 6).astype(np.float32)
    h = torch.empty((M, I), dtype=torch.bfloat16, device="cuda")
    capi.clamped_swiglu(torch.from_numpy(gu).cuda(), 7.0, h)
    ref = OS.clamped_swiglu(gu[:, :I].astype(np.float64), gu[:, I:].astype(np.float64), 7.0)
    got = bf16_np(h)
    assert np.all(np.abs(got - ref) <= 2.0 ** -8 * np.abs(ref) + 1e-6)


@pytest.mark.parametrize("H,I,T", [(256, 512, 4), (256, 512, 19), (4096, 12288, 1), (4096, 1024, 8)])
def test_dense_ffn_decode_matches_oracle(H, I, T):
    from routed_nvfp4_expert_b200 import synthetic as syn
    wl = syn.Workload("dense", T=T, H=H, I=16, E=1, k=1, Is=0, dense_I=I, sigma_w=0.02 if H == 256 else 0.0064)
    d = syn.make_dense(wl)
    x = syn.make_router_and_x(wl)["x"]
    tb = capi.bf16_tensor
    y = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(capi.dense_ffn_workspace_size(H, I, T), dtype=torch.uint8, device="cuda")
    capi.dense_ffn_bf16(7.0, tb(x), tb(d["dense_gate"]), tb(d["dense_up"]), tb(d["dense_down"]), y, ws)
    ref = OS.dense_ffn(x, d["dense_gate"], d["dense_up"], d["dense_down"], 7.0)
    assert_bf16_close(bf16_np(y), ref, what="dense y")
    assert rel_l2(bf16_np(y), ref) < 5e-3


@pytest.mark.parametrize("H,I,T", [(256, 512, 300), (4096, 1024, 4096), (4096, 12288, 640)])
def test_dense_ffn_tensor_core_matches_oracle(H, I, T):
    """T >= 128 runs the tcgen05 BF16 GEMMs (ragged last m-tile at T=300);
    the oracle checks sampled tokens, the last rows included."""
    from routed_nvfp4_expert_b200 import synthetic as syn
    wl = syn.Workload("dense", T=T, H=H, I=16, E=1, k=1, Is=0, dense_I=I, sigma_w=0.02 if H == 256 else 0.0064)
    d = syn.make_dense(wl)
    x = syn.make_router_and_x(wl)["x"]
    tb = capi.bf16_tensor
    y = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    ws = torch.empty(capi.dense_ffn_workspace_size(H, I, T), dtype=torch.uint8, device="cuda")
    capi.dense_ffn_bf16(7.0, tb(x), tb(d["dense_gate"]), tb(d["dense_up"]), tb(d["dense_down"]), y, ws)
    capi.moe_read_device_status(ws)
    tok = np.unique(np.concatenate([np.random.default_rng(T).choice(T, 12, replace=False), [T - 1, T - 2, 0]]))
    ref = OS.dense_ffn(x[tok], d["dense_gate"], d["dense_up"], d["dense_down"], 7.0)
    got = bf16_np(y)[tok]
    assert_bf16_close(got, ref, what="dense y (tensor cores)")
    assert rel_l2(got, ref) < 5e-3


@pytest.mark.parametrize("name,T", [("tiny_t4", 1), ("tiny_t4", 8), ("mid", 1), ("mid", 8)])
def test_decode_on_quantised_bank(name, T):
    """Expert banks made by quantising Gaussian weights (tensor scale from the
    amax, block scales up to 448, codes at the largest magnitude), not drawn in
    the code domain: the decode forward still matches the oracle."""
    from helpers import with_quantised_banks
    from routed_nvfp4_expert_b200 import synthetic as syn
    if name == "mid":
        wl = syn.Workload("mid", T=T, H=1024, I=512, E=32, k=8, Is=512, dense_I=64, sigma_w=0.0064)
    else:
        wl = workload(name, T)
    inp = with_quantised_banks(wl, site_inputs(wl))
    assert (inp["gate_scales"] == 0x7E).any()
    cfg = capi.config_for(wl)
    site = capi.site_to_device(inp)
    x = _x(inp)
    y = torch.empty_like(x)
    ws = capi.alloc_workspace(cfg, wl.T, capi.PATH_DECODE)
    capi.moe_forward(cfg, site, x, capi.PATH_DECODE, y, ws)
    capi.moe_read_device_status(ws)
    v = capi.moe_workspace_views(cfg, wl.T, capi.PATH_DECODE, ws)
    lg = capi.view_tensor(v.logits, (wl.T, wl.E), torch.float32).cpu().numpy()
    ref = OS.site_forward(inp, oracle_cfg(wl), "decode", gpu_logits=lg)
    assert_bf16_close(bf16_np(y), ref["y"], what=f"{name} quantised-bank y")
    assert rel_l2(bf16_np(y), ref["y"]) < 5e-3


# ------------------------------------------------------------------ tensor-core decode kernels
#
# Up to 8 tokens with H a multiple of 1024 and I a multiple of 128 run the
# routed experts on the tensor cores (weights streamed straight into
# registers, mma.sync, one B column per token of an expert); these shapes
# cover one to sixteen 128-code steps per K quarter of a gate/up tile, one to
# sixteen steps of a down tile, 1 to 64 live experts, experts shared by
# several tokens (up to 8 columns), tiles that do not divide evenly over the
# SMs, the largest supported H and I, and sites without a shared expert.

def _t1(H, I, E, k, Is, T=1, **kw):
    from routed_nvfp4_expert_b200 import synthetic as syn
    return syn.Workload(f"mma_T{T}_H{H}_I{I}_E{E}_k{k}", T=T, H=H, I=I, E=E, k=k, Is=Is, dense_I=64,
                        sigma_w=kw.pop("sigma_w", 0.0064 if H >= 2048 else 0.02), **kw)


T1_SHAPES = [(1, 1024, 128, 32, 4, 256), (1, 3072, 768, 24, 6, 256), (1, 1024, 512, 40, 16, 0),
             (1, 2048, 1536, 20, 5, 128), (1, 8192, 2048, 12, 8, 512), (3, 1024, 256, 16, 4, 128),
             (8, 2048, 512, 24, 8, 256), (5, 4096, 1024, 40, 8, 0), (8, 1024, 128, 8, 8, 64)]


@pytest.mark.parametrize("T,H,I,E,k,Is", T1_SHAPES)
def test_t1_tensor_core_forward_matches_oracle(T, H, I, E, k, Is):
    wl = _t1(H, I, E, k, Is, T=T)
    inp = site_inputs(wl)
    y, lg, ws, v = _forward(wl, inp)
    ref = OS.site_forward(inp, oracle_cfg(wl), "decode", gpu_logits=lg, want_parts=True)
    got = bf16_np(y)
    assert_bf16_close(got, ref["y"], what=f"{wl.name} y")
    assert rel_l2(got, ref["y"]) < 5e-3
    r = capi.view_tensor(v.r, (T, k, H), torch.float32)
    assert_bf16_close(bf16_np(r), ref["r"], what="r")
    # h: the SwiGLU rows of the live assignments (fp32)
    h = capi.view_tensor(v.h, (T, k, I), torch.float32).cpu().numpy().astype(np.float64)
    cache = OS.ExpertCache(inp)
    a64 = OF.bf16_value(inp["x"])
    for t in range(T):
        for j in range(k):
            wg, wu, _ = cache.get(int(ref["ids"][t][j]))
            assert_bf16_close(h[t, j], OS.clamped_swiglu(wg @ a64[t], wu @ a64[t], wl.limit), what=f"h[{t},{j}]")
    # the same input twice: bit-identical (every sum in a fixed order)
    y2, _, _, _ = _forward(wl, inp)
    assert torch.equal(y.view(torch.int16), y2.view(torch.int16))


@pytest.mark.parametrize("local", [(0, 16), (16, 32), (7, 7), (5, 21)])
def test_t1_tensor_core_local_range(local):
    wl = _t1(1024, 256, 32, 8, 256)
    inp = site_inputs(wl)
    y, lg, _, v = _forward(wl, inp, local=local)
    ref = OS.site_forward(inp, oracle_cfg(wl, local), "decode", gpu_logits=lg, want_parts=True)
    assert_bf16_close(bf16_np(y), ref["y"], what=f"local {local}")
    r = capi.view_tensor(v.r, (1, wl.k, wl.H), torch.float32).cpu().numpy()
    remote = ~((ref["ids"][0] >= local[0]) & (ref["ids"][0] < local[1]))
    assert (r[0][remote] == 0).all()


def test_t1_tensor_core_clamp_fires_and_matches_oracle():
    wl = _t1(1024, 256, 32, 8, 256, x_scale=64.0)
    inp = site_inputs(wl)
    y, lg, _, _ = _forward(wl, inp)
    ref = OS.site_forward(inp, oracle_cfg(wl), "decode", gpu_logits=lg)
    assert 0.05 * ref["clamp_total"] < ref["clamp_fired"] < ref["clamp_total"]
    assert_bf16_close(bf16_np(y), ref["y"], what="clamped y")


def test_t1_tensor_core_standalone_gemv():
    """The expert GEMV entry point at T = 1 runs the same kernels: its h and r
    match the oracle and moe_combine of r gives the routed part of y."""
    wl = _t1(3072, 768, 24, 6, 0)
    inp = site_inputs(wl)
    cfg = capi.config_for(wl)
    site = device_site(wl, inp)
    k = wl.k
    logits = torch.empty((1, wl.E), dtype=torch.float32, device="cuda")
    ids = torch.empty((1, k), dtype=torch.int32, device="cuda")
    w = torch.empty((1, k), dtype=torch.float32, device="cuda")
    capi.moe_router_topk(cfg, _x(inp), site.router_w, site.router_bias, logits, ids, w)
    buf, plan = _plan_tensors(cfg, 1)
    wsp = capi.alloc_workspace(cfg, 1, capi.PATH_PREFILL)
    capi.moe_permute(cfg, ids, plan, wsp)
    h = torch.full((k, wl.I), 3.0, dtype=torch.float32, device="cuda")
    r = torch.full((1, k, wl.H), 5.0, dtype=torch.float32, device="cuda")
    wsd = capi.alloc_workspace(cfg, 1, capi.PATH_DECODE)
    capi.nvfp4_expert_gemv(cfg, capi.PROJ_GATE_UP, _x(inp), 1, plan, None, site, h, wsd)
    capi.nvfp4_expert_gemv(cfg, capi.PROJ_DOWN, h, 1, plan, w, site, r, wsd)
    capi.moe_read_device_status(wsd)
    y = torch.empty((1, wl.H), dtype=torch.bfloat16, device="cuda")
    capi.moe_combine(r, None, y)
    ref = OS.site_forward(inp, oracle_cfg(wl), "decode", gpu_logits=logits.cpu().numpy(), want_parts=True)
    assert_bf16_close(bf16_np(r), ref["r"], what="r rows")
    assert_bf16_close(bf16_np(y), ref["y"], what="routed y")
