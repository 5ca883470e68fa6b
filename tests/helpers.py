"""Shared test helpers: cached synthetic sites, tolerance checks."""
import dataclasses
import functools

import numpy as np
import torch

from oracle import site as OS
from routed_nvfp4_expert_b200 import synthetic as syn

# Output gate for bf16 results: relative L2 <= 1e-2 and max |d| <= 2e-2.
# Where |y_ref| >= 8 the one rounding of the result to bf16 alone can move it
# by up to 2^-8 |y_ref| > 2e-2, so there the bound is 2e-2 + 2^-8 |y_ref|.
OUT_REL_L2 = 1e-2
OUT_ABS = 2e-2
OUT_REL_ELEM = 2.0 ** -8
OUT_BIG = 8.0
LOGIT_REL = 1e-5       # relative to the token's largest |logit|
WEIGHT_REL = 1e-5


def rel_l2(got, ref) -> float:
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(got - ref) / den) if den > 0 else float(np.linalg.norm(got))


def assert_bf16_close(got, ref, rel=OUT_REL_L2, what="output"):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    r = rel_l2(got, ref)
    bound = OUT_ABS + np.where(np.abs(ref) >= OUT_BIG, OUT_REL_ELEM * np.abs(ref), 0.0)
    d = np.abs(got - ref)
    bad = d > bound
    assert r <= rel, f"{what}: rel-L2 {r:.3e} > {rel:.1e}"
    assert not bad.any(), f"{what}: {bad.sum()} elements off, worst |d|={d.max():.3e}"
    return r


def bf16_np(t: torch.Tensor) -> np.ndarray:
    """torch bf16 / fp32 (any device) -> fp64 numpy."""
    return t.detach().float().cpu().numpy().astype(np.float64)


def oracle_cfg(wl, local=None):
    lb, le = local if local is not None else (0, wl.E)
    return OS.SiteConfig(wl.H, wl.I, wl.Is, wl.E, lb, le, wl.k, wl.rsf, wl.limit)


def workload(name: str, T: int | None = None, **kw):
    wl = syn.WORKLOADS[name]
    if T is not None and T != wl.T:
        wl = dataclasses.replace(wl, T=T, name=f"{name}_t{T}")
    if kw:
        wl = dataclasses.replace(wl, **kw)
    return wl


def _geom(wl):
    return (wl.H, wl.I, wl.E, wl.Is, wl.sigma_w)


@functools.lru_cache(maxsize=2)
def _weights(geom):
    H, I, E, Is, sw = geom
    wl = syn.Workload("w", T=1, H=H, I=I, E=E, k=1, Is=Is, dense_I=64, sigma_w=sw)
    out = syn.make_experts(wl)
    out.update(syn.make_shared(wl))
    return out


def site_inputs(wl):
    """Full site inputs; the expert / shared banks are cached per geometry."""
    inp = {"workload": wl}
    inp.update(syn.make_router_and_x(wl))
    inp.update(_weights(_geom(wl)))
    return inp


@functools.lru_cache(maxsize=2)
def _device_weights(geom):
    import torch as _t
    from routed_nvfp4_expert_b200 import capi
    w = _weights(geom)
    banks = {p: tuple(_t.from_numpy(w[f"{p}_{s}"]).cuda() for s in ("codes", "scales", "ts"))
             for p in ("gate", "up", "down")}
    shared = None
    if "shared_gate" in w:
        shared = tuple(capi.bf16_tensor(w[f"shared_{p}"]) for p in ("gate", "up", "down"))
    return banks, shared


def device_site(wl, inp):
    """DeviceSite for wl: cached expert / shared banks + this workload's router."""
    import torch as _t
    from routed_nvfp4_expert_b200 import capi
    banks, shared = _device_weights(_geom(wl))
    return capi.DeviceSite(_t.from_numpy(inp["router_w"]).cuda(), _t.from_numpy(inp["router_bias"]).cuda(),
                           banks, shared)


def quantised_bank(seed: int, E: int, rows: int, cols: int, sigma: float):
    """An NVFP4 bank made the way a checkpoint's would be: weights N(0, sigma)
    (fp32) quantised per expert with tensor scale ts = amax / (6 * 448), block
    scale = E4M3 round-to-nearest of amax_block / 6 / ts, code = E2M1
    round-to-nearest of w / (scale * ts). The roundings are ml_dtypes' casts,
    so this data shares nothing with either side under test. Test data only.

    Returns codes uint8 [E, rows, cols/2], scales uint8 [E, rows, cols/16],
    ts float32 [E] (the canonical layout)."""
    import ml_dtypes
    rng = np.random.default_rng(seed)
    codes = np.empty((E, rows, cols // 2), np.uint8)
    scales = np.empty((E, rows, cols // 16), np.uint8)
    ts = np.empty(E, np.float32)
    for e in range(E):
        w = (rng.standard_normal((rows, cols), dtype=np.float32) * np.float32(sigma)).astype(np.float32)
        t = np.float32(np.abs(w).max() / np.float32(6 * 448))
        blk = np.abs(w).reshape(rows, cols // 16, 16).max(axis=2)
        q = np.minimum((blk / np.float32(6)) / t, np.float32(448)).astype(np.float32)
        sb = q.astype(ml_dtypes.float8_e4m3fn)
        d = (sb.astype(np.float32) * t).astype(np.float32)
        ratio = np.where(d[:, :, None] > 0, w.reshape(rows, cols // 16, 16) / d[:, :, None], 0.0)
        ratio = np.clip(ratio.astype(np.float32), -6, 6)
        c = ratio.astype(ml_dtypes.float4_e2m1fn).view(np.uint8).reshape(rows, cols) & 0xF
        codes[e] = (c[:, 0::2] | (c[:, 1::2] << 4)).astype(np.uint8)
        scales[e] = sb.view(np.uint8)
        ts[e] = t
    return codes, scales, ts


def with_quantised_banks(wl, inp: dict, seed: int = 3) -> dict:
    """inp with its three expert banks replaced by quantised_bank() ones."""
    out = dict(inp)
    for i, (proj, rows, cols) in enumerate((("gate", wl.I, wl.H), ("up", wl.I, wl.H), ("down", wl.H, wl.I))):
        c, s, t = quantised_bank(seed * 10 + i, wl.E, rows, cols, wl.sigma_w)
        out[f"{proj}_codes"], out[f"{proj}_scales"], out[f"{proj}_ts"] = c, s, t
    return out
