"""Seeded synthetic inputs for the routed NVFP4 MoE site and the dense FFN.

This module only draws random numbers. It holds no step of the site's
arithmetic: no dequantisation, no rounding to E2M1 or E4M3, no router, no
SwiGLU. NVFP4 expert weights are drawn directly in the encoded domain:

* E2M1 nibbles: magnitude index from a fixed 128-level histogram (close to
  the code histogram of a Gaussian block quantised with its maximum mapped to
  the largest code), sign from a fair bit. Even element in the low nibble.
* E4M3 block-scale bytes (one per 16 consecutive K elements): exponent field
  12, 13 or 14 with probabilities 1/4, 1/2, 1/4 and a uniform 3-bit mantissa,
  i.e. scales in [32, 240].
* One fp32 tensor scale per expert and projection: base * (0.9 + 0.2 u),
  u ~ U[0,1). With the two histograms above the RMS of (E2M1 value x E4M3
  scale) is sqrt(8.2734 * 13750) = 337.27, so base = sigma_w / 337.27 gives
  dequantised weights of standard deviation close to sigma_w.

bf16 tensors are drawn in fp32 from numpy and rounded to bf16 by torch (a
library conversion), then kept as raw uint16 bit patterns. Every tensor has
its own stream: numpy ``SeedSequence([seed, tensor_id])``.

The CUDA path and the CPU oracle both consume exactly the bytes produced here.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch

# magnitude index histogram (units of 1/128) for E2M1 magnitudes
# {0, 0.5, 1, 1.5, 2, 3, 4, 6}
_MAG_HIST_128 = (8, 17, 16, 15, 20, 21, 19, 12)
# RMS of (E2M1 value * E4M3 block scale) under the two histograms
_RMS_CODE_TIMES_SCALE = 337.27

_TENSOR_IDS = {
    "x": 1, "router_w": 2, "router_bias": 3,
    "gate_codes": 4, "gate_scales": 5, "gate_ts": 6,
    "up_codes": 7, "up_scales": 8, "up_ts": 9,
    "down_codes": 10, "down_scales": 11, "down_ts": 12,
    "shared_gate": 13, "shared_up": 14, "shared_down": 15,
    "dense_gate": 16, "dense_up": 17, "dense_down": 18,
    "stress_set": 19, "stress_tokens": 20, "stress_column": 21,
}


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic workload: MoE site geometry plus the dense FFN beside it."""
    name: str
    T: int                 # tokens
    H: int                 # hidden size
    I: int                 # routed expert intermediate size
    E: int                 # experts (full count)
    k: int                 # top-k
    Is: int                # shared expert intermediate (0 = none)
    dense_I: int           # dense FFN intermediate size (hidden = H)
    sigma_w: float         # std of expert / shared / dense weights
    x_scale: float = 1.0   # activations are x_scale * N(0,1)
    stress: bool = False   # skewed bias on 16 experts + 1% exactly tied tokens
    rsf: float = 2.5       # routed_scaling_factor
    limit: float = 7.0     # swiglu_limit
    kind: str = "decode"   # "decode" (GEMV path), "prefill" (grouped GEMM path) or "dense" (the dense FFN)

    def with_tokens(self, T: int, name: str | None = None) -> "Workload":
        return dataclasses.replace(self, T=T, name=name or f"{self.name}_t{T}")


def _w(name, T, kind, **kw):
    base = dict(H=4096, I=1024, E=288, k=8, Is=1024, dense_I=12288, sigma_w=0.0064)
    base.update(kw)
    return Workload(name=name, T=T, kind=kind, **base)


WORKLOADS: dict[str, Workload] = {
    # tiny site: T=4, hidden 256, 16 experts (I=128), top-4, shared I=128, dense I=512
    "tiny_t4": Workload("tiny_t4", T=4, H=256, I=128, E=16, k=4, Is=128, dense_I=512,
                        sigma_w=0.02, kind="decode"),
    "decode_t1": _w("decode_t1", 1, "decode"),
    # multi-token verification steps of speculative decoding (T = 2, 4 per user)
    "decode_t2": _w("decode_t2", 2, "decode"),
    "decode_t4": _w("decode_t4", 4, "decode"),
    "decode_t8": _w("decode_t8", 8, "decode"),
    "decode_t32": _w("decode_t32", 32, "decode"),
    "decode_t64": _w("decode_t64", 64, "decode"),
    "prefill_t4096": _w("prefill_t4096", 4096, "prefill"),
    "stress_t16384": _w("stress_t16384", 16384, "prefill", x_scale=8.0, stress=True),
    # the dense BF16 FFN of the first_k_dense_replace layers at H = 4096, I = 12288
    "dense_t4096": _w("dense_t4096", 4096, "dense"),
    "dense_t1": _w("dense_t1", 1, "dense"),
}


def _rng(seed: int, name: str) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, _TENSOR_IDS[name]])))


def _to_bf16_bits(a: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def _nibble_table() -> np.ndarray:
    mags = np.repeat(np.arange(8, dtype=np.uint8), _MAG_HIST_128)   # 128 entries
    assert mags.size == 128
    b = np.arange(256, dtype=np.uint8)
    return (mags[b & 127] | ((b >> 7) << 3)).astype(np.uint8)


_NIB = _nibble_table()
# two random bytes (little-endian uint16) -> one packed byte of two nibbles
_NIB_PAIR = (_NIB[np.arange(65536) & 0xFF] | (_NIB[np.arange(65536) >> 8] << 4)).astype(np.uint8)


def _scale_table() -> np.ndarray:
    # random byte -> E4M3 byte: bits 0-2 mantissa, bits 3-4 exponent choice
    b = np.arange(256, dtype=np.int64)
    choice = (b >> 3) & 3
    exp_field = np.array([12, 13, 13, 14])[choice]
    return ((exp_field << 3) | (b & 7)).astype(np.uint8)


_SCALE = _scale_table()


def nvfp4_bank(seed: int, proj: str, E: int, rows: int, cols: int, sigma_w: float):
    """Random NVFP4 bank for E experts of shape [rows, cols] (K = cols contiguous).

    Returns codes uint8 [E, rows, cols/2], scales uint8 [E, rows, cols/16],
    tensor_scale float32 [E].
    """
    assert cols % 16 == 0
    rc = _rng(seed, f"{proj}_codes")
    rs = _rng(seed, f"{proj}_scales")
    rt = _rng(seed, f"{proj}_ts")
    codes = np.empty((E, rows, cols // 2), np.uint8)
    scales = np.empty((E, rows, cols // 16), np.uint8)
    for e in range(E):
        raw = np.frombuffer(rc.bytes(rows * cols), dtype="<u2").reshape(rows, cols // 2)
        codes[e] = _NIB_PAIR[raw]
        rawsc = np.frombuffer(rs.bytes(rows * cols // 16), dtype=np.uint8).reshape(rows, cols // 16)
        scales[e] = _SCALE[rawsc]
    base = sigma_w / _RMS_CODE_TIMES_SCALE
    ts = (base * (0.9 + 0.2 * rt.random(E))).astype(np.float32)
    return codes, scales, ts


def bf16_matrix(seed: int, name: str, rows: int, cols: int, sigma: float) -> np.ndarray:
    r = _rng(seed, name)
    return _to_bf16_bits(r.standard_normal((rows, cols), dtype=np.float32) * np.float32(sigma))


def make_router_and_x(wl: Workload, seed: int = 0) -> dict:
    """x bf16 [T, H], router_w fp32 [E, H], router_bias fp32 [E] (+ the stress set-up)."""
    T, H, E = wl.T, wl.H, wl.E
    out: dict = {}
    rx = _rng(seed, "x")
    x = rx.standard_normal((T, H), dtype=np.float32) * np.float32(wl.x_scale)
    rw = _rng(seed, "router_w")
    router_w = (rw.standard_normal((E, H), dtype=np.float32) * np.float32(1.0 / math.sqrt(H))).astype(np.float32)
    rb = _rng(seed, "router_bias")
    bias = (rb.standard_normal(E, dtype=np.float32) * np.float32(0.5)).astype(np.float32)
    if wl.stress:
        # 16 experts get bias exactly +3; their router column j* is zero; 1% of
        # tokens are 8 * e_{j*}, which gives those 16 experts exactly equal keys.
        S = np.sort(_rng(seed, "stress_set").choice(E, 16, replace=False))
        jstar = int(_rng(seed, "stress_column").integers(H))
        n_tie = max(1, round(0.01 * T))
        tie_tokens = np.sort(_rng(seed, "stress_tokens").choice(T, n_tie, replace=False))
        bias[S] = np.float32(3.0)
        router_w[S, jstar] = np.float32(0.0)
        x[tie_tokens] = 0.0
        x[tie_tokens, jstar] = 8.0
        out.update(skew_set=S, tie_column=jstar, tie_tokens=tie_tokens)
    out["x"] = _to_bf16_bits(x)
    out["router_w"] = router_w
    out["router_bias"] = bias
    return out


def make_experts(wl: Workload, seed: int = 0) -> dict:
    """NVFP4 banks: gate/up [E, I, H], down [E, H, I] (codes, scales, tensor scales)."""
    out: dict = {}
    for proj, rows, cols in (("gate", wl.I, wl.H), ("up", wl.I, wl.H), ("down", wl.H, wl.I)):
        c, s, t = nvfp4_bank(seed, proj, wl.E, rows, cols, wl.sigma_w)
        out[f"{proj}_codes"], out[f"{proj}_scales"], out[f"{proj}_ts"] = c, s, t
    return out


def make_shared(wl: Workload, seed: int = 0) -> dict:
    """BF16 shared expert: gate/up [Is, H], down [H, Is] (empty when Is == 0)."""
    if wl.Is <= 0:
        return {}
    return {
        "shared_gate": bf16_matrix(seed, "shared_gate", wl.Is, wl.H, wl.sigma_w),
        "shared_up": bf16_matrix(seed, "shared_up", wl.Is, wl.H, wl.sigma_w),
        "shared_down": bf16_matrix(seed, "shared_down", wl.H, wl.Is, wl.sigma_w),
    }


def make_site(wl: Workload, seed: int = 0, with_dense: bool = False) -> dict:
    """All inputs of one MoE site forward (and optionally the dense FFN)."""
    out: dict = {"workload": wl}
    out.update(make_router_and_x(wl, seed))
    out.update(make_experts(wl, seed))
    out.update(make_shared(wl, seed))
    if with_dense:
        out.update(make_dense(wl, seed))
    return out


def make_dense(wl: Workload, seed: int = 0) -> dict:
    """Dense BF16 FFN weights at hidden H, intermediate dense_I."""
    return {
        "dense_gate": bf16_matrix(seed, "dense_gate", wl.dense_I, wl.H, wl.sigma_w),
        "dense_up": bf16_matrix(seed, "dense_up", wl.dense_I, wl.H, wl.sigma_w),
        "dense_down": bf16_matrix(seed, "dense_down", wl.H, wl.dense_I, wl.sigma_w),
    }


def random_x(wl: Workload, T: int, seed: int) -> np.ndarray:
    """Fresh bf16 activations [T, H] (x_scale * N(0,1)), for rotating inputs."""
    r = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, 1000 + T])))
    return _to_bf16_bits(r.standard_normal((T, wl.H), dtype=np.float32) * np.float32(wl.x_scale))
