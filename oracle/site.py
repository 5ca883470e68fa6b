"""The routed MoE MLP site and the dense FFN, as a plain fp64 CPU computation.

TEST INFRASTRUCTURE: the CPU oracle. Only ``tests/``, ``__graft_entry__.smoke()``
and ``bench.py``'s CPU-baseline / reference legs import this package. The CUDA
path shares no code with it and never calls it.

What it follows (glm5next_mlp module docs, GLM-5.3-Flash MLP surface):
* "The stack this layer runs": DENSE layers run gate_proj/up_proj -> clamped
  SwiGLU -> down_proj; ROUTED layers run gate.weight -> fp32 logits ->
  router_topk -> ids[K], weights[K]; every chosen LOCAL expert runs NVFP4
  gate/up -> clamped SwiGLU -> NVFP4 down; the shared expert runs BF16 gate/up
  -> clamped SwiGLU -> BF16 down; moe_combine sums the two partials.
* "Traps this module exists to hold": the clamp is asymmetric (gate bounded
  above only, up bounded on both sides) with the limit swiglu_limit; the
  correction bias steers selection only and the emitted weight is the
  unbiased sigmoid score; routed_scaling_factor multiplies the top-k weights
  and never the shared expert; num_experts is the full count and the local
  range is separate (ids outside it contribute zero, "Why one all-reduce
  covers BOTH EP and TP").
* Constants, KERNEL_MAX_TOP_K: at most 16 experts per token.
* TensorRT-LLM PR #19136 "Test Coverage": the router gate is fp32.

Readings where the pages are silent (each is listed in the design notes):
SwiGLU is silu(min(g, L)) * clamp(u, -L, L); the bias is added to the sigmoid
score, key = fl32(fl32(sigmoid(l)) + b); equal keys go to the lower expert
index; renormalisation has no epsilon; the combine sums the k routed rows in
rank order, then the shared row; prefill runs NVFP4 activations (W4A4) with a
per-token-row second-level scale, and h is rounded to bf16 before it is
quantised.

Everything is fp64 except the selection, which runs on fp32 logits (the GPU's
own, when given) with a correctly rounded fp32 sigmoid and an fp32 add, and
the activation encoding, which is specified in IEEE fp32.

Parity pins: tests/test_oracle_pins.py (brute-force top-k over every subset,
k = 1, zero token, exact-tie tokens, bias / shared-scale / clamp invariants,
the E = k = 1 reduction to a textbook SwiGLU MLP checked with torch, the
hand-computed permutation and combine examples).
"""
from __future__ import annotations

import dataclasses

import numpy as np

from . import formats as F

MAX_TOP_K = 16          # glm5next_mlp Constants, KERNEL_MAX_TOP_K
ROWS_PER_TILE = 128     # M extent of one grouped-GEMM tile (tile_offsets)


@dataclasses.dataclass
class SiteConfig:
    """Geometry of one site; every field must be given (nothing defaulted)."""
    hidden: int
    intermediate: int
    shared_intermediate: int
    num_experts: int          # FULL count
    local_begin: int
    local_end: int
    top_k: int
    routed_scaling_factor: float
    swiglu_limit: float


# ---------------------------------------------------------------- router

def router_logits(x_bits, router_w) -> np.ndarray:
    """l[t, e] = sum_i Wr[e, i] * x[t, i], in fp64 (gate.weight applied to x)."""
    return F.bf16_value(x_bits) @ np.asarray(router_w, np.float32).astype(np.float64).T


def sigmoid_f32(logits_f32) -> np.ndarray:
    """fl32(1 / (1 + exp(-l))), evaluated in fp64 and rounded once to fp32."""
    l = np.asarray(logits_f32, np.float32).astype(np.float64)
    with np.errstate(over="ignore"):
        return (1.0 / (1.0 + np.exp(-l))).astype(np.float32)


def selection_keys(logits_f32, bias_f32) -> np.ndarray:
    """key = fl32(sigmoid_f32(l) + b): the bias enters the selection only."""
    s = sigmoid_f32(logits_f32)
    return (s + np.asarray(bias_f32, np.float32)).astype(np.float32)


def select_experts(logits_f32, bias_f32, k: int) -> np.ndarray:
    """Top-k expert ids per token, in rank order: key descending, an equal key
    goes to the lower expert index, NaN keys rank last."""
    key = selection_keys(logits_f32, bias_f32)
    T, E = key.shape
    if not 1 <= k <= min(MAX_TOP_K, E):
        raise ValueError("top_k out of range")
    nan = np.isnan(key)
    neg = np.where(nan, 0.0, -key.astype(np.float64))
    idx = np.broadcast_to(np.arange(E), (T, E))
    order = np.lexsort((idx, neg, nan), axis=-1)     # last key is primary
    return order[:, :k].astype(np.int32)


def routing_weights(logits64, ids, rsf: float) -> np.ndarray:
    """w_j = rsf * s_j / sum_{chosen} s, with s the UNBIASED sigmoid of the
    oracle's own fp64 logits; a zero denominator gives zero weights."""
    with np.errstate(over="ignore"):
        s = 1.0 / (1.0 + np.exp(-np.asarray(logits64, np.float64)))
    chosen = np.take_along_axis(s, np.asarray(ids, np.int64), axis=1)
    den = chosen.sum(axis=1, keepdims=True)
    with np.errstate(divide="ignore", invalid="ignore"):
        w = np.where(den > 0, float(rsf) * (chosen / den), 0.0)
    return w


# ---------------------------------------------------------------- MLP pieces

def clamped_swiglu(g, u, limit: float) -> np.ndarray:
    """h = silu(min(g, L)) * clamp(u, -L, L); silu(z) = z / (1 + exp(-z))."""
    gc = np.minimum(np.asarray(g, np.float64), limit)
    uc = np.clip(np.asarray(u, np.float64), -limit, limit)
    with np.errstate(over="ignore"):
        return gc / (1.0 + np.exp(-gc)) * uc


def clamp_fired(g, u, limit: float) -> np.ndarray:
    """Elements where the clamp changes an input: g > L, or |u| > L."""
    return (np.asarray(g) > limit) | (np.abs(np.asarray(u)) > limit)


def mlp(a64, wg64, wu64, wd64, limit: float, h_hook=None):
    """down(clamped_swiglu(gate a, up a)); weights are [out, in] in fp64.
    ``h_hook`` (prefill) re-encodes h before the down projection.
    Returns (out, g, u)."""
    g = a64 @ wg64.T
    u = a64 @ wu64.T
    h = clamped_swiglu(g, u, limit)
    if h_hook is not None:
        h = h_hook(h)
    return h @ wd64.T, g, u


def prefill_activation(x_bits) -> np.ndarray:
    """Prefill activations: x (bf16) encoded as NVFP4 per token row, dequantised."""
    xf = F.bf16_value(x_bits).astype(np.float32)
    c, s, t = F.quantize_rows_nvfp4(xf)
    return F.dequant_rows_nvfp4(c, s, t)


def prefill_h(h64) -> np.ndarray:
    """Prefill h: fl32, rounded to bf16, encoded as NVFP4 per row, dequantised."""
    hb = F.f32_to_bf16_bits(np.asarray(h64, np.float64).astype(np.float32))
    hf = F.bf16_value(hb).astype(np.float32)
    c, s, t = F.quantize_rows_nvfp4(hf)
    return F.dequant_rows_nvfp4(c, s, t)


# ---------------------------------------------------------------- permutation

def permute(ids, num_experts: int, rows_per_tile: int = ROWS_PER_TILE) -> dict:
    """Group the A = T*k assignments (a = t*k + j) by expert, stably.

    counts[e]        assignments of expert e
    offsets[e]       start of expert e's segment (offsets[E] = A)
    sorted[p]        assignment at sorted position p
    inv[a]           sorted position of assignment a
    tile_offsets[e]  first 128-row tile of expert e (tile_offsets[E] = tiles)
    """
    flat = np.asarray(ids, np.int64).reshape(-1)
    A = flat.size
    counts = np.bincount(flat, minlength=num_experts).astype(np.int32)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    srt = np.argsort(flat, kind="stable").astype(np.int32)
    inv = np.empty(A, np.int32)
    inv[srt] = np.arange(A, dtype=np.int32)
    tiles = (counts + rows_per_tile - 1) // rows_per_tile
    tile_offsets = np.concatenate([[0], np.cumsum(tiles)]).astype(np.int32)
    return dict(counts=counts, offsets=offsets, sorted=srt, inv=inv, tile_offsets=tile_offsets)


def combine(r_tkh, shared_th=None) -> np.ndarray:
    """moe_combine: y[t] = sum_j r[t, j] + shared[t] (shared never scaled)."""
    y = np.asarray(r_tkh, np.float64).sum(axis=1)
    if shared_th is not None:
        y = y + np.asarray(shared_th, np.float64)
    return y


# ---------------------------------------------------------------- whole site

class ExpertCache:
    """Dequantised experts, built on demand (the full bank can be GBs)."""

    def __init__(self, inp: dict):
        self.inp = inp
        self._d: dict = {}

    def get(self, e: int):
        if e not in self._d:
            i = self.inp
            self._d[e] = tuple(
                F.nvfp4_dequant(i[f"{p}_codes"][e], i[f"{p}_scales"][e], i[f"{p}_ts"][e])
                for p in ("gate", "up", "down"))
        return self._d[e]


def site_forward(inp: dict, cfg: SiteConfig, mode: str, tokens=None,
                 gpu_logits=None, cache: ExpertCache | None = None,
                 want_parts: bool = False) -> dict:
    """One routed site forward for the given tokens (default: all).

    mode 'decode'  : W4A16 -- bf16 activations go straight into the NVFP4 experts.
    mode 'prefill' : W4A4  -- x and h are NVFP4-encoded per token row.
    gpu_logits     : fp32 logits [T', E] to run the selection on (the GPU's own);
                     default: the oracle's logits rounded to fp32.
    Returns y (fp64 [T', H]) plus logits, ids, weights, and, on request, the
    per-assignment rows r[t, j] = w_j * o_j and the shared row.
    """
    x_all = np.asarray(inp["x"])
    tok = np.arange(x_all.shape[0]) if tokens is None else np.asarray(tokens)
    x_bits = x_all[tok]
    Tn, H = x_bits.shape
    k, E = cfg.top_k, cfg.num_experts
    L = float(cfg.swiglu_limit)
    cache = cache or ExpertCache(inp)

    logits64 = router_logits(x_bits, inp["router_w"])
    sel_logits = logits64.astype(np.float32) if gpu_logits is None else np.asarray(gpu_logits, np.float32)
    ids = select_experts(sel_logits, inp["router_bias"], k)
    w = routing_weights(logits64, ids, cfg.routed_scaling_factor)

    if mode == "prefill":
        a64 = prefill_activation(x_bits)
        hook = prefill_h
    elif mode == "decode":
        a64 = F.bf16_value(x_bits)
        hook = None
    else:
        raise ValueError(mode)

    r = np.zeros((Tn, k, H), np.float64)
    fired = 0
    total = 0
    for e in np.unique(ids):
        if not (cfg.local_begin <= e < cfg.local_end):
            continue                       # remote expert: contributes zero
        rows, slots = np.nonzero(ids == e)
        wg, wu, wd = cache.get(int(e))
        o, g, u = mlp(a64[rows], wg, wu, wd, L, hook)
        fired += int(clamp_fired(g, u, L).sum())
        total += g.size
        r[rows, slots] = w[rows, slots, None] * o

    shared = None
    if cfg.shared_intermediate > 0:
        xs = F.bf16_value(x_bits)
        shared, _, _ = mlp(xs, F.bf16_value(inp["shared_gate"]), F.bf16_value(inp["shared_up"]),
                           F.bf16_value(inp["shared_down"]), L)
    y = combine(r, shared)
    out = dict(y=y, logits=logits64, sel_logits=sel_logits, ids=ids, weights=w,
               clamp_fired=fired, clamp_total=total, tokens=tok)
    if want_parts:
        out.update(r=r, shared=shared)
    return out


def dense_ffn(x_bits, wg_bits, wu_bits, wd_bits, limit: float) -> np.ndarray:
    """Dense BF16 FFN: down_proj(clamped_swiglu(gate_proj x, up_proj x)), fp64."""
    y, _, _ = mlp(F.bf16_value(x_bits), F.bf16_value(wg_bits), F.bf16_value(wu_bits),
                  F.bf16_value(wd_bits), limit)
    return y
