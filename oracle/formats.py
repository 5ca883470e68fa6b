"""Number formats of the MoE site, written out plainly in fp64 / IEEE fp32.

TEST INFRASTRUCTURE: the CPU oracle. Only ``tests/``, ``__graft_entry__.smoke()``
and ``bench.py``'s CPU-baseline / reference legs import this package. The CUDA
path shares no code with it and never calls it.

Sources:
* E2M1 -- OCP Microscaling Formats (MX) Specification v1.0, FP4 (E2M1):
  1 sign bit, 2 exponent bits (bias 1), 1 mantissa bit, no Inf/NaN,
  values +-{0, 0.5, 1, 1.5, 2, 3, 4, 6}.
* E4M3 -- OCP 8-bit Floating Point Specification (OFP8), E4M3: bias 7,
  subnormals m/8 * 2^-6, S.1111.111 is NaN, no infinities, max 448.
* NVFP4 (the expert format of the glm5next_mlp module docs, section "The stack
  this layer runs": "NVFP4 gate/up -> clamped SwiGLU -> NVFP4 down"): E2M1
  values, one E4M3 scale per 16 consecutive elements along K, one fp32 scale
  per tensor; an element's value is e2m1 * e4m3 * tensor_scale. Layout
  reading: row-major [rows, K], two codes per byte, even element in the low
  nibble; scales row-major [rows, K/16].
* bf16 -- the upper 16 bits of an IEEE binary32.

Parity pins (tests/test_oracle_pins.py): exhaustive E2M1/E4M3 tables against
the specs and against ml_dtypes; encoder ties against hand-derived tables and
against ml_dtypes on every midpoint; a hand-computed activation-quant example
(tests/golden/act_quant_example.txt); a hand-computed dequant dot product.
"""
from __future__ import annotations

import numpy as np

E2M1_MAX = 6.0
E4M3_MAX = 448.0
# second-level activation scale: max |row| maps to E2M1 max * E4M3 max
ACT_ROW_SCALE_DIVISOR = np.float32(6.0 * 448.0)   # 2688


def e2m1_value(code) -> np.ndarray:
    """fp64 value of 4-bit E2M1 codes (sign = bit 3)."""
    c = np.asarray(code, dtype=np.int64) & 0xF
    sign = np.where(c & 0x8, -1.0, 1.0)
    e = (c >> 1) & 0x3
    m = (c & 0x1).astype(np.float64)
    mag = np.where(e == 0, 0.5 * m, np.ldexp(1.0 + 0.5 * m, (e - 1).astype(np.int64)))
    return sign * mag


def e4m3_value(byte) -> np.ndarray:
    """fp64 value of E4M3 ('fn' variant) bytes; 0x7F / 0xFF are NaN."""
    b = np.asarray(byte, dtype=np.int64) & 0xFF
    sign = np.where(b & 0x80, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = (b & 0x7).astype(np.float64)
    normal = np.ldexp(1.0 + m / 8.0, (e - 7).astype(np.int64))
    subnormal = np.ldexp(m / 8.0, -6)
    mag = np.where(e == 0, subnormal, normal)
    mag = np.where((e == 15) & ((b & 7) == 7), np.nan, mag)
    return sign * mag


def bf16_value(bits) -> np.ndarray:
    """fp64 value of bf16 bit patterns (exact widening)."""
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def f32_to_bf16_bits(a) -> np.ndarray:
    """Round fp32 to bf16, round-to-nearest-even on the dropped 16 bits."""
    f = np.ascontiguousarray(a, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    nan = np.isnan(f)
    r[nan] = (u[nan] >> 16).astype(np.uint16) | 0x0040   # keep NaN a (quiet) NaN
    return r


def _round_magnitude(mag: np.ndarray, grid: np.ndarray) -> np.ndarray:
    """Index into ``grid`` (ascending non-negative representable magnitudes,
    index = code) nearest to ``mag``; an exact tie goes to the even code;
    magnitudes above the last grid point saturate to it."""
    mag = np.asarray(mag, dtype=np.float64)
    hi = np.searchsorted(grid, mag, side="left")          # grid[hi-1] < mag <= grid[hi]
    hi = np.clip(hi, 1, grid.size - 1)
    lo = hi - 1
    d_lo = mag - grid[lo]
    d_hi = grid[hi] - mag
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    idx = np.where(pick_hi, hi, lo)
    idx = np.where(mag >= grid[-1], grid.size - 1, idx)
    idx = np.where(mag <= grid[0], 0, idx)
    return idx


_E2M1_GRID = e2m1_value(np.arange(8))                      # 0, .5, 1, 1.5, 2, 3, 4, 6
_E4M3_GRID = e4m3_value(np.arange(0x7F))                   # 0 .. 448, codes 0x00..0x7E


def e2m1_encode_satfinite(v) -> np.ndarray:
    """fp32 -> E2M1 code, round to nearest even, finite values beyond 6 saturate.
    The sign bit follows the input's sign (so -0.1 encodes as -0, code 0x8)."""
    f = np.asarray(v, dtype=np.float32)
    if np.isnan(f).any():
        raise ValueError("NaN has no E2M1 encoding")
    idx = _round_magnitude(np.abs(f.astype(np.float64)), _E2M1_GRID)
    return (idx | np.where(np.signbit(f), 0x8, 0)).astype(np.uint8)


def e4m3_encode_satfinite(v) -> np.ndarray:
    """fp32 -> E4M3 byte, round to nearest even, finite values beyond 448
    saturate to 448; NaN maps to 0x7F (sign kept)."""
    f = np.asarray(v, dtype=np.float32)
    nan = np.isnan(f)
    mag = np.where(nan, 0.0, np.abs(f.astype(np.float64)))
    idx = _round_magnitude(mag, _E4M3_GRID)
    out = idx | np.where(np.signbit(f), 0x80, 0)
    out = np.where(nan, 0x7F | np.where(np.signbit(f), 0x80, 0), out)
    return out.astype(np.uint8)


def unpack_nibbles(codes_u8: np.ndarray) -> np.ndarray:
    """[..., K/2] bytes -> [..., K] codes; element 2i is the low nibble."""
    c = np.asarray(codes_u8, dtype=np.uint8)
    out = np.empty(c.shape[:-1] + (c.shape[-1] * 2,), np.uint8)
    out[..., 0::2] = c & 0xF
    out[..., 1::2] = c >> 4
    return out


def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    c = np.asarray(codes, dtype=np.uint8)
    return (c[..., 0::2] & 0xF) | ((c[..., 1::2] & 0xF) << 4)


# value of every byte of packed codes: [byte, 0] = low nibble, [byte, 1] = high
_E2M1_PAIR = np.stack([e2m1_value(np.arange(256) & 0xF), e2m1_value(np.arange(256) >> 4)], axis=1)
_E4M3_ALL = e4m3_value(np.arange(256))


def nvfp4_dequant(codes_u8, scales_u8, tensor_scale) -> np.ndarray:
    """NVFP4 [rows, K] -> fp64: e2m1(code) * e4m3(block scale) * tensor_scale.
    Exact in fp64 (2 + 4 + 24 significand bits)."""
    c = np.asarray(codes_u8, dtype=np.uint8)
    rows, half = c.shape
    v = _E2M1_PAIR[c].reshape(rows, half * 2 // 16, 16)           # element order, per 16-block
    s = _E4M3_ALL[np.asarray(scales_u8, dtype=np.uint8)]           # [rows, K/16]
    return (v * (s * float(np.float32(tensor_scale)))[:, :, None]).reshape(rows, half * 2)


def quantize_rows_nvfp4(a_f32):
    """Dynamic NVFP4 encoding of activation rows, every step in IEEE fp32.

    For each row: r = max|a|; tsx = r / 2688 (2688 = 6 * 448, so r lands on the
    largest code at the largest scale). For each block of 16: sb =
    e4m3(amax_blk / 6 / tsx); d = e4m3value(sb) * tsx; code = e2m1(a / d).
    A zero row has tsx = 0: all its scales and codes are 0. A block with
    d = 0 gets codes 0.

    Returns (codes uint8 [R, K/2], block scales uint8 [R, K/16], tsx fp32 [R]).
    """
    a = np.asarray(a_f32, dtype=np.float32)
    R, K = a.shape
    assert K % 16 == 0
    absa = np.abs(a)
    r = absa.max(axis=1) if K else np.zeros(R, np.float32)
    tsx = (r / ACT_ROW_SCALE_DIVISOR).astype(np.float32)
    amax = absa.reshape(R, K // 16, 16).max(axis=2)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = ((amax / np.float32(6.0)).astype(np.float32) / tsx[:, None]).astype(np.float32)
    q = np.where(tsx[:, None] == 0, np.float32(0.0), q)
    sb = e4m3_encode_satfinite(q)
    d = (e4m3_value(sb).astype(np.float32) * tsx[:, None]).astype(np.float32)
    blocks = a.reshape(R, K // 16, 16)
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = (blocks / d[:, :, None]).astype(np.float32)
    ratio = np.where(d[:, :, None] == 0, np.float32(0.0), ratio)
    codes = e2m1_encode_satfinite(ratio).reshape(R, K)
    return pack_nibbles(codes), sb, tsx


def dequant_rows_nvfp4(codes_u8, scales_u8, tsx) -> np.ndarray:
    """Inverse of quantize_rows_nvfp4, exact in fp64."""
    v = e2m1_value(unpack_nibbles(codes_u8))
    s = np.repeat(e4m3_value(scales_u8), 16, axis=-1)
    return v * s * np.asarray(tsx, np.float32).astype(np.float64)[:, None]
