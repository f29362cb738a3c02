"""An 8-bit latent cache for the absorbed decode: the oracle's side (fp64 except the 8-bit codes).

TEST INFRASTRUCTURE: only tests/ use this file. It shares no code with the CUDA path.

Source: « Cache KV, mémoire récurrente, MLA et bas rang », trainer notes of « Le problème — Cache
KV standard »: an 8-bit cache keeps every factor of the cache size and halves the bytes per value
(2 → 1). The pages fix nothing more. Readings (each listed with its reason in the design notes):
  * The number type is FP8 E4M3 ("e4m3fn": 1 sign bit, 4 exponent bits with bias 7, 3 mantissa
    bits, subnormals, no infinities, one NaN pattern S.1111.111; largest finite value 448), the
    8-bit operand type of the B200 tensor cores.
  * Only the latent row c is narrowed. The shared RoPE key k_r (d_r = 64 values per position)
    stays in the 16-bit cache.
  * Each latent row j carries one fp32 scale s_j = max|c_j| / 448, so that the row's largest
    magnitude maps to the largest code; codes are c_j / s_j rounded to the nearest E4M3 value,
    ties to even mantissa, magnitudes above 448 saturated to 448 (a zero row keeps scale 0 and
    all-zero codes).
  * The decode attends the dequantised rows s_j · code_j exactly as the absorbed decode attends
    16-bit rows.
"""
from __future__ import annotations

import numpy as np

from . import mla_oracle as O

f64 = np.float64
E4M3_MAX = 448.0
_BIAS = 7


def e4m3_decode(codes):
    """Values of E4M3 byte codes (uint8 array) from the format definition: sign · 2^(e−7) · (1 + m/8)
    for exponent field e ≥ 1, sign · 2^(−6) · (m/8) for e = 0, NaN for the pattern x.1111.111."""
    codes = np.asarray(codes, np.uint8).astype(np.int64)
    sign = np.where(codes & 0x80, -1.0, 1.0)
    e = (codes >> 3) & 0xF
    m = (codes & 0x7).astype(f64)
    normal = sign * np.ldexp(1.0 + m / 8.0, (e - _BIAS).astype(np.int64))
    sub = sign * np.ldexp(m / 8.0, 1 - _BIAS)
    out = np.where(e == 0, sub, normal)
    return np.where((e == 0xF) & ((codes & 0x7) == 0x7), np.nan, out)


def _finite_table():
    """The 127 non-negative finite E4M3 values in increasing order, with their codes."""
    codes = np.arange(0x7F, dtype=np.uint8)   # 0x00 .. 0x7E: +0 up to 448
    return e4m3_decode(codes), codes


def e4m3_encode(v):
    """Nearest E4M3 code of each value (ties to the even code, i.e. the even mantissa), magnitudes
    beyond 448 saturated to 448. NaN inputs are not expected (the scaled rows are finite)."""
    v = np.asarray(v, f64)
    vals, codes = _finite_table()
    a = np.minimum(np.abs(v), E4M3_MAX)
    hi = np.clip(np.searchsorted(vals, a, side="left"), 0, len(vals) - 1)   # first value >= a
    lo = np.clip(hi - 1, 0, len(vals) - 1)
    d_lo, d_hi = a - vals[lo], vals[hi] - a
    # the two neighbours differ by one in the code, so "even code" is "even mantissa"
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (codes[hi] % 2 == 0))
    mag = np.where(pick_hi, codes[hi], codes[lo]).astype(np.uint8)
    neg = (v < 0) & (mag != 0)
    return np.where(neg, mag | 0x80, mag).astype(np.uint8)


def quantize_rows(c):
    """Per-row scaled E4M3 codes of latent rows c [n, d_c]: (codes uint8 [n, d_c], scales [n])."""
    c = np.asarray(c, f64)
    amax = np.abs(c).max(axis=1)
    scale = amax / E4M3_MAX
    safe = np.where(scale > 0, scale, 1.0)
    codes = e4m3_encode(c / safe[:, None])
    return codes, scale


def quantize_rows_f32(c):
    """The same quantisation with the arithmetic that decides each code done in float32, the
    precision a kernel takes that decision in: s_j = fl32(max|c_j| / 448) and code = the nearest
    E4M3 value of fl32(c_j / s_j), each operation rounded once to float32. `c` holds
    float32-representable values (bf16 rows are). Returns (codes uint8 [n, d_c], scales [n] as the
    float32 values, widened)."""
    c32 = np.asarray(c, np.float32)
    amax = np.abs(c32).max(axis=1)
    scale = (amax / np.float32(E4M3_MAX)).astype(np.float32)
    safe = np.where(scale > 0, scale, np.float32(1.0)).astype(np.float32)
    quot = (c32 / safe[:, None]).astype(np.float32)
    return e4m3_encode(quot.astype(f64)), scale.astype(f64)


def dequantize_rows(codes, scale):
    return e4m3_decode(codes) * np.asarray(scale, f64)[:, None]


def absorbed_decode_fp8(q_abs, codes, scale, k_r, seqlen, sm_scale):
    """The absorbed decode (« L'attention latente : compresser le cache », « Ce que DeepSeek fait de
    plus ») over an 8-bit latent cache: the rows are dequantised (s_j · code_j), then attended
    exactly like 16-bit rows."""
    return O.absorbed_decode(q_abs, dequantize_rows(codes, scale), k_r, seqlen, sm_scale)
