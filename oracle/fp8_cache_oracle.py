"""Float64 CPU oracle for decode attention over an FP8 (e4m3) latent cache.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline
leg of ``bench.py`` may import this module. The CUDA library never calls it and shares no
code with it.

What it computes. The MLA article on lesty.tech (section 5, the paragraph on post-training KV
quantization) says the cached latent vectors can be stored in FP8 or INT4; its 288-byte figure
for 4-bit storage counts all 576 elements of a token's cached row, so the whole row
``[c | k^R]`` is quantized. The pages fix no format. Reading taken here:

* every cached element is one OCP FP8 E4M3 byte (1 sign bit, 4 exponent bits with bias 7,
  3 mantissa bits; no infinities; exponent 15 with mantissa 7 is NaN; largest finite 448);
* one fp32 scale per tensor for the latent columns (``latent_scale``) and one for the RoPE
  columns (``rope_scale``): the value of a latent byte e is ``latent_scale * e4m3(e)``;
* writing a value v stores ``e4m3(v / scale)`` rounded to nearest, ties to the even code,
  with values beyond +-448 saturated to +-448 (NaN stays NaN).

Decode over such a cache is the bf16-cache decode (``mlra_oracle.decode``) on the dequantized
rows: the method itself is unchanged, only the cache's storage is.

Parity status: ``e4m3_decode`` and ``e4m3_encode`` are pinned by ``tests/test_oracle_fp8.py``
against the format's definition (closed-form codes), torch's float8_e4m3fn conversion and
round trips; ``dequantize_pool`` and ``decode_fp8`` against the bf16-cache oracle on rows
whose values e4m3 holds exactly.
"""
from __future__ import annotations

import math

import numpy as np

from . import mlra_oracle as O

E4M3_MAX = 448.0
E4M3_NAN = 0x7F


def e4m3_decode(code: int) -> float:
    """Value of one E4M3 byte, from the bit fields (OCP 8-bit floating point, E4M3)."""
    code = int(code) & 0xFF
    sign = -1.0 if code & 0x80 else 1.0
    exp = (code >> 3) & 0xF
    man = code & 0x7
    if exp == 0xF and man == 0x7:
        return math.nan
    if exp == 0:
        return sign * math.ldexp(man / 8.0, -6)        # subnormal: 2^(1-7) * m/8
    return sign * math.ldexp(1.0 + man / 8.0, exp - 7)


# every code's value, for table lookups
_TABLE = np.array([e4m3_decode(c) for c in range(256)], dtype=np.float64)
# finite non-negative codes in increasing order of value (0x00 .. 0x7E)
_POS_CODES = np.arange(0x7F)
_POS_VALUES = _TABLE[:0x7F]


def e4m3_decode_array(codes: np.ndarray) -> np.ndarray:
    return _TABLE[np.asarray(codes, dtype=np.uint8)]


def e4m3_encode(x: float) -> int:
    """Nearest E4M3 code to x, ties to the even code (mantissa LSB 0), saturating at +-448."""
    if math.isnan(x):
        return E4M3_NAN
    sign = 0x80 if (x < 0 or (x == 0 and math.copysign(1.0, x) < 0)) else 0
    a = min(abs(x), E4M3_MAX)
    i = int(np.searchsorted(_POS_VALUES, a))          # first value >= a
    if i < len(_POS_VALUES) and _POS_VALUES[i] == a:
        return sign | int(_POS_CODES[i])
    lo, hi = i - 1, i                                  # a lies strictly between two values
    d_lo, d_hi = a - _POS_VALUES[lo], _POS_VALUES[hi] - a
    if d_lo < d_hi or (d_lo == d_hi and _POS_CODES[lo] % 2 == 0):
        return sign | int(_POS_CODES[lo])
    return sign | int(_POS_CODES[hi])


def e4m3_encode_array(x: np.ndarray) -> np.ndarray:
    flat = np.asarray(x, dtype=np.float64).reshape(-1)
    return np.array([e4m3_encode(v) for v in flat], dtype=np.uint8).reshape(np.shape(x))


def quantize_rows(rows: np.ndarray, d_c: int, latent_scale: float, rope_scale: float) -> np.ndarray:
    """Bytes of cache rows [..][d_c + d_r] as stored: latent columns by latent_scale, RoPE
    columns by rope_scale (small inputs only: one Python call per element)."""
    rows = np.asarray(rows, dtype=np.float64)
    out = np.empty(rows.shape, dtype=np.uint8)
    out[..., :d_c] = e4m3_encode_array(rows[..., :d_c] / latent_scale)
    out[..., d_c:] = e4m3_encode_array(rows[..., d_c:] / rope_scale)
    return out


def dequantize_pool(pool_u8: np.ndarray, d_c: int, latent_scale: float, rope_scale: float) -> np.ndarray:
    """float64 values of an E4M3 cache [pages][64][d_c + d_r]."""
    v = e4m3_decode_array(pool_u8)
    v[..., :d_c] *= latent_scale
    v[..., d_c:] *= rope_scale
    return v


def decode_fp8(q, w_uk, w_uv, pool_u8, page_table, seq_lens, k, d_r, latent_scale, rope_scale,
               scale=None, form="absorbed"):
    """Decode step over an E4M3 cache: ``mlra_oracle.decode`` on the dequantized rows."""
    d_c = np.asarray(pool_u8).shape[-1] - d_r
    pool = dequantize_pool(pool_u8, d_c, latent_scale, rope_scale)
    return O.decode(q, w_uk, w_uv, pool, page_table, seq_lens, k, d_r, scale=scale, form=form)
