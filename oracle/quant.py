"""INT8 KV-cache quantiser of the oracle (numpy, fp32 decisions).

TEST INFRASTRUCTURE ONLY (tests, smoke check, CPU-baseline leg of the benchmark).

"KV Cache optimisation strategies in deployment" (yunthe.com), section
"量化压缩KV Cache的INT8与FP8方案", names an INT8 KV cache (half the memory of FP16)
without giving its scheme.  Reading used throughout this project:

  * one symmetric scale per (token, head) row of head_dim values;
  * scale = max_d |x_d| / 127, computed in fp32 from the fp16 source, then rounded to
    fp16 (round to nearest even) -- the fp16 value is what the cache stores;
  * code_d = clamp(rint(x_d / scale_fp16), -127, 127), the division in fp32 and rint
    rounding halves to even;
  * a row whose fp16 scale is 0 (all zeros, or amax so small that amax/127 rounds to
    0 in fp16) stores scale 0 and all-zero codes;
  * dequantised value = code * scale, exact in fp64.

Both the oracle and any GPU quantiser take the integer decision in fp32.
"""
import numpy as np


def quantize_rows(x_f16: np.ndarray):
    """Quantise rows of ``x_f16`` (fp16, last axis = head_dim).

    Returns ``(codes int8 [...,D], scale fp16 [...])``.
    """
    x = np.asarray(x_f16)
    if x.dtype not in (np.float16, np.float32):
        raise TypeError("quantize_rows expects float16 (or exact float32, e.g. widened bf16) input")
    x32 = x.astype(np.float32)
    amax = np.max(np.abs(x32), axis=-1)
    scale16 = (amax / np.float32(127.0)).astype(np.float32).astype(np.float16)
    s32 = scale16.astype(np.float32)[..., None]
    safe = np.where(s32 > 0, s32, np.float32(1.0))
    ratio = (x32 / safe).astype(np.float32)
    codes = np.where(s32 > 0, np.clip(np.rint(ratio), -127, 127), 0).astype(np.int8)
    return codes, scale16


def dequantize_rows(codes: np.ndarray, scale16: np.ndarray) -> np.ndarray:
    """code * scale in fp64 (exact: an 8-bit integer times an 11-bit significand)."""
    return codes.astype(np.float64) * scale16.astype(np.float64)[..., None]


# ---------------------------------------------------------------------------------------
# FP8 (E4M3) cache.  The same page and section name FP8 ("E4M1", read as E4M3, the OCP
# "fn" variant: 4 exponent bits with bias 7, 3 mantissa bits, no infinities, largest
# finite value 448).  Reading, parallel to INT8: one fp16 scale per (token, head) row,
# scale = max|x| / 448 in fp32 rounded to fp16, code = E4M3(x / scale) with the division
# in fp32 and round-to-nearest-even, saturating at +-448; scale 0 => zero codes.
# ---------------------------------------------------------------------------------------
E4M3_MAX = 448.0


def e4m3_values() -> np.ndarray:
    """The 256 code points of E4M3 as fp64 (NaN at 0x7F / 0xFF), from the format's definition."""
    c = np.arange(256)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * 2.0 ** (e - 7.0))
    mag = np.where((e == 15) & ((c & 0x7) == 7), np.nan, mag)
    return sign * mag


def e4m3_round(x) -> np.ndarray:
    """Round values (exact in fp64) to the nearest E4M3 value, ties to even, saturating."""
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    _, exp2 = np.frexp(a)                       # a = f * 2^exp2, f in [0.5, 1)
    e = np.maximum(exp2 - 1, -6)                # unbiased exponent; below 2^-6 the step is 2^-9
    step = np.ldexp(1.0, e - 3)
    r = np.minimum(np.rint(a / step) * step, E4M3_MAX)
    return np.copysign(r, x)


def e4m3_encode(values) -> np.ndarray:
    """Codes (uint8) of values that are exact E4M3 values (e.g. from e4m3_round)."""
    v = np.asarray(values, dtype=np.float64)
    table = e4m3_values()[:0x7F]                # non-negative, finite codes 0x00 .. 0x7E
    mag = np.searchsorted(table, np.abs(v))
    if not np.array_equal(table[mag], np.abs(v)):
        raise ValueError("not an E4M3 value")
    return (mag | np.where(np.signbit(v), 0x80, 0)).astype(np.uint8)


def quantize_rows_fp8(x):
    """FP8 E4M3 rows: returns (codes uint8 [...,D], scale fp16 [...])."""
    x = np.asarray(x)
    if x.dtype not in (np.float16, np.float32):
        raise TypeError("quantize_rows_fp8 expects float16 (or exact float32) input")
    x32 = x.astype(np.float32)
    amax = np.max(np.abs(x32), axis=-1)
    scale16 = (amax / np.float32(E4M3_MAX)).astype(np.float32).astype(np.float16)
    s32 = scale16.astype(np.float32)[..., None]
    safe = np.where(s32 > 0, s32, np.float32(1.0))
    ratio = (x32 / safe).astype(np.float32)
    codes = e4m3_encode(np.where(s32 > 0, e4m3_round(ratio), 0.0))
    return codes, scale16


def dequantize_rows_fp8(codes, scale16) -> np.ndarray:
    return e4m3_values()[np.asarray(codes, dtype=np.int64)] * scale16.astype(np.float64)[..., None]
