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
    if x.dtype != np.float16:
        raise TypeError("quantize_rows expects float16 input")
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
