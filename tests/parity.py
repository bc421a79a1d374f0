"""Shared helpers of the GPU parity tests: run the CUDA path and the oracle on the same
seeded inputs and compare.

Tolerances (fp32 accumulation on the GPU, fp64 in the oracle):
  * fp32 / fp16 / bf16 I/O: max |gpu - oracle| <= 2e-3, where the oracle is first rounded
    to the I/O dtype (round to nearest even), because the GPU result is rounded too.  An
    output also passes when it lies within the tolerance of the exact fp64 value (the bar as
    stated: max abs error against the oracle); with bf16 output and an 8-bit cache's 1e-2 a
    result at |o| >= 2, where one bf16 ulp is 0.0156, can differ from the rounded oracle by
    a whole ulp while within 1e-2 of the exact value.  The one other exception allowed is a
    rounding-boundary case: the exact value lies so close to the midpoint of two adjacent
    I/O values that the fp32 result rounded to the other one (|gpu - oracle_fp64| <= half an
    I/O ulp + 1e-5 relative).  Both kinds are counted, and boundary cases must stay rare.
  * INT8 and FP8 caches: the same against the oracle on the dequantised values, with 1e-2.
"""
import numpy as np
import torch

import oracle
import paged_kv_cache_384_b200 as pa

TOL = {"fp32": 2e-3, "fp16": 2e-3, "bf16": 2e-3, "int8": 1e-2}

# (I/O dtype, rounding-boundary cases accepted, outputs compared, outputs accepted on their
# distance to the exact value) of every compare() call in this process; the session summary
# (conftest.py) prints the totals.
BOUNDARY_TALLY = []
TORCH_DT = {"fp32": torch.float32, "fp16": torch.float16, "bf16": torch.bfloat16}


def round_io(x64: np.ndarray, io: str) -> np.ndarray:
    if io == "fp32":
        return x64.astype(np.float32).astype(np.float64)
    if io == "fp16":
        return x64.astype(np.float16).astype(np.float64)
    return torch.from_numpy(x64).to(torch.bfloat16).to(torch.float64).numpy()


def half_ulp(x64: np.ndarray, io: str) -> np.ndarray:
    mant = {"fp32": 23, "fp16": 10, "bf16": 7}[io]
    e = np.floor(np.log2(np.maximum(np.abs(x64), 2.0 ** -14)))
    return 2.0 ** (e - mant) / 2


def compare(gpu: torch.Tensor, ref64: np.ndarray, io: str, tol: float, max_boundary_frac=1e-3):
    """Assert parity; return (max error vs the rounded oracle, max raw error, boundary cases)."""
    g = gpu.detach().float().cpu().double().numpy()
    assert g.shape == ref64.shape
    assert np.all(np.isfinite(g)), "non-finite GPU output"
    r = round_io(ref64, io)
    err = np.abs(g - r)
    raw = np.abs(g - ref64)
    exact_ok = (err > tol) & (raw <= tol)   # within the tolerance of the exact value
    over = (err > tol) & ~exact_ok
    boundary = over & (raw <= half_ulp(ref64, io) * (1 + 1e-6) + 1e-5 * np.abs(ref64))
    hard = over & ~boundary
    if hard.any():
        idx = np.argwhere(hard)[:5]
        raise AssertionError(f"{int(hard.sum())} outputs off by > {tol}: max {err.max():.3e} at {idx.tolist()}; "
                             f"gpu {g[tuple(idx[0])]} oracle {ref64[tuple(idx[0])]}")
    assert boundary.sum() <= max(1, max_boundary_frac * g.size), f"{int(boundary.sum())} rounding-boundary cases"
    BOUNDARY_TALLY.append((io, int(boundary.sum()), int(g.size), int(exact_ok.sum())))
    return float(err.max(initial=0.0)), float(raw.max(initial=0.0)), int(boundary.sum())


class GpuCase:
    """Device copies of a workload's tensors, ready for the C ABI."""

    def __init__(self, q, k_cache, v_cache, block_tables, context_lens, scale, window=0,
                 k_scale=None, v_scale=None, device="cuda"):
        self.q = q.to(device)
        self.k_cache = k_cache.to(device)
        self.v_cache = v_cache.to(device)
        self.block_tables = block_tables.to(device=device, dtype=torch.int32).contiguous()
        self.context_lens = torch.as_tensor(context_lens, dtype=torch.int32).to(device)
        self.k_scale = None if k_scale is None else k_scale.to(device)
        self.v_scale = None if v_scale is None else v_scale.to(device)
        self.scale, self.window = scale, window
        S, H, D = self.q.shape
        self.workspace = pa.alloc_workspace(S, H, D, device)

    def decode(self, stream=None):
        out = torch.empty_like(self.q)
        pa.paged_attention_decode(out, self.q, self.k_cache, self.v_cache, self.block_tables,
                                  self.context_lens, self.scale, self.window, self.k_scale, self.v_scale,
                                  workspace=self.workspace, stream=stream)
        return out


def quantize_cache(cache_f16: torch.Tensor):
    """Oracle quantiser on a [NB, bs, H, D] fp16 cache -> (int8 codes, fp16 scales) tensors."""
    codes, scale = oracle.quant.quantize_rows(cache_f16.cpu().numpy())
    return torch.from_numpy(codes), torch.from_numpy(scale)


def oracle_decode(q, k_cache, v_cache, block_tables, context_lens, scale, window=0, k_scale=None, v_scale=None):
    return oracle.paged_decode(q, k_cache, v_cache, block_tables, context_lens, scale, window,
                               k_scale=k_scale, v_scale=v_scale)


def assert_no_device_error():
    flags = pa.device_error(clear=True)
    assert flags == 0, f"device error flags 0x{flags:x}"


def quantize_cache_fp8(cache_f16: torch.Tensor):
    """Oracle FP8 (E4M3) quantiser on a [NB, bs, H, D] fp16 cache -> (float8 codes, fp16 scales)."""
    codes, scale = oracle.quant.quantize_rows_fp8(cache_f16.cpu().numpy())
    return torch.from_numpy(codes).view(torch.float8_e4m3fn), torch.from_numpy(scale)
