"""fp64 CPU oracle for paged decode attention and its cache operations.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU-baseline /
reference leg of the benchmark may import this package.  The product library
(``paged_kv_cache_384_b200``) never imports, links or runs anything here, and this
package imports nothing from it.

Contents
  * ``paged_decode``    -- textbook softmax attention over K/V gathered through the
                           block table, fp64 (``pa_oracle.c``).
  * ``paged_prefill``   -- the same for several causal query tokens per sequence
                           (prefill / chunked prefill), fp64 (``pa_oracle.c``).
  * ``quant``           -- INT8 per-(token, head) quantiser (fp32 decisions).
  * ``cache_ops``       -- reshape_and_cache / copy_blocks placement definitions.
  * ``block_manager``   -- BlockTable / BlockManager allocator model.

Every function is pinned by ``tests/test_oracle_*.py`` against values fixed by the
pages or by mathematics (closed forms, invariances, a library attention routine on the
dense special case, brute force).
"""
import ctypes
import os

import numpy as np

from . import block_manager, cache_ops, quant  # noqa: F401
from .build import LIB, build

F32, F16, BF16, I8, FP8 = 0, 1, 2, 3, 4
_STATUS = {1: "bad argument", 2: "block-table entry out of range",
           3: "context length out of range", 4: "out of memory"}

_lib = None


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(LIB)
        lib.orc_paged_decode_gqa.restype = ctypes.c_int
        lib.orc_paged_decode_gqa.argtypes = [
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_double, ctypes.c_int, ctypes.c_int]
        lib.orc_paged_prefill.restype = ctypes.c_int
        lib.orc_paged_prefill.argtypes = [
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_double, ctypes.c_int, ctypes.c_int]
        lib.orc_f16_to_f64.restype = ctypes.c_double
        lib.orc_f16_to_f64.argtypes = [ctypes.c_uint16]
        lib.orc_bf16_to_f64.restype = ctypes.c_double
        lib.orc_bf16_to_f64.argtypes = [ctypes.c_uint16]
        lib.orc_e4m3_to_f64.restype = ctypes.c_double
        lib.orc_e4m3_to_f64.argtypes = [ctypes.c_uint8]
        _lib = lib
    return _lib


def _raw(x):
    """(contiguous numpy array holding the stored bits, dtype code) for a tensor/array."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype == torch.float32:
                return x.numpy(), F32
            if x.dtype == torch.float16:
                return x.numpy(), F16
            if x.dtype == torch.bfloat16:
                return x.view(torch.int16).numpy(), BF16
            if x.dtype == torch.int8:
                return x.numpy(), I8
            if x.dtype == torch.float8_e4m3fn:
                return x.view(torch.uint8).numpy(), FP8
            raise TypeError(f"unsupported tensor dtype {x.dtype}")
    except ImportError:  # pragma: no cover
        pass
    x = np.ascontiguousarray(x)
    codes = {np.dtype(np.float32): F32, np.dtype(np.float16): F16, np.dtype(np.int8): I8}
    if x.dtype not in codes:
        raise TypeError(f"unsupported array dtype {x.dtype} (pass bf16 as a torch tensor)")
    return x, codes[x.dtype]


def _i32(x):
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


def _u16(x):
    try:
        import torch
        if isinstance(x, torch.Tensor):
            return x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float16)).view(np.uint16)


def available_cores() -> int:
    """Host cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except (AttributeError, OSError):  # pragma: no cover
        return os.cpu_count() or 1


def _threads(threads):
    return available_cores() if threads is None else max(1, int(threads))


def paged_decode(q, k_cache, v_cache, block_tables, context_lens, scale, window=0,
                 k_scale=None, v_scale=None, threads=None):
    """Decode attention of one query token per sequence over a paged KV cache.

    q [S,Hq,D]; k_cache/v_cache [NB,bs,Hkv,D] with Hq a multiple of Hkv (grouped-query:
    query head h reads cached head h // (Hq // Hkv)); block_tables [S,MB] int; context_lens [S];
    k_scale/v_scale [NB,bs,H] fp16 for an int8 or fp8 (torch.float8_e4m3fn) cache.  Returns fp64 numpy [S,H,D].
    ``threads``: worker threads sharing the independent (sequence, head) pairs (default: every
    core this process may use); the result is bit-identical for any count.
    """
    lib = _load()
    qa, qd = _raw(q)
    ka, kd = _raw(k_cache)
    va, vd = _raw(v_cache)
    if kd != vd:
        raise TypeError("k_cache and v_cache must share a dtype")
    S, H, D = qa.shape
    NB, bs, Hc, Dc = ka.shape
    if Dc != D or H % Hc != 0 or va.shape != ka.shape:
        raise ValueError("cache shape does not match q")
    bt = _i32(block_tables).reshape(S, -1)
    cl = _i32(context_lens).reshape(S)
    MB = bt.shape[1] if bt.size else 1
    if bt.size == 0:
        bt = np.zeros((S, 1), np.int32)
    ks = vs = None
    if kd in (I8, FP8):
        ks, vs = _u16(k_scale), _u16(v_scale)
        if ks.shape != (NB, bs, Hc) or vs.shape != (NB, bs, Hc):
            raise ValueError("an int8/fp8 cache needs k_scale/v_scale of shape [NB, bs, H]")
    out = np.zeros((S, H, D), np.float64)
    st = lib.orc_paged_decode_gqa(
        out.ctypes.data, qa.ctypes.data, qd, ka.ctypes.data, va.ctypes.data, kd,
        ks.ctypes.data if ks is not None else None, vs.ctypes.data if vs is not None else None,
        bt.ctypes.data, cl.ctypes.data, S, H, Hc, D, bs, MB, NB, float(scale), int(window), _threads(threads))
    if st != 0:
        raise ValueError(f"oracle: {_STATUS.get(st, st)}")
    return out


def paged_prefill(q, k_cache, v_cache, block_tables, cu_q, context_lens, scale, window=0,
                  k_scale=None, v_scale=None, threads=None):
    """Causal attention of each sequence's newest q_len tokens over a paged KV cache.

    q [T,Hq,D] packs the sequences' query tokens (sequence s owns rows cu_q[s]..cu_q[s+1]-1);
    the chunk's own K/V are already in the cache, so query i of sequence s sits at position
    context_lens[s] - q_len + i and attends up to itself (the last ``window`` tokens if
    window > 0).  Other arguments as for ``paged_decode`` (threads share the independent
    (sequence, cached head) pairs).  Returns fp64 numpy [T,Hq,D].
    """
    lib = _load()
    qa, qd = _raw(q)
    ka, kd = _raw(k_cache)
    va, vd = _raw(v_cache)
    if kd != vd:
        raise TypeError("k_cache and v_cache must share a dtype")
    T, H, D = qa.shape
    NB, bs, Hc, Dc = ka.shape
    if Dc != D or H % Hc != 0 or va.shape != ka.shape:
        raise ValueError("cache shape does not match q")
    cu = _i32(cu_q).reshape(-1)
    S = cu.size - 1
    if S < 0 or (S > 0 and cu[-1] != T):
        raise ValueError("cu_q must have S+1 entries ending at the number of query rows")
    bt = _i32(block_tables).reshape(S, -1)
    cl = _i32(context_lens).reshape(S)
    MB = bt.shape[1] if bt.size else 1
    if bt.size == 0:
        bt = np.zeros((max(S, 1), 1), np.int32)
    ks = vs = None
    if kd in (I8, FP8):
        ks, vs = _u16(k_scale), _u16(v_scale)
        if ks.shape != (NB, bs, Hc) or vs.shape != (NB, bs, Hc):
            raise ValueError("an int8/fp8 cache needs k_scale/v_scale of shape [NB, bs, H]")
    out = np.zeros((T, H, D), np.float64)
    st = lib.orc_paged_prefill(
        out.ctypes.data, qa.ctypes.data, qd, ka.ctypes.data, va.ctypes.data, kd,
        ks.ctypes.data if ks is not None else None, vs.ctypes.data if vs is not None else None,
        bt.ctypes.data, cu.ctypes.data, cl.ctypes.data, S, H, Hc, D, bs, MB, NB, float(scale), int(window),
        _threads(threads))
    if st != 0:
        raise ValueError(f"oracle: {_STATUS.get(st, st)}")
    return out


def f16_to_f64(bits: int) -> float:
    return _load().orc_f16_to_f64(bits)


def bf16_to_f64(bits: int) -> float:
    return _load().orc_bf16_to_f64(bits)


def e4m3_to_f64(bits: int) -> float:
    return _load().orc_e4m3_to_f64(bits)
