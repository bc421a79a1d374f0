"""paged_kv_cache_384_b200 -- paged attention over a block-table KV cache on NVIDIA B200 (sm_100a).

Thin Python binding over ``libpagedattn.so`` (C ABI in ``include/pagedattn.h``).  PyTorch
only supplies device memory and the current CUDA stream; every step of the computation
runs in the library's CUDA kernels.  Functions take torch tensors, check that shapes,
dtypes and devices agree, and pass raw pointers.

    decode_workspace_bytes(num_seqs, num_heads, head_dim)
    paged_attention_decode(out, q, k_cache, v_cache, block_tables, context_lens, scale, ...)
        (grouped-query when the cache has fewer heads than q; tcgen05 kernel for 4-16 query
        heads per cached head)
    paged_attention_prefill(out, q, k_cache, v_cache, block_tables, cu_q_lens, context_lens,
                            max_q_len, scale, window=0)
    reshape_and_cache(k, v, k_cache, v_cache, slot_mapping, ...)
    reshape_and_cache_quant(k, v, k_cache, v_cache, k_scale_cache, v_scale_cache, slot_mapping)
    copy_blocks(k_cache, v_cache, src_dst_pairs, ...)
    swap_blocks(src_k, src_v, dst_k, dst_v, src_dst_pairs, ...)   (GPU <-> pinned host pools)
    BlockManager(num_blocks, block_size, free_order=None)
    slot_mapping(block_tables, seq_ids, positions, block_size)
    device_error(clear=True)

Cache layout: [num_blocks, block_size, num_heads, head_dim]; INT8 / FP8 scales
[num_blocks, block_size, num_heads] fp16.
"""
from __future__ import annotations

import ctypes

import numpy as np
import torch

from . import _lib

_L = _lib.load()

PA_F32, PA_F16, PA_BF16, PA_I8, PA_FP8_E4M3 = 0, 1, 2, 3, 4
_DTYPE = {torch.float32: PA_F32, torch.float16: PA_F16, torch.bfloat16: PA_BF16, torch.int8: PA_I8,
          torch.float8_e4m3fn: PA_FP8_E4M3}
_SCALED = (torch.int8, torch.float8_e4m3fn)
_STATUS = {0: "PA_OK", 1: "PA_ERR_INVALID_ARG", 2: "PA_ERR_UNSUPPORTED", 3: "PA_ERR_CUDA",
           4: "PA_ERR_OUT_OF_BLOCKS", 5: "PA_ERR_BAD_BLOCK"}
DEVERR = {"table": 0x1, "context": 0x2, "slot": 0x4, "pair": 0x8, "timeout": 0x10}

LIB_PATH = _lib.LIB_PATH


class PagedAttnError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{_STATUS.get(status, status)}: {message}")
        self.status = status


def _check(status: int):
    if status != 0:
        raise PagedAttnError(status, _L.pa_last_error().decode())


def version() -> str:
    return _L.pa_version().decode()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dense(name, t):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (there is no CPU path)")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


# ---------------------------------------------------------------------------------------
# Decode attention
# ---------------------------------------------------------------------------------------
def decode_workspace_bytes(num_seqs: int, num_heads: int, head_dim: int) -> int:
    """Scratch bytes paged_attention_decode needs on the current device."""
    n = _L.pa_decode_workspace_bytes(num_seqs, num_heads, head_dim)
    if n == 0 and num_seqs >= 0:
        raise PagedAttnError(1, "no workspace size (invalid sizes or no CUDA device)")
    return n


def alloc_workspace(num_seqs: int, num_heads: int, head_dim: int, device=None) -> torch.Tensor:
    """A workspace tensor (uint8) of the size paged_attention_decode needs."""
    return torch.empty(decode_workspace_bytes(num_seqs, num_heads, head_dim), dtype=torch.uint8,
                       device=device or "cuda")


def paged_attention_decode(out, q, k_cache, v_cache, block_tables, context_lens, scale, window=0,
                           k_scale=None, v_scale=None, workspace=None, stream=None):
    """out[s,h,:] = softmax(scale * q[s,h] . K_s^T) V_s over the paged cache (fp32 accumulate).

    q, out [S,Hq,D] fp32/fp16/bf16; k_cache, v_cache [NB,bs,Hkv,D] of q's dtype, or int8 /
    float8_e4m3fn with k_scale, v_scale [NB,bs,Hkv] fp16; Hq a multiple of Hkv (grouped-query
    when Hkv < Hq: query head h reads cached head h // (Hq // Hkv)); block_tables int32
    [S,MB]; context_lens int32 [S].  window > 0 attends only the last ``window`` tokens.
    ``workspace`` defaults to a fresh allocation (pass one to keep allocation off the hot path).
    """
    S, H, D = q.shape
    NB, bs, Hc, Dc = k_cache.shape
    if out.shape != q.shape or out.dtype != q.dtype or Dc != D or H % Hc != 0 or v_cache.shape != k_cache.shape:
        raise ValueError("shape/dtype mismatch between out, q and the caches")
    if k_cache.dtype != v_cache.dtype:
        raise ValueError("k_cache and v_cache must share a dtype")
    if block_tables.dtype != torch.int32 or context_lens.dtype != torch.int32:
        raise ValueError("block_tables and context_lens must be int32")
    if block_tables.dim() != 2 or block_tables.shape[0] != S or context_lens.shape != (S,):
        raise ValueError("block_tables must be [S, MB] and context_lens [S]")
    for name, t in (("out", out), ("q", q), ("k_cache", k_cache), ("v_cache", v_cache),
                    ("block_tables", block_tables), ("context_lens", context_lens)):
        _dense(name, t)
    if k_cache.dtype in _SCALED:
        if k_scale is None or v_scale is None or k_scale.dtype != torch.float16 or \
                k_scale.shape != (NB, bs, Hc) or v_scale.shape != (NB, bs, Hc):
            raise ValueError("an int8 / fp8 cache needs fp16 k_scale/v_scale of shape [NB, bs, Hkv]")
        _dense("k_scale", k_scale), _dense("v_scale", v_scale)
    if workspace is None:
        workspace = alloc_workspace(S, H, D, q.device)
    _check(_L.paged_attention_decode_gqa(
        _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(k_scale), _ptr(v_scale),
        _ptr(block_tables), _ptr(context_lens), S, H, Hc, D, bs, NB, block_tables.shape[1],
        float(scale), int(window), _DTYPE[q.dtype], _DTYPE[k_cache.dtype], _ptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)))
    return out


# ---------------------------------------------------------------------------------------
# Cache maintenance
# ---------------------------------------------------------------------------------------
def paged_attention_prefill(out, q, k_cache, v_cache, block_tables, cu_q_lens, context_lens, max_q_len: int,
                            scale: float, window: int = 0, stream=None, k_scale=None, v_scale=None):
    """Causal attention of each sequence's newest q_len tokens over the paged cache.

    q/out [T, Hq, 128] (fp16 or bf16) pack the sequences' query rows (sequence s owns rows
    cu_q_lens[s]..cu_q_lens[s+1]-1, int32 [S+1] on the GPU); the chunk's K/V must already
    be in the cache, so query i of sequence s is at position context_lens[s] - q_len + i.
    ``max_q_len`` bounds every q_len (host-known, sizes the grid).  The caches hold q's
    dtype, or int8 / float8_e4m3fn codes with fp16 k_scale / v_scale [NB, bs, Hkv].
    """
    if q.dim() != 3 or out.shape != q.shape or out.dtype != q.dtype:
        raise ValueError("q and out must be [T, Hq, D] of one dtype")
    eight_bit = k_cache.dtype in _SCALED
    if k_cache.dim() != 4 or v_cache.shape != k_cache.shape or v_cache.dtype != k_cache.dtype or \
            (k_cache.dtype != q.dtype and not eight_bit):
        raise ValueError("caches must be [NB, bs, Hkv, D] in q's dtype, or int8 / float8_e4m3fn")
    if eight_bit:
        NB_, bs_, Hkv_ = k_cache.shape[:3]
        if k_scale is None or v_scale is None or k_scale.dtype != torch.float16 or \
                k_scale.shape != (NB_, bs_, Hkv_) or v_scale.shape != (NB_, bs_, Hkv_):
            raise ValueError("an int8 / fp8 cache needs fp16 k_scale/v_scale of shape [NB, bs, Hkv]")
        _dense("k_scale", k_scale), _dense("v_scale", v_scale)
    if cu_q_lens.dtype != torch.int32 or context_lens.dtype != torch.int32 or block_tables.dtype != torch.int32:
        raise ValueError("cu_q_lens, context_lens and block_tables must be int32")
    for name, t in (("out", out), ("q", q), ("k_cache", k_cache), ("v_cache", v_cache),
                    ("block_tables", block_tables), ("cu_q_lens", cu_q_lens), ("context_lens", context_lens)):
        _dense(name, t)
    T, Hq, D = q.shape
    NB, bs, Hkv, _ = k_cache.shape
    S = context_lens.shape[0]
    if cu_q_lens.shape[0] != S + 1:
        raise ValueError("cu_q_lens must have num_seqs + 1 entries")
    if eight_bit:
        _check(_L.paged_attention_prefill_quant(
            _ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(k_scale), _ptr(v_scale), _ptr(block_tables),
            _ptr(cu_q_lens), _ptr(context_lens), S, T, int(max_q_len), Hq, Hkv, D, bs, NB, block_tables.shape[1],
            float(scale), int(window), _DTYPE[q.dtype], _DTYPE[k_cache.dtype], _stream(stream)))
        return
    _check(_L.paged_attention_prefill(_ptr(out), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
                                      _ptr(cu_q_lens), _ptr(context_lens), S, T, int(max_q_len), Hq, Hkv, D, bs,
                                      NB, block_tables.shape[1], float(scale), int(window), _DTYPE[q.dtype],
                                      _stream(stream)))


def reshape_and_cache(k, v, k_cache, v_cache, slot_mapping, k_scale=None, v_scale=None,
                      k_scale_cache=None, v_scale_cache=None, stream=None):
    """Write token t's rows k[t], v[t] ([T,H,D], token stride may exceed H*D) into slot
    slot_mapping[t] (int64; negative = skip).  int8 caches also take per-(token, head)
    fp16 scales [T,H] and the scale caches [NB,bs,H]."""
    T, H, D = k.shape
    NB, bs, Hc, Dc = k_cache.shape
    if v.shape != k.shape or (Hc, Dc) != (H, D) or v_cache.shape != k_cache.shape:
        raise ValueError("shape mismatch between k/v and the caches")
    if k.dtype != k_cache.dtype or v.dtype != k_cache.dtype or v_cache.dtype != k_cache.dtype:
        raise ValueError("k, v and the caches must share a dtype")
    if slot_mapping.dtype != torch.int64 or slot_mapping.shape != (T,):
        raise ValueError("slot_mapping must be int64 [T]")
    for name, t in (("k", k), ("v", v)):
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor (there is no CPU path)")
        if t.stride(2) != 1 or t.stride(1) != D:
            raise ValueError(f"{name} rows must be dense [H, D] blocks")
    _dense("k_cache", k_cache), _dense("v_cache", v_cache), _dense("slot_mapping", slot_mapping)
    _check(_L.reshape_and_cache(
        _ptr(k), _ptr(v), _ptr(k_cache), _ptr(v_cache), _ptr(slot_mapping), T, H, D, bs, NB,
        k.stride(0), v.stride(0), _DTYPE[k.dtype], _ptr(k_scale), _ptr(v_scale),
        _ptr(k_scale_cache), _ptr(v_scale_cache), _stream(stream)))


def reshape_and_cache_quant(k, v, k_cache, v_cache, k_scale_cache, v_scale_cache, slot_mapping, stream=None):
    """Quantise token rows k[t], v[t] ([T,H,D] fp16/bf16) to the int8 or float8_e4m3fn cache
    with one fp16 scale per (token, head), writing slot slot_mapping[t] (negative = skip)."""
    T, H, D = k.shape
    NB, bs, Hc, Dc = k_cache.shape
    if v.shape != k.shape or (Hc, Dc) != (H, D) or v_cache.shape != k_cache.shape:
        raise ValueError("shape mismatch between k/v and the caches")
    if k.dtype not in (torch.float16, torch.bfloat16) or v.dtype != k.dtype:
        raise ValueError("k and v must be fp16 or bf16")
    if k_cache.dtype not in _SCALED or v_cache.dtype != k_cache.dtype:
        raise ValueError("the caches must be int8 or float8_e4m3fn")
    if k_scale_cache.shape != (NB, bs, H) or v_scale_cache.shape != (NB, bs, H) or \
            k_scale_cache.dtype != torch.float16 or v_scale_cache.dtype != torch.float16:
        raise ValueError("scale caches must be fp16 [NB, bs, H]")
    if slot_mapping.dtype != torch.int64 or slot_mapping.shape != (T,):
        raise ValueError("slot_mapping must be int64 [T]")
    for name, t in (("k", k), ("v", v)):
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor (there is no CPU path)")
        if t.stride(2) != 1 or t.stride(1) != D:
            raise ValueError(f"{name} rows must be dense [H, D] blocks")
    for name, t in (("k_cache", k_cache), ("v_cache", v_cache), ("k_scale_cache", k_scale_cache),
                    ("v_scale_cache", v_scale_cache), ("slot_mapping", slot_mapping)):
        _dense(name, t)
    _check(_L.reshape_and_cache_quant(
        _ptr(k), _ptr(v), _DTYPE[k.dtype], _ptr(k_cache), _ptr(v_cache), _ptr(k_scale_cache),
        _ptr(v_scale_cache), _DTYPE[k_cache.dtype], _ptr(slot_mapping), T, H, D, bs, NB,
        k.stride(0), v.stride(0), _stream(stream)))


def copy_blocks(k_cache, v_cache, src_dst_pairs, k_scale_cache=None, v_scale_cache=None, stream=None):
    """k_cache[dst] = k_cache[src] (and v, and the scale pools) for each (src, dst) pair."""
    NB = k_cache.shape[0]
    if v_cache.shape != k_cache.shape or v_cache.dtype != k_cache.dtype:
        raise ValueError("k_cache and v_cache must match")
    if src_dst_pairs.dtype != torch.int64 or src_dst_pairs.dim() != 2 or src_dst_pairs.shape[1] != 2:
        raise ValueError("src_dst_pairs must be int64 [N, 2]")
    _dense("k_cache", k_cache), _dense("v_cache", v_cache), _dense("src_dst_pairs", src_dst_pairs)
    block_bytes = k_cache[0].numel() * k_cache.element_size()
    sbytes = 0 if k_scale_cache is None else k_scale_cache[0].numel() * k_scale_cache.element_size()
    _check(_L.copy_blocks(_ptr(k_cache), _ptr(v_cache), _ptr(src_dst_pairs), src_dst_pairs.shape[0], NB,
                          block_bytes, _ptr(k_scale_cache), _ptr(v_scale_cache), sbytes, _stream(stream)))


def swap_blocks(src_k, src_v, dst_k, dst_v, src_dst_pairs, src_scales=None, dst_scales=None, stream=None):
    """dst_k[d] = src_k[s] (and v, and the scale pools) for each (s, d) pair, across pools.

    One pool side is normally the GPU cache and the other a page-locked host pool
    (``torch.empty(..., pin_memory=True)``): swap-out is GPU -> host, swap-in host -> GPU.
    ``src_dst_pairs`` (int64 [N, 2]) may sit on the GPU or in pinned host memory.  The
    scale pools are given as (k_scale, v_scale) tuples, both sides or neither.  Ordered
    on ``stream``: synchronise it before reading a host destination.
    """
    if src_k.shape[1:] != dst_k.shape[1:] or src_k.dtype != dst_k.dtype:
        raise ValueError("source and destination pools must have the same block shape and dtype")
    for a, b in ((src_k, src_v), (dst_k, dst_v)):
        if a.shape != b.shape or a.dtype != b.dtype:
            raise ValueError("K and V pools must match")
    if src_dst_pairs.dtype != torch.int64 or src_dst_pairs.dim() != 2 or src_dst_pairs.shape[1] != 2:
        raise ValueError("src_dst_pairs must be int64 [N, 2]")
    if (src_scales is None) != (dst_scales is None):
        raise ValueError("pass scale pools for both sides or neither")
    for name, t in (("src_k", src_k), ("src_v", src_v), ("dst_k", dst_k), ("dst_v", dst_v),
                    ("src_dst_pairs", src_dst_pairs)) + tuple(
                        (f"scale pool {i}", t) for i, t in enumerate((src_scales or ()) + (dst_scales or ()))):
        if not (t.is_cuda or t.is_pinned()):
            raise ValueError(f"{name} must be a CUDA tensor or page-locked host memory (pin_memory=True)")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    block_bytes = src_k[0].numel() * src_k.element_size()
    sk = sv = dk = dv = None
    sbytes = 0
    if src_scales is not None:
        (sk, sv), (dk, dv) = src_scales, dst_scales
        sbytes = sk[0].numel() * sk.element_size()
    _check(_L.swap_blocks(_ptr(src_k), _ptr(src_v), _ptr(dst_k), _ptr(dst_v), _ptr(src_dst_pairs),
                          src_dst_pairs.shape[0], src_k.shape[0], dst_k.shape[0], block_bytes,
                          _ptr(sk), _ptr(sv), _ptr(dk), _ptr(dv), sbytes, _stream(stream)))


# ---------------------------------------------------------------------------------------
# Host-side helpers
# ---------------------------------------------------------------------------------------
def slot_mapping(block_tables, seq_ids, positions, block_size: int) -> torch.Tensor:
    """int64 slots of (sequence, position) pairs through host block tables (C helper)."""
    bt = np.ascontiguousarray(torch.as_tensor(block_tables).cpu().numpy(), dtype=np.int32)
    sq = np.ascontiguousarray(np.asarray(seq_ids, dtype=np.int32).reshape(-1))
    ps = np.ascontiguousarray(np.asarray(positions, dtype=np.int32).reshape(-1))
    if sq.shape != ps.shape:
        raise ValueError("seq_ids and positions must have the same length")
    out = np.empty(sq.shape, np.int64)
    _check(_L.pa_slot_mapping_host(bt.ctypes.data, bt.shape[0], bt.shape[1], block_size,
                                   sq.ctypes.data, ps.ctypes.data, sq.size, out.ctypes.data))
    return torch.from_numpy(out)


def device_error(clear: bool = True) -> int:
    """OR of PA_DEVERR_* bits raised by kernels on the current device (synchronises)."""
    flags = ctypes.c_uint32(0)
    _check(_L.pa_device_error(ctypes.byref(flags), int(clear)))
    return flags.value


def use_tensor_cores(enable: bool = True):
    """Let grouped-query decode use the tcgen05 kernel where it qualifies (default on)."""
    _check(_L.pa_decode_use_tensor_cores(int(enable)))


def profile_enable(on: bool = True):
    _check(_L.pa_profile_enable(int(on)))


def profile_read(reset: bool = True):
    """(partition_ms_total, merge_ms_total, calls) recorded since the last reset."""
    a, b, n = ctypes.c_double(), ctypes.c_double(), ctypes.c_int()
    _check(_L.pa_profile_read(ctypes.byref(a), ctypes.byref(b), ctypes.byref(n), int(reset)))
    return a.value, b.value, n.value


class BlockManager:
    """Physical-block allocator (free list popped from its end + reference counts), native.

    ``allocate(n)`` raises RuntimeError when fewer than n blocks are free; ``free(ids)``
    raises RuntimeError (changing nothing) on a double free; ``copy_on_write(id)`` returns
    the id unchanged when it is referenced at most once, else a fresh block.
    """

    def __init__(self, num_blocks: int, block_size: int, free_order=None):
        order = None
        if free_order is not None:
            order = np.ascontiguousarray(np.asarray(free_order, dtype=np.int32))
        self._h = _L.pa_bm_create(num_blocks, block_size, None if order is None else order.ctypes.data)
        if not self._h:
            raise ValueError(_L.pa_last_error().decode())
        self.num_blocks, self.block_size = num_blocks, block_size

    def __del__(self):
        h = getattr(self, "_h", None)
        if h and _L is not None:
            _L.pa_bm_destroy(h)
        self._h = None

    @staticmethod
    def _raise(st):
        if st in (4, 5):
            raise RuntimeError(_L.pa_last_error().decode())
        _check(st)

    def allocate(self, num_blocks: int = 1):
        out = np.empty(max(num_blocks, 0), np.int32)
        self._raise(_L.pa_bm_allocate(self._h, num_blocks, out.ctypes.data))
        return out.tolist()

    def free(self, block_ids):
        ids = np.ascontiguousarray(np.asarray(list(block_ids), dtype=np.int32))
        self._raise(_L.pa_bm_free(self._h, ids.ctypes.data, ids.size))

    def share(self, block_ids):
        ids = np.ascontiguousarray(np.asarray(list(block_ids), dtype=np.int32))
        self._raise(_L.pa_bm_share(self._h, ids.ctypes.data, ids.size))

    def copy_on_write(self, block_id: int) -> int:
        out = ctypes.c_int32()
        self._raise(_L.pa_bm_copy_on_write(self._h, int(block_id), ctypes.byref(out)))
        return out.value

    def usage_ratio(self) -> float:
        return _L.pa_bm_usage_ratio(self._h)

    def ref_count(self, block_id: int) -> int:
        return _L.pa_bm_ref_count(self._h, int(block_id))

    @property
    def free_blocks(self):
        n = ctypes.c_int()
        _check(_L.pa_bm_free_list(self._h, None, 0, ctypes.byref(n)))
        out = np.empty(n.value, np.int32)
        _check(_L.pa_bm_free_list(self._h, out.ctypes.data, n.value, ctypes.byref(n)))
        return out.tolist()
