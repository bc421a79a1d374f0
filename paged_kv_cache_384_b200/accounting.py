"""Byte and waste accounting for paged KV caches (host arithmetic on sizes only).

* Per-token KV bytes: 2 (K and V) x layers x heads x head_dim x element bytes
  ("KV Cache memory optimisation and PagedAttention" (yunthe.com), section
  "大模型推理KV Cache内存消耗模型").
* Waste of a contiguous reservation vs. a paged allocation ("vLLM source first look:
  PagedAttention memory design" (trdm.cn), section 一, flowchart; block-size-16 waste claim
  in "KV Cache memory optimisation and PagedAttention", section "vLLM调度器与PagedAttention协同工作").
* Algorithmic bytes of one decode call: every attended token's K and V row for every head
  is read exactly once (plus the fp16 scales of an INT8 or FP8 cache).  This is the numerator of
  the KV GB/s metric.
"""
from __future__ import annotations

from typing import Iterable

ELEM_BYTES = {"fp32": 4, "fp16": 2, "bf16": 2, "int8": 1, "fp8": 1}


def kv_bytes_per_token(layers: int, num_heads: int, head_dim: int, dtype_size: int) -> int:
    return 2 * layers * num_heads * head_dim * dtype_size


def contiguous_waste_fraction(used_tokens: int, reserved_tokens: int) -> float:
    """Share of a contiguous max-length reservation left unused."""
    return 1.0 - used_tokens / reserved_tokens


def paged_waste_fraction(used_tokens: int, block_size: int) -> float:
    """Share of the allocated blocks left unused when blocks are taken on demand."""
    if used_tokens <= 0:
        return 0.0
    allocated = -(-used_tokens // block_size) * block_size
    return (allocated - used_tokens) / allocated


def attended_tokens(context_len: int, window: int = 0) -> int:
    """Tokens one decode step reads: the whole context, or its last ``window`` tokens."""
    return min(context_len, window) if window > 0 else context_len


def decode_kv_bytes(context_lens: Iterable[int], num_heads: int, head_dim: int, cache_dtype: str,
                    window: int = 0) -> int:
    """Algorithmic K+V bytes of one decode call over a batch (scales included for 8-bit caches)."""
    e = ELEM_BYTES[cache_dtype]
    tokens = sum(attended_tokens(int(c), window) for c in context_lens)
    total = tokens * num_heads * head_dim * 2 * e
    if cache_dtype in ("int8", "fp8"):
        total += tokens * num_heads * 2 * 2  # one fp16 scale per (token, head) for K and for V
    return total


def prefill_flops(context_lens: Iterable[int], q_lens: Iterable[int], num_q_heads: int, head_dim: int,
                  window: int = 0) -> float:
    """Algorithmic FLOPs of one prefill call: query i of a sequence with ctx tokens and q_len
    queries sits at position p = ctx - q_len + i and attends p + 1 tokens (at most ``window``),
    each costing 4 * head_dim FLOPs (one multiply-add in QK^T and one in PV)."""
    rows = 0
    for ctx, ql in zip(context_lens, q_lens):
        first = int(ctx) - int(ql)
        rows += sum(attended_tokens(p + 1, window) for p in range(first, int(ctx)))
    return 4.0 * head_dim * num_q_heads * rows


def decode_unique_kv_bytes(block_tables, context_lens: Iterable[int], block_size: int, num_heads: int,
                           head_dim: int, cache_dtype: str, window: int = 0) -> int:
    """Bytes of the distinct cache rows one decode call reads: rows shared by several
    sequences (a common prompt prefix held once, "KV Cache optimisation strategies in
    deployment" (yunthe.com), section "Prefix Cache复用共享前缀的KV Cache") count once.  This
    is the least DRAM traffic the call can cause; ``decode_kv_bytes`` counts every
    sequence's rows."""
    e = ELEM_BYTES[cache_dtype]
    rows = set()
    for s, c in enumerate(context_lens):
        c = int(c)
        lo = c - attended_tokens(c, window)
        table = block_tables[s]
        for lb in range(lo // block_size, -(-c // block_size)):
            first = max(lo, lb * block_size) - lb * block_size
            last = min(c, (lb + 1) * block_size) - lb * block_size
            pb = int(table[lb])
            rows.update((pb, off) for off in range(first, last))
    per_row = num_heads * head_dim * 2 * e
    if cache_dtype in ("int8", "fp8"):
        per_row += num_heads * 2 * 2
    return len(rows) * per_row
