"""Workload recipes for paged decode attention.

Shapes follow the pages' examples: the Llama-2-70B layer of "KV Cache memory
optimisation and PagedAttention" (yunthe.com), section "大模型推理KV Cache内存消耗模型"
(64 heads x 128 dims, fp16), block_size 16 (section "PagedAttention分页内存管理原理"),
the 2000-token shared system prompt of "KV Cache optimisation strategies in deployment"
(yunthe.com), section "Prefix Cache复用共享前缀的KV Cache", and its W = 4096 sliding
window (section "Sliding Window Attention控制长序列显存").

Every draw comes from one ``torch.Generator`` seeded with ``seed``, in a fixed order:
context lengths, free-list permutation, then values (q, K cache, V cache, new K, new V).
Values are N(0, 1) drawn in fp32 and cast (round to nearest even) to the storage dtype.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Callable, List, Optional

import torch

_DT = {"fp32": torch.float32, "fp16": torch.float16, "bf16": torch.bfloat16}


@dataclass
class Workload:
    name: str
    num_seqs: int
    num_heads: int                  # query heads
    head_dim: int
    block_size: int
    num_blocks: int
    io_dtype: str                   # "fp32" | "fp16" | "bf16"
    cache_dtype: str                # io_dtype, or "int8" (values below are then the fp16 source)
    scale: float
    window: int
    context_lens: torch.Tensor      # int32 [S], newest token included
    block_tables: torch.Tensor      # int32 [S, MB], -1 past each sequence's blocks
    q: torch.Tensor                 # [S, H, D] io dtype
    k_cache: torch.Tensor           # [NB, bs, H, D] (source dtype)
    v_cache: torch.Tensor
    k_new: torch.Tensor             # [S, H, D] K/V of each sequence's newest token
    v_new: torch.Tensor
    copy_pairs: torch.Tensor        # int64 [N, 2] (src, dst) copy-on-write block copies
    tables: List[List[int]] = field(default_factory=list)
    notes: dict = field(default_factory=dict)
    num_kv_heads: int = 0           # cached heads (== num_heads unless grouped-query)

    @property
    def max_blocks_per_seq(self) -> int:
        return self.block_tables.shape[1]


def _ceil_div(a: int, b: int) -> int:
    return -(-a // b)


def _pack_tables(tables: List[List[int]], mb: Optional[int] = None) -> torch.Tensor:
    mb = max(1, max((len(t) for t in tables), default=1)) if mb is None else mb
    out = torch.full((len(tables), mb), -1, dtype=torch.int32)
    for s, t in enumerate(tables):
        if t:
            out[s, : len(t)] = torch.tensor(t, dtype=torch.int32)
    return out


def _values(gen: torch.Generator, shape, dtype: str, device) -> torch.Tensor:
    x = torch.randn(shape, generator=gen, dtype=torch.float32, device=device)
    return x.to(_DT["fp16" if dtype == "int8" else dtype])


def _generator(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def build_workload(preset: str, seed: int, bm_factory: Callable, device="cpu", **overrides) -> Workload:
    """Build preset ``preset`` with allocator class ``bm_factory(num_blocks, block_size, free_order)``.

    ``overrides`` replace preset parameters (e.g. ``num_seqs``, ``block_size``).
    Context lengths and the free-list order are drawn on the CPU generator; values on
    ``device`` (one generator per device, same seed).
    """
    if preset not in PRESETS:
        raise KeyError(f"unknown preset {preset!r}; known: {sorted(PRESETS)}")
    p = dict(PRESETS[preset])
    p.update(overrides)
    return _BUILDERS[p["kind"]](preset, seed, bm_factory, device, p)


def _build_independent(name, seed, bm_factory, device, p) -> Workload:
    """Sequences with private blocks only (tiny, Llama-2-70B layer, INT8, sliding window)."""
    S, H, D, bs = p["num_seqs"], p["num_heads"], p["head_dim"], p["block_size"]
    gcpu = _generator(seed, "cpu")
    if "context_lens" in p:
        ctx = [int(c) for c in p["context_lens"]]
    else:
        lo, hi = p["ctx_range"]
        ctx = torch.randint(lo, hi + 1, (S,), generator=gcpu).tolist()
    blocks_needed = sum(_ceil_div(c, bs) for c in ctx)
    nb = p.get("num_blocks") or math.ceil(p.get("slack", 1.1) * blocks_needed)
    nb = max(nb, blocks_needed, 1)
    free_order = torch.randperm(nb, generator=gcpu).tolist()
    bm = bm_factory(nb, bs, free_order)
    tables = [bm.allocate(_ceil_div(c, bs)) if c > 0 else [] for c in ctx]
    return _finish(name, seed, device, p, ctx, nb, tables, bm, pairs=[])


def _build_prefix_shared(name, seed, bm_factory, device, p) -> Workload:
    """Chat decode: one shared prompt prefix + private tails, then copy-on-write forks."""
    S, H, D, bs = p["num_seqs"], p["num_heads"], p["head_dim"], p["block_size"]
    prefix = p["prefix_len"]
    gcpu = _generator(seed, "cpu")
    mu, sigma = math.log(p["tail_median"]), p["tail_sigma"]
    tails = torch.exp(mu + sigma * torch.randn(S, generator=gcpu, dtype=torch.float64))
    tails = [int(min(max(round(float(t)), 1), p["tail_cap"])) for t in tails]
    n_div = p["num_diverge"]
    diverge = sorted(torch.randperm(S, generator=gcpu)[:n_div].tolist())
    if prefix % bs:
        raise ValueError("the shared prefix must fill whole blocks")
    prefix_blocks = prefix // bs
    blocks_needed = prefix_blocks + sum(_ceil_div(prefix + t, bs) - prefix_blocks for t in tails) + n_div
    nb = math.ceil(p.get("slack", 1.1) * blocks_needed)
    free_order = torch.randperm(nb, generator=gcpu).tolist()
    bm = bm_factory(nb, bs, free_order)

    shared = bm.allocate(prefix_blocks)
    tables = []
    for s in range(S):
        if s > 0:
            bm.share(shared)
        ctx = prefix + tails[s]
        own = bm.allocate(_ceil_div(ctx, bs) - prefix_blocks)
        tables.append(list(shared) + own)
    # The forks: copy-on-write of the last shared prompt block.
    pairs = []
    last = prefix_blocks - 1
    for s in diverge:
        old = tables[s][last]
        new = bm.copy_on_write(old)
        if new != old:
            pairs.append((old, new))
            tables[s][last] = new
    ctx = [prefix + t for t in tails]
    w = _finish(name, seed, device, p, ctx, nb, tables, bm, pairs)
    w.notes.update(prefix_len=prefix, tails=tails, diverge=diverge, shared_blocks=list(shared),
                   tail_sigma=sigma)
    return w


def _finish(name, seed, device, p, ctx, nb, tables, bm, pairs) -> Workload:
    S, H, D, bs = p["num_seqs"], p["num_heads"], p["head_dim"], p["block_size"]
    Hkv = p.get("num_kv_heads", H)
    gdev = _generator(seed, device)
    dt = p["dtype"]
    q = _values(gdev, (S, H, D), dt, device)
    if dt == "int8":
        q = q.to(torch.float16)
    kc = _values(gdev, (nb, bs, Hkv, D), dt, device)
    vc = _values(gdev, (nb, bs, Hkv, D), dt, device)
    kn = _values(gdev, (S, Hkv, D), dt, device)
    vn = _values(gdev, (S, Hkv, D), dt, device)
    mb = p.get("max_blocks_per_seq")
    return Workload(
        name=name, num_seqs=S, num_heads=H, head_dim=D, block_size=bs, num_blocks=nb,
        io_dtype="fp16" if dt == "int8" else dt, cache_dtype=dt,
        scale=p.get("scale", 1.0 / math.sqrt(D)), window=p.get("window", 0),
        context_lens=torch.tensor(ctx, dtype=torch.int32),
        block_tables=_pack_tables(tables, mb), q=q, k_cache=kc, v_cache=vc, k_new=kn, v_new=vn,
        copy_pairs=torch.tensor(pairs, dtype=torch.int64).reshape(-1, 2),
        tables=[list(t) for t in tables], notes={"seed": seed, "allocator": bm}, num_kv_heads=Hkv)


_BUILDERS = {"independent": _build_independent, "prefix": _build_prefix_shared}

# Workload presets.  Sizes are the full ones; tests shrink them with overrides.
PRESETS = {
    # 4 sequences, fp32, contexts {1, 15, 16, 33}, pool of 32 shuffled blocks.
    "tiny_fp32": dict(kind="independent", num_seqs=4, num_heads=4, head_dim=64, block_size=16,
                      context_lens=[1, 15, 16, 33], num_blocks=32, dtype="fp32", scale=1.0 / 8.0),
    # One Llama-2-70B attention layer: 32 sequences x 64 heads x 128, contexts U[1, 2048].
    "llama70b_fp16": dict(kind="independent", num_seqs=32, num_heads=64, head_dim=128,
                          block_size=16, ctx_range=(1, 2048), slack=1.1, dtype="fp16"),
    # Same shapes, INT8 cache (values are the fp16 source; the consumer quantises).
    "llama70b_int8": dict(kind="independent", num_seqs=32, num_heads=64, head_dim=128,
                          block_size=16, ctx_range=(1, 2048), slack=1.1, dtype="int8"),
    # The real Llama-2-70B attention layer is grouped-query (64 query heads share 8 cached
    # heads); 256 sequences keep the per-step KV stream above 1 GB like the layer above.
    "llama70b_gqa_fp16": dict(kind="independent", num_seqs=256, num_heads=64, num_kv_heads=8, head_dim=128,
                              block_size=16, ctx_range=(1, 2048), slack=1.1, dtype="fp16"),
    # High-concurrency chat: 256 sequences share a 2000-token prompt, lognormal tails
    # (median 300, sigma 1.0, cap 2048); 64 sequences fork the last shared block.
    "chat_prefix_bf16": dict(kind="prefix", num_seqs=256, num_heads=32, head_dim=128, block_size=16,
                             prefix_len=2000, tail_median=300.0, tail_sigma=1.0, tail_cap=2048,
                             num_diverge=64, slack=1.02, dtype="bf16"),
    # Long context with a sliding window: 8 x 32768 tokens, attend the last 4096.
    "sliding_window_fp16": dict(kind="independent", num_seqs=8, num_heads=32, head_dim=128,
                                block_size=16, context_lens=[32768] * 8, slack=1.0, window=4096,
                                dtype="fp16"),
}
