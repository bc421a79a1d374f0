"""GPU parity of paged_attention_decode (through the C ABI) against the fp64 oracle.

Covers the five workload recipes (tiny fp32 with a one-token append, the Llama-2-70B
layer in fp16 at full size, the chat prefix-sharing batch in bf16 with copy-on-write
forks, the INT8 cache at full size, the 32k-token sliding window with block sizes 8/16/32,
every output of each compared with the oracle)
and edge cases: empty and one-token contexts, partial blocks, unused slots and skipped
blocks poisoned with NaN, odd block sizes, head counts that force one head per CTA, a
single 32k context split over every CTA, thousands of tiny sequences, bad table entries
(reported, not faulted), and run-to-run determinism.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_384_b200 as pa
import synth
from oracle.block_manager import BlockManager as OracleBM
from oracle.block_manager import BlockTable
from parity import TOL, GpuCase, assert_no_device_error, compare, oracle_decode, quantize_cache, quantize_cache_fp8

pytestmark = pytest.mark.gpu


def _ceil(a, b):
    return -(-a // b)


def _poison_unattended(k, v, tables, ctx, bs, window=0):
    """NaN every cache row no attended token lives in (free blocks, rows past the context,
    rows before the window), so a kernel that reads one produces NaN."""
    NB = k.shape[0]
    live = torch.zeros(NB, bs, dtype=torch.bool)
    for t, c in zip(tables, ctx):
        lo = max(0, c - window) if window > 0 else 0
        for i in range(lo, c):
            live[t[i // bs], i % bs] = True
    if k.dtype in (torch.int8, torch.float8_e4m3fn):  # 8-bit codes: the NaN goes into the scales
        return live
    k[~live] = float("nan")
    v[~live] = float("nan")
    return live


def _small_case(seed, S, H, D, bs, ctx, dtype, window=0, device="cuda"):
    """Random case with shuffled blocks; int8 caches are quantised by the oracle quantiser."""
    g = torch.Generator().manual_seed(seed)
    need = sum(_ceil(c, bs) for c in ctx)
    NB = need + 5
    order = torch.randperm(NB, generator=g).tolist()
    bm = OracleBM(NB, bs, order)
    tables = [bm.allocate(_ceil(c, bs)) if c > 0 else [] for c in ctx]
    MB = max(1, max(len(t) for t in tables))
    bt = torch.full((S, MB), -1, dtype=torch.int32)
    for s, t in enumerate(tables):
        if t:
            bt[s, : len(t)] = torch.tensor(t, dtype=torch.int32)
    eight_bit = dtype.startswith("int8") or dtype.startswith("fp8")
    io = ("bf16" if dtype.endswith("-bf16") else "fp16") if eight_bit else dtype
    tdt = {"fp32": torch.float32, "fp16": torch.float16, "bf16": torch.bfloat16}[io]
    q = torch.randn(S, H, D, generator=g).to(tdt)
    src = torch.float16 if eight_bit else tdt
    k = torch.randn(NB, bs, H, D, generator=g).to(src)
    v = torch.randn(NB, bs, H, D, generator=g).to(src)
    scale = 1.0 / math.sqrt(D)
    ks = vs = None
    if eight_bit:
        quantize = quantize_cache if dtype.startswith("int8") else quantize_cache_fp8
        k, ks = quantize(k)
        v, vs = quantize(v)
        live = _poison_unattended(k, v, tables, ctx, bs, window)
        ks[~live] = float("nan")
        vs[~live] = float("nan")
    else:
        _poison_unattended(k, v, tables, ctx, bs, window)
    ref = oracle_decode(q, k, v, bt, ctx, scale, window, ks, vs)
    case = GpuCase(q, k, v, bt, ctx, scale, window, ks, vs, device)
    return case, ref, io


def _check(case, ref, io, tol=None):
    out = case.decode()
    torch.cuda.synchronize()
    assert_no_device_error()
    return compare(out, ref, io, tol if tol is not None else (TOL["int8"] if case.k_scale is not None else TOL[io]))


# ---------------------------------------------------------------------------------------
# The five recipes
# ---------------------------------------------------------------------------------------
def test_tiny_fp32_with_one_token_append(cuda_device):
    w = synth.build_workload("tiny_fp32", 0, OracleBM)
    # the library's own block manager lays the sequences out exactly like the oracle's
    assert synth.build_workload("tiny_fp32", 0, pa.BlockManager).tables == w.tables
    # decode over {1, 15, 16, 33}
    case = GpuCase(w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale)
    ref = oracle_decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale)
    _check(case, ref, "fp32")
    # append one token per sequence (a new block where the last one is full), then decode again
    bm = w.notes["allocator"]
    bs = w.block_size
    tables = [list(t) for t in w.tables]
    ctx = w.context_lens.tolist()
    for s, c in enumerate(ctx):
        if c % bs == 0:
            tables[s] += bm.allocate(1)
    oracle_slots = [BlockTable(t).get_physical_block(c, bs) * bs + BlockTable(t).get_offset(c, bs)
                    for t, c in zip(tables, ctx)]
    MB = max(len(t) for t in tables)
    bt = torch.tensor([t + [-1] * (MB - len(t)) for t in tables], dtype=torch.int32)
    gpu_slots = pa.slot_mapping(bt, list(range(len(ctx))), ctx, bs)
    assert gpu_slots.tolist() == oracle_slots
    new_ctx = [c + 1 for c in ctx]
    kc, vc = w.k_cache.clone().numpy(), w.v_cache.clone().numpy()
    oracle.cache_ops.reshape_and_cache(w.k_new.numpy(), w.v_new.numpy(), kc, vc, np.array(oracle_slots))
    ref2 = oracle_decode(w.q, torch.from_numpy(kc), torch.from_numpy(vc), bt, new_ctx, w.scale)
    case2 = GpuCase(w.q, w.k_cache, w.v_cache, bt, new_ctx, w.scale)
    pa.reshape_and_cache(w.k_new.cuda(), w.v_new.cuda(), case2.k_cache, case2.v_cache, gpu_slots.cuda())
    _check(case2, ref2, "fp32")
    assert torch.equal(case2.k_cache.cpu(), torch.from_numpy(kc))
    assert torch.equal(case2.v_cache.cpu(), torch.from_numpy(vc))


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_llama70b_layer_fp16_full_size_step(cuda_device, seed):
    """Full-size step: write each sequence's newest token, then decode; every output checked."""
    w = synth.build_workload("llama70b_fp16", seed, OracleBM)
    ctx = w.context_lens.tolist()
    bs = w.block_size
    slots = [w.tables[s][(c - 1) // bs] * bs + (c - 1) % bs for s, c in enumerate(ctx)]
    kc, vc = w.k_cache.numpy().copy(), w.v_cache.numpy().copy()
    oracle.cache_ops.reshape_and_cache(w.k_new.numpy(), w.v_new.numpy(), kc, vc, np.array(slots))
    ref = oracle_decode(w.q, torch.from_numpy(kc), torch.from_numpy(vc), w.block_tables, ctx, w.scale)
    case = GpuCase(w.q, w.k_cache, w.v_cache, w.block_tables, ctx, w.scale)
    pa.reshape_and_cache(w.k_new.cuda(), w.v_new.cuda(), case.k_cache, case.v_cache,
                         pa.slot_mapping(w.block_tables, range(len(ctx)), [c - 1 for c in ctx], bs).cuda())
    _check(case, ref, "fp16")


def test_llama70b_layer_int8_full_size(cuda_device):
    w = synth.build_workload("llama70b_int8", 0, OracleBM)
    k, ks = quantize_cache(w.k_cache)
    v, vs = quantize_cache(w.v_cache)
    ref = oracle_decode(w.q, k, v, w.block_tables, w.context_lens, w.scale, 0, ks, vs)
    case = GpuCase(w.q, k, v, w.block_tables, w.context_lens, w.scale, 0, ks, vs)
    err, raw, _ = _check(case, ref, "fp16", TOL["int8"])
    # information only: distance to attention over the unquantised fp16 cache
    ref_fp16 = oracle_decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale)
    assert np.max(np.abs(ref - ref_fp16)) < 0.1


def test_chat_prefix_bf16_with_copy_on_write(cuda_device):
    w = synth.build_workload("chat_prefix_bf16", 0, OracleBM)
    bm = w.notes["allocator"]
    last = w.notes["shared_blocks"][-1]
    assert bm.ref_count[last] == 256 - len(w.copy_pairs) and len(w.copy_pairs) == 64
    # GPU: copy-on-write block copies, then decode
    case = GpuCase(w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale)
    pa.copy_blocks(case.k_cache, case.v_cache, w.copy_pairs.cuda())
    out = case.decode()
    torch.cuda.synchronize()
    assert_no_device_error()
    # oracle: the same copies on the host, then a sampled subset of sequences
    kc = w.k_cache.view(torch.int16).numpy().copy()
    vc = w.v_cache.view(torch.int16).numpy().copy()
    oracle.cache_ops.copy_blocks(kc, vc, w.copy_pairs.numpy())
    dst = w.copy_pairs[:, 1]
    assert torch.equal(case.k_cache[dst.cuda()].cpu().view(torch.int16), torch.from_numpy(kc[dst.numpy()]))
    assert torch.equal(case.v_cache[dst.cuda()].cpu().view(torch.int16), torch.from_numpy(vc[dst.numpy()]))
    kt = torch.from_numpy(kc).view(torch.bfloat16)
    vt = torch.from_numpy(vc).view(torch.bfloat16)
    ctx = w.context_lens
    div = w.notes["diverge"]
    # every output of all 256 sequences against the oracle on the copied pool
    ref = oracle_decode(w.q, kt, vt, w.block_tables, ctx, w.scale)
    compare(out, ref, "bf16", TOL["bf16"])
    # forked sequences read copies identical to the shared block: same output as without the fork
    case_nofork = GpuCase(w.q, w.k_cache, w.v_cache, w.block_tables.clone(), ctx, w.scale)
    bt = case_nofork.block_tables
    bt[div, len(w.notes["shared_blocks"]) - 1] = last
    out2 = case_nofork.decode()
    torch.cuda.synchronize()
    assert torch.equal(out2[div].cpu(), out[div].cpu())


@pytest.mark.parametrize("bs", [8, 16, 32])
def test_sliding_window_32k_fp16(cuda_device, bs):
    w = synth.build_workload("sliding_window_fp16", 0, OracleBM, device="cuda", block_size=bs)
    case = GpuCase(w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale, w.window)
    out = case.decode()
    torch.cuda.synchronize()
    assert_no_device_error()
    # oracle on all 8 sequences: only the blocks that hold windowed tokens come back to the
    # host, packed into a small pool; every other table entry becomes -1, so a read outside
    # the window would fail in the oracle
    W = w.window
    S, MB = w.block_tables.shape
    bt = torch.full((S, MB), -1, dtype=torch.int32)
    ids = []
    for s in range(S):
        c = int(w.context_lens[s])
        first, last = (c - W) // bs, _ceil(c, bs)
        seq_ids = w.block_tables[s, first:last].tolist()
        bt[s, first:last] = torch.arange(len(ids), len(ids) + len(seq_ids), dtype=torch.int32)
        ids += seq_ids
    sel = torch.tensor(ids, device="cuda")
    kc, vc = w.k_cache[sel].cpu(), w.v_cache[sel].cpu()
    ref = oracle_decode(w.q.cpu(), kc, vc, bt, w.context_lens.cpu(), w.scale, W)
    compare(out, ref, "fp16", TOL["fp16"])


# ---------------------------------------------------------------------------------------
# Edge cases
# ---------------------------------------------------------------------------------------
DTYPES = ["fp32", "fp16", "bf16", "int8", "int8-bf16", "fp8", "fp8-bf16"]


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("bs", [1, 5, 8, 12, 16, 24, 32])
def test_dtype_headdim_blocksize_grid(cuda_device, dtype, D, bs):
    ctx = [0, 1, bs, bs + 1, 2 * bs - 1, 97, 300, 5]
    case, ref, io = _small_case(100 + bs + D, len(ctx), 8, D, bs, ctx, dtype)
    _check(case, ref, io)


@pytest.mark.parametrize("window", [1, 7, 15, 16, 17, 100, 4096])
@pytest.mark.parametrize("dtype", ["fp16", "int8"])
def test_window_edges(cuda_device, window, dtype):
    ctx = [1, 15, 16, 17, 33, 100, 257, 1000]
    case, ref, io = _small_case(window, len(ctx), 8, 128, 16, ctx, dtype, window=window)
    _check(case, ref, io)


@pytest.mark.parametrize("H", [1, 3, 5, 6, 12])
def test_head_counts_that_are_not_multiples_of_four(cuda_device, H):
    ctx = [3, 40, 129, 0, 64]
    case, ref, io = _small_case(H, len(ctx), H, 128, 16, ctx, "bf16")
    _check(case, ref, io)


def test_one_long_sequence_split_over_every_cta(cuda_device):
    case, ref, io = _small_case(7, 1, 8, 128, 16, [32768], "fp16")
    _check(case, ref, io)


def test_thousands_of_tiny_sequences(cuda_device):
    rng = np.random.default_rng(3)
    ctx = [int(c) for c in rng.integers(0, 21, 3000)]
    case, ref, io = _small_case(11, len(ctx), 4, 64, 16, ctx, "fp16")
    _check(case, ref, io)


def test_all_sequences_empty_gives_zeros(cuda_device):
    case, ref, io = _small_case(12, 4, 8, 128, 16, [0, 0, 0, 0], "fp16")
    out = case.decode()
    torch.cuda.synchronize()
    assert torch.count_nonzero(out) == 0


def test_repeated_calls_are_bitwise_deterministic(cuda_device):
    w = synth.build_workload("llama70b_fp16", 4, OracleBM, num_seqs=8)
    case = GpuCase(w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale)
    a = case.decode()
    b = case.decode()
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_side_stream(cuda_device):
    case, ref, io = _small_case(13, 6, 8, 128, 16, [5, 60, 300, 1, 17, 1024], "fp16")
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        out = case.decode(stream=s)
    s.synchronize()
    assert_no_device_error()
    compare(out, ref, io, TOL[io])


def test_bad_table_entries_are_reported_not_faulted(cuda_device):
    case, ref, io = _small_case(14, 3, 8, 128, 16, [20, 40, 9], "fp16")
    NB = case.k_cache.shape[0]
    case.block_tables[1, 1] = NB + 1000      # out of the pool
    case.block_tables[2, 0] = -7
    out = case.decode()
    torch.cuda.synchronize()
    flags = pa.device_error(clear=True)
    assert flags & pa.DEVERR["table"]
    compare(out[:1], ref[:1], io, TOL[io])   # the untouched sequence is still right


def test_context_beyond_the_table_is_clamped_and_reported(cuda_device):
    case, ref, io = _small_case(15, 2, 8, 128, 16, [20, 32], "fp16")
    MB = case.block_tables.shape[1]
    case.context_lens[1] = MB * 16 + 50
    case.decode()
    torch.cuda.synchronize()
    assert pa.device_error(clear=True) & pa.DEVERR["context"]


def test_workspace_too_small_is_rejected(cuda_device):
    case, ref, io = _small_case(16, 2, 8, 128, 16, [20, 32], "fp16")
    out = torch.empty_like(case.q)
    with pytest.raises(pa.PagedAttnError, match="workspace"):
        pa.paged_attention_decode(out, case.q, case.k_cache, case.v_cache, case.block_tables,
                                  case.context_lens, case.scale, workspace=case.workspace[:64])


def test_alternating_ring_sizes_on_one_kernel(cuda_device):
    """One kernel instantiation launched with a large, then a small, then the large
    shared-memory ring again (a regression test for the per-kernel smem limit)."""
    big, ref_big, io = _small_case(21, 3, 64, 128, 16, [40, 300, 17], "fp16")
    small, ref_small, _ = _small_case(22, 3, 1, 128, 16, [40, 300, 17], "fp16")
    for case, ref in ((big, ref_big), (small, ref_small), (big, ref_big)):
        _check(case, ref, io)
