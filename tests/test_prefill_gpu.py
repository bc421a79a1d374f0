"""GPU paged prefill / chunked-prefill attention (tcgen05) through the C ABI against the
fp64 oracle: whole prompts, chunks behind cached context and single tokens in one batch,
fp16 and bf16, 1 to 16 query heads per cached head, every block size, sliding windows,
several query and KV tiles with ragged tails, chunked = one-shot, empty sequences,
out-of-range inputs reported (not faulted), and INT8 / FP8 caches (tolerance 1e-2).  Pool rows no sequence owns hold NaN, so a
read outside the attended tokens shows up as a non-finite output."""
import math

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_384_b200 as pa
from parity import TOL, assert_no_device_error, compare, quantize_cache, quantize_cache_fp8

pytestmark = pytest.mark.gpu

DT = {"fp16": torch.float16, "bf16": torch.bfloat16}


def paged_case(seed, ctx, qlen, Hq, Hkv, bs, io, D=128, extra=5):
    """A shuffled pool holding each sequence's ctx tokens; q rows for its newest qlen tokens."""
    g = torch.Generator().manual_seed(seed)
    S = len(ctx)
    nblk = [-(-c // bs) for c in ctx]
    NB = sum(nblk) + extra
    perm = torch.randperm(NB, generator=g).tolist()
    kc = torch.full((NB, bs, Hkv, D), float("nan"), dtype=DT[io])
    vc = torch.full((NB, bs, Hkv, D), float("nan"), dtype=DT[io])
    MB = max(1, max(nblk))
    bt = torch.full((S, MB), -1, dtype=torch.int32)
    k = 0
    for s in range(S):
        K = torch.randn(ctx[s], Hkv, D, generator=g).to(DT[io])
        V = torch.randn(ctx[s], Hkv, D, generator=g).to(DT[io])
        for lb in range(nblk[s]):
            pb = perm[k]
            k += 1
            bt[s, lb] = pb
            lo, hi = lb * bs, min(ctx[s], (lb + 1) * bs)
            kc[pb, : hi - lo] = K[lo:hi]
            vc[pb, : hi - lo] = V[lo:hi]
    q = torch.randn(sum(qlen), Hq, D, generator=g).to(DT[io])
    cu = torch.tensor([0] + list(np.cumsum(qlen)), dtype=torch.int32)
    return q, kc, vc, bt, cu, torch.tensor(ctx, dtype=torch.int32)


def run_gpu(q, kc, vc, bt, cu, ctx, scale, window=0, max_q_len=None):
    out = torch.empty_like(q, device="cuda")
    mq = int((cu[1:] - cu[:-1]).max()) if max_q_len is None else max_q_len
    pa.paged_attention_prefill(out, q.cuda(), kc.cuda(), vc.cuda(), bt.cuda(), cu.cuda(), ctx.cuda(), mq, scale,
                               window)
    torch.cuda.synchronize()
    return out


def check(seed, ctx, qlen, Hq, Hkv, bs, io, window=0, D=128):
    q, kc, vc, bt, cu, cl = paged_case(seed, ctx, qlen, Hq, Hkv, bs, io, D=D)
    scale = 1 / math.sqrt(D)
    out = run_gpu(q, kc, vc, bt, cu, cl, scale, window)
    assert_no_device_error()
    ref = oracle.paged_prefill(q, kc, vc, bt, cu, cl, scale, window)
    return compare(out, ref, io, TOL[io])


@pytest.mark.parametrize("io", ["fp16", "bf16"])
@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 2), (16, 2), (8, 1)])
def test_prefill_mixed_batch(cuda_device, io, Hq, Hkv):
    # a whole prompt, a chunk behind cached context, a single token, a prompt of one block
    check(1, [37, 300, 129, 16], [37, 90, 1, 16], Hq, Hkv, 16, io)


@pytest.mark.parametrize("bs", [8, 16, 32, 64, 128])
def test_prefill_block_sizes(cuda_device, bs):
    check(2, [130, 77, 256], [130, 40, 129], 4, 2, bs, "fp16")


@pytest.mark.parametrize("window", [1, 17, 128, 300, 5000])
def test_prefill_sliding_window(cuda_device, window):
    check(3, [400, 260, 45], [400, 70, 45], 8, 2, 16, "fp16", window)
    check(4, [333], [200], 2, 2, 32, "bf16", window)


def test_prefill_sixteen_query_heads_per_cached_head(cuda_device):
    check(5, [200, 57], [200, 57], 32, 2, 16, "bf16")


@pytest.mark.parametrize("io", ["fp16", "bf16"])
def test_prefill_long_prompt_many_tiles(cuda_device, io):
    # 9 query tiles x 8 KV tiles per head, ragged in both
    check(6, [1000], [1000], 2, 2, 16, io)


def test_chunked_prefill_equals_one_shot(cuda_device):
    n = 700
    q, kc, vc, bt, cu, cl = paged_case(7, [n], [n], 8, 8, 16, "fp16")
    scale = 0.09
    whole = run_gpu(q, kc, vc, bt, cu, cl, scale)
    pieces = []
    for a, b in ((0, 130), (130, 131), (131, 512), (512, 700)):
        pieces.append(run_gpu(q[a:b].contiguous(), kc, vc, bt, torch.tensor([0, b - a], dtype=torch.int32),
                              torch.tensor([b], dtype=torch.int32), scale))
    chunked = torch.cat(pieces)
    ref = oracle.paged_prefill(q, kc, vc, bt, cu, cl, scale)
    compare(chunked, ref, "fp16", TOL["fp16"])
    compare(whole, ref, "fp16", TOL["fp16"])
    assert (chunked.float() - whole.float()).abs().max().item() <= 2e-3


def test_prefill_empty_sequences_and_loose_max_q_len(cuda_device):
    q, kc, vc, bt, cu, cl = paged_case(8, [50, 20, 90], [0, 20, 0], 4, 4, 16, "bf16")
    out = run_gpu(q, kc, vc, bt, cu, cl, 0.1, max_q_len=300)
    assert_no_device_error()
    ref = oracle.paged_prefill(q, kc, vc, bt, cu, cl, 0.1)
    compare(out, ref, "bf16", TOL["bf16"])


def test_prefill_single_tokens_match_decode(cuda_device):
    ctx = [1, 15, 16, 33, 700]
    q, kc, vc, bt, cu, cl = paged_case(9, ctx, [1] * 5, 16, 2, 16, "fp16")
    pre = run_gpu(q, kc, vc, bt, cu, cl, 0.2)
    dec = torch.empty_like(q, device="cuda")
    pa.paged_attention_decode(dec, q.cuda(), kc.cuda(), vc.cuda(), bt.cuda(), cl.cuda(), 0.2)
    torch.cuda.synchronize()
    assert (pre.float() - dec.float()).abs().max().item() <= 2e-3
    compare(pre, oracle.paged_prefill(q, kc, vc, bt, cu, cl, 0.2), "fp16", TOL["fp16"])


def test_prefill_reports_bad_lengths_and_table_entries(cuda_device):
    q, kc, vc, bt, cu, cl = paged_case(10, [40, 40], [40, 40], 2, 2, 16, "fp16")
    bad_cl = cl.clone()
    bad_cl[1] = 30                                      # fewer cached tokens than queries
    run_gpu(q, kc, vc, bt, cu, bad_cl, 0.1)
    assert pa.device_error() & pa.DEVERR["context"]
    run_gpu(q, kc, vc, bt, cu, cl, 0.1, max_q_len=20)   # q_len above the promised bound
    assert pa.device_error() & pa.DEVERR["context"]
    bad_bt = bt.clone()
    bad_bt[0, 1] = kc.shape[0] + 3                      # a block id outside the pool
    run_gpu(q, kc, vc, bad_bt, cu, cl, 0.1)
    assert pa.device_error() & pa.DEVERR["table"]
    assert_no_device_error()


def test_prefill_host_validation(cuda_device):
    q, kc, vc, bt, cu, cl = paged_case(11, [20], [20], 6, 2, 16, "fp16")   # 3 heads per cached head
    with pytest.raises(pa.PagedAttnError):
        run_gpu(q, kc, vc, bt, cu, cl, 0.1)
    q, kc, vc, bt, cu, cl = paged_case(12, [20], [20], 2, 2, 16, "fp16", D=96)
    with pytest.raises(pa.PagedAttnError):
        run_gpu(q, kc, vc, bt, cu, cl, 0.1)
    q, kc, vc, bt, cu, cl = paged_case(13, [20], [20], 2, 2, 16, "fp16", D=64)   # head_dim 64, 8-bit cache
    k, v, ks, vs = quantised(kc, vc, "int8")
    with pytest.raises(pa.PagedAttnError):
        pa.paged_attention_prefill(torch.empty_like(q, device="cuda"), q.cuda(), k.cuda(), v.cuda(), bt.cuda(),
                                   cu.cuda(), cl.cuda(), 20, 0.1, k_scale=ks.cuda(), v_scale=vs.cuda())


def test_prefill_llama70b_prompt_batch_full(cuda_device):
    """4 prompts x 2048 tokens (8192 query rows), 64 heads, bs 16, fp16: the prefill
    workload's shape, every one of the 8192 x 64 output rows against the oracle."""
    S, n, H, bs = 4, 2048, 64, 16
    g = torch.Generator().manual_seed(13)
    NB = S * n // bs + 16
    perm = torch.randperm(NB, generator=g)
    bt = perm[: S * n // bs].view(S, n // bs).to(torch.int32).contiguous()
    kc = torch.randn(NB, bs, H, 128, generator=g, dtype=torch.float16)
    vc = torch.randn(NB, bs, H, 128, generator=g, dtype=torch.float16)
    q = torch.randn(S * n, H, 128, generator=g, dtype=torch.float16)
    cu = torch.arange(0, S * n + 1, n, dtype=torch.int32)
    cl = torch.full((S,), n, dtype=torch.int32)
    scale = 1 / math.sqrt(128)
    out = run_gpu(q, kc, vc, bt, cu, cl, scale).cpu()
    assert_no_device_error()
    ref = oracle.paged_prefill(q, kc, vc, bt, cu, cl, scale)
    compare(out, ref, "fp16", TOL["fp16"])


def test_chunked_prefill_workload_full(cuda_device):
    """The chunked-prefill workload's shape: 8 sequences, 512-token chunks behind 1536 cached
    tokens, 64 heads, bs 16, fp16; every output row against the oracle."""
    S, qn, cached, H, bs = 8, 512, 1536, 64, 16
    ctx = qn + cached
    g = torch.Generator().manual_seed(17)
    nblk = ctx // bs
    NB = S * nblk + 32
    perm = torch.randperm(NB, generator=g)
    bt = perm[: S * nblk].view(S, nblk).to(torch.int32).contiguous()
    kc = torch.randn(NB, bs, H, 128, generator=g, dtype=torch.float16)
    vc = torch.randn(NB, bs, H, 128, generator=g, dtype=torch.float16)
    q = torch.randn(S * qn, H, 128, generator=g, dtype=torch.float16)
    cu = torch.arange(0, S * qn + 1, qn, dtype=torch.int32)
    cl = torch.full((S,), ctx, dtype=torch.int32)
    scale = 1 / math.sqrt(128)
    out = run_gpu(q, kc, vc, bt, cu, cl, scale).cpu()
    assert_no_device_error()
    ref = oracle.paged_prefill(q, kc, vc, bt, cu, cl, scale)
    compare(out, ref, "fp16", TOL["fp16"])


@pytest.mark.parametrize("window", [0, 40])
def test_prefill_many_short_units_per_cta(cuda_device, window):
    """More units than SMs, most of them one KV tile: every CTA walks several units, so a
    unit's rows are written while the next unit's first tile is in flight, and the q rows,
    output accumulators and score buffers change hands across units many times."""
    g = np.random.default_rng(19)
    S = 420
    ql = g.integers(1, 4, size=S).tolist()
    ctx = [q + int(g.integers(0, 300)) for q in ql]
    check(20 + window, ctx, ql, 4, 2, 16, "fp16", window)


# ---------------------------------------------------------------------------------------
# 8-bit caches: the fp16 pool of paged_case quantised by the oracle quantiser; rows no
# sequence owns keep NaN scales (and FP8 NaN codes), so reading one shows up.
# ---------------------------------------------------------------------------------------
def quantised(kc, vc, dtype):
    owned = ~torch.isnan(kc[..., 0].float())             # [NB, bs, Hkv]
    quant = quantize_cache if dtype == "int8" else quantize_cache_fp8
    k, ks = quant(torch.nan_to_num(kc.half()))
    v, vs = quant(torch.nan_to_num(vc.half()))
    ks[~owned] = float("nan")
    vs[~owned] = float("nan")
    if dtype == "fp8":
        k.view(torch.uint8)[~owned] = 0x7F                # the E4M3 NaN code
        v.view(torch.uint8)[~owned] = 0x7F
    return k, v, ks, vs


def check_8bit(seed, ctx, qlen, Hq, Hkv, bs, io, dtype, window=0):
    q, kc, vc, bt, cu, cl = paged_case(seed, ctx, qlen, Hq, Hkv, bs, "fp16")
    q = q.to(DT[io])
    k, v, ks, vs = quantised(kc, vc, dtype)
    scale = 1 / math.sqrt(128)
    out = torch.empty_like(q, device="cuda")
    pa.paged_attention_prefill(out, q.cuda(), k.cuda(), v.cuda(), bt.cuda(), cu.cuda(), cl.cuda(),
                               int((cu[1:] - cu[:-1]).max()), scale, window, k_scale=ks.cuda(), v_scale=vs.cuda())
    torch.cuda.synchronize()
    assert_no_device_error()
    ref = oracle.paged_prefill(q, k, v, bt, cu, cl, scale, window, k_scale=ks, v_scale=vs)
    return compare(out, ref, io, TOL["int8"])


@pytest.mark.parametrize("io", ["fp16", "bf16"])
@pytest.mark.parametrize("dtype", ["int8", "fp8"])
@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 2), (16, 2), (16, 1)])
def test_prefill_eight_bit_caches_mixed_batch(cuda_device, io, dtype, Hq, Hkv):
    check_8bit(31, [37, 300, 129, 16], [37, 90, 1, 16], Hq, Hkv, 16, io, dtype)


@pytest.mark.parametrize("bs", [8, 32, 64, 128])
@pytest.mark.parametrize("dtype", ["int8", "fp8"])
def test_prefill_eight_bit_block_sizes(cuda_device, bs, dtype):
    check_8bit(32, [130, 77, 256], [130, 40, 129], 4, 2, bs, "fp16", dtype)


@pytest.mark.parametrize("window", [1, 100, 5000])
def test_prefill_eight_bit_windows_and_many_tiles(cuda_device, window):
    check_8bit(33, [1000, 260], [1000, 70], 8, 2, 16, "bf16", "int8", window)
    check_8bit(34, [700], [500], 2, 2, 32, "fp16", "fp8", window)


def test_prefill_llama70b_prompt_batch_int8_full(cuda_device):
    """The prompt batch (4 x 2048 tokens, 64 heads, bs 16) over an INT8 cache: every output."""
    S, n, H, bs = 4, 2048, 64, 16
    g = torch.Generator().manual_seed(35)
    NB = S * n // bs + 16
    perm = torch.randperm(NB, generator=g)
    bt = perm[: S * n // bs].view(S, n // bs).to(torch.int32).contiguous()
    k, ks = quantize_cache(torch.randn(NB, bs, H, 128, generator=g, dtype=torch.float16))
    v, vs = quantize_cache(torch.randn(NB, bs, H, 128, generator=g, dtype=torch.float16))
    q = torch.randn(S * n, H, 128, generator=g, dtype=torch.float16)
    cu = torch.arange(0, S * n + 1, n, dtype=torch.int32)
    cl = torch.full((S,), n, dtype=torch.int32)
    scale = 1 / math.sqrt(128)
    out = torch.empty_like(q, device="cuda")
    pa.paged_attention_prefill(out, q.cuda(), k.cuda(), v.cuda(), bt.cuda(), cu.cuda(), cl.cuda(), n, scale,
                               k_scale=ks.cuda(), v_scale=vs.cuda())
    torch.cuda.synchronize()
    assert_no_device_error()
    ref = oracle.paged_prefill(q, k, v, bt, cu, cl, scale, k_scale=ks, v_scale=vs)
    compare(out, ref, "fp16", TOL["int8"])


@pytest.mark.parametrize("Hq,Hkv", [(32, 1), (64, 2), (128, 1)])
@pytest.mark.parametrize("io", ["fp16", "bf16"])
def test_prefill_multi_query(cuda_device, Hq, Hkv, io):
    """32 to 128 query heads per cached head: a unit's 128 rows are 4, 2 or 1 query tokens
    times all the query heads of one cached head."""
    check(41, [37, 300, 129, 16], [37, 90, 1, 16], Hq, Hkv, 16, io)
    check(42, [400, 45], [400, 45], Hq, Hkv, 32, io, window=100)


@pytest.mark.parametrize("io", ["fp16", "bf16"])
@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (8, 2), (32, 1)])
def test_prefill_head_dim_64(cuda_device, io, Hq, Hkv):
    """head_dim 64: the lo 64-dim halves of the operands, 4 score K-steps, a value MMA of
    N = 64; mixed batch, several tiles, a window, and ragged tails."""
    check(51, [37, 300, 129, 16], [37, 90, 1, 16], Hq, Hkv, 16, io, D=64)
    check(52, [1000, 260], [1000, 70], Hq, Hkv, 32, io, window=100, D=64)
    check(53, [130, 77], [130, 40], Hq, Hkv, 8, io, D=64)
