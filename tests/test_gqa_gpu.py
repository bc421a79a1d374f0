"""Grouped-query / multi-query paged decode on the GPU against the fp64 oracle.

query head h reads cached head h // (Hq // Hkv).  Covers group sizes 1..8 on every cache
dtype, block sizes 8/16/32, windows, NaN-poisoned unattended rows, the real Llama-2-70B
layer shape (64 query heads over 8 cached heads) at 256 sequences on every output, and
the tensor-core kernel on fp16/bf16 and on 8-bit (INT8 / FP8) caches.
"""
import math

import numpy as np
import pytest
import torch

import paged_kv_cache_384_b200 as pa
import synth
from oracle.block_manager import BlockManager as OracleBM
from parity import TOL, GpuCase, assert_no_device_error, compare, oracle_decode, quantize_cache, quantize_cache_fp8

pytestmark = pytest.mark.gpu


def _case(seed, hq, hkv, D, bs, ctx, dtype, window=0, io_name=None):
    g = torch.Generator().manual_seed(seed)
    S = len(ctx)
    NB = sum(-(-c // bs) for c in ctx) + 4
    bm = OracleBM(NB, bs, torch.randperm(NB, generator=g).tolist())
    tables = [bm.allocate(-(-c // bs)) if c else [] for c in ctx]
    MB = max(1, max(len(t) for t in tables))
    bt = torch.tensor([t + [-1] * (MB - len(t)) for t in tables], dtype=torch.int32)
    eight = dtype in ("int8", "fp8")
    io = {"fp32": torch.float32, "fp16": torch.float16, "bf16": torch.bfloat16}[io_name or ("fp16" if eight else dtype)]
    q = torch.randn(S, hq, D, generator=g).to(io)
    k = torch.randn(NB, bs, hkv, D, generator=g).to(torch.float16 if eight else io)
    v = torch.randn(NB, bs, hkv, D, generator=g).to(torch.float16 if eight else io)
    live = torch.zeros(NB, bs, dtype=torch.bool)
    for t, c in zip(tables, ctx):
        for i in range(max(0, c - window) if window else 0, c):
            live[t[i // bs], i % bs] = True
    ks = vs = None
    if eight:
        quant = quantize_cache if dtype == "int8" else quantize_cache_fp8
        k, ks = quant(k)
        v, vs = quant(v)
        ks[~live] = float("nan")
        vs[~live] = float("nan")
    else:
        k[~live] = float("nan")
        v[~live] = float("nan")
    scale = 1 / math.sqrt(D)
    ref = oracle_decode(q, k, v, bt, ctx, scale, window, ks, vs)
    ioname = {torch.float32: "fp32", torch.float16: "fp16", torch.bfloat16: "bf16"}[io]
    return GpuCase(q, k, v, bt, ctx, scale, window, ks, vs), ref, ioname


def _run(case, ref, io, tol):
    out = case.decode()
    torch.cuda.synchronize()
    assert_no_device_error()
    return compare(out, ref, io, tol)


@pytest.mark.parametrize("hq,hkv", [(2, 1), (8, 1), (8, 2), (6, 2), (12, 4), (24, 8)])
@pytest.mark.parametrize("dtype", ["fp32", "fp16", "bf16"])
def test_group_sizes(cuda_device, hq, hkv, dtype):
    ctx = [0, 1, 16, 17, 250, 1100, 33]
    case, ref, io = _case(hq * 7 + hkv, hq, hkv, 128, 16, ctx, dtype)
    _run(case, ref, io, TOL[io])


@pytest.mark.parametrize("dtype", ["int8", "fp8"])
@pytest.mark.parametrize("hq", [16, 64])
def test_eight_bit_caches(cuda_device, dtype, hq):
    ctx = [5, 300, 64, 1500]
    case, ref, io = _case(hq, hq, 8, 128, 16, ctx, dtype)
    _run(case, ref, io, TOL["int8"])


@pytest.mark.parametrize("bs", [8, 32])
@pytest.mark.parametrize("D", [64, 128])
def test_block_sizes_and_head_dims(cuda_device, bs, D):
    ctx = [3, 64, 65, 900]
    case, ref, io = _case(bs + D, 16, 2, D, bs, ctx, "bf16")
    _run(case, ref, io, TOL[io])


@pytest.mark.parametrize("window", [1, 100, 4096])
def test_window(cuda_device, window):
    ctx = [1, 99, 100, 101, 3000]
    case, ref, io = _case(window, 32, 4, 128, 16, ctx, "fp16", window=window)
    _run(case, ref, io, TOL[io])


def test_llama70b_gqa_layer_full(cuda_device):
    """64 query heads over 8 cached heads, 256 sequences of U[1, 2048] tokens: every output."""
    w = synth.build_workload("llama70b_gqa_fp16", 0, OracleBM)
    case = GpuCase(w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale)
    out = case.decode()
    torch.cuda.synchronize()
    assert_no_device_error()
    ref = oracle_decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale)
    compare(out, ref, "fp16", TOL["fp16"])


def test_head_count_mismatch_is_rejected(cuda_device):
    q = torch.zeros(1, 6, 128, dtype=torch.float16, device="cuda")
    kc = torch.zeros(4, 16, 4, 128, dtype=torch.float16, device="cuda")
    bt = torch.zeros(1, 1, dtype=torch.int32, device="cuda")
    cl = torch.ones(1, dtype=torch.int32, device="cuda")
    with pytest.raises(ValueError):
        pa.paged_attention_decode(torch.empty_like(q), q, kc, kc, bt, cl, 0.1)


@pytest.mark.parametrize("hq,hkv", [(16, 4), (64, 8), (32, 2)])
@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
@pytest.mark.parametrize("bs", [8, 16, 32])
def test_tensor_core_path(cuda_device, hq, hkv, dtype, bs):
    """Groups of 4..16 query heads on fp16/bf16 caches run as tcgen05 MMAs; the result must
    match the oracle, and the CUDA-core kernel where it applies (groups up to 8)."""
    ctx = [0, 1, 127, 128, 129, 300, 2048, 5, 700]
    case, ref, io = _case(hq + hkv + bs, hq, hkv, 128, bs, ctx, dtype)
    tc = _run(case, ref, io, TOL[io])
    if hq // hkv <= 8:
        pa.use_tensor_cores(False)
        try:
            _run(case, ref, io, TOL[io])
        finally:
            pa.use_tensor_cores(True)


def test_tensor_core_path_windows_and_long_contexts(cuda_device):
    ctx = [1, 4095, 4096, 4097, 9000, 20000]
    case, ref, io = _case(77, 64, 8, 128, 16, ctx, "bf16", window=4096)
    _run(case, ref, io, TOL[io])
    case, ref, io = _case(78, 32, 4, 128, 16, [32768], "fp16")
    _run(case, ref, io, TOL[io])


@pytest.mark.parametrize("io", ["fp16", "bf16"])
@pytest.mark.parametrize("dtype", ["int8", "fp8"])
@pytest.mark.parametrize("gq", [4, 8, 16])
@pytest.mark.parametrize("bs", [8, 16, 32])
def test_tensor_core_path_eight_bit_caches(cuda_device, io, dtype, gq, bs):
    """INT8 / FP8 caches with 4..16 query heads per cached head run on tcgen05 with the codes
    as the MMA operands (q and the weights as 8-bit digits), the per-token K scale applied to
    the score row and the V scale folded into the weight; up to 8 query heads per cached head
    two CTAs share an SM.  Unattended rows carry NaN scales.  Contexts of 0 and 1 token, and a
    batch with fewer work units than CTAs.  Parity at 1e-2 against the oracle on the
    dequantised values, and against the CUDA-core kernel where it applies."""
    ctx = [0, 1, 127, 128, 129, 300, 2048, 5, 700]
    case, ref, ioname = _case(gq * 10 + bs, 8 * gq, 8, 128, bs, ctx, dtype, io_name=io)
    _run(case, ref, ioname, TOL["int8"])
    if gq <= 8:
        pa.use_tensor_cores(False)
        try:
            _run(case, ref, ioname, TOL["int8"])
        finally:
            pa.use_tensor_cores(True)


@pytest.mark.parametrize("dtype", ["int8", "fp8"])
def test_tensor_core_eight_bit_windows_and_long_contexts(cuda_device, dtype):
    ctx = [1, 4095, 4096, 4097, 9000, 20000]
    case, ref, io = _case(91, 64, 8, 128, 16, ctx, dtype, window=4096)
    _run(case, ref, io, TOL["int8"])
    case, ref, io = _case(92, 64, 8, 128, 16, [32768], dtype)
    _run(case, ref, io, TOL["int8"])


def test_llama70b_gqa_layer_int8_full(cuda_device):
    """The grouped-query Llama-2-70B layer (256 sequences, 64 query heads over 8 cached heads)
    with an INT8 cache written by the oracle quantiser: every output."""
    w = synth.build_workload("llama70b_gqa_fp16", 0, OracleBM)
    k, ks = quantize_cache(w.k_cache)
    v, vs = quantize_cache(w.v_cache)
    case = GpuCase(w.q, k, v, w.block_tables, w.context_lens, w.scale, 0, ks, vs)
    out = case.decode()
    torch.cuda.synchronize()
    assert_no_device_error()
    ref = oracle_decode(w.q, k, v, w.block_tables, w.context_lens, w.scale, 0, ks, vs)
    compare(out, ref, "fp16", TOL["int8"])


@pytest.mark.parametrize("hq,hkv", [(32, 1), (64, 1), (64, 2), (48, 1), (40, 1)])
@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_multi_query_above_sixteen_heads(cuda_device, hq, hkv, dtype):
    """More than 16 query heads per cached head: query sub-groups of up to 16 (10 for 40)
    on the tensor cores, each reading the same cached head."""
    ctx = [0, 1, 127, 128, 129, 300, 2048, 5, 700]
    case, ref, io = _case(hq + hkv, hq, hkv, 128, 16, ctx, dtype)
    _run(case, ref, io, TOL[io])


def test_multi_query_windows_block_sizes_and_eight_bit(cuda_device):
    case, ref, io = _case(93, 64, 1, 128, 32, [1, 4095, 4096, 4097, 9000], "fp16", window=4096)
    _run(case, ref, io, TOL[io])
    case, ref, io = _case(94, 32, 1, 128, 8, [32768], "bf16")
    _run(case, ref, io, TOL[io])
    case, ref, io = _case(95, 256, 8, 128, 16, [3, 500, 2048, 129], "int8")
    _run(case, ref, io, TOL["int8"])


@pytest.mark.parametrize("hq,hkv", [(16, 4), (64, 8), (32, 2), (64, 1)])
@pytest.mark.parametrize("dtype", ["fp16", "bf16"])
def test_tensor_core_path_head_dim_64(cuda_device, hq, hkv, dtype):
    """head_dim 64 on the tensor cores (half the score MMA steps; the value MMA's upper 64
    rows are unused), against the oracle and, for groups up to 8, the CUDA-core kernel."""
    ctx = [0, 1, 127, 128, 129, 300, 2048, 5, 700]
    case, ref, io = _case(hq * 3 + hkv, hq, hkv, 64, 16, ctx, dtype)
    _run(case, ref, io, TOL[io])
    if hq // hkv <= 8:
        pa.use_tensor_cores(False)
        try:
            _run(case, ref, io, TOL[io])
        finally:
            pa.use_tensor_cores(True)
    case, ref, io = _case(hq * 5 + hkv, hq, hkv, 64, 32, [1, 4095, 4096, 9000], dtype, window=4096)
    _run(case, ref, io, TOL[io])
