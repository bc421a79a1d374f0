"""The allocation-free decode entry point, through the C ABI.

paged_attention_decode_static_scratch serves callers that cannot allocate device memory
themselves (a plugin inside a framework that owns all device memory, or a loop that
cannot afford cudaMalloc's device synchronisation): its scratch is a fixed array inside
the library.  Here it must give the same results as paged_attention_decode with a
caller-provided workspace, on two different batches called back to back (the second call
finds the first call's leftovers in the shared array), on an INT8 cache (its per-row
scales passed through), and on the largest batch the array takes; one more sequence must
be refused.  This file is collected last on purpose.
"""
import ctypes

import pytest
import torch

import paged_kv_cache_384_b200 as pa
import synth
from oracle.block_manager import BlockManager as OracleBM
from parity import TOL, GpuCase, quantize_cache

pytestmark = pytest.mark.gpu

_DT = {torch.float32: 0, torch.float16: 1, torch.bfloat16: 2, torch.int8: 3, torch.float8_e4m3fn: 4}


def _static_scratch_decode(case):
    out = torch.empty_like(case.q)
    S, H, D = case.q.shape
    NB, bs = case.k_cache.shape[:2]
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    ks = None if case.k_scale is None else P(case.k_scale)
    vs = None if case.v_scale is None else P(case.v_scale)
    st = pa._L.paged_attention_decode_static_scratch(
        P(out), P(case.q), P(case.k_cache), P(case.v_cache), ks, vs, P(case.block_tables),
        P(case.context_lens), S, H, D, bs, NB, case.block_tables.shape[1], case.scale, case.window,
        _DT[case.q.dtype], _DT[case.k_cache.dtype], ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, pa._L.pa_last_error().decode()
    return out


def _case(preset, seed, **kw):
    w = synth.build_workload(preset, seed, OracleBM, **kw)
    return GpuCase(w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale, w.window), w.io_dtype


def test_static_scratch_matches_the_workspace_entry_point_twice_in_a_row(cuda_device):
    cases = [_case("llama70b_fp16", 21, num_seqs=12), _case("chat_prefix_bf16", 22, num_seqs=40, num_diverge=0)]
    results = []
    for case, io in cases:                      # two calls in a row on the shared scratch
        results.append((_static_scratch_decode(case), case, io))
    for got, case, io in results:
        ref = case.decode()                     # caller-provided workspace
        torch.cuda.synchronize()
        err = (got.float() - ref.float()).abs().max().item()
        assert err <= TOL[io], err
    assert pa.device_error(clear=True) == 0


def test_static_scratch_rejects_batches_larger_than_the_array(cuda_device):
    S, H, D = 4096, 64, 128
    assert pa.decode_workspace_bytes(S, H, D) > 16 << 20
    dummy = torch.empty(16, dtype=torch.float16, device="cuda")
    p = ctypes.c_void_p(dummy.data_ptr())
    st = pa._L.paged_attention_decode_static_scratch(p, p, p, p, None, None, p, p, S, H, D, 16, 8, 1, 0.1, 0, 1, 1,
                                                     None)
    assert st == 1
    assert "scratch" in pa._L.pa_last_error().decode()


def _compare_with_workspace_entry_point(case, io, tol):
    got = _static_scratch_decode(case)
    ref = case.decode()
    torch.cuda.synchronize()
    err = (got.float() - ref.float()).abs().max().item()
    assert err <= tol, err
    assert pa.device_error(clear=True) == 0


def test_static_scratch_int8_cache_with_scales(cuda_device):
    w = synth.build_workload("llama70b_int8", 23, OracleBM, num_seqs=8)
    k, ks = quantize_cache(w.k_cache)
    v, vs = quantize_cache(w.v_cache)
    case = GpuCase(w.q, k, v, w.block_tables, w.context_lens, w.scale, 0, ks, vs)
    for _ in range(2):
        _compare_with_workspace_entry_point(case, "fp16", TOL["int8"])


def test_static_scratch_at_the_size_limit(cuda_device):
    """The largest number of 64-head sequences whose scratch fits the 16 MiB array runs and
    matches; one sequence more is refused."""
    H, D, limit = 64, 128, 16 << 20
    S = 1
    while pa.decode_workspace_bytes(S + 1, H, D) <= limit:
        S += 1
    assert pa.decode_workspace_bytes(S, H, D) > limit - 64 * 1024   # close to the limit
    g = torch.Generator().manual_seed(24)
    ctx = torch.randint(1, 80, (S,), generator=g)
    nblk = [-(-int(c) // 16) for c in ctx]
    NB = sum(nblk) + 7
    perm = torch.randperm(NB, generator=g).tolist()
    bt = torch.full((S, max(nblk)), -1, dtype=torch.int32)
    k = 0
    for s, n in enumerate(nblk):
        bt[s, :n] = torch.tensor(perm[k:k + n], dtype=torch.int32)
        k += n
    q = torch.randn(S, H, D, generator=g).half()
    kc = torch.randn(NB, 16, H, D, generator=g).half()
    vc = torch.randn(NB, 16, H, D, generator=g).half()
    case = GpuCase(q, kc, vc, bt, ctx, D ** -0.5)
    for _ in range(2):
        _compare_with_workspace_entry_point(case, "fp16", TOL["fp16"])
    # one sequence more no longer fits
    big = torch.empty(16, dtype=torch.float16, device="cuda")
    p = ctypes.c_void_p(big.data_ptr())
    st = pa._L.paged_attention_decode_static_scratch(p, p, p, p, None, None, p, p, S + 1, H, D, 16, 8, 1, 0.1, 0,
                                                     1, 1, None)
    assert st == 1 and "scratch" in pa._L.pa_last_error().decode()
