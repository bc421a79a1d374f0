"""GPU quantise-on-write (reshape_and_cache_quant) and decode over the 8-bit caches it fills.

The INT8 and FP8 (E4M3) codes and fp16 scales must equal the oracle quantiser's bit for bit
(both take every rounding decision in fp32); decode over the GPU-written cache must match
the oracle on the dequantised values within the quantised-cache tolerance (1e-2).
"""
import math

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_384_b200 as pa
from oracle.block_manager import BlockManager as OracleBM
from parity import TOL, GpuCase, assert_no_device_error, compare, oracle_decode

pytestmark = pytest.mark.gpu

CODE_DT = {"int8": torch.int8, "fp8": torch.float8_e4m3fn}


def _oracle_quant(x: torch.Tensor, kind: str):
    a = x.float().numpy() if x.dtype == torch.bfloat16 else x.numpy()   # bf16 widens exactly
    if kind == "int8":
        codes, scale = oracle.quant.quantize_rows(a)
        return codes.view(np.uint8), scale
    codes, scale = oracle.quant.quantize_rows_fp8(a)
    return codes, scale


@pytest.mark.parametrize("kind", ["int8", "fp8"])
@pytest.mark.parametrize("src", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("D", [64, 128])
def test_quantise_on_write_is_bit_exact(cuda_device, kind, src, D):
    g = torch.Generator().manual_seed(D + (src == torch.bfloat16))
    NB, bs, H, T = 24, 16, 8, 60
    k = (torch.randn(T, H, D, generator=g) * torch.rand(T, H, 1, generator=g) * 4).to(src)
    v = (torch.randn(T, H, D, generator=g) * 0.01).to(src)
    k[3, 2] = 0                                   # zero row: scale 0, codes 0
    k[5, 1, :4] = torch.tensor([2.5, -2.5, 3.5, 0.5]) * (k[5, 1].float().abs().max() / 127)  # near ties
    slots = torch.randperm(NB * bs, generator=g)[:T]
    slots[7] = -1
    kc = torch.zeros(NB, bs, H, D, dtype=torch.uint8)
    vc = torch.zeros_like(kc)
    ksc = torch.zeros(NB, bs, H, dtype=torch.float16)
    vsc = torch.zeros_like(ksc)
    ck, sk = _oracle_quant(k, kind)
    cv, sv = _oracle_quant(v, kind)
    rk, rv, rks, rvs = kc.numpy().copy(), vc.numpy().copy(), ksc.numpy().copy(), vsc.numpy().copy()
    oracle.cache_ops.reshape_and_cache(ck, cv, rk, rv, slots.numpy(), sk, sv, rks, rvs)
    d = dict(kc=kc.cuda().view(CODE_DT[kind]), vc=vc.cuda().view(CODE_DT[kind]), ks=ksc.cuda(), vs=vsc.cuda())
    pa.reshape_and_cache_quant(k.cuda(), v.cuda(), d["kc"], d["vc"], d["ks"], d["vs"], slots.cuda())
    torch.cuda.synchronize()
    assert_no_device_error()
    assert np.array_equal(d["kc"].view(torch.uint8).cpu().numpy(), rk)
    assert np.array_equal(d["vc"].view(torch.uint8).cpu().numpy(), rv)
    assert np.array_equal(d["ks"].cpu().numpy().view(np.uint16), rks.view(np.uint16))
    assert np.array_equal(d["vs"].cpu().numpy().view(np.uint16), rvs.view(np.uint16))


@pytest.mark.parametrize("kind", ["int8", "fp8"])
@pytest.mark.parametrize("io", [torch.float16, torch.bfloat16])
def test_decode_over_a_gpu_quantised_cache(cuda_device, kind, io):
    """Prefill-style fill of the whole cache through the quantiser, then decode."""
    g = torch.Generator().manual_seed(7)
    S, H, D, bs = 6, 16, 128, 16
    ctx = [1, 17, 200, 513, 64, 1000]
    NB = sum(-(-c // bs) for c in ctx) + 3
    bm = OracleBM(NB, bs, torch.randperm(NB, generator=g).tolist())
    tables = [bm.allocate(-(-c // bs)) for c in ctx]
    MB = max(len(t) for t in tables)
    bt = torch.tensor([t + [-1] * (MB - len(t)) for t in tables], dtype=torch.int32)
    T = sum(ctx)
    k = torch.randn(T, H, D, generator=g).to(io)
    v = torch.randn(T, H, D, generator=g).to(io)
    q = torch.randn(S, H, D, generator=g).to(io)
    slots = pa.slot_mapping(bt, [s for s, c in enumerate(ctx) for _ in range(c)],
                            [i for c in ctx for i in range(c)], bs)
    kc = torch.zeros(NB, bs, H, D, dtype=torch.uint8, device="cuda").view(CODE_DT[kind])
    vc = torch.zeros_like(kc)
    ks = torch.zeros(NB, bs, H, dtype=torch.float16, device="cuda")
    vs = torch.zeros_like(ks)
    pa.reshape_and_cache_quant(k.cuda(), v.cuda(), kc, vc, ks, vs, slots.cuda())
    case = GpuCase(q, kc, vc, bt, ctx, 1 / math.sqrt(D), 0, ks, vs)
    out = case.decode()
    torch.cuda.synchronize()
    assert_no_device_error()
    ref = oracle_decode(q, kc.cpu(), vc.cpu(), bt, ctx, 1 / math.sqrt(D), 0, ks.cpu(), vs.cpu())
    compare(out, ref, "fp16" if io == torch.float16 else "bf16", TOL["int8"])
    # and the dequantised cache stays close to the unquantised attention
    ref_full = oracle_decode(q, _dense_cache(k, slots, NB, bs), _dense_cache(v, slots, NB, bs), bt, ctx,
                             1 / math.sqrt(D))
    assert np.max(np.abs(ref - ref_full)) < (0.05 if kind == "int8" else 0.15)


def _dense_cache(x, slots, NB, bs):
    T, H, D = x.shape
    c = torch.zeros(NB * bs, H, D, dtype=torch.float32)
    c[slots] = x.float()
    return c.view(NB, bs, H, D)
