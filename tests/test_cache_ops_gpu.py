"""GPU reshape_and_cache and copy_blocks through the C ABI: bit-exact against the oracle's
placement definitions, including padding slots, fused-QKV strides, INT8 scales, the
byte-granular copy path and out-of-range indices (reported, not faulted)."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_384_b200 as pa
import synth
from oracle.block_manager import BlockManager as OracleBM
from parity import assert_no_device_error

pytestmark = pytest.mark.gpu

DT = {"fp32": torch.float32, "fp16": torch.float16, "bf16": torch.bfloat16}


def _bits(t):
    return t.cpu().view(torch.uint8).numpy() if t.dtype != torch.int8 else t.cpu().numpy().view(np.uint8)


@pytest.mark.parametrize("dtype", ["fp32", "fp16", "bf16"])
@pytest.mark.parametrize("fused", [False, True])
def test_reshape_and_cache_bit_exact(cuda_device, dtype, fused):
    g = torch.Generator().manual_seed(1)
    NB, bs, H, D, T = 40, 16, 8, 128, 50
    kc = torch.randn(NB, bs, H, D, generator=g).to(DT[dtype])
    vc = torch.randn(NB, bs, H, D, generator=g).to(DT[dtype])
    qkv = torch.randn(T, 3, H, D, generator=g).to(DT[dtype])
    if fused:   # K and V rows taken straight out of a fused QKV tensor (token stride 3*H*D)
        k, v = qkv[:, 1], qkv[:, 2]
    else:
        k, v = qkv[:, 1].contiguous(), qkv[:, 2].contiguous()
    slots = torch.randperm(NB * bs, generator=g)[:T]
    slots[::7] = -1                                  # padding tokens
    ref_k = _bits(kc).reshape(NB, bs, H, -1).copy()
    ref_v = _bits(vc).reshape(NB, bs, H, -1).copy()
    oracle.cache_ops.reshape_and_cache(_bits(k.contiguous()).reshape(T, H, -1), _bits(v.contiguous()).reshape(T, H, -1),
                                       ref_k, ref_v, slots.numpy())
    kd, vd = kc.cuda(), vc.cuda()
    pa.reshape_and_cache(k.cuda() if not fused else qkv.cuda()[:, 1], v.cuda() if not fused else qkv.cuda()[:, 2],
                         kd, vd, slots.cuda())
    torch.cuda.synchronize()
    assert_no_device_error()
    assert np.array_equal(_bits(kd).reshape(ref_k.shape), ref_k)
    assert np.array_equal(_bits(vd).reshape(ref_v.shape), ref_v)


def test_reshape_and_cache_int8_with_scales(cuda_device):
    g = torch.Generator().manual_seed(2)
    NB, bs, H, D, T = 12, 16, 8, 64, 20
    kc = torch.randint(-127, 128, (NB, bs, H, D), generator=g, dtype=torch.int8)
    vc = torch.randint(-127, 128, (NB, bs, H, D), generator=g, dtype=torch.int8)
    ksc = torch.rand(NB, bs, H, generator=g).half()
    vsc = torch.rand(NB, bs, H, generator=g).half()
    k, ks = oracle.quant.quantize_rows(torch.randn(T, H, D, generator=g).half().numpy())
    v, vs = oracle.quant.quantize_rows(torch.randn(T, H, D, generator=g).half().numpy())
    slots = torch.randperm(NB * bs, generator=g)[:T]
    rk, rv, rks, rvs = kc.numpy().copy(), vc.numpy().copy(), ksc.numpy().copy(), vsc.numpy().copy()
    oracle.cache_ops.reshape_and_cache(k, v, rk, rv, slots.numpy(), ks, vs, rks, rvs)
    d = [t.cuda() for t in (kc, vc, ksc, vsc)]
    pa.reshape_and_cache(torch.from_numpy(k).cuda(), torch.from_numpy(v).cuda(), d[0], d[1], slots.cuda(),
                         torch.from_numpy(ks).cuda(), torch.from_numpy(vs).cuda(), d[2], d[3])
    torch.cuda.synchronize()
    assert_no_device_error()
    for got, ref in zip(d, (rk, rv, rks, rvs)):
        assert np.array_equal(got.cpu().numpy(), ref)


def test_reshape_and_cache_reports_out_of_range_slots(cuda_device):
    NB, bs, H, D = 4, 16, 2, 64
    kc = torch.zeros(NB, bs, H, D, dtype=torch.float16, device="cuda")
    vc = torch.zeros_like(kc)
    k = torch.ones(2, H, D, dtype=torch.float16, device="cuda")
    pa.reshape_and_cache(k, k, kc, vc, torch.tensor([3, NB * bs + 5], device="cuda"))
    torch.cuda.synchronize()
    assert pa.device_error(clear=True) & pa.DEVERR["slot"]
    assert torch.count_nonzero(kc) == H * D     # only the valid token landed


def test_copy_blocks_chat_forks_bit_exact(cuda_device):
    w = synth.build_workload("chat_prefix_bf16", 1, OracleBM, num_seqs=32, num_diverge=12)
    kd, vd = w.k_cache.cuda(), w.v_cache.cuda()
    pa.copy_blocks(kd, vd, w.copy_pairs.cuda())
    kc = w.k_cache.view(torch.int16).numpy().copy()
    vc = w.v_cache.view(torch.int16).numpy().copy()
    oracle.cache_ops.copy_blocks(kc, vc, w.copy_pairs.numpy())
    torch.cuda.synchronize()
    assert_no_device_error()
    assert np.array_equal(kd.cpu().view(torch.int16).numpy(), kc)
    assert np.array_equal(vd.cpu().view(torch.int16).numpy(), vc)


def test_copy_blocks_int8_pools_with_scales(cuda_device):
    g = torch.Generator().manual_seed(3)
    NB, bs, H, D = 20, 16, 8, 128
    pools = [torch.randint(-127, 128, (NB, bs, H, D), generator=g, dtype=torch.int8) for _ in range(2)]
    scales = [torch.rand(NB, bs, H, generator=g).half() for _ in range(2)]
    pairs = torch.tensor([[0, 10], [3, 11], [7, 19], [2, 12]])
    ref = [p.numpy().copy() for p in pools] + [s.numpy().copy() for s in scales]
    oracle.cache_ops.copy_blocks(ref[0], ref[1], pairs.numpy(), ref[2], ref[3])
    d = [t.cuda() for t in pools + scales]
    pa.copy_blocks(d[0], d[1], pairs.cuda(), d[2], d[3])
    torch.cuda.synchronize()
    assert_no_device_error()
    for got, r in zip(d, ref):
        assert np.array_equal(got.cpu().numpy(), r)


def test_copy_blocks_byte_path_for_odd_block_sizes(cuda_device):
    g = torch.Generator().manual_seed(4)
    NB = 9
    k = torch.randint(-127, 128, (NB, 3, 5), generator=g, dtype=torch.int8)   # 15-byte blocks
    v = torch.randint(-127, 128, (NB, 3, 5), generator=g, dtype=torch.int8)
    pairs = torch.tensor([[1, 4], [2, 8]])
    rk, rv = k.numpy().copy(), v.numpy().copy()
    oracle.cache_ops.copy_blocks(rk, rv, pairs.numpy())
    kd, vd = k.cuda(), v.cuda()
    pa.copy_blocks(kd, vd, pairs.cuda())
    torch.cuda.synchronize()
    assert np.array_equal(kd.cpu().numpy(), rk) and np.array_equal(vd.cpu().numpy(), rv)


def test_copy_blocks_reports_out_of_range_pairs(cuda_device):
    k = torch.zeros(4, 16, 2, 64, dtype=torch.float16, device="cuda")
    v = torch.zeros_like(k)
    k[1] = 1.0
    pa.copy_blocks(k, v, torch.tensor([[1, 2], [1, 9]], device="cuda"))
    torch.cuda.synchronize()
    assert pa.device_error(clear=True) & pa.DEVERR["pair"]
    assert torch.equal(k[2], k[1])
