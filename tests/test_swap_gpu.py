"""GPU swap_blocks through the C ABI: whole blocks moved between the GPU pool and a
page-locked host pool (swap-out, swap-in), bit-exact against the oracle's block-move
definition, with and without 8-bit scale pools, pairs held on either side, the byte path
for odd block sizes, out-of-range pairs (reported, not faulted) and pageable memory
(rejected on the host)."""
import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_384_b200 as pa
from parity import assert_no_device_error

pytestmark = pytest.mark.gpu


def _u8(t):
    return t.detach().cpu().contiguous().view(torch.uint8).numpy()


def _pools(g, nb, shape, dtype, device, pin=False):
    if dtype == torch.int8:
        k = torch.randint(-127, 128, (nb,) + shape, generator=g, dtype=torch.int8)
        v = torch.randint(-127, 128, (nb,) + shape, generator=g, dtype=torch.int8)
    else:
        k = torch.randn((nb,) + shape, generator=g).to(dtype)
        v = torch.randn((nb,) + shape, generator=g).to(dtype)
    if device == "cuda":
        return k.cuda(), v.cuda()
    return (k.pin_memory(), v.pin_memory()) if pin else (k, v)


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16, torch.float32])
@pytest.mark.parametrize("pairs_on", ["cuda", "host"])
def test_swap_out_and_in_bit_exact(cuda_device, dtype, pairs_on):
    g = torch.Generator().manual_seed(11)
    bs, H, D = 16, 8, 128
    gk, gv = _pools(g, 200, (bs, H, D), dtype, "cuda")
    hk, hv = _pools(g, 64, (bs, H, D), dtype, "cpu", pin=True)
    src = torch.randperm(200, generator=g)[:40]
    dst = torch.randperm(64, generator=g)[:40]
    out_pairs = torch.stack([src, dst], 1).to(torch.int64)
    want_hk, want_hv = _u8(hk).reshape(64, -1).copy(), _u8(hv).reshape(64, -1).copy()
    oracle.cache_ops.swap_blocks(_u8(gk).reshape(200, -1), _u8(gv).reshape(200, -1), want_hk, want_hv,
                                 out_pairs.numpy())
    pairs = out_pairs.cuda() if pairs_on == "cuda" else out_pairs.pin_memory()
    pa.swap_blocks(gk, gv, hk, hv, pairs)                       # swap-out
    torch.cuda.synchronize()
    assert_no_device_error()
    assert np.array_equal(_u8(hk).reshape(64, -1), want_hk)
    assert np.array_equal(_u8(hv).reshape(64, -1), want_hv)

    # swap-in into different GPU blocks
    back_dst = torch.randperm(200, generator=g)[:40]
    in_pairs = torch.stack([dst, back_dst], 1).to(torch.int64)
    want_gk, want_gv = _u8(gk).reshape(200, -1).copy(), _u8(gv).reshape(200, -1).copy()
    oracle.cache_ops.swap_blocks(want_hk, want_hv, want_gk, want_gv, in_pairs.numpy())
    pairs = in_pairs.cuda() if pairs_on == "cuda" else in_pairs.pin_memory()
    pa.swap_blocks(hk, hv, gk, gv, pairs)                       # swap-in
    torch.cuda.synchronize()
    assert_no_device_error()
    assert np.array_equal(_u8(gk).reshape(200, -1), want_gk)
    assert np.array_equal(_u8(gv).reshape(200, -1), want_gv)


@pytest.mark.parametrize("code", [torch.int8, torch.float8_e4m3fn])
def test_swap_8bit_pools_carry_their_scales(cuda_device, code):
    g = torch.Generator().manual_seed(12)
    bs, H, D = 16, 8, 64
    gk, gv = _pools(g, 30, (bs, H, D), torch.int8, "cuda")
    gk, gv = gk.view(code), gv.view(code)
    gks, gvs = torch.rand(30, bs, H, generator=g).half().cuda(), torch.rand(30, bs, H, generator=g).half().cuda()
    hk = torch.zeros(10, bs, H, D, dtype=torch.int8).pin_memory().view(code)
    hv = torch.zeros(10, bs, H, D, dtype=torch.int8).pin_memory().view(code)
    hks, hvs = torch.zeros(10, bs, H).half().pin_memory(), torch.zeros(10, bs, H).half().pin_memory()
    pairs = torch.tensor([[3, 9], [29, 0], [0, 4]], dtype=torch.int64)
    want = [np.zeros((10, bs * H * D), np.uint8), np.zeros((10, bs * H * D), np.uint8),
            np.zeros((10, bs * H * 2), np.uint8), np.zeros((10, bs * H * 2), np.uint8)]
    oracle.cache_ops.swap_blocks(_u8(gk).reshape(30, -1), _u8(gv).reshape(30, -1), want[0], want[1], pairs.numpy(),
                                 (_u8(gks).reshape(30, -1), _u8(gvs).reshape(30, -1)), (want[2], want[3]))
    pa.swap_blocks(gk, gv, hk, hv, pairs.cuda(), (gks, gvs), (hks, hvs))
    torch.cuda.synchronize()
    assert_no_device_error()
    for got, w in zip((hk, hv, hks, hvs), want):
        assert np.array_equal(_u8(got).reshape(10, -1), w)


def test_swap_device_to_device_and_byte_path(cuda_device):
    # block bytes 3*5*7*2 = 210, not a multiple of 16: the byte-granular path
    g = torch.Generator().manual_seed(13)
    a_k, a_v = _pools(g, 17, (3, 5, 7), torch.float16, "cuda")
    b_k, b_v = _pools(g, 11, (3, 5, 7), torch.float16, "cpu", pin=True)
    pairs = torch.tensor([[16, 10], [0, 0], [5, 3]], dtype=torch.int64)
    want_k, want_v = _u8(b_k).reshape(11, -1).copy(), _u8(b_v).reshape(11, -1).copy()
    oracle.cache_ops.swap_blocks(_u8(a_k).reshape(17, -1), _u8(a_v).reshape(17, -1), want_k, want_v, pairs.numpy())
    pa.swap_blocks(a_k, a_v, b_k, b_v, pairs.cuda())
    torch.cuda.synchronize()
    assert np.array_equal(_u8(b_k).reshape(11, -1), want_k) and np.array_equal(_u8(b_v).reshape(11, -1), want_v)
    # two GPU pools (e.g. a defragmenting move): same call, no host memory involved
    c_k, c_v = torch.zeros(11, 3, 5, 7, dtype=torch.float16, device="cuda"), torch.zeros_like(b_v).cuda()
    pa.swap_blocks(a_k, a_v, c_k, c_v, pairs.cuda())
    torch.cuda.synchronize()
    assert_no_device_error()
    for i, (s, d) in enumerate(pairs.tolist()):
        assert torch.equal(c_k[d], a_k[s]) and torch.equal(c_v[d], a_v[s])


def test_swap_reports_out_of_range_pairs(cuda_device):
    g = torch.Generator().manual_seed(14)
    gk, gv = _pools(g, 8, (16, 2, 64), torch.float16, "cuda")
    hk, hv = torch.zeros(4, 16, 2, 64).half().pin_memory(), torch.zeros(4, 16, 2, 64).half().pin_memory()
    pairs = torch.tensor([[7, 4], [8, 0], [1, 1]], dtype=torch.int64).cuda()   # dst 4 and src 8 are outside
    pa.swap_blocks(gk, gv, hk, hv, pairs)
    torch.cuda.synchronize()
    assert pa.device_error() & pa.DEVERR["pair"]
    assert torch.equal(hk[1], gk[1].cpu()) and not hk[0].any()


def test_swap_rejects_pageable_host_memory(cuda_device):
    gk, gv = torch.zeros(4, 16, 2, 64).half().cuda(), torch.zeros(4, 16, 2, 64).half().cuda()
    hk, hv = torch.zeros(4, 16, 2, 64).half(), torch.zeros(4, 16, 2, 64).half()   # not pinned
    pairs = torch.tensor([[0, 0]], dtype=torch.int64).cuda()
    with pytest.raises(ValueError):
        pa.swap_blocks(gk, gv, hk, hv, pairs)
    # the library itself refuses pageable memory too (the binding's check bypassed)
    import ctypes
    st = pa._L.swap_blocks(ctypes.c_void_p(gk.data_ptr()), ctypes.c_void_p(gv.data_ptr()),
                           ctypes.c_void_p(hk.data_ptr()), ctypes.c_void_p(hv.data_ptr()),
                           ctypes.c_void_p(pairs.data_ptr()), 1, 4, 4, hk[0].numel() * 2,
                           None, None, None, None, 0, None)
    assert st == 1 and b"pageable" in pa._L.pa_last_error()
    torch.cuda.synchronize()
