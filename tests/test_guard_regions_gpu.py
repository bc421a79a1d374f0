"""Guard regions: no kernel writes outside the buffers it is given.

Every buffer a call may write (its output, the decode workspace, the cache pools and their
scale pools, a page-locked host pool) is handed over as the middle of a larger allocation
whose head and tail hold a canary byte pattern.  After the call the canaries must be
unchanged byte for byte, and inputs the call only reads must be unchanged as a whole.
Edge-touching work is chosen on purpose: the first and last slot of a pool, the first and
last block in copy pairs, sequences whose rows reach the end of ``out``.
"""
import math

import pytest
import torch

import paged_kv_cache_384_b200 as pa
from parity import assert_no_device_error, quantize_cache

pytestmark = pytest.mark.gpu

GUARD = 4096        # bytes of canary on each side (a multiple of 256: the inner slice stays aligned)
CANARY = 0xA5


class Guarded:
    """A tensor of ``shape``/``dtype`` living between two canary regions of one allocation."""

    def __init__(self, shape, dtype, device="cuda", pinned=False, init=None):
        es = torch.empty((), dtype=dtype).element_size()
        n = math.prod(shape)
        self.g = GUARD // es
        self.buf = torch.empty(self.g + n + self.g, dtype=dtype, device=device if not pinned else "cpu")
        if pinned:
            self.buf = self.buf.pin_memory()
        self.buf.view(torch.uint8).fill_(CANARY)
        self.t = self.buf[self.g:self.g + n].view(shape)
        if init is not None:
            self.t.copy_(init)

    def intact(self) -> bool:
        raw = self.buf.view(torch.uint8)
        gb = self.g * self.buf.element_size()
        return bool((raw[:gb] == CANARY).all()) and bool((raw[-gb:] == CANARY).all())


def _pool(seed, NB, bs, H, D, dtype):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(NB, bs, H, D, generator=g).to(dtype), torch.randn(NB, bs, H, D, generator=g).to(dtype)


def _tables(seed, ctx, bs, NB):
    g = torch.Generator().manual_seed(seed)
    perm = torch.randperm(NB, generator=g).tolist()
    nblk = [-(-c // bs) for c in ctx]
    bt = torch.full((len(ctx), max(1, max(nblk))), -1, dtype=torch.int32)
    k = 0
    for s, n in enumerate(nblk):
        bt[s, :n] = torch.tensor(perm[k:k + n], dtype=torch.int32)
        k += n
    return bt


@pytest.mark.parametrize("hq,hkv,dtype", [(8, 8, torch.float16), (16, 2, torch.bfloat16), (64, 8, torch.float16),
                                          (8, 8, torch.float32), (8, 8, torch.int8)])
def test_decode_writes_only_out_and_workspace(cuda_device, hq, hkv, dtype):
    bs, D = 16, 128
    ctx = [1, 700, 33, 2048, 0, 129]          # the last rows of out belong to a split segment
    NB = sum(-(-c // bs) for c in ctx) + 2
    io = torch.float16 if dtype == torch.int8 else dtype
    k, v = _pool(1, NB, bs, hkv, D, io)
    ks = vs = None
    if dtype == torch.int8:
        k, ks = quantize_cache(k)
        v, vs = quantize_cache(v)
    kc, vc = Guarded(k.shape, k.dtype, init=k.cuda()), Guarded(v.shape, v.dtype, init=v.cuda())
    kcs = None if ks is None else Guarded(ks.shape, ks.dtype, init=ks.cuda())
    vcs = None if vs is None else Guarded(vs.shape, vs.dtype, init=vs.cuda())
    q = torch.randn(len(ctx), hq, D, generator=torch.Generator().manual_seed(2)).to(io).cuda()
    out = Guarded(q.shape, q.dtype)
    ws_bytes = pa.decode_workspace_bytes(len(ctx), hq, D)
    ws = Guarded((ws_bytes,), torch.uint8)
    bt = _tables(3, ctx, bs, NB).cuda()
    cl = torch.tensor(ctx, dtype=torch.int32, device="cuda")
    pa.paged_attention_decode(out.t, q, kc.t, vc.t, bt, cl, D ** -0.5, 0, None if kcs is None else kcs.t,
                              None if vcs is None else vcs.t, workspace=ws.t)
    torch.cuda.synchronize()
    assert_no_device_error()
    assert out.intact() and ws.intact()
    assert kc.intact() and vc.intact() and torch.equal(kc.t.cpu(), k) and torch.equal(vc.t.cpu(), v)
    if kcs is not None:
        assert kcs.intact() and vcs.intact()
    assert torch.isfinite(out.t.float()).all()


@pytest.mark.parametrize("quant", [False, True])
def test_cache_writes_stay_inside_the_pools(cuda_device, quant):
    NB, bs, H, D = 9, 16, 8, 128
    T = 5
    slots = torch.tensor([0, NB * bs - 1, 17, -1, 5 * bs + 3], dtype=torch.int64, device="cuda")  # first and last slot
    g = torch.Generator().manual_seed(4)
    k_new = torch.randn(T, H, D, generator=g).half().cuda()
    v_new = torch.randn(T, H, D, generator=g).half().cuda()
    if quant:
        kc = Guarded((NB, bs, H, D), torch.int8)
        vc = Guarded((NB, bs, H, D), torch.int8)
        ksc = Guarded((NB, bs, H), torch.float16)
        vsc = Guarded((NB, bs, H), torch.float16)
        pa.reshape_and_cache_quant(k_new, v_new, kc.t, vc.t, ksc.t, vsc.t, slots)
        pools = (kc, vc, ksc, vsc)
    else:
        kc = Guarded((NB, bs, H, D), torch.float16)
        vc = Guarded((NB, bs, H, D), torch.float16)
        pa.reshape_and_cache(k_new, v_new, kc.t, vc.t, slots)
        pools = (kc, vc)
    torch.cuda.synchronize()
    assert_no_device_error()
    assert all(p.intact() for p in pools)
    if not quant:
        assert torch.equal(kc.t.view(NB * bs, H, D)[NB * bs - 1], k_new[1])
        assert torch.equal(vc.t.view(NB * bs, H, D)[0], v_new[0])


@pytest.mark.parametrize("dtype", [torch.float16, torch.int8])
def test_copy_blocks_writes_only_destination_blocks(cuda_device, dtype):
    NB, bs, H, D = 10, 16, 8, 128
    k, v = _pool(5, NB, bs, H, D, torch.float16)
    scales = None
    if dtype == torch.int8:
        k, ks = quantize_cache(k)
        v, vs = quantize_cache(v)
        scales = (Guarded(ks.shape, ks.dtype, init=ks.cuda()), Guarded(vs.shape, vs.dtype, init=vs.cuda()))
    kc, vc = Guarded(k.shape, k.dtype, init=k.cuda()), Guarded(v.shape, v.dtype, init=v.cuda())
    # the first and last block as targets; no source is also a target
    pairs = torch.tensor([[3, NB - 1], [4, 0], [7, 6]], dtype=torch.int64)
    pa.copy_blocks(kc.t, vc.t, pairs.cuda(), *(s.t for s in scales) if scales else ())
    torch.cuda.synchronize()
    assert_no_device_error()
    assert kc.intact() and vc.intact()
    if scales:
        assert scales[0].intact() and scales[1].intact()
    want = k.clone()
    for s_, d_ in pairs.tolist():
        want[d_] = k[s_]
    assert torch.equal(kc.t.cpu(), want)


def test_prefill_writes_only_out(cuda_device):
    bs, Hq, Hkv, D = 16, 8, 2, 128
    ctx, qlen = [40, 300, 5], [40, 17, 5]
    NB = sum(-(-c // bs) for c in ctx) + 1
    k, v = _pool(6, NB, bs, Hkv, D, torch.float16)
    kc, vc = k.cuda(), v.cuda()
    q = torch.randn(sum(qlen), Hq, D, generator=torch.Generator().manual_seed(7)).half().cuda()
    out = Guarded(q.shape, q.dtype)
    bt = _tables(8, ctx, bs, NB).cuda()
    cu = torch.tensor([0, 40, 57, 62], dtype=torch.int32, device="cuda")
    cl = torch.tensor(ctx, dtype=torch.int32, device="cuda")
    pa.paged_attention_prefill(out.t, q, kc, vc, bt, cu, cl, max(qlen), D ** -0.5)
    torch.cuda.synchronize()
    assert_no_device_error()
    assert out.intact()
    assert torch.equal(kc.cpu(), k) and torch.equal(vc.cpu(), v)


def test_swap_writes_only_destination_blocks_on_both_sides(cuda_device):
    NB, NH, bs, H, D = 8, 5, 16, 4, 128
    k, v = _pool(9, NB, bs, H, D, torch.float16)
    gk, gv = Guarded(k.shape, k.dtype, init=k.cuda()), Guarded(v.shape, v.dtype, init=v.cuda())
    hk = Guarded((NH, bs, H, D), torch.float16, pinned=True)
    hv = Guarded((NH, bs, H, D), torch.float16, pinned=True)
    out_pairs = torch.tensor([[0, NH - 1], [NB - 1, 0], [3, 2]], dtype=torch.int64).cuda()
    pa.swap_blocks(gk.t, gv.t, hk.t, hv.t, out_pairs)
    torch.cuda.synchronize()
    assert hk.intact() and hv.intact()
    in_pairs = torch.tensor([[NH - 1, NB - 1], [0, 0]], dtype=torch.int64).cuda()
    pa.swap_blocks(hk.t, hv.t, gk.t, gv.t, in_pairs)
    torch.cuda.synchronize()
    assert_no_device_error()
    assert gk.intact() and gv.intact() and hk.intact() and hv.intact()
    assert torch.equal(gk.t[NB - 1].cpu(), k[0]) and torch.equal(gk.t[0].cpu(), k[NB - 1])
