"""Pins of the fp64 prefill / chunked-prefill oracle against things other than itself (CPU).

* a naive pure-Python causal attention (tiny sizes) and torch's
  scaled_dot_product_attention with an explicit position mask, under shuffled block tables;
* the whole-prompt case against the library's is_causal path;
* q_len == 1 against the (separately pinned) decode oracle;
* chunking invariance: a prompt prefilled in chunks equals one-shot prefill, bit for bit;
* closed forms (first query sees one token; constant values) and the sliding window
  against a banded mask;
* grouped-query heads against multi-head with repeated K/V;
* an 8-bit cache against the library routine on dequantised values.
An off-by-one in the causal bound, queries placed at the wrong positions, a window that
keeps one token too many or too few, or a wrong kv-head mapping fails one of these.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from test_oracle_decode import _pack


def _case(rng, ctx, qlen, H=2, D=8):
    K = [rng.standard_normal((c, H, D)) for c in ctx]
    V = [rng.standard_normal((c, H, D)) for c in ctx]
    q = rng.standard_normal((sum(qlen), H, D))
    cu = np.concatenate([[0], np.cumsum(qlen)]).astype(np.int32)
    return K, V, q, cu


def _masked_sdpa(q, K, V, ctx, scale, window=0):
    """Library attention for one sequence: q [n, H, D] at positions ctx-n..ctx-1."""
    n = q.shape[0]
    pos_q = np.arange(ctx - n, ctx)[:, None]
    pos_k = np.arange(ctx)[None, :]
    allowed = pos_k <= pos_q
    if window > 0:
        allowed &= pos_k > pos_q - window
    qt = torch.as_tensor(q).permute(1, 0, 2)
    kt = torch.as_tensor(K).permute(1, 0, 2)
    vt = torch.as_tensor(V).permute(1, 0, 2)
    return F.scaled_dot_product_attention(qt, kt, vt, attn_mask=torch.as_tensor(allowed),
                                          scale=scale).permute(1, 0, 2).numpy()


def _naive(q, K, V, ctx, scale):
    """Triple loop, plain Python floats."""
    n, H, D = q.shape
    out = np.zeros_like(q)
    for i in range(n):
        p = ctx - n + i
        for h in range(H):
            s = [scale * sum(q[i, h, d] * K[j, h, d] for d in range(D)) for j in range(p + 1)]
            m = max(s)
            e = [math.exp(x - m) for x in s]
            z = sum(e)
            for d in range(D):
                out[i, h, d] = sum(e[j] * V[j, h, d] for j in range(p + 1)) / z
    return out


def test_prefill_matches_a_naive_loop_on_tiny_inputs():
    rng = np.random.default_rng(0)
    ctx, qlen = [7, 12], [7, 4]
    K, V, q, cu = _case(rng, ctx, qlen)
    kc, vc, bt = _pack(K, V, ctx, 4, rng)
    got = oracle.paged_prefill(torch.from_numpy(q.astype(np.float32)), torch.from_numpy(kc.astype(np.float32)),
                               torch.from_numpy(vc.astype(np.float32)), bt, cu, ctx, 0.4)
    q32 = q.astype(np.float32).astype(np.float64)
    for s in range(2):
        ref = _naive(q32[cu[s]:cu[s + 1]], K[s].astype(np.float32).astype(np.float64),
                     V[s].astype(np.float32).astype(np.float64), ctx[s], 0.4)
        assert np.abs(got[cu[s]:cu[s + 1]] - ref).max() < 1e-12


@pytest.mark.parametrize("bs", [1, 8, 16, 32])
def test_prefill_matches_masked_library_attention(bs):
    rng = np.random.default_rng(bs)
    ctx, qlen = [33, 1, 50, 16], [33, 1, 17, 5]
    K, V, q, cu = _case(rng, ctx, qlen, H=3, D=16)
    K = [k.astype(np.float32).astype(np.float64) for k in K]
    V = [v.astype(np.float32).astype(np.float64) for v in V]
    kc, vc, bt = _pack(K, V, ctx, bs, rng)
    q32 = q.astype(np.float32)
    got = oracle.paged_prefill(torch.from_numpy(q32), torch.from_numpy(kc.astype(np.float32)),
                               torch.from_numpy(vc.astype(np.float32)), bt, cu, ctx, 0.25)
    for s in range(len(ctx)):
        ref = _masked_sdpa(q32[cu[s]:cu[s + 1]].astype(np.float64), K[s], V[s], ctx[s], 0.25)
        assert np.abs(got[cu[s]:cu[s + 1]] - ref).max() < 1e-12


def test_whole_prompt_equals_library_is_causal():
    rng = np.random.default_rng(3)
    n, H, D = 40, 2, 32
    q = torch.randn(n, H, D, dtype=torch.float32, generator=torch.Generator().manual_seed(3))
    K = torch.randn(n, H, D, generator=torch.Generator().manual_seed(4))
    V = torch.randn(n, H, D, generator=torch.Generator().manual_seed(5))
    kc, vc, bt = _pack([K.double().numpy()], [V.double().numpy()], [n], 16, rng)
    got = oracle.paged_prefill(q, torch.from_numpy(kc.astype(np.float32)), torch.from_numpy(vc.astype(np.float32)),
                               bt, [0, n], [n], 1 / math.sqrt(D))
    ref = F.scaled_dot_product_attention(q.double().transpose(0, 1), K.double().transpose(0, 1),
                                         V.double().transpose(0, 1), is_causal=True).transpose(0, 1)
    assert np.abs(got - ref.numpy()).max() < 1e-12


def test_single_query_is_decode():
    rng = np.random.default_rng(4)
    ctx = [5, 17, 64]
    K, V, q, cu = _case(rng, ctx, [1, 1, 1], H=4, D=16)
    kc, vc, bt = _pack(K, V, ctx, 16, rng)
    args = (torch.from_numpy(kc.astype(np.float32)), torch.from_numpy(vc.astype(np.float32)), bt)
    q32 = torch.from_numpy(q.astype(np.float32))
    for w in (0, 7):
        a = oracle.paged_prefill(q32, *args, cu, ctx, 0.3, window=w)
        b = oracle.paged_decode(q32, *args, ctx, 0.3, window=w)
        assert np.array_equal(a, b)


def test_chunked_prefill_equals_one_shot_bit_for_bit():
    rng = np.random.default_rng(5)
    n = 45
    K, V, q, _ = _case(rng, [n], [n], H=2, D=8)
    kc, vc, bt = _pack(K, V, [n], 8, rng)
    kt, vt = torch.from_numpy(kc.astype(np.float32)), torch.from_numpy(vc.astype(np.float32))
    q32 = torch.from_numpy(q.astype(np.float32))
    whole = oracle.paged_prefill(q32, kt, vt, bt, [0, n], [n], 0.5, window=13)
    pieces = []
    for a, b in ((0, 9), (9, 10), (10, 32), (32, 45)):     # chunk boundaries inside and at blocks
        pieces.append(oracle.paged_prefill(q32[a:b], kt, vt, bt, [0, b - a], [b], 0.5, window=13))
    assert np.array_equal(np.concatenate(pieces), whole)


def test_closed_forms():
    rng = np.random.default_rng(6)
    n, H, D = 9, 2, 4
    K, V, q, _ = _case(rng, [n], [n], H, D)
    V[0][:] = 0.75                                           # constant values
    kc, vc, bt = _pack(K, V, [n], 4, rng)
    kt, vt = torch.from_numpy(kc.astype(np.float32)), torch.from_numpy(vc.astype(np.float32))
    got = oracle.paged_prefill(torch.from_numpy(q.astype(np.float32)), kt, vt, bt, [0, n], [n], 1.0)
    assert np.abs(got - 0.75).max() < 1e-15
    V2 = [rng.standard_normal((n, H, D))]
    kc, vc, bt = _pack(K, V2, [n], 4, rng)
    got = oracle.paged_prefill(torch.from_numpy(q.astype(np.float32)), torch.from_numpy(kc.astype(np.float32)),
                               torch.from_numpy(vc.astype(np.float32)), bt, [0, n], [n], 1.0)
    assert np.array_equal(got[0], V2[0][0].astype(np.float32).astype(np.float64))  # first query sees token 0 only
    got_w1 = oracle.paged_prefill(torch.from_numpy(q.astype(np.float32)), torch.from_numpy(kc.astype(np.float32)),
                                  torch.from_numpy(vc.astype(np.float32)), bt, [0, n], [n], 1.0, window=1)
    assert np.array_equal(got_w1, V2[0].astype(np.float32).astype(np.float64))   # window 1: each sees itself


@pytest.mark.parametrize("window", [1, 5, 16])
def test_window_matches_banded_mask(window):
    rng = np.random.default_rng(7 + window)
    ctx, qlen = [30, 21], [12, 21]
    K, V, q, cu = _case(rng, ctx, qlen, H=2, D=8)
    K = [k.astype(np.float32).astype(np.float64) for k in K]
    V = [v.astype(np.float32).astype(np.float64) for v in V]
    kc, vc, bt = _pack(K, V, ctx, 16, rng)
    q32 = q.astype(np.float32)
    got = oracle.paged_prefill(torch.from_numpy(q32), torch.from_numpy(kc.astype(np.float32)),
                               torch.from_numpy(vc.astype(np.float32)), bt, cu, ctx, 0.3, window=window)
    for s in range(2):
        ref = _masked_sdpa(q32[cu[s]:cu[s + 1]].astype(np.float64), K[s], V[s], ctx[s], 0.3, window)
        assert np.abs(got[cu[s]:cu[s + 1]] - ref).max() < 1e-12


def test_grouped_query_equals_repeated_kv():
    rng = np.random.default_rng(9)
    ctx, qlen, Hkv, G, D = [20, 35], [20, 6], 2, 3, 8
    K, V, _, cu = _case(rng, ctx, qlen, H=Hkv, D=D)
    q = rng.standard_normal((sum(qlen), Hkv * G, D)).astype(np.float32)
    kc, vc, bt = _pack(K, V, ctx, 8, rng)
    kt, vt = torch.from_numpy(kc.astype(np.float32)), torch.from_numpy(vc.astype(np.float32))
    got = oracle.paged_prefill(torch.from_numpy(q), kt, vt, bt, cu, ctx, 0.35)
    rep = oracle.paged_prefill(torch.from_numpy(q), kt.repeat_interleave(G, dim=2), vt.repeat_interleave(G, dim=2),
                               bt, cu, ctx, 0.35)
    assert np.array_equal(got, rep)


def test_int8_cache_matches_library_on_dequantised_values():
    rng = np.random.default_rng(10)
    ctx, qlen, H, D = [24], [10], 2, 16
    K, V, q, cu = _case(rng, ctx, qlen, H, D)
    kq, ks = oracle.quant.quantize_rows(K[0].astype(np.float16))
    vq, vs = oracle.quant.quantize_rows(V[0].astype(np.float16))
    kdq = oracle.quant.dequantize_rows(kq, ks)
    vdq = oracle.quant.dequantize_rows(vq, vs)
    perm_rng = np.random.default_rng(11)
    kc, vc, bt = _pack([kq.astype(np.float64)], [vq.astype(np.float64)], ctx, 8, perm_rng, fill=0)
    ksc, vsc, _ = _pack([ks[..., None].astype(np.float64)], [vs[..., None].astype(np.float64)], ctx, 8,
                        np.random.default_rng(11), fill=0)
    got = oracle.paged_prefill(torch.from_numpy(q.astype(np.float32)), torch.from_numpy(kc.astype(np.int8)),
                               torch.from_numpy(vc.astype(np.int8)), bt, cu, ctx, 0.3,
                               k_scale=ksc[..., 0].astype(np.float16), v_scale=vsc[..., 0].astype(np.float16))
    ref = _masked_sdpa(q.astype(np.float32).astype(np.float64), kdq, vdq, ctx[0], 0.3)
    assert np.abs(got - ref).max() < 1e-12


def test_rejects_more_queries_than_context():
    kc = torch.zeros(2, 4, 1, 8)
    with pytest.raises(ValueError):
        oracle.paged_prefill(torch.zeros(5, 1, 8), kc, kc, [[0, 1]], [0, 5], [4], 1.0)


def test_threads_share_out_pairs_without_changing_a_bit():
    """Worker threads give the single-threaded prefill result bit for bit."""
    g = torch.Generator().manual_seed(31)
    ctx, qlen, bs, Hq, Hkv, D = [9, 40, 1, 70], [9, 5, 1, 33], 8, 6, 3, 16
    NB = sum(-(-c // bs) for c in ctx) + 2
    perm = torch.randperm(NB, generator=g)
    MB = max(-(-c // bs) for c in ctx)
    bt = torch.full((len(ctx), MB), -1, dtype=torch.int32)
    k = 0
    for s, c in enumerate(ctx):
        for lb in range(-(-c // bs)):
            bt[s, lb] = int(perm[k])
            k += 1
    kc = torch.randn(NB, bs, Hkv, D, generator=g)
    vc = torch.randn(NB, bs, Hkv, D, generator=g)
    q = torch.randn(sum(qlen), Hq, D, generator=g)
    cu = torch.tensor([0] + list(np.cumsum(qlen)), dtype=torch.int32)
    for window in (0, 7):
        one = oracle.paged_prefill(q, kc, vc, bt, cu, ctx, 0.25, window, threads=1)
        for n in (2, 4, 32):
            many = oracle.paged_prefill(q, kc, vc, bt, cu, ctx, 0.25, window, threads=n)
            assert np.array_equal(one.view(np.uint64), many.view(np.uint64))
