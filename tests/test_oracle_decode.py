"""Pins of the fp64 decode oracle against things other than itself (CPU only).

* exact fp16 / bf16 decoding vs numpy / torch conversions of every bit pattern;
* the dense special case vs torch's scaled_dot_product_attention (a library routine) on
  contiguous K/V, under shuffled block tables and several block sizes;
* closed forms: one token, identical keys, constant values, one dominant key, empty context;
* invariances: physical block permutation, block_size repacking, window >= context;
* the window against the library routine on the truncated sequence;
* the INT8 path against the library routine on dequantised values.
A dropped term, a wrong sign or stride, a transposed operand or an off-by-one window
fails at least one of these.
"""
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle


def _pack(K, V, ctx, bs, rng, extra_blocks=3, fill=np.nan):
    """Place logical K/V [S][n_s, H, D] into a shuffled pool [NB, bs, H, D] (test-side)."""
    S = len(ctx)
    H, D = K[0].shape[1], K[0].shape[2]
    nblocks = [-(-c // bs) for c in ctx]
    NB = sum(nblocks) + extra_blocks
    perm = rng.permutation(NB)
    kc = np.full((NB, bs, H, D), fill, np.float64)
    vc = np.full((NB, bs, H, D), fill, np.float64)
    MB = max(1, max(nblocks))
    bt = np.full((S, MB), -1, np.int32)
    k = 0
    for s in range(S):
        for lb in range(nblocks[s]):
            pb = perm[k]
            k += 1
            bt[s, lb] = pb
            lo, hi = lb * bs, min(ctx[s], (lb + 1) * bs)
            kc[pb, : hi - lo] = K[s][lo:hi]
            vc[pb, : hi - lo] = V[s][lo:hi]
    return kc, vc, bt


def _as_f32_tensor(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))


def _sdpa(q, K, V, scale):
    """Library attention of one query per head: q [H, D], K/V [n, H, D] (fp64)."""
    qt = torch.as_tensor(q, dtype=torch.float64)[:, None, :]          # [H, 1, D]
    kt = torch.as_tensor(K, dtype=torch.float64).permute(1, 0, 2)     # [H, n, D]
    vt = torch.as_tensor(V, dtype=torch.float64).permute(1, 0, 2)
    return F.scaled_dot_product_attention(qt, kt, vt, scale=scale)[:, 0, :].numpy()


def _random_case(rng, S=3, H=2, D=8, max_ctx=40):
    ctx = [int(c) for c in rng.integers(1, max_ctx + 1, S)]
    q = rng.standard_normal((S, H, D)).astype(np.float32)
    K = [rng.standard_normal((c, H, D)).astype(np.float32) for c in ctx]
    V = [rng.standard_normal((c, H, D)).astype(np.float32) for c in ctx]
    return ctx, q, K, V


def test_f16_decoder_matches_numpy_for_every_bit_pattern():
    bits = np.arange(65536, dtype=np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([oracle.f16_to_f64(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


def test_bf16_decoder_matches_torch_for_every_bit_pattern():
    bits = torch.arange(65536, dtype=torch.int32).to(torch.int16)
    ref = bits.view(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([oracle.bf16_to_f64(int(b) & 0xFFFF) for b in bits.tolist()])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


@pytest.mark.parametrize("bs", [1, 3, 8, 16, 32])
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_dense_special_case_matches_library_attention(bs, seed):
    rng = np.random.default_rng(seed)
    ctx, q, K, V = _random_case(rng)
    kc, vc, bt = _pack(K, V, ctx, bs, rng)
    scale = 1.0 / math.sqrt(q.shape[2])
    out = oracle.paged_decode(_as_f32_tensor(q), _as_f32_tensor(kc), _as_f32_tensor(vc), bt, ctx, scale)
    for s in range(len(ctx)):
        ref = _sdpa(q[s], K[s], V[s], scale)
        np.testing.assert_allclose(out[s], ref, rtol=0, atol=1e-12)


def test_identity_table_with_block_size_equal_context_is_dense_attention():
    rng = np.random.default_rng(7)
    H, D, n = 2, 8, 37
    q = rng.standard_normal((1, H, D)).astype(np.float32)
    K = rng.standard_normal((1, n, H, D)).astype(np.float32)
    V = rng.standard_normal((1, n, H, D)).astype(np.float32)
    out = oracle.paged_decode(_as_f32_tensor(q), _as_f32_tensor(K), _as_f32_tensor(V), [[0]], [n], 0.3)
    np.testing.assert_allclose(out[0], _sdpa(q[0], K[0], V[0], 0.3), rtol=0, atol=1e-12)


def test_single_token_returns_its_value_row_exactly():
    rng = np.random.default_rng(1)
    q = rng.standard_normal((1, 2, 8)).astype(np.float32)
    K = [rng.standard_normal((1, 2, 8)).astype(np.float32)]
    V = [rng.standard_normal((1, 2, 8)).astype(np.float32)]
    kc, vc, bt = _pack(K, V, [1], 16, rng)
    out = oracle.paged_decode(_as_f32_tensor(q), _as_f32_tensor(kc), _as_f32_tensor(vc), bt, [1], 0.5)
    assert np.array_equal(out[0], V[0][0].astype(np.float64))


def test_identical_keys_give_the_mean_of_values():
    rng = np.random.default_rng(2)
    n, H, D = 29, 2, 8
    q = rng.standard_normal((1, H, D)).astype(np.float32)
    k = rng.standard_normal((1, H, D)).astype(np.float32)
    K = [np.repeat(k, n, axis=0)]
    V = [rng.standard_normal((n, H, D)).astype(np.float32)]
    kc, vc, bt = _pack(K, V, [n], 8, rng)
    out = oracle.paged_decode(_as_f32_tensor(q), _as_f32_tensor(kc), _as_f32_tensor(vc), bt, [n], 0.7)
    np.testing.assert_allclose(out[0], V[0].astype(np.float64).mean(axis=0), rtol=0, atol=1e-13)


def test_constant_values_are_returned_unchanged():
    rng = np.random.default_rng(3)
    n, H, D = 21, 2, 8
    q = rng.standard_normal((1, H, D)).astype(np.float32)
    K = [rng.standard_normal((n, H, D)).astype(np.float32)]
    c = rng.standard_normal((1, H, D)).astype(np.float32)
    V = [np.repeat(c, n, axis=0)]
    kc, vc, bt = _pack(K, V, [n], 16, rng)
    out = oracle.paged_decode(_as_f32_tensor(q), _as_f32_tensor(kc), _as_f32_tensor(vc), bt, [n], 0.4)
    np.testing.assert_allclose(out[0], c[0].astype(np.float64), rtol=0, atol=1e-14)


def test_one_dominant_key_selects_its_value():
    rng = np.random.default_rng(4)
    n, H, D = 33, 1, 8
    q = np.zeros((1, H, D), np.float32)
    q[0, 0, 0] = 1.0
    K = [np.zeros((n, H, D), np.float32)]
    K[0][17, 0, 0] = 60.0  # score 60 above every other key (scale 1)
    V = [rng.standard_normal((n, H, D)).astype(np.float32)]
    kc, vc, bt = _pack(K, V, [n], 16, rng)
    out = oracle.paged_decode(_as_f32_tensor(q), _as_f32_tensor(kc), _as_f32_tensor(vc), bt, [n], 1.0)
    np.testing.assert_allclose(out[0, 0], V[0][17, 0].astype(np.float64), rtol=0, atol=n * math.exp(-60) * 10)


def test_empty_context_gives_zeros():
    q = torch.randn(2, 2, 8)
    kc = torch.randn(4, 16, 2, 8)
    out = oracle.paged_decode(q, kc, kc, [[0], [1]], [0, 5], 0.3)
    assert np.all(out[0] == 0.0)
    assert np.all(np.isfinite(out[1]))


@pytest.mark.parametrize("seed", [0, 1])
def test_physical_block_permutation_is_invisible(seed):
    rng = np.random.default_rng(seed)
    ctx, q, K, V = _random_case(rng, S=4, max_ctx=70)
    kc, vc, bt = _pack(K, V, ctx, 16, rng, fill=0.0)
    base = oracle.paged_decode(_as_f32_tensor(q), _as_f32_tensor(kc), _as_f32_tensor(vc), bt, ctx, 0.35)
    perm = rng.permutation(kc.shape[0])           # new id of old block b is perm[b]
    kc2 = np.empty_like(kc); vc2 = np.empty_like(vc)
    kc2[perm] = kc; vc2[perm] = vc
    bt2 = np.where(bt >= 0, perm[np.maximum(bt, 0)], -1).astype(np.int32)
    moved = oracle.paged_decode(_as_f32_tensor(q), _as_f32_tensor(kc2), _as_f32_tensor(vc2), bt2, ctx, 0.35)
    assert np.array_equal(base, moved)


def test_block_size_repacking_is_invisible():
    rng = np.random.default_rng(5)
    ctx, q, K, V = _random_case(rng, S=3, max_ctx=100)
    outs = []
    for bs in (1, 8, 16, 32):
        kc, vc, bt = _pack(K, V, ctx, bs, rng)
        outs.append(oracle.paged_decode(_as_f32_tensor(q), _as_f32_tensor(kc), _as_f32_tensor(vc), bt, ctx, 0.35))
    for o in outs[1:]:
        assert np.array_equal(outs[0], o)


def test_window_covering_the_context_equals_full_attention():
    rng = np.random.default_rng(6)
    ctx, q, K, V = _random_case(rng, S=3, max_ctx=50)
    kc, vc, bt = _pack(K, V, ctx, 16, rng)
    args = (_as_f32_tensor(q), _as_f32_tensor(kc), _as_f32_tensor(vc), bt, ctx, 0.35)
    full = oracle.paged_decode(*args)
    assert np.array_equal(full, oracle.paged_decode(*args, window=max(ctx)))
    assert np.array_equal(full, oracle.paged_decode(*args, window=10 ** 6))


@pytest.mark.parametrize("window", [1, 5, 16, 17, 31])
def test_window_attends_exactly_the_last_w_tokens(window):
    rng = np.random.default_rng(window)
    ctx, q, K, V = _random_case(rng, S=3, max_ctx=60)
    kc, vc, bt = _pack(K, V, ctx, 16, rng)
    out = oracle.paged_decode(_as_f32_tensor(q), _as_f32_tensor(kc), _as_f32_tensor(vc), bt, ctx, 0.35, window=window)
    for s, c in enumerate(ctx):
        lo = max(0, c - window)
        np.testing.assert_allclose(out[s], _sdpa(q[s], K[s][lo:c], V[s][lo:c], 0.35), rtol=0, atol=1e-12)


def test_int8_cache_dequantises_with_per_row_scales():
    rng = np.random.default_rng(8)
    S, H, D, bs, n = 2, 8, 16, 8, 19
    q = rng.standard_normal((S, H, D)).astype(np.float32)
    NB = 2 * (-(-n // bs)) + 1
    kq = rng.integers(-127, 128, (NB, bs, H, D)).astype(np.int8)
    vq = rng.integers(-127, 128, (NB, bs, H, D)).astype(np.int8)
    ks = (rng.random((NB, bs, H)) * 0.05 + 1e-3).astype(np.float16)
    vs = (rng.random((NB, bs, H)) * 0.05 + 1e-3).astype(np.float16)
    bt = rng.permutation(NB)[: 2 * (-(-n // bs))].reshape(2, -1).astype(np.int32)
    out = oracle.paged_decode(_as_f32_tensor(q), torch.from_numpy(kq), torch.from_numpy(vq), bt, [n, n], 0.25,
                              k_scale=torch.from_numpy(ks), v_scale=torch.from_numpy(vs))
    for s in range(S):
        rows = [(bt[s, i // bs], i % bs) for i in range(n)]
        Kd = np.stack([kq[pb, off].astype(np.float64) * ks[pb, off].astype(np.float64)[:, None] for pb, off in rows])
        Vd = np.stack([vq[pb, off].astype(np.float64) * vs[pb, off].astype(np.float64)[:, None] for pb, off in rows])
        np.testing.assert_allclose(out[s], _sdpa(q[s], Kd, Vd, 0.25), rtol=0, atol=1e-12)


def test_half_precision_inputs_are_read_exactly():
    rng = np.random.default_rng(9)
    ctx, q, K, V = _random_case(rng, S=2, max_ctx=30)
    kc, vc, bt = _pack(K, V, ctx, 16, rng, fill=0.0)
    for dt in (torch.float16, torch.bfloat16):
        qt, kt, vt = (torch.from_numpy(x.astype(np.float32)).to(dt) for x in (q, kc, vc))
        out = oracle.paged_decode(qt, kt, vt, bt, ctx, 0.35)
        ref = oracle.paged_decode(qt.float(), kt.float(), vt.float(), bt, ctx, 0.35)
        assert np.array_equal(out, ref)


def test_out_of_range_table_entry_is_an_error():
    q = torch.randn(1, 1, 8)
    kc = torch.randn(2, 4, 1, 8)
    with pytest.raises(ValueError, match="block-table"):
        oracle.paged_decode(q, kc, kc, [[0, 5]], [6], 0.3)
    with pytest.raises(ValueError, match="context"):
        oracle.paged_decode(q, kc, kc, [[0, 1]], [9], 0.3)


# ---------------------------------------------------------------------------------------
# Grouped-query attention (query head h reads cached head h // (Hq // Hkv))
# ---------------------------------------------------------------------------------------
@pytest.mark.parametrize("hq,hkv", [(8, 2), (8, 1), (6, 3), (4, 4)])
def test_gqa_equals_multi_head_on_a_repeated_cache(hq, hkv):
    rng = np.random.default_rng(hq * 10 + hkv)
    S, D, bs = 3, 8, 8
    ctx = [5, 17, 30]
    NB = sum(-(-c // bs) for c in ctx) + 2
    q = rng.standard_normal((S, hq, D)).astype(np.float32)
    kc = rng.standard_normal((NB, bs, hkv, D)).astype(np.float32)
    vc = rng.standard_normal((NB, bs, hkv, D)).astype(np.float32)
    bt = rng.permutation(NB)[: sum(-(-c // bs) for c in ctx)]
    tables, k = [], 0
    for c in ctx:
        n = -(-c // bs)
        tables.append(list(bt[k:k + n]) + [-1] * (4 - n))
        k += n
    bt = np.array(tables, np.int32)
    g = hq // hkv
    gqa = oracle.paged_decode(_as_f32_tensor(q), _as_f32_tensor(kc), _as_f32_tensor(vc), bt, ctx, 0.3)
    kx = torch.from_numpy(kc).repeat_interleave(g, dim=2)   # library expansion of the shared heads
    vx = torch.from_numpy(vc).repeat_interleave(g, dim=2)
    mha = oracle.paged_decode(_as_f32_tensor(q), kx, vx, bt, ctx, 0.3)
    assert np.array_equal(gqa, mha)


def test_gqa_dense_case_matches_library_attention():
    rng = np.random.default_rng(11)
    hq, hkv, D, n = 8, 2, 16, 29
    q = rng.standard_normal((1, hq, D)).astype(np.float32)
    K = rng.standard_normal((1, n, hkv, D)).astype(np.float32)
    V = rng.standard_normal((1, n, hkv, D)).astype(np.float32)
    out = oracle.paged_decode(_as_f32_tensor(q), _as_f32_tensor(K), _as_f32_tensor(V), [[0]], [n], 0.25)
    qt = torch.from_numpy(q[0]).double()[None, :, None, :]                  # [1, Hq, 1, D]
    kt = torch.from_numpy(K[0]).double().permute(1, 0, 2)[None]             # [1, Hkv, n, D]
    vt = torch.from_numpy(V[0]).double().permute(1, 0, 2)[None]
    ref = F.scaled_dot_product_attention(qt, kt, vt, scale=0.25, enable_gqa=True)[0, :, 0, :].numpy()
    np.testing.assert_allclose(out[0], ref, rtol=0, atol=1e-12)


def test_threads_share_out_pairs_without_changing_a_bit():
    """Several worker threads give the single-threaded result bit for bit, on a batch with
    empty, windowed, grouped-query and 8-bit cases, and the same error status when an item
    fails (the lowest failing (sequence, head) pair decides it)."""
    rng = np.random.default_rng(21)
    ctx = [0, 1, 17, 40, 3, 64, 33]
    K = [rng.standard_normal((c, 2, 16)) for c in ctx]
    V = [rng.standard_normal((c, 2, 16)) for c in ctx]
    kc, vc, bt = _pack(K, V, ctx, 8, rng)
    q = rng.standard_normal((len(ctx), 6, 16)).astype(np.float32)
    kt, vt = _as_f32_tensor(kc), _as_f32_tensor(vc)
    for window in (0, 9):
        one = oracle.paged_decode(q, kt, vt, bt, ctx, 0.3, window, threads=1)
        for n in (2, 5, 64):
            many = oracle.paged_decode(q, kt, vt, bt, ctx, 0.3, window, threads=n)
            assert np.array_equal(one.view(np.uint64), many.view(np.uint64))
    bad = bt.copy()
    bad[5, 2] = kc.shape[0] + 3             # sequence 5: an entry outside the pool
    ctx_bad = list(ctx)
    ctx_bad[6] = bt.shape[1] * 8 + 1        # sequence 6: a context beyond its table
    for n in (1, 3, 16):
        with pytest.raises(ValueError, match="block-table entry"):
            oracle.paged_decode(q, kt, vt, bad, ctx_bad, 0.3, threads=n)
    ctx_bad[2] = -1                          # now an earlier pair fails on its context
    for n in (1, 3, 16):
        with pytest.raises(ValueError, match="context length"):
            oracle.paged_decode(q, kt, vt, bad, ctx_bad, 0.3, threads=n)
