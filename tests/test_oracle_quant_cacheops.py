"""Pins of the oracle's INT8 quantiser and cache-maintenance definitions (CPU only).

Quantiser (reading of "KV Cache optimisation strategies in deployment" (yunthe.com),
section "量化压缩KV Cache的INT8与FP8方案", which names INT8 without a scheme): brute
force over every finite fp16 value checks the dequantisation error bound, the code
range, symmetry, that the row maximum maps to +-127, and ties-to-even on exact halves.
Cache operations: the page's flat address h*D + (pb*bs + off)*H*D ("KV Cache memory
optimisation and PagedAttention" (yunthe.com), section "PagedAttention注意力计算流程").
"""
import numpy as np
import pytest

from oracle import cache_ops, quant


def _all_finite_f16():
    v = np.arange(65536, dtype=np.uint16).view(np.float16)
    return v[np.isfinite(v)]


def test_every_fp16_value_dequantises_within_half_a_step():
    x = _all_finite_f16()
    # rows [x, m]: m = 1.0 sets the scale unless |x| is larger
    rows = np.stack([x, np.full_like(x, 1.0)], axis=1)
    codes, scale = quant.quantize_rows(rows)
    deq = quant.dequantize_rows(codes, scale)
    s = scale.astype(np.float64)
    assert np.all(np.abs(codes.astype(np.int32)) <= 127)
    err = np.abs(deq - rows.astype(np.float64))
    # |x / s| <= 127 * (1 + 2^-11) so rounding to the nearest code is within s/2 (+ the fp32 division)
    assert np.all(err <= s[:, None] * (0.5 + 1e-3))


def test_row_maximum_maps_to_127():
    rng = np.random.default_rng(0)
    rows = rng.standard_normal((4096, 128)).astype(np.float16)
    codes, scale = quant.quantize_rows(rows)
    amax_idx = np.argmax(np.abs(rows.astype(np.float32)), axis=1)
    top = np.abs(codes[np.arange(4096), amax_idx].astype(np.int32))
    assert np.all(top == 127)
    assert np.all(scale > 0)


def test_quantiser_is_odd_symmetric():
    rng = np.random.default_rng(1)
    rows = rng.standard_normal((512, 64)).astype(np.float16)
    c1, s1 = quant.quantize_rows(rows)
    c2, s2 = quant.quantize_rows(-rows)
    assert np.array_equal(s1, s2)
    assert np.array_equal(c1.astype(np.int32), -c2.astype(np.int32))


def test_exact_halves_round_to_even():
    s = 2.0 ** -7                       # 127 * s is exact in fp16, amax / 127 = s exactly
    row = np.array([127 * s, 2.5 * s, 3.5 * s, -2.5 * s, 0.5 * s, 1.5 * s, 0.0, -0.5 * s], np.float16)
    codes, scale = quant.quantize_rows(row[None, :])
    assert float(scale[0]) == s
    assert codes[0].tolist() == [127, 2, 4, -2, 0, 2, 0, 0]


def test_zero_row_has_zero_scale_and_codes():
    codes, scale = quant.quantize_rows(np.zeros((3, 16), np.float16))
    assert np.all(scale == 0) and np.all(codes == 0)


def test_tiny_row_whose_scale_underflows_stores_zeros():
    row = np.array([[2.0 ** -24, 0.0]], np.float16)  # amax / 127 rounds to 0 in fp16
    codes, scale = quant.quantize_rows(row)
    assert scale[0] == 0 and np.all(codes == 0)


def test_reshape_and_cache_follows_the_pages_flat_address():
    rng = np.random.default_rng(2)
    NB, bs, H, D, T = 5, 4, 3, 8, 7
    kc = np.zeros((NB, bs, H, D), np.float32)
    vc = np.zeros((NB, bs, H, D), np.float32)
    k = rng.standard_normal((T, H, D)).astype(np.float32)
    v = rng.standard_normal((T, H, D)).astype(np.float32)
    slots = np.array([0, 19, 5, -1, 7, 12, 3])
    cache_ops.reshape_and_cache(k, v, kc, vc, slots)
    flat_k, flat_v = kc.reshape(-1), vc.reshape(-1)
    for t, slot in enumerate(slots):
        if slot < 0:
            continue
        pb, off = slot // bs, slot % bs
        for h in range(H):
            addr = h * D + (pb * bs + off) * H * D   # the page's address expression
            assert np.array_equal(flat_k[addr: addr + D], k[t, h])
            assert np.array_equal(flat_v[addr: addr + D], v[t, h])
    written = {int(s) for s in slots if s >= 0}
    untouched = [s for s in range(NB * bs) if s not in written]
    assert np.all(kc.reshape(NB * bs, -1)[untouched] == 0)


def test_copy_blocks_duplicates_whole_blocks_and_nothing_else():
    rng = np.random.default_rng(3)
    NB, bs, H, D = 6, 4, 2, 8
    kc = rng.standard_normal((NB, bs, H, D)).astype(np.float32)
    vc = rng.standard_normal((NB, bs, H, D)).astype(np.float32)
    k0, v0 = kc.copy(), vc.copy()
    pairs = np.array([[1, 4], [2, 5]])
    cache_ops.copy_blocks(kc, vc, pairs)
    assert np.array_equal(kc[4], k0[1]) and np.array_equal(kc[5], k0[2])
    assert np.array_equal(vc[4], v0[1]) and np.array_equal(vc[5], v0[2])
    for b in (0, 1, 2, 3):
        assert np.array_equal(kc[b], k0[b]) and np.array_equal(vc[b], v0[b])



def _memmove_swap(src, dst, pairs):
    """Byte model of a block swap written with raw memmove on flat buffers."""
    import ctypes
    src_b, dst_b = src.view(np.uint8).reshape(-1), dst.view(np.uint8).reshape(-1)
    blk = src[0].nbytes
    for s, d in pairs:
        ctypes.memmove(dst_b.ctypes.data + d * blk, src_b.ctypes.data + s * blk, blk)


def test_swap_blocks_matches_a_memmove_model_between_pools_of_different_sizes():
    rng = np.random.default_rng(5)
    bs, H, D = 4, 3, 8
    gk = rng.integers(0, 256, (9, bs, H, D), dtype=np.uint8)
    gv = rng.integers(0, 256, (9, bs, H, D), dtype=np.uint8)
    gks = rng.integers(0, 1 << 16, (9, bs, H), dtype=np.uint16)
    gvs = rng.integers(0, 1 << 16, (9, bs, H), dtype=np.uint16)
    hk, hv = np.zeros((5, bs, H, D), np.uint8), np.zeros((5, bs, H, D), np.uint8)
    hks, hvs = np.zeros((5, bs, H), np.uint16), np.zeros((5, bs, H), np.uint16)
    pairs = [(7, 0), (2, 4), (8, 1)]
    want = [x.copy() for x in (hk, hv, hks, hvs)]
    for s_, w in zip((gk, gv, gks, gvs), want):
        _memmove_swap(s_, w, pairs)
    cache_ops.swap_blocks(gk, gv, hk, hv, np.array(pairs), (gks, gvs), (hks, hvs))
    for got, w in zip((hk, hv, hks, hvs), want):
        assert np.array_equal(got, w)
    assert not hk[2].any() and not hk[3].any()  # blocks not named by a pair stay as they were


def test_swap_out_then_in_restores_blocks_at_their_new_ids():
    rng = np.random.default_rng(6)
    g = rng.standard_normal((2, 8, 2, 2, 4)).astype(np.float32)
    gk, gv = g[0].copy(), g[1].copy()
    hk, hv = np.full((4, 2, 2, 4), np.nan, np.float32), np.full((4, 2, 2, 4), np.nan, np.float32)
    out_pairs = np.array([[1, 3], [6, 0]])
    cache_ops.swap_blocks(gk, gv, hk, hv, out_pairs)
    gk[[1, 6]] = 0  # the GPU blocks are reused by someone else meanwhile
    back = np.array([[3, 5], [0, 2]])  # swap-in lands in other free GPU blocks
    cache_ops.swap_blocks(hk, hv, gk, gv, back)
    assert np.array_equal(gk[5], g[0][1]) and np.array_equal(gk[2], g[0][6])
    assert np.array_equal(gv[5], g[1][1]) and np.array_equal(gv[2], g[1][6])


# ---------------------------------------------------------------------------------------
# FP8 (E4M3) quantiser
# ---------------------------------------------------------------------------------------
def test_e4m3_code_points_match_torch_and_the_c_decoder():
    import oracle
    import torch
    mine = quant.e4m3_values()
    lib = torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    c = np.array([oracle.e4m3_to_f64(i) for i in range(256)])
    for other in (lib, c):
        assert np.array_equal(np.isnan(mine), np.isnan(other))
        assert np.array_equal(mine[~np.isnan(mine)], other[~np.isnan(other)])
    assert np.nanmax(mine) == 448.0


def test_e4m3_rounding_matches_torch_on_a_dense_sweep():
    import torch
    rng = np.random.default_rng(5)
    x = np.concatenate([rng.standard_normal(300000).astype(np.float32) * np.float32(40),
                        (rng.random(100000).astype(np.float32) - np.float32(0.5)) * np.float32(0.03),
                        np.float32([2 ** -10, -2 ** -10, 3 * 2 ** -10, 448, -448, 2 ** -6, 0.0, -0.0])])
    x = x[np.abs(x) <= 448]
    mine = quant.e4m3_round(x)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn)
    assert np.array_equal(quant.e4m3_encode(mine), ref.view(torch.uint8).numpy())


def test_fp8_quantiser_properties_on_every_fp16_value():
    x = _all_finite_f16()
    rows = np.stack([x, np.full_like(x, 1.0)], axis=1)
    codes, scale = quant.quantize_rows_fp8(rows)
    deq = quant.dequantize_rows_fp8(codes, scale)
    s = scale.astype(np.float64)[:, None]
    ratio = rows.astype(np.float64) / s
    # E4M3 has 3 mantissa bits: relative error <= 2^-4 for normal values, absolute <= 2^-10 * s below
    err = np.abs(deq - rows.astype(np.float64))
    bound = np.maximum(np.abs(rows.astype(np.float64)) * 2.0 ** -4, 2.0 ** -10 * s) * (1 + 1e-3)
    assert np.all(err <= bound + 1e-3 * s * 2.0 ** -9)
    top = np.argmax(np.abs(rows.astype(np.float32)), axis=1)
    assert np.all(np.abs(quant.e4m3_values()[codes[np.arange(len(x)), top]]) == 448.0)
    assert np.all(np.isfinite(ratio))


def test_fp8_zero_row():
    codes, scale = quant.quantize_rows_fp8(np.zeros((2, 8), np.float16))
    assert np.all(codes == 0) and np.all(scale == 0)
