"""Host-side checks that need no GPU.

* Golden values printed on the pages pin the byte / waste accounting used by the
  benchmark (tests/golden/*.json, each with its source).
* The C ABI: the library loads, exports every function declared in include/*.h, and its
  host-side validation rejects bad arguments with the documented status before touching
  CUDA (so these calls are safe without a GPU).
"""
import ctypes
import glob
import json
import math
import os
import re

import pytest

from paged_kv_cache_384_b200 import accounting

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
GOLDEN = os.path.join(ROOT, "tests", "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def test_llama2_70b_kv_bytes_per_token_and_batch_total():
    g = _golden("kv_bytes_llama2_70b.json")
    per_token = accounting.kv_bytes_per_token(g["layers"], g["num_heads"], g["head_dim"], g["dtype_size"])
    assert per_token == 2_621_440                         # exactly 2.5 MiB
    assert round(per_token / 2 ** 20, 1) == g["printed_per_token_mb"]
    total = per_token * g["batch"] * g["seq_len"]
    assert round(total / 2 ** 30) == g["printed_total_gb"]


def test_flowchart_contiguous_waste_and_paged_waste():
    g = _golden("flowchart_block_tables.json")
    for used, printed in zip(g["used_tokens"], g["printed_waste_percent"]):
        w = accounting.contiguous_waste_fraction(used, g["reserved_tokens"])
        assert abs(100 * w - printed) < 2.0                # page rounds 75.6 -> 75, 41.4 -> 40
    b = _golden("block_size_waste.json")
    for used in g["used_tokens"]:
        assert 100 * accounting.paged_waste_fraction(used, b["block_size"]) < b["printed_max_waste_percent"]


def test_decode_byte_count():
    assert accounting.decode_kv_bytes([3, 5], 2, 64, "fp16") == 8 * 2 * 64 * 2 * 2
    assert accounting.decode_kv_bytes([10, 2], 1, 64, "fp16", window=4) == 6 * 64 * 2 * 2
    assert accounting.decode_kv_bytes([4], 8, 128, "int8") == 4 * 8 * (128 * 2 + 4)


# ---------------------------------------------------------------------------------------
# C ABI
# ---------------------------------------------------------------------------------------
def _declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^\s*[A-Za-z_][\w\s\*]*?\b([A-Za-z_]\w*)\s*\(", text, flags=re.M):
            name = m.group(1)
            if name not in {"if", "while", "for", "return", "sizeof"}:
                names.add(name)
    return names


def test_library_exports_every_declared_function():
    from paged_kv_cache_384_b200 import _lib
    lib = ctypes.CDLL(_lib.LIB_PATH)
    declared = _declared_functions()
    assert {"paged_attention_decode", "reshape_and_cache", "copy_blocks"} <= declared
    missing = [n for n in sorted(declared) if not hasattr(lib, n)]
    assert not missing, missing
    assert set(_lib.SIGNATURES) >= declared


@pytest.fixture(scope="module")
def L():
    from paged_kv_cache_384_b200 import _lib
    return _lib.load()


def _decode(L, **kw):
    a = dict(out=16, q=16, k=16, v=16, ks=None, vs=None, bt=16, cl=16, S=1, H=4, D=64, bs=16, NB=4,
             MB=2, scale=0.125, window=0, io=0, cache=0, ws=16, wsb=1 << 20)
    a.update(kw)
    P = lambda x: None if x is None else ctypes.c_void_p(x)
    return L.paged_attention_decode(P(a["out"]), P(a["q"]), P(a["k"]), P(a["v"]), P(a["ks"]), P(a["vs"]),
                                    P(a["bt"]), P(a["cl"]), a["S"], a["H"], a["D"], a["bs"], a["NB"], a["MB"],
                                    a["scale"], a["window"], a["io"], a["cache"], P(a["ws"]), a["wsb"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(q=None), 1), (dict(out=None), 1), (dict(bt=None), 1), (dict(ws=None), 1),
    (dict(D=96), 2), (dict(bs=0), 2), (dict(bs=64), 2), (dict(H=0), 1), (dict(S=-1), 1),
    (dict(NB=0), 1), (dict(MB=0), 1), (dict(window=-1), 1), (dict(scale=float("nan")), 1),
    (dict(io=0, cache=1), 1), (dict(io=3, cache=3), 1), (dict(io=1, cache=3, H=4), 2),
    (dict(io=1, cache=3, H=8), 1),             # int8 without scales
    (dict(q=24), 1),                           # misaligned
    (dict(NB=1 << 28, bs=16), 1),              # slot index overflows int32
])
def test_decode_host_validation(L, kw, status):
    assert _decode(L, **kw) == status
    assert L.pa_last_error().decode()


def test_decode_with_no_sequences_is_a_no_op(L):
    assert _decode(L, S=0, q=None, out=None) == 0


def test_cache_ops_host_validation(L):
    P = ctypes.c_void_p
    # negative token count
    assert L.reshape_and_cache(P(16), P(16), P(16), P(16), P(16), -1, 4, 64, 16, 4, 256, 256, 1,
                               None, None, None, None, None) == 1
    # int8 without scale pointers
    assert L.reshape_and_cache(P(16), P(16), P(16), P(16), P(16), 1, 4, 64, 16, 4, 256, 256, 3,
                               None, None, None, None, None) == 1
    # stride shorter than a row
    assert L.reshape_and_cache(P(16), P(16), P(16), P(16), P(16), 1, 4, 64, 16, 4, 128, 256, 1,
                               None, None, None, None, None) == 1
    # zero tokens: nothing to do
    assert L.reshape_and_cache(P(16), P(16), P(16), P(16), P(16), 0, 4, 64, 16, 4, 256, 256, 1,
                               None, None, None, None, None) == 0
    # one scale pool only
    assert L.copy_blocks(P(16), P(16), P(16), 1, 4, 4096, P(16), None, 64, None) == 1
    assert L.copy_blocks(P(16), P(16), P(16), 0, 4, 4096, None, None, 0, None) == 0
    assert L.copy_blocks(None, P(16), P(16), 1, 4, 4096, None, None, 0, None) == 1


def test_workspace_query_rejects_bad_sizes(L):
    assert L.pa_decode_workspace_bytes(1, 4, 96) == 0
    assert L.pa_decode_workspace_bytes(-1, 4, 64) == 0


def test_gqa_host_validation(L):
    P = lambda x: None if x is None else ctypes.c_void_p(x)
    def call(hq, hkv, io=1, cache=1):
        return L.paged_attention_decode_gqa(P(16), P(16), P(16), P(16), None, None, P(16), P(16), 1, hq, hkv, 128,
                                            16, 4, 2, 0.1, 0, io, cache, P(16), 1 << 20, None)
    assert call(6, 4) == 1              # query heads not a multiple of cached heads
    assert call(8, 0) == 1
    assert call(64, 8, 3, 3) == 1       # int8 queries are not a thing


def test_prefill_host_validation(L):
    P = ctypes.c_void_p
    def call(T=40, mq=40, hq=8, hkv=2, D=128, bs=16, dt=1, ptr=16):
        p = P(ptr) if ptr else None
        return L.paged_attention_prefill(p, p, p, p, p, p, p, 1, T, mq, hq, hkv, D, bs, 64, 8, 0.1, 0, dt, None)
    assert call(hq=6, hkv=4) == 1       # query heads not a multiple of cached heads
    assert call(hq=12, hkv=4) == 2      # 3 query heads per cached head: unsupported
    assert call(hq=48, hkv=2) == 2      # 24 per cached head: not a power of two
    assert call(hq=512, hkv=2) == 2     # 256 per cached head: more than a unit's 128 rows
    assert call(D=96) == 2              # head_dim 128 or 64 only
    assert call(D=64, ptr=0) == 1       # head_dim 64 gets past the shape checks
    assert call(bs=12) == 2             # block size must divide 128 in steps of 8
    assert call(dt=0) == 2              # fp32 I/O is not a tensor-core type here
    assert call(T=-1) == 1
    assert call(ptr=0) == 1             # NULL pointers
    assert call(ptr=24) == 1            # not 16-byte aligned
    assert call(T=0) == 0               # nothing to do
    assert call(mq=0) == 0
    assert call(T=1 << 28) == 2         # T * Hq = 2^31: output row indices would overflow
    assert L.pa_last_error().decode()


def test_prefill_quant_host_validation(L):
    P = ctypes.c_void_p
    def call(cache=3, ks=16, vs=16, io=1, D=128):
        p = P(16)
        k = P(ks) if ks else None
        v = P(vs) if vs else None
        return L.paged_attention_prefill_quant(p, p, p, p, k, v, p, p, p, 1, 40, 40, 8, 2, D, 16, 64, 8, 0.1, 0,
                                               io, cache, None)
    assert call(cache=1) == 1           # a 16-bit cache belongs to paged_attention_prefill
    assert call(ks=0) == 1              # an 8-bit cache needs both scale pools
    assert call(vs=17) == 1             # fp16 scales must be 2-byte aligned
    assert call(io=0) == 2              # fp32 I/O is not a tensor-core type here
    assert call(D=64) == 2              # 8-bit codes: head_dim 128 only
    assert L.pa_last_error().decode()


def test_swap_host_validation(L):
    P = ctypes.c_void_p
    def call(n=1, nsrc=4, ndst=4, bb=4096, scales=(None, None, None, None), sb=0, pairs=16):
        return L.swap_blocks(P(16), P(16), P(16), P(16), P(pairs) if pairs else None, n, nsrc, ndst, bb,
                             *[P(x) if x else None for x in scales], sb, None)
    assert call(n=-1) == 1
    assert call(nsrc=0) == 1
    assert call(bb=0) == 1
    assert call(scales=(16, 16, 16, None), sb=64) == 1   # all four scale pools or none
    assert call(scales=(16, 16, 16, 16), sb=0) == 1
    assert call(pairs=0) == 1                            # NULL pair array
    assert call(pairs=20) == 1                           # pairs not 8-byte aligned
    assert call(n=70000) == 2                            # more pairs than one launch takes
    assert call(n=0) == 0                                # nothing to do



def test_prefill_binding_refuses_before_any_launch():
    """The Python binding only marshals: tensors that are not dense CUDA tensors of the right
    shapes and dtypes are refused on the host (there is no CPU path to fall back to)."""
    import torch
    import paged_kv_cache_384_b200 as pa
    T, Hq, Hkv, D, S, NB, bs = 8, 4, 2, 128, 2, 4, 16
    q = torch.zeros(T, Hq, D, dtype=torch.float16)
    kc = torch.zeros(NB, bs, Hkv, D, dtype=torch.float16)
    bt = torch.zeros(S, 2, dtype=torch.int32)
    cu = torch.tensor([0, 4, 8], dtype=torch.int32)
    cl = torch.tensor([4, 4], dtype=torch.int32)
    with pytest.raises(ValueError, match="CUDA tensor"):
        pa.paged_attention_prefill(torch.empty_like(q), q, kc, kc.clone(), bt, cu, cl, 4, 0.1)
    with pytest.raises(ValueError, match="one dtype"):
        pa.paged_attention_prefill(torch.empty_like(q, dtype=torch.bfloat16), q, kc, kc.clone(), bt, cu, cl, 4, 0.1)
    with pytest.raises(ValueError, match="q's dtype"):
        pa.paged_attention_prefill(torch.empty_like(q), q, kc.to(torch.bfloat16), kc.to(torch.bfloat16), bt, cu, cl,
                                   4, 0.1)
    with pytest.raises(ValueError, match="int32"):
        pa.paged_attention_prefill(torch.empty_like(q), q, kc, kc.clone(), bt, cu.long(), cl, 4, 0.1)


def test_prefill_flop_count():
    """4 * head_dim FLOPs per (query row, attended token): a whole prompt of n tokens attends
    n(n+1)/2 tokens per head; a chunk behind cached context attends the suffix of that sum;
    a window caps every row; and the count equals a brute-force walk of the causal mask."""
    D, H = 128, 3
    assert accounting.prefill_flops([5], [5], H, D) == 4 * D * H * 15
    assert accounting.prefill_flops([8], [3], H, D) == 4 * D * H * (6 + 7 + 8)
    assert accounting.prefill_flops([8], [3], H, D, window=4) == 4 * D * H * 12
    ctx, ql, window = [9, 4, 17], [4, 4, 1], 6
    brute = 0
    for c, q in zip(ctx, ql):
        for i in range(q):
            pos = c - q + i
            brute += sum(1 for tok in range(c) if tok <= pos and pos - tok < window)
    assert accounting.prefill_flops(ctx, ql, H, D, window) == 4 * D * H * brute
