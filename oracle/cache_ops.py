"""Oracle definitions of the two cache-maintenance operations (numpy, byte exact).

TEST INFRASTRUCTURE ONLY (tests, smoke check, CPU-baseline leg of the benchmark).

Cache layout [num_blocks, block_size, num_heads, head_dim]: the pseudocode kernel on
"KV Cache memory optimisation and PagedAttention" (yunthe.com), section
"PagedAttention注意力计算流程", addresses a row at (pb*block_size + off)*H*D + h*D, so a
*slot* ``pb*block_size + off`` names one token row of H*D contiguous values.

Arrays may be of any element dtype (raw bit views such as uint16 for bf16 are fine);
everything here is placement and copying, no arithmetic on values.
"""
import numpy as np


def reshape_and_cache(k, v, k_cache, v_cache, slot_mapping, k_scale=None, v_scale=None,
                      k_scale_cache=None, v_scale_cache=None):
    """Write token t's K/V rows ([T, H, D]) into slot ``slot_mapping[t]`` of the caches.

    New tokens are appended to the cache one row per token ("vLLM source first look:
    PagedAttention memory design" (trdm.cn), section 一: the cache grows by one row per
    generated token; the block it lands in was allocated on demand, "KV Cache memory
    optimisation and PagedAttention", section "vLLM调度器与PagedAttention协同工作").
    Reading: a negative slot marks a padding token and is skipped.
    Per-(token, head) scales ([T, H]) go to the scale caches ([NB, bs, H]) the same way.
    Updates the caches in place and returns them.
    """
    bs = k_cache.shape[1]
    for t, slot in enumerate(np.asarray(slot_mapping).tolist()):
        if slot < 0:
            continue
        pb, off = divmod(int(slot), bs)
        k_cache[pb, off] = k[t]
        v_cache[pb, off] = v[t]
        if k_scale_cache is not None:
            k_scale_cache[pb, off] = k_scale[t]
            v_scale_cache[pb, off] = v_scale[t]
    return k_cache, v_cache


def copy_blocks(k_cache, v_cache, pairs, k_scale_cache=None, v_scale_cache=None):
    """Copy whole physical blocks src -> dst, pair by pair, for K, V (and scales).

    "vLLM source first look: PagedAttention memory design" (trdm.cn), section 二,
    BlockManager.copy_on_write: the new block receives a copy of the old block's KV
    data.  Pairs are applied in order (the GPU entry point requires distinct
    destinations that are never also sources, under which order does not matter).
    Updates in place and returns the caches.
    """
    for src, dst in np.asarray(pairs).reshape(-1, 2).tolist():
        k_cache[dst] = k_cache[src].copy()
        v_cache[dst] = v_cache[src].copy()
        if k_scale_cache is not None:
            k_scale_cache[dst] = k_scale_cache[src].copy()
            v_scale_cache[dst] = v_scale_cache[src].copy()
    return k_cache, v_cache


def swap_blocks(src_k, src_v, dst_k, dst_v, pairs, src_scales=None, dst_scales=None):
    """Move whole blocks between two pools: dst[d] = src[s] for each (s, d) pair.

    "KV Cache memory optimisation and PagedAttention" (yunthe.com), section
    "vLLM调度器与PagedAttention协同工作", item 3: when GPU memory runs short a preempted
    request's KV blocks are moved out to CPU memory (swap-out) and brought back later
    (swap-in); section "vLLM部署配置与PagedAttention参数调优" sizes that CPU pool
    (swap_space).  The operation is a block copy between two pools that may differ in
    size; the scale pools ((k, v) tuples, [NB, bs, H]) follow their blocks.
    Pairs apply in order.  Updates the destination pools in place and returns them.
    """
    for s, d in np.asarray(pairs).reshape(-1, 2).tolist():
        dst_k[d] = src_k[s]
        dst_v[d] = src_v[s]
        if src_scales is not None:
            dst_scales[0][d] = src_scales[0][s]
            dst_scales[1][d] = src_scales[1][s]
    return dst_k, dst_v
