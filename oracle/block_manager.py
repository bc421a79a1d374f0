"""Oracle model of the block table and the physical-block allocator.

TEST INFRASTRUCTURE ONLY (tests, smoke check, CPU-baseline leg of the benchmark).

Follows "vLLM source first look: PagedAttention memory design" (trdm.cn), section 二
(BlockTable and BlockManager), and the three-level mapping of "KV Cache memory
optimisation and PagedAttention" (yunthe.com), section "PagedAttention分页内存管理原理"
(logical block table, physical block table = per-block allocation state, allocator).

The page's Python lost its comparison operators and decorators in extraction.  The
readings taken here:
  * get_physical_block raises IndexError when ``token // block_size >= len(block_ids)``;
  * allocate raises RuntimeError when fewer than ``n`` blocks are free, and pops from
    the END of the free list (last freed, first reused);
  * free decrements each reference count, returns a block to the END of the free list
    when its count reaches 0, and raises RuntimeError on a count that would go
    negative (double free).  Refinement: the whole request is validated first, so a
    failed free changes nothing;
  * copy_on_write returns the same id when the count is <= 1; otherwise it allocates a
    new block (count 1), decrements the old one and returns the new id -- the caller
    then copies the block's KV data (copy_blocks);
  * share (fork) adds one reference to each given block: the pages say requests share
    the physical blocks of a common prompt under reference counting ("KV Cache memory
    optimisation and PagedAttention", section "vLLM调度器与PagedAttention协同工作",
    shared prefixes) but print no method for it;
  * usage_ratio = 1 - free / num_blocks.
"""
from collections import Counter


class BlockTable:
    """Per-sequence logical -> physical block list (section 二, BlockTable)."""

    def __init__(self, block_ids=None, num_tokens=0):
        self.block_ids = list(block_ids or [])
        self.num_tokens = num_tokens

    @property
    def num_blocks(self):
        return len(self.block_ids)

    def append_block(self, physical_block_id):
        self.block_ids.append(physical_block_id)

    def get_physical_block(self, token_idx, block_size):
        block_idx = token_idx // block_size
        if block_idx >= len(self.block_ids):
            raise IndexError(f"token {token_idx}: logical block {block_idx} not allocated")
        return self.block_ids[block_idx]

    def get_offset(self, token_idx, block_size):
        return token_idx % block_size


class BlockManager:
    """Free list + reference counts (section 二, BlockManager)."""

    def __init__(self, num_blocks, block_size, free_order=None):
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.free_blocks = list(range(num_blocks)) if free_order is None else list(free_order)
        if sorted(self.free_blocks) != list(range(num_blocks)):
            raise ValueError("free_order must be a permutation of range(num_blocks)")
        self.ref_count = [0] * num_blocks

    def allocate(self, num_blocks=1):
        if len(self.free_blocks) < num_blocks:
            raise RuntimeError(f"out of blocks: need {num_blocks}, {len(self.free_blocks)} free")
        allocated = []
        for _ in range(num_blocks):
            block_id = self.free_blocks.pop()
            self.ref_count[block_id] = 1
            allocated.append(block_id)
        return allocated

    def free(self, block_ids):
        need = Counter(block_ids)
        for block_id, n in need.items():
            if not 0 <= block_id < self.num_blocks or self.ref_count[block_id] < n:
                raise RuntimeError(f"block {block_id}: reference count would go negative")
        for block_id in block_ids:
            self.ref_count[block_id] -= 1
            if self.ref_count[block_id] == 0:
                self.free_blocks.append(block_id)

    def share(self, block_ids):
        for block_id in block_ids:
            if not 0 <= block_id < self.num_blocks or self.ref_count[block_id] <= 0:
                raise RuntimeError(f"block {block_id} is not allocated")
        for block_id in block_ids:
            self.ref_count[block_id] += 1

    def copy_on_write(self, block_id):
        if self.ref_count[block_id] <= 1:
            return block_id
        new_block_id = self.allocate(1)[0]
        self.ref_count[block_id] -= 1
        return new_block_id

    def usage_ratio(self):
        return 1.0 - len(self.free_blocks) / self.num_blocks
