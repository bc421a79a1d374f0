"""Block table / block manager: brute-force semantics (CPU only).

The oracle's BlockManager follows "vLLM source first look: PagedAttention memory design"
(trdm.cn), section 二.  It is checked against a naive model that only tracks, for every
block, the multiset of owners (sequences) holding it -- reference count = number of
owners, free list = blocks with no owner.  The native BlockManager of the library is
then checked against the oracle's, operation by operation (identical ids, identical
errors, identical free lists).
"""
import json
import os
import random
from collections import Counter

import pytest

from oracle.block_manager import BlockManager as OracleBM
from oracle.block_manager import BlockTable

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


class NaiveModel:
    def __init__(self, num_blocks):
        self.num_blocks = num_blocks
        self.owners = [Counter() for _ in range(num_blocks)]

    def refs(self, b):
        return sum(self.owners[b].values())


def _random_ops(seed, bm_cls, num_blocks=24, steps=600, check_model=True):
    rng = random.Random(seed)
    order = list(range(num_blocks))
    rng.shuffle(order)
    bm = bm_cls(num_blocks, 16, order)
    model = NaiveModel(num_blocks)
    seqs = {}          # seq id -> list of blocks
    next_id = 0
    log = []
    for _ in range(steps):
        op = rng.choice(["alloc", "alloc", "free", "fork", "cow", "double_free", "exhaust"])
        if op == "alloc":
            n = rng.randint(1, 4)
            try:
                ids = bm.allocate(n)
            except RuntimeError:
                log.append(("alloc-fail", n))
                assert sum(1 for b in range(num_blocks) if model.refs(b) == 0) < n
                continue
            seqs[next_id] = list(ids)
            for b in ids:
                assert model.refs(b) == 0
                model.owners[b][next_id] += 1
            log.append(("alloc", tuple(ids)))
            next_id += 1
        elif op == "free" and seqs:
            sid = rng.choice(sorted(seqs))
            ids = seqs.pop(sid)
            bm.free(ids)
            for b in ids:
                model.owners[b][sid] -= 1
                if model.owners[b][sid] == 0:
                    del model.owners[b][sid]
            log.append(("free", tuple(ids)))
        elif op == "fork" and seqs:
            sid = rng.choice(sorted(seqs))
            ids = list(seqs[sid])
            bm.share(ids)
            seqs[next_id] = ids
            for b in ids:
                model.owners[b][next_id] += 1
            log.append(("fork", tuple(ids)))
            next_id += 1
        elif op == "cow" and seqs:
            sid = rng.choice(sorted(seqs))
            i = rng.randrange(len(seqs[sid]))
            old = seqs[sid][i]
            shared = model.refs(old) > 1
            try:
                new = bm.copy_on_write(old)
            except RuntimeError:
                assert shared and not any(model.refs(b) == 0 for b in range(num_blocks))
                log.append(("cow-fail", old))
                continue
            if not shared:
                assert new == old
            else:
                assert new != old and model.refs(new) == 0
                model.owners[old][sid] -= 1
                if model.owners[old][sid] == 0:
                    del model.owners[old][sid]
                model.owners[new][sid] += 1
                seqs[sid][i] = new
            log.append(("cow", old, new))
        elif op == "double_free":
            free_now = [b for b in range(num_blocks) if model.refs(b) == 0]
            if free_now:
                b = rng.choice(free_now)
                before = (list(bm.free_blocks), [bm_ref(bm, x) for x in range(num_blocks)])
                with pytest.raises(RuntimeError):
                    bm.free([b])
                after = (list(bm.free_blocks), [bm_ref(bm, x) for x in range(num_blocks)])
                assert before == after   # a failed free changes nothing
                log.append(("double-free", b))
        elif op == "exhaust":
            n_free = sum(1 for b in range(num_blocks) if model.refs(b) == 0)
            with pytest.raises(RuntimeError):
                bm.allocate(n_free + 1)
            log.append(("exhaust", n_free))
        if check_model:
            free_list = list(bm.free_blocks)
            assert len(free_list) == len(set(free_list))
            assert sorted(free_list) == [b for b in range(num_blocks) if model.refs(b) == 0]
            for b in range(num_blocks):
                assert bm_ref(bm, b) == model.refs(b)
            assert abs(bm.usage_ratio() - (1 - len(free_list) / num_blocks)) < 1e-15
    return log, list(bm.free_blocks), [bm_ref(bm, b) for b in range(num_blocks)]


def bm_ref(bm, b):
    return bm.ref_count[b] if isinstance(bm.ref_count, list) else bm.ref_count(b)


@pytest.mark.parametrize("seed", range(8))
def test_oracle_block_manager_matches_owner_model(seed):
    _random_ops(seed, OracleBM)


def test_allocate_pops_the_end_of_the_free_list():
    bm = OracleBM(6, 16, [5, 4, 3, 2, 1, 0])
    assert bm.allocate(2) == [0, 1]
    bm.free([0])
    assert bm.allocate(1) == [0]          # last freed, first reused


def test_copy_on_write_of_an_unshared_block_is_the_same_block():
    bm = OracleBM(4, 16)
    (b,) = bm.allocate(1)
    assert bm.copy_on_write(b) == b
    bm.share([b])
    nb = bm.copy_on_write(b)
    assert nb != b and bm.ref_count[b] == 1 and bm.ref_count[nb] == 1


def test_block_table_lookup_on_the_flowchart_tables():
    with open(os.path.join(GOLDEN, "flowchart_block_tables.json")) as f:
        g = json.load(f)
    bs = 16
    for ids in g["block_tables"]:
        t = BlockTable(ids)
        for i in range(len(ids) * bs):
            assert t.get_physical_block(i, bs) == ids[i // bs]
            assert t.get_offset(i, bs) == i % bs
        with pytest.raises(IndexError):
            t.get_physical_block(len(ids) * bs, bs)


def test_native_block_manager_matches_the_oracle_operation_by_operation():
    pa = pytest.importorskip("paged_kv_cache_384_b200")
    for seed in range(6):
        a = _random_ops(seed, OracleBM, check_model=False)
        b = _random_ops(seed, pa.BlockManager, check_model=True)
        assert a == b


def test_native_block_manager_rejects_bad_free_orders():
    pa = pytest.importorskip("paged_kv_cache_384_b200")
    with pytest.raises(ValueError):
        pa.BlockManager(4, 16, [0, 1, 1, 2])
    bm = pa.BlockManager(4, 16)
    with pytest.raises(RuntimeError):
        bm.free([7])
    with pytest.raises(RuntimeError):
        bm.share([0])            # not allocated


def test_slot_mapping_helper_matches_the_oracle_block_table():
    pa = pytest.importorskip("paged_kv_cache_384_b200")
    rng = random.Random(3)
    bs = 16
    tables = [[rng.randrange(100) for _ in range(rng.randint(1, 5))] for _ in range(6)]
    mb = max(len(t) for t in tables)
    packed = [t + [-1] * (mb - len(t)) for t in tables]
    seq, pos, ref = [], [], []
    for s, t in enumerate(tables):
        bt = BlockTable(t)
        for i in range(len(t) * bs):
            seq.append(s)
            pos.append(i)
            ref.append(bt.get_physical_block(i, bs) * bs + bt.get_offset(i, bs))
    got = pa.slot_mapping(packed, seq, pos, bs)
    assert got.tolist() == ref
    with pytest.raises(Exception):
        pa.slot_mapping(packed, [0], [len(tables[0]) * bs], bs)  # -1 entry / outside the table
