"""Prefix caching (CPU): the oracle model pinned to its readings, and the native block
manager matched to it bit for bit under random operations.

Reading (the pages give the idea, not the lookup): full blocks registered under a
caller key; a registered block released to refcount 0 waits in an evictable queue
(least recently released first) instead of the free stack; allocation uses the free
stack first, then evicts; a new sequence shares the registered blocks of its leading
keys up to the first miss.
"""
import numpy as np
import pytest

import paged_kv_cache_403_b200 as pa
from oracle.block_manager import BlockManagerModel, OutOfBlocks

B = 16


def keys_for(prompt_id, n, offset=0):
    # a stand-in for a hash chain: distinct per (prompt, block index)
    return [(prompt_id << 32) | (offset + i) for i in range(n)]


# ------------------------------------------------------------------ model pins
def test_shared_system_prompt_is_reused_not_reallocated():
    bm = BlockManagerModel(1024, B)
    a = bm.seq_add()
    bm.reserve_slots([a], [2048 + 50])
    assert bm.register(a, keys_for(7, 128)) == 128
    free_before = bm.num_free()
    b, hits = bm.seq_add_cached(keys_for(7, 131))          # 3 trailing keys are unknown
    assert hits == 128 and bm.length(b) == 2048
    assert bm.num_free() == free_before                      # nothing allocated
    assert bm.table(b) == bm.table(a)[:128]
    assert all(bm.refcount[x] == 2 for x in bm.table(b))
    slots, cow = bm.reserve_slots([b], [20])                 # private suffix: new blocks, no copies
    assert cow == [] and len(bm.table(b)) == 130
    assert slots[0] == bm.table(b)[128] * B


def test_released_cached_blocks_wait_in_the_queue_and_are_found_again():
    bm = BlockManagerModel(512, B)
    a = bm.seq_add()
    bm.reserve_slots([a], [64 + 5])                          # 4 full blocks + 1 partial
    bm.register(a, keys_for(1, 4))
    full, tail = bm.table(a)[:4], bm.table(a)[4]
    bm.seq_free(a)
    assert list(bm.evictable) == full                        # released in logical order
    assert bm.free_stack[-1] == tail                         # the unregistered tail is simply free
    assert bm.num_free() == 512
    c, hits = bm.seq_add_cached(keys_for(1, 4))
    assert hits == 4 and bm.table(c) == full and not bm.evictable


def test_eviction_takes_the_least_recently_released_block():
    bm = BlockManagerModel(6, B)
    a = bm.seq_add()
    bm.reserve_slots([a], [32])
    bm.register(a, keys_for(1, 2))
    b = bm.seq_add()
    bm.reserve_slots([b], [32])
    bm.register(b, keys_for(2, 2))
    table_a, table_b = bm.table(a), bm.table(b)
    bm.seq_free(b)                                           # released first
    bm.seq_free(a)
    order = list(bm.evictable)
    assert order == table_b + table_a
    c = bm.seq_add()
    bm.reserve_slots([c], [32])                              # 2 free blocks left: no eviction
    assert len(bm.evictable) == 4
    bm.reserve_slots([c], [16])                              # free stack empty: evict the front
    assert len(bm.evictable) == 3 and bm.table(c)[-1] == order[0]
    _, hits = bm.seq_add_cached(keys_for(2, 2))              # prompt 2's first block is gone
    assert hits == 0


def test_registration_rules():
    bm = BlockManagerModel(64, B)
    a = bm.seq_add()
    bm.reserve_slots([a], [40])
    with pytest.raises(Exception):
        bm.register(a, keys_for(1, 3))                       # the third block is partial
    assert bm.register(a, keys_for(1, 2)) == 2
    assert bm.register(a, keys_for(1, 2)) == 0               # already registered
    b = bm.seq_add()
    bm.reserve_slots([b], [16])
    assert bm.register(b, keys_for(1, 1)) == 0               # key taken by another block


def test_out_of_blocks_rolls_back_an_eviction():
    bm = BlockManagerModel(4, B)
    a = bm.seq_add()
    bm.reserve_slots([a], [32])
    bm.register(a, keys_for(1, 2))
    bm.seq_free(a)
    c = bm.seq_add()
    snapshot = (list(bm.free_stack), list(bm.evictable), dict(bm.block_of))
    with pytest.raises(OutOfBlocks):
        bm.reserve_slots([c], [16 * 5])                      # needs 5 blocks, 4 exist
    assert (list(bm.free_stack), list(bm.evictable), dict(bm.block_of)) == snapshot


# ------------------------------------------------------------------ library vs model
class Lib:
    def __init__(self, nb, order):
        self.p = pa.pa_pool_create(1, nb, B, 1, 64, "f16", None, None, order)
        self.nb = nb


def state(lib, bm, live):
    assert [int(x) for x in pa.pa_free_list(lib.p)] == bm.free_stack
    assert [int(x) for x in pa.pa_prefix_evictable(lib.p)] == list(bm.evictable)
    assert pa.pa_num_free_blocks(lib.p) == bm.num_free()
    for s in live:
        ln, t = pa.pa_seq_info(lib.p, s)
        assert ln == bm.length(s) and [int(x) for x in t] == bm.table(s)
    st = pa.pa_pool_stats(lib.p)
    assert st["num_cached"] == len(bm.block_of) and st["num_evictable"] == len(bm.evictable)


@pytest.mark.parametrize("seed,nb", [(0, 160), (1, 160), (2, 32), (3, 32)])
def test_library_matches_model_with_prefix_caching(seed, nb):
    rng = np.random.default_rng(seed)
    order = rng.permutation(nb)
    lib, bm = Lib(nb, order), BlockManagerModel(nb, B, order)
    live, prompts = [], 6
    for _ in range(1200):
        op = int(rng.integers(0, 7))          # 5 and 6 retire: sequences come and go
        if op == 0 or not live:
            s1, s2 = pa.pa_seq_add(lib.p), bm.seq_add()
            assert s1 == s2
            live.append(s1)
        elif op == 1:                                         # append
            k = int(rng.integers(1, min(len(live), 4) + 1))
            sel = [int(x) for x in rng.choice(live, size=k, replace=False)]
            nt = [int(x) for x in rng.integers(0, 40, size=k)]
            e1 = e2 = None
            try:
                r1 = pa.pa_reserve_slots(lib.p, sel, nt)
                r1 = ([int(x) for x in r1[0]], [tuple(int(v) for v in c) for c in r1[1]])
            except pa.PaError as e:
                e1 = e.status
            try:
                r2 = bm.reserve_slots(sel, nt)
            except OutOfBlocks:
                e2 = pa.PA_ERR_OUT_OF_BLOCKS
            assert e1 == e2
            if e1 is None:
                assert r1 == r2
        elif op == 2:                                         # register some full blocks
            s = int(rng.choice(live))
            nfull = bm.length(s) // B
            if nfull:
                n = int(rng.integers(1, nfull + 1))
                keys = keys_for(int(rng.integers(0, prompts)), n)
                assert pa.pa_prefix_register(lib.p, s, keys) == bm.register(s, keys)
        elif op == 3:                                         # admit through the cache
            keys = keys_for(int(rng.integers(0, prompts)), int(rng.integers(1, 12)))
            r1, r2 = pa.pa_seq_add_cached(lib.p, keys), bm.seq_add_cached(keys)
            assert r1 == r2
            live.append(r1[0])
        elif op == 4:
            p = int(rng.choice(live))
            c1, c2 = pa.pa_seq_fork(lib.p, p), bm.seq_fork(p)
            assert c1 == c2
            live.append(c1)
        else:
            s = int(rng.choice(live))
            live.remove(s)
            pa.pa_seq_free(lib.p, s)
            bm.seq_free(s)
        state(lib, bm, live)
    st = pa.pa_pool_stats(lib.p)
    assert st["cache_hits"] > 0
    if nb == 32:
        assert st["cache_evictions"] > 0            # the small pool forces reclaiming cached blocks
    pa.pa_pool_destroy(lib.p)


def test_library_rejects_partial_block_registration():
    p = pa.pa_pool_create(1, 16, B, 1, 64, "f16")
    s = pa.pa_seq_add(p)
    pa.pa_reserve_slots(p, [s], [20])
    with pytest.raises(pa.PaError) as e:
        pa.pa_prefix_register(p, s, keys_for(1, 2))
    assert e.value.status == pa.PA_ERR_INVALID_ARG
    assert pa.pa_prefix_register(p, s, keys_for(1, 1)) == 1
    pa.pa_pool_destroy(p)


# ------------------------------------------------------------------ planted mistakes
def _policy_battery(cls):
    checks = [test_shared_system_prompt_is_reused_not_reallocated,
              test_released_cached_blocks_wait_in_the_queue_and_are_found_again,
              test_eviction_takes_the_least_recently_released_block, test_registration_rules,
              test_out_of_blocks_rolls_back_an_eviction]
    import sys
    mod = sys.modules[__name__]
    real = mod.BlockManagerModel
    try:
        mod.BlockManagerModel = cls
        for c in checks:
            try:
                c()
            except Exception:
                return False
        return True
    finally:
        mod.BlockManagerModel = real


class EvictNewest(BlockManagerModel):          # LIFO eviction instead of least recently released
    def alloc(self):
        if not self.free_stack and self.evictable:
            b, _ = self.evictable.popitem(last=True)
            del self.block_of[self.key_of.pop(b)]
            self.refcount[b] = 1
            return b
        return super().alloc()


class CachedBlocksFreed(BlockManagerModel):    # released cached blocks go back on the free stack
    def free(self, b):
        super().free(b)
        if b in self.evictable:
            del self.evictable[b]
            del self.block_of[self.key_of.pop(b)]
            self.free_stack.append(b)


class EvictBeforeFree(BlockManagerModel):      # reclaims cached blocks while free ones remain
    def alloc(self):
        if self.evictable:
            b, _ = self.evictable.popitem(last=False)
            del self.block_of[self.key_of.pop(b)]
            self.refcount[b] = 1
            return b
        return super().alloc()


class HitSkipsGap(BlockManagerModel):          # keeps walking keys after a miss
    def seq_add_cached(self, keys):
        sid = self.seq_add()
        for k in keys:
            b = self.block_of.get(int(k))
            if b is None:
                continue
            if self.refcount[b] == 0:
                del self.evictable[b]
            self.refcount[b] += 1
            self.tables[sid].append(b)
        self.lengths[sid] = len(self.tables[sid]) * self.block_size
        return sid, len(self.tables[sid])


def test_policy_pins_accept_the_model():
    assert _policy_battery(BlockManagerModel)


@pytest.mark.parametrize("mutant", [EvictNewest, CachedBlocksFreed, EvictBeforeFree, HitSkipsGap],
                         ids=lambda c: c.__name__)
def test_policy_pins_reject_planted_mistake(mutant):
    assert not _policy_battery(mutant)
