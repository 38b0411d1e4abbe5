"""Pins for the oracle's block-manager model (CPU only).

The pages fix block counts and byte totals for a concrete model ("A concrete
memory example", tests/golden/memory_example.json), the 50-token / 4-block case
and the 12, 87, 301, 44 placement ("How PagedAttention works"), that finished
requests return their blocks at once, that tail waste stays under one block and
that a diverging sharer gets a private copy.  Random operation sequences check
the bookkeeping invariants; planted mistakes (subclasses with one step changed)
must each fail at least one pin.
"""
import json
import os

import numpy as np
import pytest

from oracle.block_manager import BlockManagerModel, DoubleFree, InvalidArgument, OutOfBlocks

MIB = 1 << 20
GIB = 1 << 30


def golden(golden_dir):
    return json.load(open(os.path.join(golden_dir, "memory_example.json")))


def kv_bytes_per_token(m):
    # keys and values, every layer, every KV head, head_dim elements
    return 2 * m["num_layers"] * m["num_kv_heads"] * m["head_dim"] * m["elem_bytes"]


def add_with_tokens(bm, n):
    s = bm.seq_add()
    bm.reserve_slots([s], [n])
    return s


# ------------------------------------------------------------------ page figures
def check_request_table(cls, g):
    B = g["block_size"]
    bm = cls(4096, B, order=np.random.default_rng(0).permutation(4096))
    per_tok = kv_bytes_per_token(g["model"])
    total_blocks = 0
    seqs = {}
    for name, r in g["requests"].items():
        s = add_with_tokens(bm, r["live_tokens"])
        seqs[name] = s
        nblk = len(bm.table(s))
        if nblk != r["blocks"] or nblk * B * per_tok != r["allocated_mib"] * MIB:
            return False
        total_blocks += nblk
    if total_blocks != g["total"]["blocks"] or bm.num_free() != 4096 - total_blocks:
        return False
    if total_blocks * B * per_tok != g["total"]["allocated_mib"] * MIB:
        return False
    used = set()
    for s in seqs.values():
        used.update(bm.table(s))
    return len(used) == total_blocks


def test_memory_example_figures(golden_dir):
    g = golden(golden_dir)
    per_tok = kv_bytes_per_token(g["model"])
    assert per_tok == g["kv_bytes_per_token"] == 128 * 1024
    live = sum(r["live_tokens"] for r in g["requests"].values())
    assert live == g["total"]["live_tokens"]
    assert live * per_tok == g["live_mib"] * MIB
    assert g["total"]["allocated_mib"] * MIB - live * per_tok == g["tail_mib"] * MIB
    assert g["contiguous_reservation_tokens"] * per_tok == g["contiguous_mib_per_request"] * MIB
    assert 4 * g["contiguous_reservation_tokens"] * per_tok == g["contiguous_gib_for_four"] * GIB


def test_request_table_block_counts(golden_dir):
    assert check_request_table(BlockManagerModel, golden(golden_dir))


def check_fifty_tokens(cls, g):
    f = g["fifty_tokens"]
    phys = f["physical_blocks"]
    rest = [b for b in range(400) if b not in phys]
    bm = cls(400, g["block_size"], order=phys + rest)
    s = bm.seq_add()
    slots, cow = bm.reserve_slots([s], [f["tokens"]])
    if cow or bm.table(s) != phys or bm.length(s) != f["tokens"]:
        return False
    # positions 0..49 in order: block 12 rows 0..15, block 87 rows 0..15, block 301 rows
    # 0..15, then block 44 rows 0..1 (three full blocks and one holding two tokens)
    expect = (list(range(12 * 16, 13 * 16)) + list(range(87 * 16, 88 * 16))
              + list(range(301 * 16, 302 * 16)) + [44 * 16, 44 * 16 + 1])
    return (slots == expect and f["full_blocks"] == 3
            and f["tokens"] - f["full_blocks"] * 16 == f["tokens_in_last"])


def test_fifty_tokens_in_blocks_12_87_301_44(golden_dir):
    assert check_fifty_tokens(BlockManagerModel, golden(golden_dir))


def check_finished_blocks_return(cls, g):
    B = g["block_size"]
    bm = cls(1024, B)
    seqs = {n: add_with_tokens(bm, r["live_tokens"]) for n, r in g["requests"].items()}
    b_blocks = bm.table(seqs["B"])
    free_before = bm.num_free()
    bm.seq_free(seqs["B"])
    if bm.num_free() != free_before + g["requests"]["B"]["blocks"]:
        return False
    # a new request of the same size reuses exactly those blocks (most recent first)
    e = add_with_tokens(bm, g["requests"]["B"]["live_tokens"])
    return bm.table(e) == b_blocks[::-1] and bm.num_free() == free_before


def test_finished_request_returns_blocks(golden_dir):
    assert check_finished_blocks_return(BlockManagerModel, golden(golden_dir))


def check_tail_waste(cls):
    rng = np.random.default_rng(1)
    for B in (1, 7, 16, 32):
        bm = cls(20000, B)
        for L in list(rng.integers(1, 600, size=30)) + [1, B, B + 1, 2 * B - 1, 2 * B]:
            s = add_with_tokens(bm, int(L))
            n = len(bm.table(s))
            if not (0 <= n * B - L < B and (n - 1) * B < L <= n * B):
                return False
            bm.seq_free(s)
        if bm.num_free() != 20000:
            return False
    return True


def test_tail_waste_under_one_block():
    assert check_tail_waste(BlockManagerModel)


# ------------------------------------------------------------------ copy-on-write
def check_cow_partial_tail(cls):
    bm = cls(64, 16)
    p = add_with_tokens(bm, 20)                  # tail block holds 4 tokens
    tail = bm.table(p)[-1]
    c = bm.seq_fork(p)
    if bm.refcount[tail] != 2 or bm.table(c) != bm.table(p):
        return False
    slots, cow = bm.reserve_slots([c], [1])
    new = bm.table(c)[-1]
    return (len(cow) == 1 and cow[0] == (tail, new) and new != tail
            and bm.table(p)[-1] == tail and bm.refcount[tail] == 1 and bm.refcount[new] == 1
            and slots == [new * 16 + 4] and bm.length(c) == 21 and bm.length(p) == 20
            and bm.table(c)[0] == bm.table(p)[0] and bm.refcount[bm.table(p)[0]] == 2)


def test_cow_on_partial_shared_tail():
    assert check_cow_partial_tail(BlockManagerModel)


def check_cow_full_tail(cls):
    bm = cls(64, 16)
    p = add_with_tokens(bm, 32)                  # two full blocks: next token opens a block
    c = bm.seq_fork(p)
    slots, cow = bm.reserve_slots([c], [1])
    return (cow == [] and len(bm.table(c)) == 3 and bm.table(c)[:2] == bm.table(p)
            and slots == [bm.table(c)[2] * 16])


def test_full_shared_tail_needs_no_copy():
    assert check_cow_full_tail(BlockManagerModel)


def check_prefix_2040(cls):
    """64 sequences share a 2040-token prefix whose last block is partial (8 of 16)."""
    bm = cls(1024, 16)
    root = add_with_tokens(bm, 2040)
    seqs = [root] + [bm.seq_fork(root) for _ in range(63)]
    shared_tail = bm.table(root)[-1]
    if bm.refcount[shared_tail] != 64 or any(bm.refcount[b] != 64 for b in bm.table(root)):
        return False
    slots, cow = bm.reserve_slots(seqs, [1] * 64)
    # the first 63 writers copy; the last one finds the block private and writes in place
    if len(cow) != 63 or any(src != shared_tail for src, _ in cow):
        return False
    if bm.table(seqs[-1])[-1] != shared_tail or bm.refcount[shared_tail] != 1:
        return False
    dsts = [d for _, d in cow]
    return (len(set(dsts)) == 63 and all(bm.table(s)[-1] == d for s, d in zip(seqs, dsts))
            and slots[:63] == [d * 16 + 8 for d in dsts] and slots[63] == shared_tail * 16 + 8)


def test_prefix_with_partial_last_block_copies_on_write():
    assert check_prefix_2040(BlockManagerModel)


def test_parent_and_child_in_one_batch():
    bm = BlockManagerModel(64, 16)
    p = add_with_tokens(bm, 5)
    c = bm.seq_fork(p)
    tail = bm.table(p)[0]
    slots, cow = bm.reserve_slots([p, c], [1, 1])
    assert len(cow) == 1 and cow[0][0] == tail          # parent wrote first and copied
    assert bm.table(c)[0] == tail and bm.refcount[tail] == 1
    assert slots == [cow[0][1] * 16 + 5, tail * 16 + 5]


# ------------------------------------------------------------------ errors
def check_errors(cls):
    bm = cls(8, 16)
    s = add_with_tokens(bm, 100)                 # 7 blocks
    snapshot = (list(bm.free_stack), list(bm.refcount), bm.table(s), bm.length(s))
    t = bm.seq_add()
    try:
        bm.reserve_slots([s, t], [13, 20])       # s fits in its tail... t needs 2 blocks: 1 free
        return False
    except OutOfBlocks:
        pass
    if (list(bm.free_stack), list(bm.refcount), bm.table(s), bm.length(s)) != snapshot \
            or bm.length(t) != 0:
        return False
    b = bm.alloc()
    bm.free(b)
    try:
        bm.free(b)
        return False
    except DoubleFree:
        pass
    return bm.num_free() == 1


def test_out_of_blocks_and_double_free():
    assert check_errors(BlockManagerModel)


def test_invalid_arguments():
    bm = BlockManagerModel(8, 16)
    s = bm.seq_add()
    with pytest.raises(InvalidArgument):
        bm.reserve_slots([s, s], [1, 1])
    with pytest.raises(InvalidArgument):
        bm.reserve_slots([99], [1])
    with pytest.raises(InvalidArgument):
        bm.free(8)
    with pytest.raises(InvalidArgument):
        BlockManagerModel(4, 16, order=[0, 1, 1, 2])


# ------------------------------------------------------------------ invariants
def check_invariants(bm):
    NB = bm.num_blocks
    free = bm.free_stack
    if len(set(free)) != len(free):
        return False
    in_free = set(free)
    for b in range(NB):
        if (bm.refcount[b] == 0) != (b in in_free):
            return False
    refs = sum(bm.refcount)
    entries = sum(len(t) for t in bm.tables.values())
    if refs != entries:
        return False
    for s, t in bm.tables.items():
        L = bm.lengths[s]
        if len(t) != -(-L // bm.block_size) or any(bm.refcount[b] < 1 for b in t):
            return False
    return len(free) + sum(1 for r in bm.refcount if r > 0) == NB


def check_random_ops(cls, seed=0, n_ops=400):
    rng = np.random.default_rng(seed)
    bm = cls(200, 8, order=rng.permutation(200))
    live = []
    for _ in range(n_ops):
        op = rng.integers(0, 4)
        try:
            if op == 0 or not live:
                live.append(bm.seq_add())
            elif op == 1:
                k = int(rng.integers(1, min(len(live), 5) + 1))
                sel = list(rng.choice(live, size=k, replace=False))
                bm.reserve_slots(sel, list(rng.integers(0, 30, size=k)))
            elif op == 2:
                live.append(bm.seq_fork(int(rng.choice(live))))
            else:
                s = int(rng.choice(live))
                live.remove(s)
                bm.seq_free(s)
        except OutOfBlocks:
            pass
        if not check_invariants(bm):
            return False
    return True


@pytest.mark.parametrize("seed", range(5))
def test_invariants_under_random_operations(seed):
    assert check_random_ops(BlockManagerModel, seed)


# ------------------------------------------------------------------ planted mistakes
def battery(cls, g):
    checks = [lambda: check_request_table(cls, g), lambda: check_fifty_tokens(cls, g),
              lambda: check_finished_blocks_return(cls, g), lambda: check_tail_waste(cls),
              lambda: check_cow_partial_tail(cls), lambda: check_cow_full_tail(cls),
              lambda: check_prefix_2040(cls), lambda: check_errors(cls),
              lambda: all(check_random_ops(cls, s, 200) for s in range(3))]
    for c in checks:
        try:
            if not c():
                return False
        except Exception:
            return False
    return True


class FifoFree(BlockManagerModel):          # reuse the oldest freed block instead of the newest
    def free(self, b):
        self._check_block(b)
        if self.refcount[b] == 0:
            raise DoubleFree(b)
        self.refcount[b] -= 1
        if self.refcount[b] == 0:
            self.free_stack.insert(0, b)


class NoCopyOnWrite(BlockManagerModel):     # writes into a shared tail
    def _append_one(self, sid, cow_pairs):
        B = self.block_size
        L = self.lengths[sid]
        if L % B == 0:
            self.tables[sid].append(self.alloc())
        self.lengths[sid] = L + 1
        return self.tables[sid][L // B] * B + L % B


class CowWithoutDecref(BlockManagerModel):  # leaks a reference on every copy
    def _append_one(self, sid, cow_pairs):
        B = self.block_size
        L = self.lengths[sid]
        t = self.tables[sid]
        if L % B == 0:
            t.append(self.alloc())
        elif self.refcount[t[-1]] > 1:
            new = self.alloc()
            cow_pairs.append((t[-1], new))
            t[-1] = new
        self.lengths[sid] = L + 1
        return t[L // B] * B + L % B


class OffByOneBoundary(BlockManagerModel):  # opens a block one token late
    def _append_one(self, sid, cow_pairs):
        B = self.block_size
        L = self.lengths[sid]
        t = self.tables[sid]
        if L % B == 1 or not t:
            t.append(self.alloc())
        self.lengths[sid] = L + 1
        return t[L // B] * B + L % B


class ForkWithoutIncref(BlockManagerModel):
    def seq_fork(self, parent):
        child = self.seq_add()
        self.tables[child] = list(self.tables[parent])
        self.lengths[child] = self.lengths[parent]
        return child


class NoRollback(BlockManagerModel):        # partial appends survive a failed call
    def reserve_slots(self, seq_ids, ntok):
        slots, cow = [], []
        for s, n in zip(seq_ids, ntok):
            for _ in range(int(n)):
                slots.append(self._append_one(int(s), cow))
        return slots, cow


class FreeNeverPushes(BlockManagerModel):
    def free(self, b):
        self._check_block(b)
        if self.refcount[b] == 0:
            raise DoubleFree(b)
        self.refcount[b] -= 1


MUTANTS = [FifoFree, NoCopyOnWrite, CowWithoutDecref, OffByOneBoundary, ForkWithoutIncref,
           NoRollback, FreeNeverPushes]


def test_battery_accepts_model(golden_dir):
    assert battery(BlockManagerModel, golden(golden_dir))


@pytest.mark.parametrize("mutant", MUTANTS, ids=lambda c: c.__name__)
def test_battery_rejects_planted_mistake(mutant, golden_dir):
    assert not battery(mutant, golden(golden_dir))
