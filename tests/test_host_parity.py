"""Native block manager (libpa, C++) vs the oracle's model (Python), bit for bit.

Both run the same schedule of each workload -- prefill, decode reservations,
forks and copy-on-write, retirements and admissions -- and must agree on every
slot, copy pair, block table, length, refcount and on the free stack itself.
Host only: no device memory is touched.
"""
import numpy as np
import pytest

import paged_kv_cache_403_b200 as pa
from oracle.block_manager import BlockManagerModel, DoubleFree, OutOfBlocks
from synthetic import workloads as wl


class Lib:
    def __init__(self, nb, bs, order):
        self.p = pa.pa_pool_create(1, nb, bs, 1, 64, "f16", None, None, order)
        self.nb = nb

    def add(self):
        return pa.pa_seq_add(self.p)

    def fork(self, s):
        return pa.pa_seq_fork(self.p, s)

    def free(self, s):
        pa.pa_seq_free(self.p, s)

    def reserve(self, sids, ntok):
        slots, cow = pa.pa_reserve_slots(self.p, sids, ntok)
        return [int(x) for x in slots], [tuple(int(v) for v in c) for c in cow]

    def table(self, s):
        return [int(b) for b in pa.pa_seq_info(self.p, s)[1]]

    def length(self, s):
        return pa.pa_seq_info(self.p, s)[0]

    def free_list(self):
        return [int(b) for b in pa.pa_free_list(self.p)]

    def refcounts(self):
        return [pa.pa_block_refcount(self.p, b) for b in range(self.nb)]


class Model:
    def __init__(self, nb, bs, order):
        self.m = BlockManagerModel(nb, bs, order)

    def add(self):
        return self.m.seq_add()

    def fork(self, s):
        return self.m.seq_fork(s)

    def free(self, s):
        self.m.seq_free(s)

    def reserve(self, sids, ntok):
        return self.m.reserve_slots(sids, ntok)

    def table(self, s):
        return self.m.table(s)

    def length(self, s):
        return self.m.length(s)

    def free_list(self):
        return list(self.m.free_stack)

    def refcounts(self):
        return list(self.m.refcount)


def both(nb, bs, order):
    return Lib(nb, bs, order), Model(nb, bs, order)


def same_state(a, b, sids):
    assert a.free_list() == b.free_list()
    for s in sids:
        assert a.table(s) == b.table(s)
        assert a.length(s) == b.length(s)


def run_static(recipe):
    sh = recipe["shape"]
    a, b = both(sh.num_blocks, sh.block_size, recipe["order"])
    lens = [int(x) for x in recipe["lens"]]
    sa = [a.add() for _ in lens]
    sb = [b.add() for _ in lens]
    assert sa == sb
    assert a.reserve(sa, lens) == b.reserve(sb, lens)
    assert a.reserve(sa, [1] * len(sa)) == b.reserve(sb, [1] * len(sb))
    same_state(a, b, sa)
    assert a.refcounts() == b.refcounts()
    return a, sa


def test_tiny():
    a, sids = run_static(wl.tiny())
    # 50/17/3/33 tokens + 1 appended: 4 + 2 + 1 + 3 = 10 blocks out of 64
    assert [len(a.table(s)) for s in sids] == [4, 2, 1, 3]
    assert len(a.free_list()) == 54


def test_worked_example():
    a, sids = run_static(wl.worked_example())
    # blocks after the prompts: 244 / 27 / 132 / 5 = 408; one more token each leaves them unchanged
    assert [len(a.table(s)) for s in sids] == [244, 27, 132, 5]
    assert len(a.free_list()) == 4096 - 408


@pytest.mark.parametrize("bs", [16, 32])
def test_large_pool(bs):
    r = wl.large_pool(block_size=bs)
    a, sids = run_static(r)
    expect = [-(-(int(L) + 1) // bs) for L in r["lens"]]
    assert [len(a.table(s)) for s in sids] == expect


def test_continuous_batch_64_steps():
    r = wl.continuous_batch()
    sh, sched = r["shape"], r["schedule"]
    a, b = both(sh.num_blocks, sh.block_size, r["order"])
    n = len(sched.initial)
    sa = [a.add() for _ in range(n)]
    sb = [b.add() for _ in range(n)]
    init = [int(x) for x in sched.initial]
    assert a.reserve(sa, init) == b.reserve(sb, init)
    pending = []
    for t, events in enumerate(sched.events):
        for slot, plen in pending:
            sa[slot], sb[slot] = a.add(), b.add()
            assert sa[slot] == sb[slot]
            assert a.reserve([sa[slot]], [plen]) == b.reserve([sb[slot]], [plen])
        pending = []
        assert a.reserve(sa, [1] * n) == b.reserve(sb, [1] * n)
        if t % 16 == 0:
            same_state(a, b, sa)
        for slot, plen in events:
            a.free(sa[slot])
            b.free(sb[slot])
            pending.append((slot, plen))
    live = [s for i, s in enumerate(sa) if i not in {slot for slot, _ in pending}]
    same_state(a, b, live)
    assert a.refcounts() == b.refcounts()
    assert sum(len(e) for e in sched.events) > 0       # the schedule did retire sequences


def test_prefix_sharing_and_copy_on_write():
    r = wl.prefix_sharing()
    sh = r["shape"]
    a, b = both(sh.num_blocks, sh.block_size, r["order"])
    ra, rb = a.add(), b.add()
    assert a.reserve([ra], [r["prefix"]]) == b.reserve([rb], [r["prefix"]])
    n = len(r["suffix"])
    sa = [ra] + [a.fork(ra) for _ in range(n - 1)]
    sb = [rb] + [b.fork(rb) for _ in range(n - 1)]
    assert all(x == 64 for x in [a.refcounts()[blk] for blk in a.table(ra)])
    suffix = [int(x) for x in r["suffix"]]
    assert a.reserve(sa, suffix) == b.reserve(sb, suffix)
    assert a.reserve(sa, [1] * n) == b.reserve(sb, [1] * n)
    lens = [a.length(s) for s in sa]
    victim = next(i for i, L in enumerate(lens) if L % 16)
    ca, cb = a.fork(sa[victim]), b.fork(sb[victim])
    ra_, rb_ = a.reserve(sa + [ca], [1] * (n + 1)), b.reserve(sb + [cb], [1] * (n + 1))
    assert ra_ == rb_
    assert len(ra_[1]) == 1                             # exactly one copy-on-write pair
    same_state(a, b, sa + [ca])
    assert a.refcounts() == b.refcounts()


def test_random_operations_including_failures():
    rng = np.random.default_rng(123)
    a, b = both(300, 16, rng.permutation(300))
    live = []
    for _ in range(1500):
        op = int(rng.integers(0, 5))
        if op == 0 or not live:
            x, y = a.add(), b.add()
            assert x == y
            live.append(x)
        elif op == 1:
            k = int(rng.integers(1, min(len(live), 6) + 1))
            sel = [int(s) for s in rng.choice(live, size=k, replace=False)]
            ntok = [int(t) for t in rng.integers(0, 40, size=k)]
            ea = eb = None
            try:
                ra = a.reserve(sel, ntok)
            except pa.PaError as e:
                ea = e.status
            try:
                rb = b.reserve(sel, ntok)
            except OutOfBlocks:
                eb = pa.PA_ERR_OUT_OF_BLOCKS
            assert ea == eb
            if ea is None:
                assert ra == rb
        elif op == 2:
            p = int(rng.choice(live))
            x, y = a.fork(p), b.fork(p)
            assert x == y
            live.append(x)
        else:
            s = int(rng.choice(live))
            live.remove(s)
            a.free(s)
            b.free(s)
        same_state(a, b, live)
    assert a.refcounts() == b.refcounts()


def test_out_of_blocks_leaves_state_unchanged():
    a, b = both(8, 16, None)
    s = a.add()
    b.add()
    a.reserve([s], [100])
    b.reserve([s], [100])
    t = a.add()
    b.add()
    before = (a.free_list(), a.refcounts(), a.table(s), a.length(s))
    with pytest.raises(pa.PaError) as e:
        a.reserve([s, t], [13, 20])
    assert e.value.status == pa.PA_ERR_OUT_OF_BLOCKS
    with pytest.raises(OutOfBlocks):
        b.reserve([s, t], [13, 20])
    assert (a.free_list(), a.refcounts(), a.table(s), a.length(s)) == before
    same_state(a, b, [s, t])


def test_double_free_and_injected_allocation_failure():
    p = pa.pa_pool_create(1, 4, 16, 1, 64, "f16")
    blk = pa.pa_alloc_block(p)
    pa.pa_free_block(p, blk)
    with pytest.raises(pa.PaError) as e:
        pa.pa_free_block(p, blk)
    assert e.value.status == pa.PA_ERR_DOUBLE_FREE
    s = pa.pa_seq_add(p)
    pa.pa_reserve_slots(p, [s], [20])                 # 2 blocks
    before = (list(pa.pa_free_list(p)), pa.pa_seq_info(p, s)[0])
    pa.pa_debug_fail_alloc_after(p, 0)
    with pytest.raises(pa.PaError) as e:
        pa.pa_reserve_slots(p, [s], [20])             # needs one more block: injected failure
    assert e.value.status == pa.PA_ERR_OUT_OF_BLOCKS
    assert (list(pa.pa_free_list(p)), pa.pa_seq_info(p, s)[0]) == before
    pa.pa_reserve_slots(p, [s], [20])                 # injection was one-shot
    st = pa.pa_pool_stats(p)
    assert st["num_free"] == 1 and st["num_tokens"] == 40 and st["peak_used"] == 3
    pa.pa_pool_destroy(p)


def test_invalid_arguments_rejected():
    p = pa.pa_pool_create(1, 4, 16, 1, 64, "f16")
    s = pa.pa_seq_add(p)
    for call in (lambda: pa.pa_reserve_slots(p, [s, s], [1, 1]),
                 lambda: pa.pa_reserve_slots(p, [99], [1]),
                 lambda: pa.pa_free_block(p, 4),
                 lambda: pa.pa_incref_block(p, 0),
                 lambda: pa.pa_seq_fork(p, 42),
                 lambda: pa.pa_pool_create(1, 3, 16, 1, 64, "f16", None, None, [0, 1, 1])):
        with pytest.raises(pa.PaError) as e:
            call()
        assert e.value.status == pa.PA_ERR_INVALID_ARG
    pa.pa_reserve_slots(p, [s], [40])
    with pytest.raises(pa.PaError):
        pa.pa_build_block_tables(p, [s], 2)           # 3 blocks do not fit a width of 2
    t, ln = pa.pa_build_block_tables(p, [s], 5)
    assert ln.tolist() == [40] and t[0, 3:].tolist() == [-1, -1]
    pa.pa_pool_destroy(p)


def test_duplicate_ids_rejected_without_change_and_next_call_unaffected():
    p = pa.pa_pool_create(1, 8, 16, 1, 64, "f16")
    a, b = pa.pa_seq_add(p), pa.pa_seq_add(p)
    pa.pa_reserve_slots(p, [a, b], [3, 5])
    free_before = pa.pa_free_list(p).tolist()
    with pytest.raises(pa.PaError) as e:
        pa.pa_reserve_slots(p, [a, b, a], [1, 1, 1])
    assert e.value.status == pa.PA_ERR_INVALID_ARG and "duplicate" in str(e.value)
    assert pa.pa_seq_info(p, a)[0] == 3 and pa.pa_seq_info(p, b)[0] == 5
    assert pa.pa_free_list(p).tolist() == free_before
    slots, _ = pa.pa_reserve_slots(p, [b, a], [1, 1])     # the same ids again, once each
    ta, tb = pa.pa_seq_info(p, a)[1], pa.pa_seq_info(p, b)[1]
    assert slots.tolist() == [int(tb[0]) * 16 + 5, int(ta[0]) * 16 + 3]
    pa.pa_pool_destroy(p)


def test_counts_far_beyond_the_pool_fail_cleanly():
    """Counts near INT32_MAX on many sequences are refused as out of blocks before any
    block is taken (no host memory is sized by them), and the pool is unchanged."""
    p = pa.pa_pool_create(1, 64, 16, 1, 64, "f16")
    seqs = [pa.pa_seq_add(p) for _ in range(8)]
    pa.pa_reserve_slots(p, seqs, [5] * 8)
    before = (pa.pa_free_list(p).tolist(), [pa.pa_seq_info(p, s)[0] for s in seqs], pa.pa_pool_stats(p))
    huge = 2**31 - 1 - 5
    # the refusal comes before any slot is written, so a small output buffer is enough
    slot_out = np.empty(1024, np.int64)
    for ntok in ([huge] * 8, [1] * 7 + [huge], [56 * 16 + 12] + [0] * 7):
        with pytest.raises(pa.PaError) as e:
            pa.pa_reserve_slots(p, seqs, ntok, slot_out=slot_out)
        assert e.value.status == pa.PA_ERR_OUT_OF_BLOCKS and "no change made" in str(e.value)
        assert (pa.pa_free_list(p).tolist(), [pa.pa_seq_info(p, s)[0] for s in seqs],
                pa.pa_pool_stats(p)) == before
    # exactly what is left still fits: 56 free blocks, 11 more tokens fill each tail
    slots, _ = pa.pa_reserve_slots(p, seqs, [56 * 16 + 11] + [11] * 7)
    assert len(slots) == 56 * 16 + 11 * 8 and pa.pa_num_free_blocks(p) == 0
    pa.pa_pool_destroy(p)
