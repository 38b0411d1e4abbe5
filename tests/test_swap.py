"""Preemption with swap: bookkeeping (CPU, library vs oracle model, bit-exact) and the
device round trip (GPU, host buffer and restored blocks vs the oracle's cache model)."""
import math

import numpy as np
import pytest
import torch

import paged_kv_cache_403_b200 as pa
from oracle.block_manager import BlockManagerModel, InvalidArgument, OutOfBlocks

B = 16


def test_swap_bookkeeping_matches_model_under_random_operations():
    rng = np.random.default_rng(5)
    nb = 32
    order = rng.permutation(nb)
    lib = pa.pa_pool_create(1, nb, B, 1, 64, "f16", None, None, order)
    bm = BlockManagerModel(nb, B, order)
    live, swapped = [], []
    outs = {"out": 0, "in": 0, "oom": 0}
    for _ in range(1500):
        op = int(rng.integers(0, 6))
        if op == 0 or not (live or swapped):
            s1, s2 = pa.pa_seq_add(lib), bm.seq_add()
            assert s1 == s2
            live.append(s1)
        elif op == 1 and live:
            s = int(rng.choice(live))
            n = int(rng.integers(1, 40))
            e1 = e2 = None
            try:
                r1 = pa.pa_reserve_slots(lib, [s], [n])
            except pa.PaError as e:
                e1 = e.status
            try:
                r2 = bm.reserve_slots([s], [n])
            except OutOfBlocks:
                e2 = pa.PA_ERR_OUT_OF_BLOCKS
            assert e1 == e2
            if e1 is None:
                assert [int(x) for x in r1[0]] == r2[0]
        elif op == 2 and live:
            s = int(rng.choice(live))
            pa.pa_swap_out(lib, s)
            assert bm.swap_out(s) is not None
            live.remove(s)
            swapped.append(s)
            outs["out"] += 1
        elif op == 3 and swapped:
            s = int(rng.choice(swapped))
            e1 = e2 = None
            try:
                pa.pa_swap_in(lib, s)
            except pa.PaError as e:
                e1 = e.status
            try:
                bm.swap_in(s)
            except OutOfBlocks:
                e2 = pa.PA_ERR_OUT_OF_BLOCKS
            assert e1 == e2
            if e1 is None:
                swapped.remove(s)
                live.append(s)
                outs["in"] += 1
            else:
                outs["oom"] += 1
        elif op == 4 and (live or swapped):
            s = int(rng.choice(live + swapped))
            pa.pa_seq_free(lib, s)
            bm.seq_free(s)
            (live if s in live else swapped).remove(s)
        assert [int(x) for x in pa.pa_free_list(lib)] == bm.free_stack
        for s in live + swapped:
            ln, t = pa.pa_seq_info(lib, s)
            assert ln == bm.length(s) and [int(x) for x in t] == bm.table(s)
    assert outs["out"] > 10 and outs["in"] > 10 and outs["oom"] > 0
    pa.pa_pool_destroy(lib)


def test_swapped_sequence_refuses_appends_and_tables():
    p = pa.pa_pool_create(1, 8, B, 1, 64, "f16")
    s = pa.pa_seq_add(p)
    pa.pa_reserve_slots(p, [s], [40])
    pa.pa_swap_out(p, s)
    assert pa.pa_num_free_blocks(p) == 8 and pa.pa_seq_info(p, s)[0] == 40
    for call in (lambda: pa.pa_reserve_slots(p, [s], [1]), lambda: pa.pa_seq_fork(p, s),
                 lambda: pa.pa_build_block_tables(p, [s], 4), lambda: pa.pa_swap_out(p, s)):
        with pytest.raises(pa.PaError):
            call()
    pa.pa_swap_in(p, s)
    assert len(pa.pa_seq_info(p, s)[1]) == 3
    pa.pa_pool_destroy(p)


def test_model_swap_rules():
    bm = BlockManagerModel(8, B)
    a = bm.seq_add()
    bm.reserve_slots([a], [40])
    blocks = bm.table(a)
    assert bm.swap_out(a) == blocks and bm.num_free() == 8 and bm.length(a) == 40
    with pytest.raises(InvalidArgument):
        bm.reserve_slots([a], [1])
    b = bm.seq_add()
    bm.reserve_slots([b], [16 * 6])
    with pytest.raises(OutOfBlocks):
        bm.swap_in(a)                               # needs 3, 2 free: nothing changes
    assert bm.num_free() == 2 and bm.table(a) == []
    bm.seq_free(b)
    assert len(bm.swap_in(a)) == 3


@pytest.mark.gpu
@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_swap_round_trip_on_gpu(dtype):
    """Swap a sequence out, let another sequence overwrite its old blocks, swap it back
    in: the host buffer and the restored blocks equal the oracle's copies bit for bit and
    attention over the restored sequence matches the oracle."""
    from oracle.cache_model import append_rows, empty_pools, swap_buffer, swap_restore
    import oracle
    from paged_kv_cache_403_b200.engine import PagedCache
    from synthetic import values as sv

    L, NB, H, D = 2, 48, 2, 128
    order = np.random.default_rng(3).permutation(NB)
    cache = PagedCache(L, NB, B, H, D, dtype, order)
    bm = BlockManagerModel(NB, B, order)
    kref, vref = empty_pools(L, NB, H, B, D, dtype)
    rng = np.random.default_rng(4)

    def write(sid, n):
        slots, _ = cache.reserve([sid], [n])
        oslots, _ = bm.reserve_slots([sid], [n])
        assert [int(x) for x in slots] == oslots
        for layer in range(L):
            k = sv.narrow(rng.standard_normal((n, H, D)).astype(np.float32), dtype)
            v = sv.narrow(rng.standard_normal((n, H, D)).astype(np.float32), dtype)
            t = lambda a: torch.from_numpy(a.view(np.int16) if dtype == "bf16" else a).cuda()  # noqa: E731
            kk, vv = t(k), t(v)
            if dtype == "bf16":
                kk, vv = kk.view(torch.bfloat16), vv.view(torch.bfloat16)
            cache.append(layer, kk, vv, torch.from_numpy(np.ascontiguousarray(slots)).cuda())
            append_rows(kref, vref, layer, oslots, k, v)

    a, b = cache.add(), cache.add()
    assert (a, b) == (bm.seq_add(), bm.seq_add())
    write(a, 150)
    write(b, 40)
    nbytes = pa.pa_swap_bytes(cache.pool, a)
    assert nbytes == 10 * L * 2 * H * B * D * 2
    buf = torch.empty(nbytes, dtype=torch.uint8).pin_memory()
    pa.pa_swap_out(cache.pool, a, buf)
    old = bm.swap_out(a)
    torch.cuda.synchronize()
    expect = swap_buffer(kref, vref, old)
    got = buf.numpy().view(expect.dtype).reshape(expect.shape)
    assert np.array_equal(got, expect)
    write(b, 300)                                  # reuses (overwrites) a's old blocks
    assert set(bm.table(b)) & set(old)
    pa.pa_swap_in(cache.pool, a, buf)
    new = bm.swap_in(a)
    swap_restore(kref, vref, new, expect)
    torch.cuda.synchronize()
    assert [int(x) for x in cache.info(a)[1]] == new
    hk = cache.k_pool.cpu()
    hv = cache.v_pool.cpu()
    if dtype == "bf16":
        hk, hv = hk.view(torch.int16), hv.view(torch.int16)
    assert np.array_equal(hk.numpy().view(kref.dtype), kref) and np.array_equal(hv.numpy().view(vref.dtype), vref)
    # attention over the restored sequence
    tables, lens = cache.tables([a], 12)
    q = sv.narrow(rng.standard_normal((1, 4, D)).astype(np.float32), dtype)
    qt = torch.from_numpy(q.view(np.int16) if dtype == "bf16" else q).cuda()
    if dtype == "bf16":
        qt = qt.view(torch.bfloat16)
    out = torch.empty((1, 4, D), dtype=torch.float32, device="cuda")
    cache.decode(1, qt, out, torch.from_numpy(tables).cuda(), torch.from_numpy(lens).cuda())
    ref = oracle.paged_decode(kref[1], vref[1], dtype, tables, lens, q, 1 / math.sqrt(D))
    assert np.abs(out.cpu().numpy() - ref).max() <= 2e-3
    assert pa.pa_device_error(clear=True) == 0
