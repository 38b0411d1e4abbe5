"""Pins for the oracle's cache-content model of 16-bit and fp32 pools (CPU only).

``oracle.cache_model.append_rows``, ``swap_buffer`` and ``swap_restore`` decide the
expected pools of every bit-exact comparison of the GPU path, so they are pinned
here against what the pages fix, not against themselves:

* "What problem does PagedAttention solve, and what is continuous batching?",
  section "How PagedAttention works": a 50-token request in blocks of 16 sits in
  physical blocks 12, 87, 301 and 44, in that order -- three full blocks and one
  holding two tokens.  The written rows must be exactly there, and nowhere else.
* "Continuous Batching & Paged Attention", section "Paged attention borrows a trick
  from operating systems": a growing request is given another block when its last
  one fills, so reading a sequence back through its block table (position j in
  table[j // B], row j % B) returns its tokens in order, however they were appended.
* first page, section "What happens when the KV cache is full?": a preempted
  request's cache can be offloaded and brought back; after the round trip, into
  whatever blocks are free then, the sequence reads back unchanged.

Every written element carries its own identity (kind, layer, sequence, position,
head, dim) as an integer code, so a misplaced, mislabelled or reordered row names
itself.  Planted mistakes (a swapped divmod, keys written to the value pool, a
padding row written anyway, the wrong layer, reversed heads; a swap record with K
and V or the blocks in the wrong order, or layer-major; a restore in reverse order
or with K and V exchanged) must each fail at least one pin.
"""
import numpy as np
import pytest

from oracle import cache_model as cm
from oracle.block_manager import BlockManagerModel

B = 16
NL, H, D = 2, 2, 8
SENTINEL = 0xFFFF            # never a code: codes are 1 .. 2*NL*4*64*H*D
STORAGE = {"f32": np.float32, "f16": np.float16, "bf16": np.uint16}


def code(kind, layer, seq, pos, head, dim):
    """Identity of one element as a positive integer below 2^15 (kind 0 = K, 1 = V)."""
    return 1 + (((((kind * NL + layer) * 4 + seq) * 64 + pos) * H + head) * D + dim)


def as_storage(codes, dtype):
    """Integer codes as elements of the pool's storage type: fp32 holds them as exact
    values, the 16-bit types as raw bit patterns (a bit copy is all a write does)."""
    codes = np.asarray(codes)
    if dtype == "f32":
        return codes.astype(np.float32)
    return codes.astype(np.uint16).view(STORAGE[dtype])


def as_codes(arr, dtype):
    if dtype == "f32":
        return arr.astype(np.int64)
    return arr.view(np.uint16).astype(np.int64)


def rows_for(kind, layer, seq, positions):
    """[n][H][D] code rows for the given positions of one sequence."""
    p = np.asarray(positions)[:, None, None]
    h = np.arange(H)[None, :, None]
    d = np.arange(D)[None, None, :]
    return code(kind, layer, seq, p, h, d)


def fresh_pools(num_blocks, dtype):
    kp, vp = cm.empty_pools(NL, num_blocks, H, B, D, dtype)
    fill = np.float32(-1.0) if dtype == "f32" else np.uint16(SENTINEL).view(STORAGE[dtype])
    kp[...] = fill
    vp[...] = fill
    return kp, vp


def untouched(pool, dtype, mask):
    """Every element outside ``mask`` (bool [NL][NB][B], per (layer, block, row)) still
    holds the fill value."""
    c = as_codes(pool, dtype)
    fill = -1 if dtype == "f32" else SENTINEL
    rest = ~np.broadcast_to(mask[:, :, None, :, None], pool.shape)
    return bool(np.all(c[rest] == fill))


# ------------------------------------------------------------------ the pins
def check_fifty_tokens_land_in_12_87_301_44(append_rows, dtype):
    """The page's example, read literally: positions 0-15 are rows 0-15 of block 12,
    16-31 of block 87, 32-47 of block 301, 48-49 rows 0-1 of block 44."""
    rest = [b for b in range(400) if b not in (12, 87, 301, 44)]
    bm = BlockManagerModel(400, B, order=[12, 87, 301, 44] + rest)
    s = bm.seq_add()
    slots, _ = bm.reserve_slots([s], [50])
    kp, vp = fresh_pools(400, dtype)
    layer = 1
    # one padding row (slot -1) rides along and must be written nowhere
    pad = np.full((1, H, D), 7, np.int64)
    k = np.concatenate([rows_for(0, layer, s, range(50)), pad])
    v = np.concatenate([rows_for(1, layer, s, range(50)), pad])
    append_rows(kp, vp, layer, np.array(list(slots) + [-1], np.int64), as_storage(k, dtype), as_storage(v, dtype))
    placement = [(12, r, r) for r in range(16)] + [(87, r, 16 + r) for r in range(16)] + \
                [(301, r, 32 + r) for r in range(16)] + [(44, 0, 48), (44, 1, 49)]
    mask = np.zeros((NL, 400, B), bool)
    for kind, pool in ((0, kp), (1, vp)):
        c = as_codes(pool, dtype)
        for blk, row, pos in placement:
            want = rows_for(kind, layer, s, [pos])[0]
            if not np.array_equal(c[layer, blk, :, row, :], want):
                return False
            mask[layer, blk, row] = True
        if not untouched(pool, dtype, mask):
            return False
    return True


def _grow(bm, kp, vp, append_rows, dtype, seqs, steps, rng):
    """Prefill then decode steps over several sequences, with padding rows (slot -1)
    mixed into the batches; returns the number of tokens of each sequence."""
    lens = {s: 0 for s in seqs}
    for step in range(steps):
        ids = list(seqs)
        ntok = [int(rng.integers(1, 40)) if step == 0 else 1 for _ in ids]
        slots, cow = bm.reserve_slots(ids, ntok)
        assert not cow
        pos = [(s, lens[s] + t) for s, n in zip(ids, ntok) for t in range(n)]
        for s, n in zip(ids, ntok):
            lens[s] += n
        for layer in range(NL):
            k = [rows_for(0, layer, s, [p])[0] for s, p in pos]
            v = [rows_for(1, layer, s, [p])[0] for s, p in pos]
            # a padding row, written nowhere, at a random place in the batch
            at = int(rng.integers(0, len(pos) + 1))
            sl = list(slots[:at]) + [-1] + list(slots[at:])
            k.insert(at, np.full((H, D), 7, np.int64))
            v.insert(at, np.full((H, D), 7, np.int64))
            append_rows(kp, vp, layer, np.array(sl, np.int64), as_storage(np.array(k), dtype),
                        as_storage(np.array(v), dtype))
    return lens


def check_gather_through_table(append_rows, dtype, seed=0):
    """Four sequences grown in interleaved steps over a shuffled pool: reading position j
    of a sequence from row j % B of block table[j // B] gives its K and V rows in order,
    in both layers, and no other (layer, block, row) of either pool was written."""
    rng = np.random.default_rng(seed)
    nb = 64
    bm = BlockManagerModel(nb, B, order=rng.permutation(nb))
    seqs = [bm.seq_add() for _ in range(4)]
    kp, vp = fresh_pools(nb, dtype)
    lens = _grow(bm, kp, vp, append_rows, dtype, seqs, steps=20, rng=rng)
    mask = np.zeros((NL, nb, B), bool)
    for kind, pool in ((0, kp), (1, vp)):
        c = as_codes(pool, dtype)
        for s in seqs:
            table = bm.table(s)
            if len(table) != -(-lens[s] // B):
                return False
            for layer in range(NL):
                got = np.stack([c[layer, table[j // B], :, j % B, :] for j in range(lens[s])])
                if not np.array_equal(got, rows_for(kind, layer, s, range(lens[s]))):
                    return False
                for j in range(lens[s]):
                    mask[layer, table[j // B], j % B] = True
        if not untouched(pool, dtype, mask):
            return False
    return True


def check_swap_record(append_rows, swap_buffer, dtype):
    """The host record of a swapped-out sequence holds, for its i-th block in logical
    order and each layer, the keys then the values of positions i*B .. i*B+B-1 (the
    record layout [block][layer][K, V][head][row][dim], a reading: block-major so one
    block restores into any free block)."""
    rng = np.random.default_rng(3)
    nb = 32
    bm = BlockManagerModel(nb, B, order=rng.permutation(nb))
    s = bm.seq_add()
    kp, vp = fresh_pools(nb, dtype)
    n = 50
    slots, _ = bm.reserve_slots([s], [n])
    for layer in range(NL):
        append_rows(kp, vp, layer, slots, as_storage(rows_for(0, layer, s, range(n)), dtype),
                    as_storage(rows_for(1, layer, s, range(n)), dtype))
    blocks = bm.swap_out(s)
    buf = np.asarray(swap_buffer(kp, vp, blocks))
    if buf.shape != (len(blocks), NL, 2, H, B, D):
        return False
    c = as_codes(buf, dtype)
    fill = -1 if dtype == "f32" else SENTINEL
    for i in range(len(blocks)):
        for layer in range(NL):
            for kind in (0, 1):
                for r in range(B):
                    pos = i * B + r
                    got = c[i, layer, kind, :, r, :]
                    want = rows_for(kind, layer, s, [pos])[0] if pos < n else np.full((H, D), fill)
                    if not np.array_equal(got, want):
                        return False
    return True


def check_swap_round_trip(append_rows, swap_buffer, swap_restore, dtype):
    """Swap a 50-token sequence out, let another sequence take and overwrite some of its
    freed blocks, swap it back in (into the blocks the block manager hands out then,
    in its allocation order), restore, and read it through its new table: its rows are
    back in order, and the other sequence's rows are intact."""
    rng = np.random.default_rng(5)
    nb = 24
    bm = BlockManagerModel(nb, B, order=rng.permutation(nb))
    a = bm.seq_add()
    kp, vp = fresh_pools(nb, dtype)
    n = 50
    slots, _ = bm.reserve_slots([a], [n])
    for layer in range(NL):
        append_rows(kp, vp, layer, slots, as_storage(rows_for(0, layer, a, range(n)), dtype),
                    as_storage(rows_for(1, layer, a, range(n)), dtype))
    old = bm.swap_out(a)
    buf = np.array(swap_buffer(kp, vp, old), copy=True)
    b = bm.seq_add()                                  # reuses the freed blocks, newest first
    nb_tok = 33
    slots_b, _ = bm.reserve_slots([b], [nb_tok])
    for layer in range(NL):
        append_rows(kp, vp, layer, slots_b, as_storage(rows_for(0, layer, b, range(nb_tok)), dtype),
                    as_storage(rows_for(1, layer, b, range(nb_tok)), dtype))
    new = bm.swap_in(a)
    if new == old or len(new) != len(old):
        return False
    swap_restore(kp, vp, new, buf)
    for kind, pool in ((0, kp), (1, vp)):
        c = as_codes(pool, dtype)
        for s, L in ((a, n), (b, nb_tok)):
            table = bm.table(s)
            for layer in range(NL):
                got = np.stack([c[layer, table[j // B], :, j % B, :] for j in range(L)])
                if not np.array_equal(got, rows_for(kind, layer, s, range(L))):
                    return False
    return True


DTYPES = ["f32", "f16", "bf16"]


@pytest.mark.parametrize("dtype", DTYPES)
def test_fifty_tokens_land_in_blocks_12_87_301_44(dtype):
    assert check_fifty_tokens_land_in_12_87_301_44(cm.append_rows, dtype)


@pytest.mark.parametrize("dtype", DTYPES)
@pytest.mark.parametrize("seed", [0, 1])
def test_gather_through_table_reproduces_written_rows(dtype, seed):
    assert check_gather_through_table(cm.append_rows, dtype, seed)


@pytest.mark.parametrize("dtype", DTYPES)
def test_swap_record_layout(dtype):
    assert check_swap_record(cm.append_rows, cm.swap_buffer, dtype)


@pytest.mark.parametrize("dtype", DTYPES)
def test_swap_round_trip_into_other_blocks(dtype):
    assert check_swap_round_trip(cm.append_rows, cm.swap_buffer, cm.swap_restore, dtype)


def test_empty_swap_record():
    kp, vp = fresh_pools(4, "bf16")
    buf = cm.swap_buffer(kp, vp, [])
    assert buf.shape == (0, NL, 2, H, B, D)
    cm.swap_restore(kp, vp, [], buf)
    assert untouched(kp, "bf16", np.zeros((NL, 4, B), bool))


# ------------------------------------------------------------------ planted mistakes
def battery(append_rows=cm.append_rows, swap_buffer=cm.swap_buffer, swap_restore=cm.swap_restore):
    checks = []
    for dtype in DTYPES:
        checks += [lambda dt=dtype: check_fifty_tokens_land_in_12_87_301_44(append_rows, dt),
                   lambda dt=dtype: check_gather_through_table(append_rows, dt, 0),
                   lambda dt=dtype: check_swap_record(append_rows, swap_buffer, dt),
                   lambda dt=dtype: check_swap_round_trip(append_rows, swap_buffer, swap_restore, dt)]
    for c in checks:
        try:
            if not c():
                return False
        except Exception:
            return False
    return True


def append_divmod_swapped(k_pool, v_pool, layer, slots, k_rows, v_rows):
    bs = k_pool.shape[3]
    for i, slot in enumerate(slots):
        if int(slot) < 0:
            continue
        off, blk = divmod(int(slot), bs)
        k_pool[layer, blk, :, off, :] = k_rows[i]
        v_pool[layer, blk, :, off, :] = v_rows[i]


def append_k_into_v(k_pool, v_pool, layer, slots, k_rows, v_rows):
    cm.append_rows(k_pool, v_pool, layer, slots, v_rows, k_rows)


def append_writes_padding(k_pool, v_pool, layer, slots, k_rows, v_rows):
    bs = k_pool.shape[3]
    for i, slot in enumerate(slots):
        blk, off = divmod(int(slot), bs)
        k_pool[layer, blk, :, off, :] = k_rows[i]
        v_pool[layer, blk, :, off, :] = v_rows[i]


def append_layer_zero(k_pool, v_pool, layer, slots, k_rows, v_rows):
    cm.append_rows(k_pool, v_pool, 0, slots, k_rows, v_rows)


def append_heads_reversed(k_pool, v_pool, layer, slots, k_rows, v_rows):
    cm.append_rows(k_pool, v_pool, layer, slots, np.asarray(k_rows)[:, ::-1], np.asarray(v_rows)[:, ::-1])


def buffer_kv_swapped(k_pool, v_pool, blocks):
    return cm.swap_buffer(v_pool, k_pool, blocks)


def buffer_reversed(k_pool, v_pool, blocks):
    return cm.swap_buffer(k_pool, v_pool, list(blocks)[::-1])


def buffer_layer_major(k_pool, v_pool, blocks):
    buf = cm.swap_buffer(k_pool, v_pool, blocks)
    return np.ascontiguousarray(np.swapaxes(buf, 0, 1)).reshape(buf.shape)


def restore_reversed(k_pool, v_pool, blocks, buf):
    cm.swap_restore(k_pool, v_pool, list(blocks)[::-1], buf)


def restore_kv_swapped(k_pool, v_pool, blocks, buf):
    cm.swap_restore(v_pool, k_pool, blocks, buf)


MUTANTS = {
    "append_divmod_swapped": dict(append_rows=append_divmod_swapped),
    "append_k_into_v": dict(append_rows=append_k_into_v),
    "append_writes_padding": dict(append_rows=append_writes_padding),
    "append_layer_zero": dict(append_rows=append_layer_zero),
    "append_heads_reversed": dict(append_rows=append_heads_reversed),
    "buffer_kv_swapped": dict(swap_buffer=buffer_kv_swapped),
    "buffer_reversed": dict(swap_buffer=buffer_reversed),
    "buffer_layer_major": dict(swap_buffer=buffer_layer_major),
    "restore_reversed": dict(swap_restore=restore_reversed),
    "restore_kv_swapped": dict(swap_restore=restore_kv_swapped),
}


def test_battery_accepts_model():
    assert battery()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_battery_rejects_planted_mistake(name):
    assert not battery(**MUTANTS[name])
