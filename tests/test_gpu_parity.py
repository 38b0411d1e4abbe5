"""GPU path vs oracle, through the C ABI (pytest -m gpu).

Bit-exact: block tables, lengths, slots, copy pairs, the whole key/value pools
after appends and copy-on-write.  Attention: max-abs 1e-5 (fp32 cache) or 2e-3
(fp16 / bf16 cache) against the fp64 oracle with fp32 output; with output in the
cache's own type the bound adds half an ulp of that type at the reference value.
"""
import math

import numpy as np
import pytest
import torch

import paged_kv_cache_403_b200 as pa
from paged_kv_cache_403_b200.engine import PagedCache
from paged_kv_cache_403_b200.runners import ContinuousBatch, run_prefix_sharing, run_static
from synthetic import values as sv
from synthetic import workloads as wl

from oracle_replay import OracleRun, check_close, device_generated_rows, histories_attention, sequence_attention

pytestmark = pytest.mark.gpu

DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


def host(t):
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def widen(t):
    return t.detach().cpu().to(torch.float64).numpy()


@pytest.fixture(autouse=True)
def clean_device_error():
    pa.pa_device_error(clear=True)
    yield
    assert pa.pa_device_error(clear=True) == 0


# ------------------------------------------------------------------ generator
@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_device_generator_matches_host(dtype):
    from synthetic import gpu as sgpu
    rng = np.random.default_rng(0)
    uids = rng.integers(0, 1 << 22, size=257).astype(np.int32)
    toks = rng.integers(0, 1 << 20, size=257).astype(np.int32)
    for kind, layer, scale in [(sv.KIND_K, 0, 1.0), (sv.KIND_V, 31, 0.088), (sv.KIND_Q, 7, 2.5)]:
        out = torch.empty((257, 8, 128), dtype=DT[dtype], device="cuda")
        sgpu.fill_rows(out, kind, 12345, layer, torch.from_numpy(uids).cuda(), torch.from_numpy(toks).cuda(),
                       scale, dtype)
        ref = sv.rows(kind, 12345, layer, uids, toks, 8, 128, scale, dtype)
        assert np.array_equal(host(out), ref)


# ------------------------------------------------------------------ static workloads
def replay_static(recipe, layers=None):
    sh = recipe["shape"]
    o = OracleRun(sh, recipe["order"], recipe["seed"])
    lens = [int(L) for L in recipe["lens"]]
    sids = [o.bm.seq_add() for _ in lens]
    o.prefill(sids, list(range(len(lens))), lens)
    mb = max(-(-(L + 1) // sh.block_size) for L in lens)
    return o, o.decode_step(sids, list(range(len(lens))), mb, layers)


@pytest.mark.parametrize("out", ["f32", "native"])
@pytest.mark.parametrize("split", [0, 32])
def test_tiny(out, split):
    r = wl.tiny()
    cache, _, rec = run_static(r, split_tokens=split, out_dtype=torch.float32 if out == "f32" else None)
    o, ref = replay_static(r)
    assert np.array_equal(rec.slots, ref["slots"]) and np.array_equal(rec.tables, ref["tables"])
    assert np.array_equal(rec.lens, ref["lens"])
    assert np.array_equal(host(cache.k_pool), o.k) and np.array_equal(host(cache.v_pool), o.v)
    assert [int((t >= 0).sum()) for t in rec.tables] == [4, 2, 1, 3]
    check_close(widen(rec.outputs[0]), ref["outputs"][0], "f32", "f32", "tiny")


@pytest.mark.parametrize("out", ["f32", "native"])
def test_worked_example(out):
    r = wl.worked_example()
    cache, _, rec = run_static(r, split_tokens=1024, out_dtype=torch.float32 if out == "f32" else None)
    o, ref = replay_static(r)
    assert np.array_equal(rec.slots, ref["slots"]) and np.array_equal(rec.tables, ref["tables"])
    assert np.array_equal(host(cache.k_pool), o.k) and np.array_equal(host(cache.v_pool), o.v)
    blocks = [int((t >= 0).sum()) for t in rec.tables]
    assert blocks == [244, 27, 132, 5] and sum(blocks) == 408
    # bytes of those blocks in the device pools, scaled to the pages' 32-layer model: 816 MiB
    per_block_layer = (cache.k_pool[0, 0].numel() * cache.k_pool.element_size()
                       + cache.v_pool[0, 0].numel() * cache.v_pool.element_size())
    assert sum(blocks) * per_block_layer * 32 == 816 * 2 ** 20
    err = check_close(widen(rec.outputs[0]), ref["outputs"][0], "f32" if out == "f32" else "f16", "f16",
                      "worked example")
    print(f"worked example max err {err:.3g}")


def test_prefix_sharing_with_copy_on_write():
    r = wl.prefix_sharing()
    cache, _, res = run_prefix_sharing(r, split_tokens=512, out_dtype=torch.float32)
    sh = r["shape"]
    o = OracleRun(sh, r["order"], r["seed"])
    n, prefix = len(r["suffix"]), r["prefix"]
    root = o.bm.seq_add()
    o.prefill([root], [0], [prefix])
    sids = [root] + [o.bm.seq_fork(root) for _ in range(n - 1)]
    uids = list(range(n))
    suffix = [int(x) for x in r["suffix"]]
    slots, cow = o.bm.reserve_slots(sids, suffix)
    assert not cow
    o.write(slots, np.repeat(uids, suffix), np.concatenate([prefix + np.arange(x) for x in suffix]))
    mb = res["step1"].tables.shape[1]
    ref1 = o.decode_step(sids, uids, mb)
    victim = next(i for i, L in enumerate(o.bm.lengths[s] for s in sids) if L % sh.block_size)
    assert victim == res["victim"]
    child = o.bm.seq_fork(sids[victim])
    ref2 = o.decode_step(sids + [child], uids + [n], mb)
    for rec, ref in [(res["step1"], ref1), (res["step2"], ref2)]:
        assert np.array_equal(rec.slots, ref["slots"]) and np.array_equal(rec.tables, ref["tables"])
        assert np.array_equal(rec.cow, ref["cow"])
        check_close(widen(rec.outputs[0]), ref["outputs"][0], "f32", "f16", "prefix sharing")
    assert len(res["step2"].cow) == 1
    assert np.array_equal(host(cache.k_pool), o.k) and np.array_equal(host(cache.v_pool), o.v)


def test_prefix_with_partial_shared_block_copies_for_each_writer():
    """2040-token prefix (last block half full) shared by 64 sequences: 63 copies."""
    sh = wl.Shape(1, 16, 8, 2, 64, "bf16", 512, kv_scale=1.0)
    order = np.random.default_rng(9).permutation(512)
    from paged_kv_cache_403_b200.runners import DeviceGen, decode_step, prefill
    cache = PagedCache.from_shape(sh, order)
    gen = DeviceGen(77, sh)
    root = cache.add()
    prefill(cache, gen, [root], [0], [2040])
    sids = [root] + [cache.fork(root) for _ in range(63)]
    rec = decode_step(cache, gen, sids, list(range(64)), 8, 128, out_dtype=torch.float32)
    assert len(rec.cow) == 63
    o = OracleRun(sh, order, 77)
    oroot = o.bm.seq_add()
    o.prefill([oroot], [0], [2040])
    osids = [oroot] + [o.bm.seq_fork(oroot) for _ in range(63)]
    ref = o.decode_step(osids, list(range(64)), 128)
    assert np.array_equal(rec.cow, ref["cow"]) and np.array_equal(rec.slots, ref["slots"])
    assert np.array_equal(host(cache.k_pool), o.k) and np.array_equal(host(cache.v_pool), o.v)
    check_close(widen(rec.outputs[0]), ref["outputs"][0], "f32", "bf16", "partial prefix")


# ------------------------------------------------------------------ continuous batch
def test_continuous_batch_reduced_full_replay():
    """24 sequences, 10 steps, stops at p = 0.05 so sequences retire and are admitted."""
    r = wl.continuous_batch(seed=31, n=24, steps=10, p_stop=0.05, lo=20, hi=700)
    assert sum(len(e) for e in r["schedule"].events[:9]) > 0
    cb = ContinuousBatch(r, max_blocks=48)
    sh = r["shape"]
    o = OracleRun(sh, r["order"], r["seed"])
    n = len(r["schedule"].initial)
    osids = [o.bm.seq_add() for _ in range(n)]
    ouids = list(range(n))
    o.prefill(osids, ouids, [int(x) for x in r["schedule"].initial])
    next_uid, pending = n, []
    for t in range(10):
        rec = cb.step(split_tokens=128, out_dtype=torch.float32)
        for slot, plen in pending:
            osids[slot] = o.bm.seq_add()
            ouids[slot] = next_uid
            next_uid += 1
            o.prefill([osids[slot]], [ouids[slot]], [plen])
        pending = []
        ref = o.decode_step(osids, ouids, 48)
        assert np.array_equal(rec.slots, ref["slots"]) and np.array_equal(rec.tables, ref["tables"])
        check_close(widen(rec.outputs[0]), ref["outputs"][0], "f32", "bf16", f"step {t}")
        for slot, plen in r["schedule"].events[t]:
            o.bm.seq_free(osids[slot])
            pending.append((slot, plen))
    assert np.array_equal(host(cb.cache.k_pool), o.k) and np.array_equal(host(cb.cache.v_pool), o.v)


@pytest.mark.slow
@pytest.mark.parametrize("split", [2048, 4096])
def test_continuous_batch_full_size_sampled(split):
    """256 sequences, 64 steps, bf16 output, split 4096 as timed by the benchmark (and
    2048): sampled sequences of steps 0 and 21, and every sequence of the last step
    (after retirements and admissions), checked against the oracle on regenerated
    histories."""
    r = wl.continuous_batch()
    sh = r["shape"]
    cb = ContinuousBatch(r)
    rng = np.random.default_rng(0)
    for t in range(64):
        rec = cb.step(split_tokens=split)
        if t == 63:
            ref = histories_attention(sh, r["seed"], 0, rec.uids, rec.lens, rec.positions,
                                      device_generated_rows(sh, r["seed"], 0))
            err = check_close(widen(rec.outputs[0]), ref, "bf16", "bf16", f"step {t}, all sequences")
            print(f"continuous batch split {split}: step 63, all {len(rec.lens)} sequences, max err {err:.3g}")
        elif t in (0, 21):
            lens = rec.lens
            picks = set(rng.choice(len(lens), size=5, replace=False).tolist())
            picks |= {int(np.argmax(lens)), int(np.argmin(lens))}
            out = widen(rec.outputs[0])
            for i in sorted(picks):
                ref = sequence_attention(sh, r["seed"], 0, rec.uids[i], int(lens[i]), rec.uids[i],
                                         int(rec.positions[i]))
                check_close(out[i], ref, "bf16", "bf16", f"step {t} seq {i}")
    # sampled pool rows equal the regenerated rows (slot of the latest token of a few sequences)
    for i in range(0, 256, 37):
        L = int(rec.lens[i])
        blk = int(rec.tables[i][(L - 1) // 16])
        got = host(cb.cache.k_pool[0, blk, :, (L - 1) % 16])
        exp = sv.rows(sv.KIND_K, r["seed"], 0, [rec.uids[i]], [L - 1], 8, 128, sh.kv_scale, "bf16")[0]
        assert np.array_equal(got, exp)


@pytest.mark.slow
@pytest.mark.parametrize("bs,split", [(16, 2048), (32, 2048), (16, 4096), (32, 4096)])
def test_large_pool_sampled(bs, split):
    """384 sequences, lognormal lengths, 32 layers (~100 GB), split-K: ranges of at most
    4096 tokens as the benchmark times them (only sequences over 4096 tokens split), and
    2048."""
    r = wl.large_pool(block_size=bs)
    sh = r["shape"]
    cache, _, rec = run_static(r, split_tokens=split, keep_layers={0, 31})
    lens = rec.lens
    assert (lens > 4096).any()
    picks = [int(np.argmax(lens)), int(np.argmin(lens)), int(np.argsort(lens)[len(lens) // 2])]
    picks += [int(i) for i in np.nonzero(lens > 4096)[0][:2]]
    out = widen(rec.outputs[0])
    for i in picks:
        ref = sequence_attention(sh, r["seed"], 0, rec.uids[i], int(lens[i]), rec.uids[i], int(rec.positions[i]))
        check_close(out[i], ref, "f16", "f16", f"layer 0 seq {i}")
    # every sequence of the last layer
    ref = histories_attention(sh, r["seed"], 31, rec.uids, lens, rec.positions,
                              device_generated_rows(sh, r["seed"], 31))
    err = check_close(widen(rec.outputs[31]), ref, "f16", "f16", "layer 31, all sequences")
    print(f"large pool B{bs} split {split}: layer 31, all {len(lens)} sequences, max err {err:.3g}")
    del cache
    torch.cuda.empty_cache()


# ------------------------------------------------------------------ prefix caching on the GPU
@pytest.mark.parametrize("cache_on", [True, False])
def test_shared_prompt_with_prefix_cache(cache_on):
    """Requests share a 256-token system prompt; with the cache its 16 blocks are written
    once and shared by every later admission.  Attention over the shared blocks matches
    the oracle on each request's regenerated history (system prompt + own tokens)."""
    from paged_kv_cache_403_b200.runners import SharedPromptBatch
    r = wl.shared_prompt_batch(seed=61, n=12, steps=6, system=256, p_stop=0.15)
    sh, sysl, sys_uid = r["shape"], r["system"], r["system_uid"]
    sb = SharedPromptBatch(r, max_blocks=272, cache=cache_on)
    st = pa.pa_pool_stats(sb.cache.pool)
    if cache_on:
        assert st["num_cached"] == sysl // 16 and st["cache_hits"] == (12 - 1) * (sysl // 16)
    else:
        assert st["num_cached"] == 0
    for t in range(6):
        rec = sb.step(split_tokens=512, out_dtype=torch.float32)
        out = widen(rec.outputs[0])
        for i in range(len(rec.lens)):
            uid = rec.uids[i]
            ref = sequence_attention(sh, r["seed"], 0, uid, int(rec.lens[i]), uid, int(rec.positions[i]),
                                     writer=lambda p, u=uid: (sys_uid, p) if p < sysl else (u, p))
            check_close(out[i], ref, "f32", "bf16", f"step {t} seq {i}")
        if cache_on:   # every live sequence starts with the same 16 physical blocks
            first = {tuple(row[:sysl // 16]) for row in rec.tables}
            assert len(first) == 1
    admitted = sum(len(e) for e in r["schedule"].events[:5])
    assert admitted > 0
    if cache_on:
        assert pa.pa_pool_stats(sb.cache.pool)["cache_hits"] == (12 - 1 + admitted) * (sysl // 16)
