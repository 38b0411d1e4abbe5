"""Paged chunked-prefill attention on the GPU (tcgen05) vs the fp64 oracle, through the
C ABI.  Tolerance: max-abs 2e-3 (fp16 / bf16 cache, fp32 output)."""
import math

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_403_b200 as pa
from paged_kv_cache_403_b200.engine import PagedCache
from synthetic import values as sv

from oracle_replay import check_close

pytestmark = pytest.mark.gpu
DT = {"f16": torch.float16, "bf16": torch.bfloat16}


def dev(a, dtype):
    t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16) if dtype == "bf16" else np.ascontiguousarray(a))
    return (t.view(torch.bfloat16) if dtype == "bf16" else t).cuda()


@pytest.fixture(autouse=True)
def clean_device_error():
    pa.pa_device_error(clear=True)
    yield
    assert pa.pa_device_error(clear=True) == 0


def prefill_case(lens, chunks, B=16, hq=8, hkv=2, dtype="bf16", kv_scale=None, seed=0, fill=None, k_rows=None,
                 q_rows=None):
    """k_rows(total, rng) / q_rows(total, rng): optional fp32 replacements for the random
    keys / queries (the oracle gets the same host rows)."""
    d = 128
    kv_scale = 1 / math.sqrt(d) if kv_scale is None else kv_scale
    rng = np.random.default_rng(seed)
    nb = sum(-(-L // B) for L in lens) + 4
    order = rng.permutation(nb)
    cache = PagedCache(1, nb, B, hkv, d, dtype, order)
    if fill is not None:
        cache.k_pool.fill_(fill)
        cache.v_pool.fill_(fill)
    sids = [cache.add() for _ in lens]
    slots, _ = cache.reserve(sids, lens)
    k = sv.narrow((rng.standard_normal((sum(lens), hkv, d)) * kv_scale).astype(np.float32), dtype)
    v = sv.narrow((rng.standard_normal((sum(lens), hkv, d)) * kv_scale).astype(np.float32), dtype)
    if k_rows is not None:
        k = sv.narrow(k_rows(sum(lens), rng).astype(np.float32), dtype)
    cache.append(0, dev(k, dtype), dev(v, dtype), torch.from_numpy(np.ascontiguousarray(slots)).cuda())
    max_blocks = max(-(-L // B) for L in lens)
    tables, ln = cache.tables(sids, max_blocks)
    q_start = np.concatenate([[0], np.cumsum(chunks)]).astype(np.int32)
    q = sv.narrow(rng.standard_normal((int(q_start[-1]), hq, d)).astype(np.float32), dtype)
    if q_rows is not None:
        q = sv.narrow(q_rows(int(q_start[-1]), rng).astype(np.float32), dtype)
    # oracle's own pool (host): the same rows placed by the oracle's block-manager replay
    from oracle.block_manager import BlockManagerModel
    from oracle.cache_model import append_rows, empty_pools
    bm = BlockManagerModel(nb, B, order)
    osids = [bm.seq_add() for _ in lens]
    oslots, _ = bm.reserve_slots(osids, lens)
    kp, vp = empty_pools(1, nb, hkv, B, d, dtype)
    append_rows(kp, vp, 0, oslots, k, v)
    otables, olens = bm.dense_tables(osids, max_blocks)
    assert np.array_equal(np.array(otables), tables)
    oracle_args = (kp[0], vp[0], dtype, np.array(otables, np.int32), np.array(olens, np.int32), q_start)
    ref = oracle.paged_prefill(*oracle_args, q, 1 / math.sqrt(d))
    return dict(oracle_args=oracle_args, cache=cache, tables=torch.from_numpy(tables).cuda(), lens=torch.from_numpy(ln).cuda(),
                q_start=torch.from_numpy(q_start).cuda(), q=dev(q, dtype), ref=ref, max_q=int(max(chunks)),
                hq=hq, d=d, dtype=dtype, q_np=q, tables_np=tables, lens_np=ln)


def run(c, out_dtype=torch.float32):
    out = torch.full((c["q"].shape[0], c["hq"], c["d"]), float("nan"), dtype=out_dtype, device="cuda")
    pa.pa_prefill_attention(c["cache"].pool, 0, c["q"], out, c["tables"], c["lens"], c["q_start"], c["max_q"],
                            1 / math.sqrt(c["d"]))
    torch.cuda.synchronize()
    return out.cpu().to(torch.float64).numpy()


@pytest.mark.parametrize("dtype", ["bf16", "f16"])
@pytest.mark.parametrize("B", [16, 32])
def test_prefill_matches_oracle(dtype, B):
    lens = [300, 64, 65, 1000, 37]
    chunks = [100, 64, 1, 257, 37]           # mid-context chunk, whole prompts, a single token
    c = prefill_case(lens, chunks, B=B, dtype=dtype)
    err = check_close(run(c), c["ref"], "f32", dtype, "prefill")
    print(f"prefill {dtype} B{B} max err {err:.3g}")


@pytest.mark.parametrize("hq,hkv", [(2, 2), (4, 2), (8, 2), (16, 2)])
def test_prefill_gqa_groups(hq, hkv):
    c = prefill_case([200, 129], [70, 129], hq=hq, hkv=hkv)
    check_close(run(c), c["ref"], "f32", "bf16", f"gqa {hq}/{hkv}")


def test_prefill_native_output_and_unit_scale_values():
    c = prefill_case([150, 90], [150, 33], kv_scale=1.0, seed=3)
    check_close(run(c, torch.bfloat16), c["ref"], "bf16", "bf16", "native out, N(0,1) values")


def test_prefill_single_token_chunk_equals_decode():
    c = prefill_case([77, 300], [1, 1], seed=4)
    pre = run(c)
    out = torch.empty((2, c["hq"], c["d"]), dtype=torch.float32, device="cuda")
    c["cache"].decode(0, c["q"], out, c["tables"], c["lens"])
    torch.cuda.synchronize()
    check_close(pre, c["ref"], "f32", "bf16", "chunk of one")
    assert np.abs(pre - out.cpu().numpy()).max() <= 2e-3


def test_prefill_unused_slots_holding_nan():
    c = prefill_case([100, 47], [20, 47], fill=float("nan"), seed=5)
    out = run(c)
    assert np.isfinite(out).all()
    check_close(out, c["ref"], "f32", "bf16", "nan pool")


def test_prefill_rejects_unsupported_shapes():
    cache = PagedCache(1, 8, 16, 2, 64, "bf16")
    t = torch.zeros((1, 1), dtype=torch.int32, device="cuda")
    q = torch.zeros((4, 4, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(pa.PaError) as e:
        pa.pa_prefill_attention(cache.pool, 0, q, torch.zeros((4, 4, 64), device="cuda"), t,
                                torch.ones(1, dtype=torch.int32, device="cuda"),
                                torch.tensor([0, 4], dtype=torch.int32, device="cuda"), 4, 0.1)
    assert e.value.status == pa.PA_ERR_UNSUPPORTED


@pytest.mark.parametrize("B", [16, 32])
def test_prefill_key_tile_and_cta_boundaries(B):
    """Keys around the 128-key tile edges and query chunks around the 64-token CTA span
    (256 rows / GQA 4), including a chunk that starts exactly on a tile edge."""
    lens = [127, 128, 129, 255, 256, 257, 384, 1024]
    chunks = [63, 64, 65, 127, 128, 1, 256, 200]
    c = prefill_case(lens, chunks, B=B, seed=6)
    check_close(run(c), c["ref"], "f32", "bf16", f"boundaries B{B}")


def test_prefill_empty_chunks_in_the_batch():
    """Sequences without queries this pass (chunk 0) sit between ones with queries."""
    c = prefill_case([50, 300, 40, 129], [0, 77, 0, 129], seed=7)
    check_close(run(c), c["ref"], "f32", "bf16", "empty chunks")


def test_prefill_rising_scores_and_large_queries():
    """Keys whose scores keep rising along each sequence move the running maximum on
    almost every tile (the warp-wide rescale of O in TMEM, agreed by both threads of a
    row); a second case uses large query norms (very peaky rows)."""
    d = 128
    qdir = np.random.default_rng(8).standard_normal(d)
    qdir /= np.linalg.norm(qdir)
    lens = [900, 1500]

    def ramp_keys(total, rng):
        pos = np.concatenate([np.arange(L) / L for L in lens])
        return ((-20 + 60 * pos)[:, None, None] * qdir[None, None, :] / 3 + rng.standard_normal((total, 2, d)) * 0.05)

    c = prefill_case(lens, [300, 129], seed=9, k_rows=ramp_keys,
                     q_rows=lambda total, rng: np.tile(qdir * 12, (total, 8, 1)))
    check_close(run(c), c["ref"], "f32", "bf16", "rising scores")
    c2 = prefill_case([600, 257], [257, 257], seed=10, q_rows=lambda total, rng: rng.standard_normal((total, 8, d)) * 12)
    check_close(run(c2), c2["ref"], "f32", "bf16", "large queries")


def test_prefill_long_sequence():
    """An 8,704-token sequence: 68 key tiles for the last chunk's queries."""
    c = prefill_case([8704, 600], [512, 96], seed=12)
    check_close(run(c), c["ref"], "f32", "bf16", "long sequence")


@pytest.mark.slow
def test_chunked_prefill_workload_full_size_sampled():
    """The benchmarked chunked-prefill workload (32 sequences, 512-token chunks) in the
    launch configuration bench.py times; three sequences checked against the oracle on
    regenerated histories."""
    import bench
    from synthetic import workloads as wl
    r = wl.chunked_prefill()
    sh = r["shape"]
    c = bench.prefill_setup(torch, r)
    out = torch.empty((c["rows"], sh.num_q_heads, sh.head_dim), dtype=torch.float32, device="cuda")
    pa.pa_prefill_attention(c["cache"].pool, 0, c["q"], out, c["tables"], c["lens"], c["q_start"], c["max_q"],
                            1 / math.sqrt(sh.head_dim))
    got = out.cpu().numpy()
    q_start = c["q_start"].cpu().numpy()
    for s in (0, int(np.argmax(r["lens"])), len(r["lens"]) - 1):
        L, C = int(r["lens"][s]), int(r["chunks"][s])
        k = sv.rows(sv.KIND_K, r["seed"], 0, np.full(L, s), np.arange(L), sh.num_kv_heads, sh.head_dim,
                    sh.kv_scale, sh.dtype)
        v = sv.rows(sv.KIND_V, r["seed"], 0, np.full(L, s), np.arange(L), sh.num_kv_heads, sh.head_dim,
                    sh.kv_scale, sh.dtype)
        nblk = -(-L // 16)
        pad = nblk * 16 - L
        shp = (nblk, 16, sh.num_kv_heads, sh.head_dim)
        kp = np.concatenate([k, np.zeros((pad,) + k.shape[1:], k.dtype)]).reshape(shp).transpose(0, 2, 1, 3)
        vp = np.concatenate([v, np.zeros((pad,) + v.shape[1:], v.dtype)]).reshape(shp).transpose(0, 2, 1, 3)
        q = sv.rows(sv.KIND_Q, r["seed"], 0, np.full(C, s), np.arange(L - C, L), sh.num_q_heads, sh.head_dim,
                    sh.q_scale, sh.dtype)
        ref = oracle.paged_prefill(np.ascontiguousarray(kp), np.ascontiguousarray(vp), sh.dtype,
                                   np.arange(nblk, dtype=np.int32)[None], [L], [0, C], q, 1 / math.sqrt(sh.head_dim))
        check_close(got[q_start[s]:q_start[s + 1]], ref, "f32", "bf16", f"chunked prefill seq {s}")
