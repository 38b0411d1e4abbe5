"""Edge cases of the GPU path through the C ABI (pytest -m gpu)."""
import math

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_403_b200 as pa
from oracle.cache_model import append_rows, copy_blocks, empty_pools
from paged_kv_cache_403_b200.engine import PagedCache
from synthetic import values as sv

from oracle_replay import check_close

pytestmark = pytest.mark.gpu
DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}


def host(t):
    t = t.detach().cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def dev(a, dtype):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype == "bf16":
        t = t.view(torch.bfloat16)
    return t.cuda()


@pytest.fixture(autouse=True)
def clean_device_error():
    pa.pa_device_error(clear=True)
    yield
    assert pa.pa_device_error(clear=True) == 0


class Case:
    """Sequences with given host K/V/q, placed through the library, and the oracle result."""

    def __init__(self, lens, B=16, hq=8, hkv=2, d=128, dtype="bf16", order=None, nb=None, seed=0,
                 kv_scale=1.0, q_scale=1.0, k_override=None, fill=None):
        self.lens, self.B, self.hq, self.hkv, self.d, self.dtype = list(lens), B, hq, hkv, d, dtype
        nb = nb or sum(-(-L // B) for L in lens) + 8
        rng = np.random.default_rng(seed)
        self.k = [sv.narrow((rng.standard_normal((L, hkv, d)) * kv_scale).astype(np.float32), dtype)
                  for L in lens]
        if k_override is not None:
            self.k = [sv.narrow(k_override(i, L).astype(np.float32), dtype) for i, L in enumerate(lens)]
        self.v = [sv.narrow((rng.standard_normal((L, hkv, d)) * kv_scale).astype(np.float32), dtype)
                  for L in lens]
        self.q = sv.narrow((rng.standard_normal((len(lens), hq, d)) * q_scale).astype(np.float32), dtype)
        self.cache = PagedCache(1, nb, B, hkv, d, dtype, order)
        if fill is not None:                 # what unused slots hold before anything is written
            self.cache.k_pool.fill_(fill)
            self.cache.v_pool.fill_(fill)
        self.sids = [self.cache.add() for _ in lens]
        slots, _ = self.cache.reserve(self.sids, self.lens)
        kk = np.concatenate(self.k) if lens else np.zeros((0, hkv, d))
        vv = np.concatenate(self.v) if lens else np.zeros((0, hkv, d))
        self.cache.append(0, dev(kk, dtype), dev(vv, dtype), torch.from_numpy(slots).cuda())
        self.max_blocks = max(-(-L // B) for L in lens)
        t, ln = self.cache.tables(self.sids, self.max_blocks)
        self.tables_host, self.lens_host = t, ln
        self.tables, self.lens_dev = torch.from_numpy(t).cuda(), torch.from_numpy(ln).cuda()

    def run(self, split=0, out="f32", q=None):
        n = len(self.lens)
        out_t = torch.empty((n, self.hq, self.d), dtype=DT[out] if out != "native" else DT[self.dtype],
                            device="cuda")
        ws = self.cache.workspace(n, self.hq, self.max_blocks, split)
        self.cache.decode(0, dev(self.q if q is None else q, self.dtype), out_t, self.tables, self.lens_dev,
                          1.0 / math.sqrt(self.d), split, ws)
        torch.cuda.synchronize()
        return out_t.cpu().to(torch.float64).numpy()

    def oracle(self):
        outs = []
        for i, L in enumerate(self.lens):
            nblk = -(-L // self.B)
            pad = nblk * self.B - L
            k = np.concatenate([self.k[i], np.zeros((pad, self.hkv, self.d), self.k[i].dtype)])
            v = np.concatenate([self.v[i], np.zeros((pad, self.hkv, self.d), self.v[i].dtype)])
            kp = np.ascontiguousarray(k.reshape(nblk, self.B, self.hkv, self.d).transpose(0, 2, 1, 3))
            vp = np.ascontiguousarray(v.reshape(nblk, self.B, self.hkv, self.d).transpose(0, 2, 1, 3))
            outs.append(oracle.paged_decode(kp, vp, self.dtype, np.arange(nblk, dtype=np.int32)[None],
                                            [L], self.q[i:i + 1], 1.0 / math.sqrt(self.d))[0])
        return np.stack(outs)


def test_placement_invariance_bit_identical():
    """Identity placement, a shuffled pool and the pages' 12, 87, 301, 44 table give
    the same bits: paging changes where data lives, never the result."""
    lens = [50]
    order_pages = [12, 87, 301, 44] + [b for b in range(400) if b not in (12, 87, 301, 44)]
    a = Case(lens, nb=400, order=list(range(400)))
    b = Case(lens, nb=400, order=list(np.random.default_rng(5).permutation(400)))
    c = Case(lens, nb=400, order=order_pages)
    assert c.tables_host[0].tolist() == [12, 87, 301, 44]
    oa, ob, oc = a.run(), b.run(), c.run()
    assert np.array_equal(oa, ob) and np.array_equal(oa, oc)
    check_close(oa, a.oracle(), "f32", "bf16", "placement")


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_single_token_returns_its_value(dtype):
    c = Case([1, 1, 1], dtype=dtype, hq=4, hkv=2, d=64)
    out = c.run()
    for i in range(3):
        for h in range(4):
            assert np.array_equal(out[i, h], sv.to_float64(c.v[i][0, h // 2], dtype))


@pytest.mark.parametrize("split", [0, 16, 512])
def test_block_and_split_boundaries(split):
    lens = [1, 15, 16, 17, 31, 32, 33, 511, 512, 513, 1023, 1024, 1025, 2047, 2048, 2049]
    c = Case(lens, order=list(np.random.default_rng(1).permutation(sum(-(-L // 16) for L in lens) + 8)))
    check_close(c.run(split), c.oracle(), "f32", "bf16", f"split {split}")


def test_maximum_length_split_and_unsplit():
    c = Case([16384, 3], hq=32, hkv=8, dtype="f16", kv_scale=1 / math.sqrt(128),
             order=list(np.random.default_rng(2).permutation(1024 + 1 + 8)))
    ref = c.oracle()
    o0 = c.run(0)
    for split in (4096, 512, 16):
        check_close(c.run(split), ref, "f32", "f16", f"split {split}")
    check_close(o0, ref, "f32", "f16", "unsplit")


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("B", [16, 32])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("hq,hkv", [(4, 4), (8, 4), (8, 2), (32, 4)])
def test_shapes(dtype, B, d, hq, hkv):
    lens = [7, 40, 300, 65]
    c = Case(lens, B=B, hq=hq, hkv=hkv, d=d, dtype=dtype,
             order=list(np.random.default_rng(3).permutation(sum(-(-L // B) for L in lens) + 8)))
    ref = c.oracle()
    check_close(c.run(0), ref, "f32", dtype, "shapes")
    check_close(c.run(2 * B), ref, "f32", dtype, "shapes split")
    check_close(c.run(0, out="native"), ref, dtype, dtype, "shapes native out")


def test_peaky_and_increasing_scores():
    """Large query norms and scores that keep rising along the sequence exercise the
    running-maximum updates of the online softmax."""
    d = 128
    qdir = np.random.default_rng(4).standard_normal(d)
    qdir /= np.linalg.norm(qdir)

    def keys(i, L):
        ramp = np.linspace(-30, 60, L)[:, None, None]          # score grows with position
        noise = np.random.default_rng(10 + i).standard_normal((L, 2, d)) * 0.05
        return ramp * qdir[None, None, :] / 4 + noise

    c = Case([700, 33, 2100], hq=8, hkv=2, d=d, dtype="f32", k_override=keys)
    q = np.tile((qdir * 16).astype(np.float32), (3, 8, 1))
    c.q = q
    ref = c.oracle()
    for split in (0, 64):
        check_close(c.run(split), ref, "f32", "f32", f"peaky split {split}")
    c2 = Case([1000, 257], hq=8, hkv=2, q_scale=25.0)
    check_close(c2.run(0), c2.oracle(), "f32", "bf16", "large q")


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
@pytest.mark.parametrize("B", [16, 32])
def test_unused_slots_holding_nan_do_not_leak(dtype, B):
    """Pools whose unused slots hold NaN (memory never written): every tail block has
    NaN rows past the sequence end; outputs must stay finite and match the oracle."""
    lens = [1, 5, 17, 31, 33, 100, 511]
    c = Case(lens, B=B, dtype=dtype, fill=float("nan"),
             order=list(np.random.default_rng(8).permutation(sum(-(-L // B) for L in lens) + 8)))
    ref = c.oracle()
    for split in (0, 2 * B):
        out = c.run(split)
        assert np.isfinite(out).all()
        check_close(out, ref, "f32", dtype, f"nan pool split {split}")


def test_empty_batch_launches_nothing():
    c = Case([5])
    before = pa.pa_launch_count()
    out = torch.empty((0, 8, 128), dtype=torch.float32, device="cuda")
    q = torch.empty((0, 8, 128), dtype=torch.bfloat16, device="cuda")
    c.cache.decode(0, q, out, c.tables[:0], c.lens_dev[:0], 0.1)
    pa.pa_append_kv(c.cache.pool, 0, q, q, torch.empty(0, dtype=torch.int64, device="cuda"))
    assert pa.pa_launch_count() == before


def test_invalid_arguments_rejected_before_launch():
    c = Case([40])
    before = pa.pa_launch_count()
    q = dev(c.q, "bf16")
    out = torch.empty((1, 8, 128), dtype=torch.float32, device="cuda")
    bad = [
        dict(split_tokens=24),                                              # not a multiple of 16
        dict(split_tokens=16),                                              # workspace missing
        dict(out=torch.empty((1, 8, 128), dtype=torch.float16, device="cuda")),   # wrong out dtype
    ]
    for kw in bad:
        with pytest.raises(pa.PaError) as e:
            pa.pa_decode_attention(c.cache.pool, 0, q, kw.get("out", out), c.tables, c.lens_dev, 0.1,
                                   kw.get("split_tokens", 0))
        assert e.value.status == pa.PA_ERR_INVALID_ARG
    with pytest.raises(pa.PaError) as e:
        pa.pa_decode_attention(c.cache.pool, 1, q, out, c.tables, c.lens_dev, 0.1)   # layer
    assert e.value.status == pa.PA_ERR_INVALID_ARG
    odd = PagedCache(1, 8, 16, 2, 96, "bf16")
    q96 = torch.zeros((1, 8, 96), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(pa.PaError) as e:
        pa.pa_decode_attention(odd.pool, 0, q96, torch.zeros((1, 8, 96), device="cuda"), c.tables,
                               c.lens_dev, 0.1)
    assert e.value.status == pa.PA_ERR_UNSUPPORTED
    q6 = torch.zeros((1, 6, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(pa.PaError) as e:
        pa.pa_decode_attention(c.cache.pool, 0, q6, torch.zeros((1, 6, 128), device="cuda"), c.tables,
                               c.lens_dev, 0.1)
    assert e.value.status == pa.PA_ERR_UNSUPPORTED
    assert pa.pa_launch_count() == before


def test_bad_tables_and_slots_set_the_error_word_without_faulting():
    c = Case([40, 9])
    t = c.tables.clone()
    t[1, 0] = 10 ** 6                                # block id far outside the pool
    out = torch.empty((2, 8, 128), dtype=torch.float32, device="cuda")
    c.cache.decode(0, dev(c.q, "bf16"), out, t, c.lens_dev, 0.1)
    assert pa.pa_device_error(clear=True) & 1
    lens = c.lens_dev.clone()
    lens[0] = 10 ** 5                                # longer than its table
    c.cache.decode(0, dev(c.q, "bf16"), out, c.tables, lens, 0.1)
    assert pa.pa_device_error(clear=True) & 2
    k = torch.zeros((1, 2, 128), dtype=torch.bfloat16, device="cuda")
    c.cache.append(0, k, k, torch.tensor([10 ** 9], dtype=torch.int64, device="cuda"))
    assert pa.pa_device_error(clear=True) & 8
    assert pa.pa_device_error() == 0


@pytest.mark.parametrize("dtype", ["f32", "f16", "bf16"])
def test_append_and_copy_blocks_bit_exact_multi_layer(dtype):
    """3 layers: appends with a skipped (negative) slot, then copy-on-write copies."""
    L, NB, B, H, D = 3, 40, 16, 2, 64
    order = np.random.default_rng(6).permutation(NB)
    cache = PagedCache(L, NB, B, H, D, dtype, order)
    kref, vref = empty_pools(L, NB, H, B, D, dtype)
    rng = np.random.default_rng(7)
    s = cache.add()
    slots, _ = cache.reserve([s], [37])
    slots = slots.copy()
    slots[5] = -1
    for layer in range(L):
        k = sv.narrow(rng.standard_normal((37, H, D)).astype(np.float32), dtype)
        v = sv.narrow(rng.standard_normal((37, H, D)).astype(np.float32), dtype)
        cache.append(layer, dev(k, dtype), dev(v, dtype), torch.from_numpy(slots).cuda())
        append_rows(kref, vref, layer, slots, k, v)
    child = cache.fork(s)
    slots2, cow = cache.reserve([child], [1])
    assert len(cow) == 1
    cache.copy_blocks(cow)
    copy_blocks(kref, vref, cow)
    torch.cuda.synchronize()
    assert np.array_equal(host(cache.k_pool), kref) and np.array_equal(host(cache.v_pool), vref)
