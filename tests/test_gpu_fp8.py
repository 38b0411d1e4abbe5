"""FP8 KV cache (E4M3 codes, one power-of-two scale per (token, KV head) row) on the
GPU, through the C ABI (pytest -m gpu).

Appends, block copies and swaps must match the oracle bit for bit (codes and scale
bytes).  Decode attention is compared with the fp64 oracle over the exactly
dequantised cache, which the oracle builds itself from the same host rows
(oracle.fp8.quantize_rows), never from device data.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_403_b200 as pa
from oracle import fp8 as F
from oracle.cache_model import (append_rows_fp8, copy_blocks, copy_scales, empty_pools, empty_scales,
                                swap_buffer_fp8)
from paged_kv_cache_403_b200.engine import PagedCache
from synthetic import values as sv

from oracle_replay import check_close

pytestmark = pytest.mark.gpu
DT = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}
D = 128


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


def quantize(rows, act):
    """Oracle-side codes and scale bytes of host rows stored in `act`."""
    return F.quantize_rows(oracle.widen(rows, act).astype(np.float32))


class Fp8Case:
    """Sequences with host K/V/q rows, appended through the library into an FP8 pool."""

    def __init__(self, lens, B=16, hq=8, hkv=2, act="bf16", nb=None, seed=0, kv_scale=1.0, q_scale=1.0,
                 order=None, fill=None, k_rows=None, v_rows=None, q=None):
        self.lens, self.B, self.hq, self.hkv, self.act = list(lens), B, hq, hkv, act
        nb = nb or sum(-(-L // B) for L in lens) + 8
        if order is None:
            order = np.random.default_rng(seed + 100).permutation(nb)
        rng = np.random.default_rng(seed)
        gen = lambda L: sv.narrow((rng.standard_normal((L, hkv, D)) * kv_scale).astype(np.float32), act)  # noqa
        self.k = [gen(L) if k_rows is None else sv.narrow(k_rows(i, L).astype(np.float32), act)
                  for i, L in enumerate(lens)]
        self.v = [gen(L) if v_rows is None else sv.narrow(v_rows(i, L).astype(np.float32), act)
                  for i, L in enumerate(lens)]
        self.q = sv.narrow((rng.standard_normal((len(lens), hq, D)) * q_scale).astype(np.float32), act) \
            if q is None else sv.narrow(q.astype(np.float32), act)
        self.cache = PagedCache(1, nb, B, hkv, D, "fp8", order, act_dtype=act)
        if fill is not None:                     # what never-written slots hold
            self.cache.k_pool.fill_(fill[0])
            self.cache.v_pool.fill_(fill[0])
            self.cache.scales.fill_(fill[1])
        self.sids = [self.cache.add() for _ in lens]
        slots, _ = self.cache.reserve(self.sids, self.lens)
        self.cache.append(0, dev(np.concatenate(self.k), act), dev(np.concatenate(self.v), act),
                          torch.from_numpy(slots).cuda())
        self.max_blocks = max(-(-L // B) for L in lens)
        t, ln = self.cache.tables(self.sids, self.max_blocks)
        self.tables, self.lens_dev = torch.from_numpy(t).cuda(), torch.from_numpy(ln).cuda()

    def run(self, split=0, out="f32"):
        n = len(self.lens)
        out_t = torch.empty((n, self.hq, D), dtype=DT[out], device="cuda")
        ws = self.cache.workspace(n, self.hq, self.max_blocks, split)
        self.cache.decode(0, dev(self.q, self.act), out_t, self.tables, self.lens_dev, 1.0 / math.sqrt(D), split,
                          ws)
        torch.cuda.synchronize()
        return out_t.cpu().to(torch.float64).numpy()

    def oracle(self):
        outs = []
        for i, L in enumerate(self.lens):
            nblk = -(-L // self.B)
            pad = nblk * self.B - L
            kc, ks = quantize(self.k[i], self.act)
            vc, vs = quantize(self.v[i], self.act)
            lay = lambda a: np.ascontiguousarray(                                          # noqa: E731
                np.concatenate([a, np.zeros((pad,) + a.shape[1:], a.dtype)])
                .reshape((nblk, self.B) + a.shape[1:]).swapaxes(1, 2))
            outs.append(oracle.paged_decode_fp8(lay(kc), lay(vc), lay(ks), lay(vs),
                                                np.arange(nblk, dtype=np.int32)[None], [L], self.q[i:i + 1],
                                                self.act, 1.0 / math.sqrt(D))[0])
        return np.stack(outs)


# ------------------------------------------------------------------ append / copy / swap
def special_rows(rng, n, hkv, d, act):
    """Rows that reach the corners of the quantiser: zeros, a single spike, tiny and huge
    magnitudes, exact 448 * 2^k maxima, rounding ties, negative values that round to -0."""
    rows = rng.standard_normal((n, hkv, d)).astype(np.float32)
    rows[0] = 0.0
    rows[1] = 0.0
    rows[1, :, 3] = -7.5
    rows[2] *= 1e-3
    rows[3] *= 3e3 if act == "bf16" else 30.0
    rows[4, :, 0] = 448.0 * 2.0 ** -6                       # amax exactly 448 * 2^X
    rows[5, :, :] = -2.0 ** -21                             # X = -10: -2^-11 rounds to -0 (0x80)
    rows[5, :, 1] = 448.0 * 2.0 ** -10
    lower = rng.integers(0, 0x7E, size=(hkv, d)).astype(np.uint8)          # a code and the next one up
    mid = (F.e4m3_decode(lower) + F.e4m3_decode(lower + 1)) / 2
    rows[6] = mid * rng.choice([-1.0, 1.0], size=(hkv, d)) * 2.0 ** -3      # exact rounding ties
    rows[6, :, 0] = 448.0 * 2.0 ** -3
    if act == "bf16":
        rows[7] *= 1e-30                                    # far below fp16 range
        rows[8] *= 1e30
    return sv.narrow(rows, act)


@pytest.mark.parametrize("act", ["f16", "bf16"])
@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("B", [16, 32])
def test_append_copy_bit_exact(act, d, B):
    NL, NB, H = 2, 24, 2
    order = np.random.default_rng(6).permutation(NB)
    cache = PagedCache(NL, NB, B, H, d, "fp8", order, act_dtype=act)
    kref, vref = empty_pools(NL, NB, H, B, d, "fp8")
    sref = empty_scales(NL, NB, H, B)
    rng = np.random.default_rng(7)
    s = cache.add()
    n = 3 * B + 5
    slots, _ = cache.reserve([s], [n])
    slots = slots.copy()
    slots[9] = -1                                            # a skipped row
    for layer in range(NL):
        k = special_rows(rng, n, H, d, act)
        v = sv.narrow(rng.standard_normal((n, H, d)).astype(np.float32) * 0.3, act)
        cache.append(layer, dev(k, act), dev(v, act), torch.from_numpy(slots).cuda())
        append_rows_fp8(kref, vref, sref, layer, slots, k, v, act)
    child = cache.fork(s)
    _, cow = cache.reserve([child], [1])
    assert len(cow) == 1
    cache.copy_blocks(cow)
    copy_blocks(kref, vref, cow)
    copy_scales(sref, cow)
    torch.cuda.synchronize()
    assert np.array_equal(host(cache.k_pool), kref) and np.array_equal(host(cache.v_pool), vref)
    assert np.array_equal(host(cache.scales), sref)


def test_swap_round_trip_bit_exact():
    NL, NB, B, H = 3, 20, 16, 2
    cache = PagedCache(NL, NB, B, H, D, "fp8", np.arange(NB), act_dtype="f16")
    kref, vref = empty_pools(NL, NB, H, B, D, "fp8")
    sref = empty_scales(NL, NB, H, B)
    rng = np.random.default_rng(9)
    s = cache.add()
    slots, _ = cache.reserve([s], [40])
    for layer in range(NL):
        k = sv.narrow(rng.standard_normal((40, H, D)).astype(np.float32), "f16")
        v = sv.narrow(rng.standard_normal((40, H, D)).astype(np.float32), "f16")
        cache.append(layer, dev(k, "f16"), dev(v, "f16"), torch.from_numpy(slots).cuda())
        append_rows_fp8(kref, vref, sref, layer, slots, k, v, "f16")
    _, table = cache.info(s)
    nbytes = pa.pa_swap_bytes(cache.pool, s)
    assert nbytes == 3 * NL * 2 * H * B * (D + 1)
    buf = torch.empty(nbytes, dtype=torch.uint8, pin_memory=True)
    pa.pa_swap_out(cache.pool, s, buf)
    torch.cuda.synchronize()
    assert np.array_equal(buf.numpy(), swap_buffer_fp8(kref, vref, sref, table))
    cache.k_pool.zero_()
    cache.scales.zero_()
    other = cache.add()
    cache.reserve([other], [16])                             # take a block so the sequence moves
    pa.pa_swap_in(cache.pool, s, buf)
    _, table2 = cache.info(s)
    torch.cuda.synchronize()
    kp, vp, sc = host(cache.k_pool), host(cache.v_pool), host(cache.scales)
    for b_old, b_new in zip(table, table2):
        assert np.array_equal(kp[:, b_new], kref[:, b_old]) and np.array_equal(vp[:, b_new], vref[:, b_old])
        assert np.array_equal(sc[:, b_new], sref[:, b_old])


# ------------------------------------------------------------------ decode
@pytest.mark.parametrize("act", ["f16", "bf16"])
@pytest.mark.parametrize("B", [16, 32])
@pytest.mark.parametrize("hq,hkv", [(4, 4), (8, 4), (8, 2), (32, 4), (32, 8), (16, 8), (12, 6)])
def test_decode_shapes(act, B, hq, hkv):
    """Groups of 2 and 4 run several KV heads per CTA (4, 2, or 2 with unused columns for
    6 KV heads); groups of 1 and 8 one head per CTA."""
    c = Fp8Case([7, 40, 300, 65], B=B, hq=hq, hkv=hkv, act=act, seed=3)
    ref = c.oracle()
    check_close(c.run(0), ref, "f32", act, "fp8 shapes")
    check_close(c.run(2 * B), ref, "f32", act, "fp8 shapes split")
    check_close(c.run(0, out=act), ref, act, act, "fp8 shapes native out")


@pytest.mark.parametrize("split", [0, 16, 512])
def test_decode_block_and_split_boundaries(split):
    lens = [1, 15, 16, 17, 31, 32, 33, 511, 512, 513, 1023, 1024, 1025, 2047, 2048, 2049]
    c = Fp8Case(lens, seed=1)
    check_close(c.run(split), c.oracle(), "f32", "bf16", f"fp8 split {split}")


def test_single_token_returns_its_dequantised_value():
    """One token: the output is that token's dequantised value row.  Not bit-exact: the
    output and the denominator keep separate running references (max of s + X_v and of
    s), and the final factor 2^(m_o - m) comes from an fp32 difference of the two, so it
    may be off by an ulp of the score, a relative 2^-20 at most here."""
    c = Fp8Case([1, 1, 1], hq=4, hkv=2, act="f16", seed=2)
    out = c.run()
    for i in range(3):
        vc, vs = quantize(c.v[i], "f16")
        val = F.dequantize(vc, vs)[0]
        for h in range(4):
            np.testing.assert_allclose(out[i, h], val[h // 2], rtol=2.0 ** -20, atol=0)


@pytest.mark.parametrize("B", [16, 32])
def test_unused_slots_holding_nan_codes_do_not_leak(B):
    """Never-written slots hold NaN codes (0x7F) and the largest scale byte."""
    lens = [1, 5, 17, 31, 33, 100, 511]
    c = Fp8Case(lens, B=B, fill=(0x7F, 255), seed=8)
    ref = c.oracle()
    for split in (0, 2 * B):
        out = c.run(split)
        assert np.isfinite(out).all()
        check_close(out, ref, "f32", "bf16", f"nan codes split {split}")


@pytest.mark.parametrize("act,q_scale", [("bf16", 1e-6), ("bf16", 3e5), ("f16", 1e-3), ("f16", 200.0)])
def test_query_magnitudes(act, q_scale):
    """The query is prescaled by a power of two before it is rounded to fp16, so tiny and
    (for bf16) beyond-fp16 queries keep their bits; the scores then are huge or flat."""
    c = Fp8Case([300, 47, 1000], act=act, q_scale=q_scale / 8, seed=4)
    ref = c.oracle()
    for split in (0, 64):
        out = c.run(split)
        assert np.isfinite(out).all()
        check_close(out, ref, "f32", act, f"q scale {q_scale}")


def test_row_scales_spanning_many_octaves():
    """Value rows whose magnitudes grow by 2^40 along the sequence (and keys that shrink):
    the value-exponent reference moves up tile after tile and rescales the output."""
    def grow(i, L):
        mag = np.exp2(np.linspace(-20, 20, L))[:, None, None]
        return np.random.default_rng(30 + i).standard_normal((L, 2, D)) * mag

    def shrink(i, L):
        mag = np.exp2(np.linspace(4, -30, L))[:, None, None]
        return np.random.default_rng(40 + i).standard_normal((L, 2, D)) * mag

    c = Fp8Case([700, 64, 2100], act="bf16", k_rows=shrink, v_rows=grow, seed=5)
    ref = c.oracle()
    scale = np.abs(ref).max(axis=-1, keepdims=True)
    for split in (0, 128):
        out = c.run(split)
        err = np.abs(out - ref) / np.maximum(scale, 1e-30)
        assert err.max() < 1e-5, err.max()                   # relative to each head's output range


def contiguous_pool(rows, B):
    """[L][heads][d] rows -> [blocks][heads][B][d] with an identity table, zero padded."""
    L = rows.shape[0]
    pad = np.zeros((-L % B,) + rows.shape[1:], rows.dtype)
    return np.ascontiguousarray(np.concatenate([rows, pad]).reshape((-1, B) + rows.shape[1:]).swapaxes(1, 2))


def test_quantisation_error_against_the_unquantised_oracle():
    """Context, not parity: the FP8 cache's attention stays close to the bf16 cache's.
    Each cached element moves by at most 2^-4 of itself (half a quantum of a 3-bit
    mantissa), so the value part of the output moves by at most 2^-4 max|v|; the key
    part perturbs the weights.  Checked: max error under 2^-4 max|v|, and an RMS error
    of a few percent of the output's RMS."""
    c = Fp8Case([300, 1000, 77], hq=32, hkv=8, act="bf16", seed=6)
    out = c.run()
    exact = [oracle.paged_decode(contiguous_pool(c.k[i], 16), contiguous_pool(c.v[i], 16), "bf16",
                                 np.arange(-(-L // 16), dtype=np.int32)[None], [L], c.q[i:i + 1],
                                 1.0 / math.sqrt(D))[0] for i, L in enumerate(c.lens)]
    exact = np.stack(exact)
    vmax = max(np.abs(oracle.widen(v, "bf16")).max() for v in c.v)
    assert np.abs(out - exact).max() < 2.0 ** -4 * vmax
    rms = np.sqrt(np.mean((out - exact) ** 2)) / np.sqrt(np.mean(exact ** 2))
    assert rms < 0.05, rms


def test_fp8_pool_rejections():
    c = Fp8Case([40])
    q = dev(c.q, "bf16")
    before = pa.pa_launch_count()
    with pytest.raises(pa.PaError) as e:                     # out dtype neither f32 nor bf16
        pa.pa_decode_attention(c.cache.pool, 0, q, torch.empty((1, 8, D), dtype=torch.float16, device="cuda"),
                               c.tables, c.lens_dev, 0.1)
    assert e.value.status == pa.PA_ERR_INVALID_ARG
    qs = torch.tensor([0, 1], dtype=torch.int32, device="cuda")
    with pytest.raises(pa.PaError) as e:                     # no tensor-core prefill over FP8
        pa.pa_prefill_attention(c.cache.pool, 0, q, torch.empty((1, 8, D), device="cuda"), c.tables, c.lens_dev,
                                qs, 1, 0.1)
    assert e.value.status == pa.PA_ERR_UNSUPPORTED
    k = torch.zeros((1, 4, 2, 16, D), dtype=torch.uint8, device="cuda")
    p = pa.pa_pool_create(1, 4, 16, 2, D, "fp8", k, k.clone(), act_dtype="bf16")
    with pytest.raises(pa.PaError) as e:                     # scales never attached
        pa.pa_decode_attention(p, 0, q, torch.empty((1, 8, D), device="cuda"), c.tables[:, :1], c.lens_dev, 0.1)
    assert e.value.status == pa.PA_ERR_INVALID_ARG
    pa.pa_pool_destroy(p)
    with pytest.raises(pa.PaError) as e:                     # FP8 needs a 16-bit activation type
        pa.pa_pool_create(1, 4, 16, 2, D, "fp8", act_dtype="f32")
    assert e.value.status == pa.PA_ERR_INVALID_ARG
    assert pa.pa_launch_count() == before


# ------------------------------------------------------------------ full sizes
@pytest.mark.slow
@pytest.mark.parametrize("split", [2048, 4096])
def test_continuous_batch_fp8_full_size_sampled(split):
    """256 sequences, 64 steps, FP8 cache, bf16 output, split 4096 (the benchmark's
    default) and 2048; sampled sequences against the oracle
    over their regenerated, oracle-quantised histories, and sampled cache rows bit-exact
    against the oracle's quantiser."""
    from oracle_replay import sequence_attention_fp8
    from paged_kv_cache_403_b200.runners import ContinuousBatch
    from synthetic import workloads as wl
    r = wl.continuous_batch()
    sh = r["shape"]
    cb = ContinuousBatch(r, kv_fp8=True)
    rng = np.random.default_rng(0)
    for t in range(64):
        rec = cb.step(split_tokens=split)
        if t in (0, 33, 63):
            lens = rec.lens
            picks = set(rng.choice(len(lens), size=5, replace=False).tolist())
            picks |= {int(np.argmax(lens)), int(np.argmin(lens))}
            out = rec.outputs[0].detach().cpu().to(torch.float64).numpy()
            for i in sorted(picks):
                ref = sequence_attention_fp8(sh, r["seed"], 0, rec.uids[i], int(lens[i]), rec.uids[i],
                                             int(rec.positions[i]))
                check_close(out[i], ref, "bf16", "bf16", f"step {t} seq {i}")
    kp, sc = host(cb.cache.k_pool), host(cb.cache.scales)
    for i in range(0, 256, 37):
        L = int(rec.lens[i])
        blk, off = int(rec.tables[i][(L - 1) // 16]), (L - 1) % 16
        row = sv.rows(sv.KIND_K, r["seed"], 0, [rec.uids[i]], [L - 1], 8, 128, sh.kv_scale, "bf16")
        codes, scales = quantize(row, "bf16")
        assert np.array_equal(kp[0, blk, :, off], codes[0]) and np.array_equal(sc[0, blk, :, 0, off], scales[0])


@pytest.mark.slow
@pytest.mark.parametrize("split", [2048, 4096])
def test_large_pool_fp8_sampled(split):
    """384 sequences, lognormal lengths, 32 layers, block 32, FP8 cache (~50 GB), split 4096
    (the benchmark's default) and 2048; layers 0 and 31 sampled against the oracle."""
    from oracle_replay import sequence_attention_fp8
    from paged_kv_cache_403_b200.runners import run_static
    from synthetic import workloads as wl
    r = wl.large_pool(block_size=32)
    sh = r["shape"]
    cache, _, rec = run_static(r, split_tokens=split, keep_layers={0, 31}, kv_fp8=True)
    lens = rec.lens
    picks = [int(np.argmax(lens)), int(np.argmin(lens)), int(np.argsort(lens)[len(lens) // 2])]
    picks += [int(i) for i in np.nonzero(lens > 4096)[0][:2]]
    for layer in (0, 31):
        out = rec.outputs[layer].detach().cpu().to(torch.float64).numpy()
        for i in picks:
            ref = sequence_attention_fp8(sh, r["seed"], layer, rec.uids[i], int(lens[i]), rec.uids[i],
                                         int(rec.positions[i]))
            check_close(out[i], ref, "f16", "f16", f"layer {layer} seq {i}")
    del cache
    torch.cuda.empty_cache()
