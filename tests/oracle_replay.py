"""Replays a workload on the oracle side (test helper; imports only oracle/ and synthetic/).

Inputs are regenerated on the host from the seeded generators; nothing here reads
data produced by the CUDA path.  Expected outputs come from oracle.paged_decode.
"""
from __future__ import annotations

import math

import numpy as np

import oracle
from oracle.block_manager import BlockManagerModel
from oracle.cache_model import append_rows, copy_blocks, empty_pools
from synthetic import values as sv

TOL = {"f32": 1e-5, "f16": 2e-3, "bf16": 2e-3}   # max-abs, fp32 output
ULP = {"f32": 2.0 ** -23, "f16": 2.0 ** -10, "bf16": 2.0 ** -7}


def narrow_bound(ref: np.ndarray, out_dtype: str, kv_dtype: str) -> np.ndarray:
    """Allowed |gpu - oracle| when the result is stored in `out_dtype`: the arithmetic
    tolerance plus half an ulp of the output format at the reference value."""
    mag = np.maximum(np.abs(ref), 2.0 ** -14)
    ulp = ULP[out_dtype] * 2.0 ** np.floor(np.log2(mag))
    return TOL[kv_dtype] + (0.5 * ulp if out_dtype != "f32" else 0.0)


def check_close(gpu: np.ndarray, ref: np.ndarray, out_dtype: str, kv_dtype: str, what: str = ""):
    err = np.abs(gpu.astype(np.float64) - ref)
    bound = narrow_bound(ref, out_dtype, kv_dtype)
    bad = err > bound
    assert not bad.any(), (f"{what}: {bad.sum()} elements over tolerance; max err {err.max():.3g} "
                           f"at {np.unravel_index(err.argmax(), err.shape)}")
    return float(err.max())


class OracleRun:
    """Oracle-side mirror: block manager model + host pools + fp64 attention."""

    def __init__(self, shape, order, seed):
        self.shape, self.seed = shape, seed
        self.bm = BlockManagerModel(shape.num_blocks, shape.block_size, order)
        self.k, self.v = empty_pools(shape.num_layers, shape.num_blocks, shape.num_kv_heads,
                                     shape.block_size, shape.head_dim, shape.dtype)

    def rows(self, kind, layer, uids, toks):
        s = self.shape
        heads = s.num_q_heads if kind == sv.KIND_Q else s.num_kv_heads
        scale = s.q_scale if kind == sv.KIND_Q else s.kv_scale
        return sv.rows(kind, self.seed, layer, uids, toks, heads, s.head_dim, scale, s.dtype)

    def write(self, slots, uids, toks):
        for layer in range(self.shape.num_layers):
            append_rows(self.k, self.v, layer, slots, self.rows(sv.KIND_K, layer, uids, toks),
                        self.rows(sv.KIND_V, layer, uids, toks))

    def prefill(self, sids, uids, lens):
        slots, cow = self.bm.reserve_slots(sids, lens)
        assert not cow
        self.write(slots, np.repeat(uids, lens), np.concatenate([np.arange(L) for L in lens]))
        return slots

    def decode_step(self, sids, uids, max_blocks, layers=None):
        positions = [self.bm.length(s) for s in sids]
        slots, cow = self.bm.reserve_slots(sids, [1] * len(sids))
        copy_blocks(self.k, self.v, cow)
        self.write(slots, uids, positions)
        tables, lens = self.bm.dense_tables(sids, max_blocks)
        tables = np.array(tables, np.int32)
        lens = np.array(lens, np.int32)
        outs = {}
        for layer in (range(self.shape.num_layers) if layers is None else layers):
            q = self.rows(sv.KIND_Q, layer, uids, positions)
            outs[layer] = oracle.paged_decode(self.k[layer], self.v[layer], self.shape.dtype, tables, lens, q,
                                              1.0 / math.sqrt(self.shape.head_dim))
        return dict(slots=np.array(slots, np.int64), cow=np.array(cow, np.int32).reshape(-1, 2),
                    tables=tables, lens=lens, outputs=outs, positions=np.array(positions))


def sequence_attention(shape, seed, layer, uid, length, q_uid, q_pos, writer=None):
    """fp64 attention of one query against one sequence's regenerated history.

    writer(pos) -> (uid, token) names who wrote position pos (default: uid, pos).
    The history is laid into a contiguous pool with an identity block table.
    """
    B, hkv, d = shape.block_size, shape.num_kv_heads, shape.head_dim
    pos = np.arange(length)
    if writer is None:
        wu, wt = np.full(length, uid), pos
    else:
        wu, wt = map(np.array, zip(*[writer(p) for p in pos]))
    k = sv.rows(sv.KIND_K, seed, layer, wu, wt, hkv, d, shape.kv_scale, shape.dtype)
    v = sv.rows(sv.KIND_V, seed, layer, wu, wt, hkv, d, shape.kv_scale, shape.dtype)
    nblk = -(-length // B)
    pad = nblk * B - length
    if pad:
        k = np.concatenate([k, np.zeros((pad, hkv, d), k.dtype)])
        v = np.concatenate([v, np.zeros((pad, hkv, d), v.dtype)])
    kp = np.ascontiguousarray(k.reshape(nblk, B, hkv, d).transpose(0, 2, 1, 3))
    vp = np.ascontiguousarray(v.reshape(nblk, B, hkv, d).transpose(0, 2, 1, 3))
    q = sv.rows(sv.KIND_Q, seed, layer, [q_uid], [q_pos], shape.num_q_heads, d, shape.q_scale, shape.dtype)
    return oracle.paged_decode(kp, vp, shape.dtype, np.arange(nblk, dtype=np.int32)[None], np.array([length]),
                               q, 1.0 / math.sqrt(d))[0]


def sequence_attention_fp8(shape, seed, layer, uid, length, q_uid, q_pos):
    """As sequence_attention, over an FP8 cache: the regenerated rows (in the workload's
    type) are quantised by the oracle's own quantiser, then attended in fp64."""
    from oracle.fp8 import quantize_rows
    B, hkv, d = shape.block_size, shape.num_kv_heads, shape.head_dim
    pos = np.arange(length)
    wu = np.full(length, uid)
    kc, ks = quantize_rows(oracle.widen(sv.rows(sv.KIND_K, seed, layer, wu, pos, hkv, d, shape.kv_scale, shape.dtype),
                                        shape.dtype).astype(np.float32))
    vc, vs = quantize_rows(oracle.widen(sv.rows(sv.KIND_V, seed, layer, wu, pos, hkv, d, shape.kv_scale, shape.dtype),
                                        shape.dtype).astype(np.float32))
    nblk = -(-length // B)
    pad = nblk * B - length
    lay = lambda a: np.ascontiguousarray(np.concatenate([a, np.zeros((pad,) + a.shape[1:], a.dtype)])  # noqa: E731
                                         .reshape((nblk, B) + a.shape[1:]).swapaxes(1, 2))
    q = sv.rows(sv.KIND_Q, seed, layer, [q_uid], [q_pos], shape.num_q_heads, d, shape.q_scale, shape.dtype)
    return oracle.paged_decode_fp8(lay(kc), lay(vc), lay(ks), lay(vs), np.arange(nblk, dtype=np.int32)[None],
                                   np.array([length]), q, shape.dtype, 1.0 / math.sqrt(d))[0]


STORAGE = {"f32": np.float32, "f16": np.float16, "bf16": np.uint16}


def histories_attention(shape, seed, layer, uids, lens, q_positions, rows=None):
    """fp64 attention of every sequence of a batch against its whole regenerated history
    (position p of sequence i written by uid uids[i] as token p), in one oracle call.

    rows(kind, uids, toks) -> host storage rows [len][num_kv_heads][head_dim]; by default
    the host generator.  Each history is laid into its own run of blocks of a contiguous
    host pool with an identity-like block table, so this checks the GPU's gather through
    its own shuffled tables against plain contiguous reads.
    """
    B, hkv, d = shape.block_size, shape.num_kv_heads, shape.head_dim
    if rows is None:
        def rows(kind, u, t):
            return sv.rows(kind, seed, layer, u, t, hkv, d, shape.kv_scale, shape.dtype)
    lens = np.asarray(lens, np.int64)
    nblk = -(-lens // B)
    first = np.concatenate([[0], np.cumsum(nblk)[:-1]]).astype(np.int64)
    kp = np.zeros((int(nblk.sum()), hkv, B, d), STORAGE[shape.dtype])
    vp = np.zeros_like(kp)
    for i, (uid, L) in enumerate(zip(uids, lens)):
        L = int(L)
        toks = np.arange(L)
        u = np.full(L, int(uid))
        for kind, pool in ((sv.KIND_K, kp), (sv.KIND_V, vp)):
            r = np.asarray(rows(kind, u, toks))
            pad = int(nblk[i]) * B - L
            if pad:
                r = np.concatenate([r, np.zeros((pad, hkv, d), r.dtype)])
            pool[first[i]:first[i] + nblk[i]] = r.reshape(int(nblk[i]), B, hkv, d).transpose(0, 2, 1, 3)
    tables = np.full((len(lens), int(nblk.max())), -1, np.int32)
    for i in range(len(lens)):
        tables[i, :nblk[i]] = first[i] + np.arange(nblk[i])
    q = sv.rows(sv.KIND_Q, seed, layer, np.asarray(uids), np.asarray(q_positions), shape.num_q_heads, d,
                shape.q_scale, shape.dtype)
    return oracle.paged_decode(kp, vp, shape.dtype, tables, lens.astype(np.int32), q, 1.0 / math.sqrt(d))


def device_generated_rows(shape, seed, layer):
    """rows() for histories_attention drawn by the device implementation of the seeded
    input generator (synthetic/csrc/synth_gen.cu, bit-identical to the host one and
    tested against it), then copied to the host: the same inputs, made fast enough to
    regenerate whole full-size batches."""
    import torch
    from synthetic import gpu as sgpu
    dt = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}[shape.dtype]

    def rows(kind, u, t):
        out = torch.empty((len(u), shape.num_kv_heads, shape.head_dim), dtype=dt, device="cuda")
        sgpu.fill_rows(out, kind, seed, layer, torch.from_numpy(np.asarray(u, np.int32)).cuda(),
                       torch.from_numpy(np.asarray(t, np.int32)).cuda(), shape.kv_scale, shape.dtype)
        h = out.cpu()
        return h.view(torch.int16).numpy().view(np.uint16) if dt == torch.bfloat16 else h.numpy()
    return rows
