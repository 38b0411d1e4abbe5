"""Pins for the oracle's fp64 paged decode attention (CPU only).

Each pin ties the oracle to something other than itself: the number formats'
definitions (exhaustive), closed forms of softmax attention, hand-expanded
brute force, placement invariance from the pages' block-table example, and
torch's scaled_dot_product_attention in float64 as an independent library
routine.  The planted-mistake tests compile mutated copies of oracle.c and
check that these pins reject every mutant.
"""
import math
import os
import subprocess
import tempfile

import numpy as np
import pytest
import torch

import oracle
from synthetic import values as sv

ORACLE_C = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")


def contiguous_to_pool(kv, block_size, order=None, num_blocks=None):
    """Lay one sequence's [L][Hkv][d] rows into blocks; returns (pool, table)."""
    L, hkv, d = kv.shape
    nblk = -(-L // block_size)
    num_blocks = num_blocks or nblk
    order = list(range(nblk)) if order is None else list(order)
    pool = np.zeros((num_blocks, hkv, block_size, d), kv.dtype)
    for j in range(L):
        pool[order[j // block_size], :, j % block_size, :] = kv[j]
    return pool, np.array(order[:nblk], np.int32)


def run_one(k, v, q, scale, block_size=16, order=None, num_blocks=None, dtype="f32",
            fn=None):
    """Oracle on a single sequence given contiguous K/V [L][Hkv][d] and q [Hq][d]."""
    kp, table = contiguous_to_pool(k, block_size, order, num_blocks)
    vp, _ = contiguous_to_pool(v, block_size, order, num_blocks)
    fn = fn or oracle.paged_decode
    return fn(kp, vp, dtype, table[None, :], np.array([k.shape[0]], np.int32), q[None], scale)[0]


# ---------------------------------------------------------------- number formats
def test_half_decoder_exhaustive():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    got = oracle.widen(bits.view(np.float16), "f16")
    ref = bits.view(np.float16).astype(np.float64)
    assert np.array_equal(got, ref, equal_nan=True)


def test_bf16_decoder_exhaustive():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    got = oracle.widen(bits, "bf16")
    ref = torch.from_numpy(bits.astype(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(got, ref, equal_nan=True)


# ---------------------------------------------------------------- closed forms
def test_single_token_returns_its_value_exactly():
    rng = np.random.default_rng(0)
    k = rng.standard_normal((1, 2, 8)).astype(np.float32)
    v = rng.standard_normal((1, 2, 8)).astype(np.float32)
    q = rng.standard_normal((4, 8)).astype(np.float32)
    o = run_one(k, v, q, 0.3)
    for h in range(4):
        assert np.array_equal(o[h], v[0, h // 2].astype(np.float64))


def test_equal_keys_give_mean_of_values():
    rng = np.random.default_rng(1)
    L = 37
    k = np.repeat(rng.standard_normal((1, 1, 16)).astype(np.float32), L, axis=0)
    v = rng.standard_normal((L, 1, 16)).astype(np.float32)
    q = rng.standard_normal((1, 16)).astype(np.float32)
    o = run_one(k, v, q, 1.0)
    np.testing.assert_allclose(o[0], v[:, 0].astype(np.float64).mean(axis=0), rtol=0, atol=1e-13)


def test_zero_query_gives_mean_of_values():
    rng = np.random.default_rng(2)
    L = 53
    k = rng.standard_normal((L, 1, 16)).astype(np.float32)
    v = rng.standard_normal((L, 1, 16)).astype(np.float32)
    q = np.zeros((1, 16), np.float32)
    o = run_one(k, v, q, 1.0)
    np.testing.assert_allclose(o[0], v[:, 0].astype(np.float64).mean(axis=0), rtol=0, atol=1e-13)


def test_dominant_key_selects_its_value():
    rng = np.random.default_rng(3)
    L, d = 40, 16
    q = rng.standard_normal((1, d)).astype(np.float32)
    k = (rng.standard_normal((L, 1, d)) * 0.01).astype(np.float32)
    k[17, 0] = q[0] * 10.0           # score margin ~ 10*|q|^2 ~ 160 >> log(L)
    v = rng.standard_normal((L, 1, d)).astype(np.float32)
    o = run_one(k, v, q, 1.0)
    np.testing.assert_allclose(o[0], v[17, 0].astype(np.float64), rtol=0, atol=1e-12)


def test_large_scores_do_not_overflow():
    # scores of order 1e3: exp without subtracting the maximum would overflow
    rng = np.random.default_rng(4)
    L, d = 20, 8
    k = (rng.standard_normal((L, 1, d)) * 30).astype(np.float32)
    v = rng.standard_normal((L, 1, d)).astype(np.float32)
    q = (rng.standard_normal((1, d)) * 30).astype(np.float32)
    o = run_one(k, v, q, 1.0)
    z = (k[:, 0].astype(np.float64) @ q[0].astype(np.float64))
    w = np.exp(z - z.max())
    ref = (w[:, None] * v[:, 0].astype(np.float64)).sum(0) / w.sum()
    assert np.all(np.isfinite(o))
    np.testing.assert_allclose(o[0], ref, rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("L", [1, 2, 3])
def test_brute_force_hand_expanded(L):
    """d = 2, one head: softmax written out term by term with math.exp."""
    rng = np.random.default_rng(10 + L)
    k = rng.standard_normal((L, 1, 2)).astype(np.float32)
    v = rng.standard_normal((L, 1, 2)).astype(np.float32)
    q = rng.standard_normal((1, 2)).astype(np.float32)
    scale = 0.7
    q0, q1 = float(q[0, 0]), float(q[0, 1])
    e = [math.exp(scale * (q0 * float(k[j, 0, 0]) + q1 * float(k[j, 0, 1]))) for j in range(L)]
    den = sum(e)
    ref = [sum(e[j] * float(v[j, 0, c]) for j in range(L)) / den for c in range(2)]
    o = run_one(k, v, q, scale, block_size=2)
    np.testing.assert_allclose(o[0], ref, rtol=1e-13, atol=1e-15)


# ---------------------------------------------------------------- paging
def test_pages_block_table_example_matches_contiguous(golden_dir):
    """50 tokens in physical blocks 12, 87, 301, 44 == the same tokens placed contiguously."""
    import json
    g = json.load(open(os.path.join(golden_dir, "memory_example.json")))["fifty_tokens"]
    rng = np.random.default_rng(5)
    L, hkv, hq, d = g["tokens"], 2, 4, 16
    k = rng.standard_normal((L, hkv, d)).astype(np.float32)
    v = rng.standard_normal((L, hkv, d)).astype(np.float32)
    q = rng.standard_normal((hq, d)).astype(np.float32)
    phys = g["physical_blocks"]
    assert len(phys) == g["blocks"] == -(-L // 16)
    o_paged = run_one(k, v, q, 0.25, order=phys, num_blocks=400)
    o_contig = run_one(k, v, q, 0.25)
    o_shuffled = run_one(k, v, q, 0.25, order=list(np.random.default_rng(6).permutation(64)),
                         num_blocks=64)
    assert np.array_equal(o_paged, o_contig)
    assert np.array_equal(o_shuffled, o_contig)


def test_matches_torch_sdpa_float64_gqa_ragged():
    """Several ragged sequences, GQA 4, shuffled pool, vs torch SDPA in float64."""
    rng = np.random.default_rng(7)
    B, hq, hkv, d, scale = 16, 8, 2, 32, 1 / math.sqrt(32)
    lens = [1, 15, 16, 17, 70]
    nb = 64
    order = rng.permutation(nb)
    kp = np.zeros((nb, hkv, B, d), np.float32)
    vp = np.zeros_like(kp)
    tables = np.full((len(lens), 8), -1, np.int32)
    ks, vs = [], []
    nxt = 0
    for s, L in enumerate(lens):
        k = rng.standard_normal((L, hkv, d)).astype(np.float32)
        v = rng.standard_normal((L, hkv, d)).astype(np.float32)
        ks.append(k)
        vs.append(v)
        for b in range(-(-L // B)):
            tables[s, b] = order[nxt]
            nxt += 1
        for j in range(L):
            kp[tables[s, j // B], :, j % B] = k[j]
            vp[tables[s, j // B], :, j % B] = v[j]
    q = rng.standard_normal((len(lens), hq, d)).astype(np.float32)
    out = oracle.paged_decode(kp, vp, "f32", tables, np.array(lens, np.int32), q, scale)
    for s, L in enumerate(lens):
        qt = torch.from_numpy(q[s]).double()[None, :, None, :]              # [1][hq][1][d]
        kt = torch.from_numpy(ks[s]).double().permute(1, 0, 2)[None]       # [1][hkv][L][d]
        vt = torch.from_numpy(vs[s]).double().permute(1, 0, 2)[None]
        ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=scale,
                                                               enable_gqa=True)
        np.testing.assert_allclose(out[s], ref[0, :, 0].numpy(), rtol=1e-12, atol=1e-13)


@pytest.mark.parametrize("dtype", ["f16", "bf16"])
def test_narrow_types_read_exactly(dtype):
    """fp16 / bf16 pools: the oracle equals SDPA on the exactly widened values."""
    rng = np.random.default_rng(8)
    L, hkv, hq, d = 33, 1, 2, 16
    k = sv.narrow(rng.standard_normal((L, hkv, d)).astype(np.float32), dtype)
    v = sv.narrow(rng.standard_normal((L, hkv, d)).astype(np.float32), dtype)
    q = sv.narrow(rng.standard_normal((hq, d)).astype(np.float32), dtype)
    o = run_one(k, v, q, 0.25, dtype=dtype)
    kt = torch.from_numpy(sv.to_float64(k, dtype)).permute(1, 0, 2)[None]
    vt = torch.from_numpy(sv.to_float64(v, dtype)).permute(1, 0, 2)[None]
    qt = torch.from_numpy(sv.to_float64(q, dtype))[None, :, None, :]
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=0.25, enable_gqa=True)
    np.testing.assert_allclose(o, ref[0, :, 0].numpy(), rtol=1e-12, atol=1e-13)


def test_rejects_invalid_tables():
    kp = np.zeros((4, 1, 16, 8), np.float32)
    q = np.zeros((1, 1, 8), np.float32)
    with pytest.raises(ValueError):
        oracle.paged_decode(kp, kp, "f32", np.array([[9]], np.int32), np.array([3], np.int32), q, 1.0)
    with pytest.raises(ValueError):
        oracle.paged_decode(kp, kp, "f32", np.array([[0]], np.int32), np.array([17], np.int32), q, 1.0)
    with pytest.raises(ValueError):
        oracle.paged_decode(kp, kp, "f32", np.array([[0]], np.int32), np.array([0], np.int32), q, 1.0)


# ---------------------------------------------------------------- planted mistakes
MUTANTS = {
    "gqa_modulo": ("const int g = h / group;\n        const int L = lens[s];",
                   "const int g = h % num_kv_heads;\n        const int L = lens[s];"),
    "gather_swapped": ("j / block_size];\n            size_t row", "j % block_size];\n            size_t row"),
    "row_offset": ("size_t row = (((size_t)blk * num_kv_heads + g) * block_size + j % block_size) * head_dim;",
                   "size_t row = (((size_t)blk * num_kv_heads + g) * block_size + j / block_size) * head_dim;"),
    "no_scale": ("acc += qh[i] * K[(size_t)j * head_dim + i];\n            z[j] = scale * acc;",
                 "acc += qh[i] * K[(size_t)j * head_dim + i];\n            z[j] = acc;"),
    "no_max_shift": ("for (int j = 0; j < L; ++j) {\n            z[j] = exp(z[j] - zmax);",
                     "for (int j = 0; j < L; ++j) {\n            z[j] = exp(z[j]);"),
    "k_transposed": ("acc += qh[i] * K[(size_t)j * head_dim + i];",
                     "acc += qh[i] * K[(size_t)i * head_dim + j % head_dim];"),
    "v_for_k": ("K[(size_t)j * head_dim + i] = load_elem(k_pool", "K[(size_t)j * head_dim + i] = load_elem(v_pool"),
    "half_bias": ("expo - 25", "expo - 24"),
    "no_normalise": ("o[i] = acc / denom;", "o[i] = acc;"),
}


def _compile_mutant(name):
    src = open(ORACLE_C).read()
    old, new = (x.replace("\\n", "\n") for x in MUTANTS[name])
    assert src.count(old) == 1, name
    tmpd = tempfile.mkdtemp()
    c = os.path.join(tmpd, "m.c")
    so = os.path.join(tmpd, "m.so")
    open(c, "w").write(src.replace(old, new))
    subprocess.run(["gcc", "-std=c11", "-O1", "-fPIC", "-shared", "-o", so, c, "-lm"], check=True)
    return so


def _mutant_decode(so):
    import ctypes
    L = ctypes.CDLL(so)
    L.oracle_paged_decode.restype = ctypes.c_int
    L.oracle_paged_decode.argtypes = oracle.lib().oracle_paged_decode.argtypes

    def fn(k_layer, v_layer, dtype, tables, lens, q, scale, n_threads=1):
        k = np.ascontiguousarray(k_layer)
        v = np.ascontiguousarray(v_layer)
        t = np.ascontiguousarray(tables, dtype=np.int32)
        ln = np.ascontiguousarray(lens, dtype=np.int32)
        qq = np.ascontiguousarray(q)
        out = np.empty(qq.shape, np.float64)
        p = lambda a: a.ctypes.data_as(ctypes.c_void_p)  # noqa: E731
        rc = L.oracle_paged_decode(p(k), p(v), {"f32": 0, "f16": 1, "bf16": 2}[dtype],
                                   k.shape[0], k.shape[2], k.shape[1], k.shape[3], p(t),
                                   t.shape[1], p(ln), t.shape[0], p(qq), qq.shape[1],
                                   float(scale), p(out), 1)
        if rc:
            raise ValueError
        return out
    return fn


def _pins_pass(fn):
    """A compact battery of the pins above, run against an arbitrary implementation."""
    rng = np.random.default_rng(99)
    try:
        # SDPA comparison, GQA, multi-block, shuffled placement, fp32 and fp16
        for dtype in ("f32", "f16"):
            L, hkv, hq, d, B = 41, 2, 4, 8, 16
            k = sv.narrow((rng.standard_normal((L, hkv, d)) * 3).astype(np.float32), dtype)
            v = sv.narrow(rng.standard_normal((L, hkv, d)).astype(np.float32), dtype)
            q = sv.narrow(rng.standard_normal((hq, d)).astype(np.float32), dtype)
            o = run_one(k, v, q, 0.5, block_size=B, order=[5, 2, 7], num_blocks=8, dtype=dtype,
                        fn=fn)
            kt = torch.from_numpy(sv.to_float64(k, dtype)).permute(1, 0, 2)[None]
            vt = torch.from_numpy(sv.to_float64(v, dtype)).permute(1, 0, 2)[None]
            qt = torch.from_numpy(sv.to_float64(q, dtype))[None, :, None, :]
            ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=0.5,
                                                                   enable_gqa=True)
            if not np.allclose(o, ref[0, :, 0].numpy(), rtol=1e-10, atol=1e-12):
                return False
        # large scores
        L, d = 20, 8
        k = (rng.standard_normal((L, 1, d)) * 30).astype(np.float32)
        v = rng.standard_normal((L, 1, d)).astype(np.float32)
        q = (rng.standard_normal((1, d)) * 30).astype(np.float32)
        o = run_one(k, v, q, 1.0, fn=fn)
        z = k[:, 0].astype(np.float64) @ q[0].astype(np.float64)
        w = np.exp(z - z.max())
        ref = (w[:, None] * v[:, 0].astype(np.float64)).sum(0) / w.sum()
        if not np.allclose(o[0], ref, rtol=1e-10, atol=1e-12):
            return False
    except ValueError:
        return False
    return True


def test_pins_accept_the_oracle():
    assert _pins_pass(oracle.paged_decode)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_reject_planted_mistake(name):
    """Run the battery on the mutant in a child process: some mutants read out of
    bounds and crash, which also counts as rejected."""
    import sys
    so = _compile_mutant(name)
    here = os.path.dirname(os.path.abspath(__file__))
    code = ("import sys; sys.path[:0] = [%r, %r]; import test_oracle_attention as t; "
            "sys.exit(0 if t._pins_pass(t._mutant_decode(%r)) else 1)"
            % (here, os.path.dirname(here), so))
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, timeout=300)
    assert r.returncode != 0, f"mutant {name} passed every pin"


def test_whole_batch_helper_matches_per_sequence_helper():
    """The full-size GPU checks attend over a whole batch's regenerated histories in one
    oracle call; each row must equal the per-sequence oracle call bit for bit."""
    from oracle_replay import histories_attention, sequence_attention
    from synthetic import workloads as wl
    r = wl.worked_example()
    sh = r["shape"]
    uids, lens = [3, 9, 1, 4], [70, 17, 33, 1]
    pos = [L - 1 for L in lens]
    batch = histories_attention(sh, r["seed"], 0, uids, lens, pos)
    for i in range(4):
        one = sequence_attention(sh, r["seed"], 0, uids[i], lens[i], uids[i], pos[i])
        assert np.array_equal(batch[i], one)
