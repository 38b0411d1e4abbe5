"""Pins for the oracle's fp64 paged chunked-prefill attention (CPU only).

A chunk is the last C tokens of a sequence; query i sits at position L - C + i and
attends to keys 0..L - C + i.  Pinned against: the decode oracle (C = 1), torch
SDPA in float64 with the bottom-right-aligned causal mask and with is_causal for a
whole prompt, causality itself (future keys do not matter), and planted mutants.
"""
import math
import os
import subprocess
import sys
import tempfile

import numpy as np
import pytest
import torch

import oracle
from synthetic import values as sv

ORACLE_C = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")


def build_case(lens, chunks, hq, hkv, d, B=16, dtype="f32", seed=0, nb_extra=5):
    rng = np.random.default_rng(seed)
    nblk = [-(-L // B) for L in lens]
    nb = sum(nblk) + nb_extra
    order = rng.permutation(nb)
    kp = np.zeros((nb, hkv, B, d), np.float32)
    vp = np.zeros_like(kp)
    tables = np.full((len(lens), max(nblk)), -1, np.int32)
    ks, vs, nxt = [], [], 0
    for s, L in enumerate(lens):
        k = rng.standard_normal((L, hkv, d)).astype(np.float32)
        v = rng.standard_normal((L, hkv, d)).astype(np.float32)
        ks.append(k)
        vs.append(v)
        for b in range(nblk[s]):
            tables[s, b] = order[nxt]
            nxt += 1
        for j in range(L):
            kp[tables[s, j // B], :, j % B] = k[j]
            vp[tables[s, j // B], :, j % B] = v[j]
    q_start = np.concatenate([[0], np.cumsum(chunks)]).astype(np.int32)
    q = rng.standard_normal((q_start[-1], hq, d)).astype(np.float32)
    if dtype != "f32":
        kp, vp, q = sv.narrow(kp, dtype), sv.narrow(vp, dtype), sv.narrow(q, dtype)
        ks = [sv.narrow(k, dtype) for k in ks]
        vs = [sv.narrow(v, dtype) for v in vs]
    return dict(kp=kp, vp=vp, tables=tables, lens=np.array(lens, np.int32), q_start=q_start, q=q, ks=ks,
                vs=vs, dtype=dtype)


def run(c, scale, fn=None):
    fn = fn or oracle.paged_prefill
    return fn(c["kp"], c["vp"], c["dtype"], c["tables"], c["lens"], c["q_start"], c["q"], scale)


def sdpa_reference(c, scale):
    outs = []
    for s, L in enumerate(c["lens"]):
        q0, q1 = c["q_start"][s], c["q_start"][s + 1]
        C = q1 - q0
        if C == 0:
            continue
        qt = torch.from_numpy(sv.to_float64(c["q"][q0:q1], c["dtype"])).permute(1, 0, 2)[None]   # [1][hq][C][d]
        kt = torch.from_numpy(sv.to_float64(c["ks"][s], c["dtype"])).permute(1, 0, 2)[None]      # [1][hkv][L][d]
        vt = torch.from_numpy(sv.to_float64(c["vs"][s], c["dtype"])).permute(1, 0, 2)[None]
        i = torch.arange(C)[:, None]
        j = torch.arange(int(L))[None, :]
        mask = j <= (int(L) - C + i)                       # bottom-right aligned causal mask
        o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=scale,
                                                             enable_gqa=True)
        outs.append(o[0].permute(1, 0, 2).numpy())
    return np.concatenate(outs)


def test_single_query_chunk_equals_decode():
    c = build_case([1, 17, 50, 129], [1, 1, 1, 1], hq=8, hkv=2, d=32)
    pre = run(c, 0.2)
    dec = oracle.paged_decode(c["kp"], c["vp"], "f32", c["tables"], c["lens"], c["q"], 0.2)
    assert np.array_equal(pre, dec)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_matches_sdpa_bottom_right_causal(dtype):
    c = build_case([40, 100, 7, 65], [13, 100, 7, 1], hq=8, hkv=2, d=32, dtype=dtype, seed=1)
    np.testing.assert_allclose(run(c, 0.25), sdpa_reference(c, 0.25), rtol=1e-12, atol=1e-13)


def test_whole_prompt_is_causal_self_attention():
    c = build_case([64], [64], hq=4, hkv=4, d=16, seed=2)
    qt = torch.from_numpy(c["q"].astype(np.float64)).permute(1, 0, 2)[None]
    kt = torch.from_numpy(c["ks"][0].astype(np.float64)).permute(1, 0, 2)[None]
    vt = torch.from_numpy(c["vs"][0].astype(np.float64)).permute(1, 0, 2)[None]
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=True, scale=0.3)
    np.testing.assert_allclose(run(c, 0.3), ref[0].permute(1, 0, 2).numpy(), rtol=1e-12, atol=1e-13)


def test_future_keys_do_not_matter():
    c = build_case([48], [16], hq=2, hkv=1, d=16, seed=3)
    base = run(c, 0.5)
    # change every key and value after position 32 + 4 (query 4 of the chunk)
    for j in range(37, 48):
        blk = c["tables"][0, j // 16]
        c["kp"][blk, :, j % 16] += 5.0
        c["vp"][blk, :, j % 16] -= 3.0
    moved = run(c, 0.5)
    assert np.array_equal(moved[:5], base[:5])           # queries at positions 32..36
    assert not np.allclose(moved[5:], base[5:])


def test_rejects_invalid_chunks():
    c = build_case([10], [3], hq=1, hkv=1, d=8)
    c["q_start"] = np.array([0, 11], np.int32)             # chunk longer than the sequence
    c["q"] = np.zeros((11, 1, 8), np.float32)
    with pytest.raises(ValueError):
        run(c, 1.0)


# ------------------------------------------------------------------ planted mistakes
MUTANTS = {
    "not_causal": ("const int nkeys = p + 1;", "const int nkeys = L;"),
    "no_offset": ("const int p = L - C + (int)(row - q_start[s]);", "const int p = (int)(row - q_start[s]);"),
    "off_by_one": ("const int nkeys = p + 1;", "const int nkeys = p;"),
    "gqa": ("const int g = h / group;\\n        int s = 0;", "const int g = h % num_kv_heads;\\n        int s = 0;"),
}


def _battery(fn):
    try:
        c = build_case([40, 100, 7, 65], [13, 100, 7, 1], hq=8, hkv=2, d=32, seed=1)
        if not np.allclose(run(c, 0.25, fn), sdpa_reference(c, 0.25), rtol=1e-10, atol=1e-12):
            return False
        c = build_case([1, 17, 50, 129], [1, 1, 1, 1], hq=8, hkv=2, d=32)
        dec = oracle.paged_decode(c["kp"], c["vp"], "f32", c["tables"], c["lens"], c["q"], 0.2)
        return bool(np.allclose(run(c, 0.2, fn), dec, rtol=1e-12, atol=1e-14))
    except ValueError:
        return False


def _mutant_fn(so):
    import ctypes
    lib = ctypes.CDLL(so)
    lib.oracle_paged_prefill.restype = ctypes.c_int
    lib.oracle_paged_prefill.argtypes = oracle.lib().oracle_paged_prefill.argtypes

    def fn(k, v, dtype, tables, lens, q_start, q, scale):
        k, v = np.ascontiguousarray(k), np.ascontiguousarray(v)
        t = np.ascontiguousarray(tables, np.int32)
        ln = np.ascontiguousarray(lens, np.int32)
        qs = np.ascontiguousarray(q_start, np.int32)
        qq = np.ascontiguousarray(q)
        out = np.empty(qq.shape, np.float64)
        p = lambda a: a.ctypes.data_as(ctypes.c_void_p)  # noqa: E731
        rc = lib.oracle_paged_prefill(p(k), p(v), {"f32": 0, "f16": 1, "bf16": 2}[dtype], k.shape[0], k.shape[2],
                                      k.shape[1], k.shape[3], p(t), t.shape[1], p(ln), p(qs), ln.shape[0], p(qq),
                                      qq.shape[1], float(scale), p(out), 1)
        if rc:
            raise ValueError
        return out
    return fn


def test_battery_accepts_oracle():
    assert _battery(oracle.paged_prefill)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_battery_rejects_planted_mistake(name):
    src = open(ORACLE_C).read()
    old, new = (x.replace("\\n", "\n") for x in MUTANTS[name])
    assert src.count(old) == 1, name
    d = tempfile.mkdtemp()
    c_path, so = os.path.join(d, "m.c"), os.path.join(d, "m.so")
    open(c_path, "w").write(src.replace(old, new))
    subprocess.run(["gcc", "-std=c11", "-O1", "-fPIC", "-shared", "-o", so, c_path, "-lm"], check=True)
    here = os.path.dirname(os.path.abspath(__file__))
    code = ("import sys; sys.path[:0] = [%r, %r]; import test_oracle_prefill as t; "
            "sys.exit(0 if t._battery(t._mutant_fn(%r)) else 1)" % (here, os.path.dirname(here), so))
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, timeout=300)
    assert r.returncode != 0, f"mutant {name} passed every pin"
