"""Counter-based synthetic K/V/q values (host side, numpy).

Seeded input generator shared by the oracle side and the GPU side; it holds none
of the attention or paging arithmetic.  Every element of every synthetic tensor is
a pure function of (seed, kind, sequence uid, layer, token position, head, dim), so
any sequence's keys and values can be regenerated on the host for a sampled check
without ever reading device memory.

Generator definition (implemented a second time, independently, in
``synthetic/csrc/synth_gen.cu`` for filling device memory):

* counter  c = kind<<62 | uid<<40 | layer<<34 | token<<14 | head<<8 | dim
  (kind 0 = K, 1 = V, 2 = Q; uid < 2^22, layer < 64, token < 2^20, head < 64,
  dim < 256).
* z = SplitMix64 output number c of the stream seeded with ``seed``:
  z = mix64(seed + (c + 1) * 0x9E3779B97F4A7C15), with mix64 the SplitMix64
  finaliser (Steele, Lea & Flood, "Fast splittable pseudorandom number
  generators", OOPSLA 2014; seed-0 outputs 0xe220a8397b1dcdaf,
  0x6e789e6aa1b965f4, 0x06c45d188009454f).
* s = sum of the four 16-bit fields of z (Irwin-Hall sum of four discrete
  uniforms), centred: s - 131070, an integer in [-131070, 131070], exact in fp32.
* v32 = fp32(s - 131070) * fp32(scale / sqrt((2^32 - 1) / 3)): one IEEE fp32
  multiply, so the value has mean 0 and standard deviation ``scale`` and is an
  approximately normal variate with no transcendental function involved.
* stored value = v32 rounded to nearest-even into the storage type (fp32 keeps
  it, fp16 / bf16 round it).

Because the arithmetic is integer plus one correctly rounded fp32 multiply plus
one correctly rounded narrowing, both implementations give the same bits.
"""
from __future__ import annotations

import math

import numpy as np

GOLDEN_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

KIND_K, KIND_V, KIND_Q = 0, 1, 2
DTYPES = ("f32", "f16", "bf16")
ELEM_BYTES = {"f32": 4, "f16": 2, "bf16": 2}


def mix64(z: np.ndarray) -> np.ndarray:
    """SplitMix64 finaliser on uint64 arrays (wrapping arithmetic)."""
    z = np.asarray(z, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = (z ^ (z >> np.uint64(30))) * _M1
        z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def splitmix64(seed: int, index: np.ndarray) -> np.ndarray:
    """Output number ``index`` (0-based) of the SplitMix64 stream seeded with ``seed``."""
    idx = np.asarray(index, dtype=np.uint64)
    with np.errstate(over="ignore"):
        state = np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + (idx + np.uint64(1)) * GOLDEN_GAMMA
    return mix64(state)


def counters(kind: int, uid, layer, token, head, dim) -> np.ndarray:
    """Pack the element coordinates into the 64-bit counter (broadcasting)."""
    u = np.uint64
    uid = np.asarray(uid, dtype=np.uint64)
    token = np.asarray(token, dtype=np.uint64)
    head = np.asarray(head, dtype=np.uint64)
    dim = np.asarray(dim, dtype=np.uint64)
    layer = np.asarray(layer, dtype=np.uint64)
    if np.any(uid >= u(1 << 22)) or np.any(token >= u(1 << 20)) or np.any(layer >= u(64)) \
            or np.any(head >= u(64)) or np.any(dim >= u(256)):
        raise ValueError("coordinate out of the counter's field range")
    return ((u(kind) << u(62)) | (uid << u(40)) | (layer << u(34)) | (token << u(14))
            | (head << u(8)) | dim)


def unit_scale_f32(scale: float) -> np.float32:
    """fp32 multiplier mapping the centred Irwin-Hall sum to standard deviation ``scale``."""
    return np.float32(scale / math.sqrt((2.0 ** 32 - 1.0) / 3.0))


def values_f32(seed: int, ctr: np.ndarray, scale: float) -> np.ndarray:
    """fp32 values for the given counters (before narrowing to the storage type)."""
    z = splitmix64(seed, ctr)
    m = np.uint64(0xFFFF)
    s = ((z & m) + ((z >> np.uint64(16)) & m) + ((z >> np.uint64(32)) & m)
         + ((z >> np.uint64(48)) & m)).astype(np.int64) - 131070
    return s.astype(np.float32) * unit_scale_f32(scale)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bfloat16 (nearest, ties to even); returns uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    nan = (u & np.uint64(0x7FFFFFFF)) > np.uint64(0x7F800000)
    r = (u + np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    r = np.where(nan, (u >> np.uint64(16)) | np.uint64(0x40), r)
    return r.astype(np.uint16)


def narrow(x32: np.ndarray, dtype: str) -> np.ndarray:
    """Storage representation: float32 / float16 arrays, bf16 as uint16 bit patterns."""
    if dtype == "f32":
        return np.ascontiguousarray(x32, dtype=np.float32)
    if dtype == "f16":
        return x32.astype(np.float16)
    if dtype == "bf16":
        return f32_to_bf16_bits(x32)
    raise ValueError(dtype)


def to_float64(stored: np.ndarray, dtype: str) -> np.ndarray:
    """Exact widening of stored values to float64 (bf16 bits are the top half of fp32)."""
    if dtype == "bf16":
        return (stored.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return stored.astype(np.float64)


def rows(kind: int, seed: int, layer: int, uids, tokens, num_heads: int, head_dim: int,
         scale: float, dtype: str) -> np.ndarray:
    """Rows [n][num_heads][head_dim] for row i = (uids[i], tokens[i]) in storage form."""
    uids = np.asarray(uids, dtype=np.int64).reshape(-1, 1, 1)
    tokens = np.asarray(tokens, dtype=np.int64).reshape(-1, 1, 1)
    h = np.arange(num_heads, dtype=np.int64).reshape(1, -1, 1)
    d = np.arange(head_dim, dtype=np.int64).reshape(1, 1, -1)
    ctr = counters(kind, uids, layer, tokens, h, d)
    return narrow(values_f32(seed, ctr, scale), dtype)


def to_torch(stored: np.ndarray, dtype: str):
    """Wrap a storage array as a CPU torch tensor of the matching dtype (no copy for bf16 view)."""
    import torch
    t = torch.from_numpy(np.ascontiguousarray(stored))
    if dtype == "bf16":
        return t.view(torch.bfloat16)
    return t
