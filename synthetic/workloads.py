"""Seeded workload recipes for the five decode workloads (host side).

Holds only random draws and sizes: sequence lengths, the shuffled order of the
physical block pool, stop draws of the continuous batch, prefix/suffix lengths.
Nothing here allocates blocks or computes attention; both the GPU path and the
oracle consume these recipes.  Every draw comes from
``numpy.random.default_rng(seed)`` with seed = workload number (1..5) unless a
caller passes another.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np


@dataclass
class Shape:
    """Cache geometry of one workload."""
    num_layers: int
    block_size: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    dtype: str            # "f32" | "f16" | "bf16"
    num_blocks: int
    kv_scale: float       # standard deviation of synthetic K and V values
    q_scale: float = 1.0  # standard deviation of synthetic q values


def tiny(seed: int = 1) -> dict:
    """4 sequences of 50/17/3/33 tokens, block 16, 4 q / 2 KV heads, d64, fp32, 64-block pool."""
    rng = np.random.default_rng(seed)
    shape = Shape(1, 16, 4, 2, 64, "f32", 64, kv_scale=1.0)
    return dict(name="tiny", seed=seed, shape=shape, lens=np.array([50, 17, 3, 33]),
                order=rng.permutation(shape.num_blocks).astype(np.int32))


def worked_example(seed: int = 2, steps: int = 0) -> dict:
    """The pages' four requests (3900/420/2100/70 tokens), 32 q / 8 KV heads, d128, fp16.
    ``steps``: decode steps the pool must also hold (each appends one token per request)."""
    rng = np.random.default_rng(seed)
    shape = Shape(1, 16, 32, 8, 128, "f16", 4096 + 4 * -(-steps // 16), kv_scale=1.0 / math.sqrt(128.0))
    return dict(name="worked_example", seed=seed, shape=shape,
                lens=np.array([3900, 420, 2100, 70]),
                order=rng.permutation(shape.num_blocks).astype(np.int32))


@dataclass
class ContinuousSchedule:
    """Continuous-batch schedule: fixed batch slots, Bernoulli stops, uniform replacements.

    ``initial[i]`` is the prompt length of the sequence first held by slot i.
    ``events[t]`` lists (slot, new_prompt_len) pairs: after step t the sequence in
    that slot stops and, at step t+1, a new sequence with that prompt length takes
    the slot.  Sequence uids are issued in order of admission: 0..n-1 for the
    initial batch, then n, n+1, ... in (step, slot) order.
    """
    initial: np.ndarray
    events: list = field(default_factory=list)


def continuous_schedule(n: int, steps: int, seed: int, lo: int = 128, hi: int = 4096,
                        p_stop: float = 1.0 / 200.0) -> ContinuousSchedule:
    """Draw order: initial lengths; then per step one uniform per slot (stop if < p),
    then one length per stopping slot in ascending slot order."""
    rng = np.random.default_rng(seed)
    initial = rng.integers(lo, hi + 1, size=n)
    events = []
    for _ in range(steps):
        stops = np.nonzero(rng.random(n) < p_stop)[0]
        events.append([(int(s), int(rng.integers(lo, hi + 1))) for s in stops])
    return ContinuousSchedule(initial=initial, events=events)


def continuous_batch(seed: int = 3, n: int = 256, steps: int = 64, p_stop: float = 1.0 / 200.0,
                     lo: int = 128, hi: int = 4096) -> dict:
    """256 sequences, lengths U[128, 4096], block 16, 32 q / 8 KV heads, d128, bf16.

    Pool: every slot can hold a maximum-length sequence plus the steps' appends, so
    the pool never runs out (n * ceil((hi + steps) / 16) blocks; 66,560 at the
    default sizes)."""
    shape = Shape(1, 16, 32, 8, 128, "bf16",
                  num_blocks=n * ((hi + max(steps, 64) + 15) // 16), kv_scale=1.0 / math.sqrt(128.0))
    order = np.random.default_rng(seed + 1000).permutation(shape.num_blocks).astype(np.int32)
    return dict(name="continuous_batch", seed=seed, shape=shape, order=order,
                schedule=continuous_schedule(n, steps, seed, lo, hi, p_stop))


def prefix_sharing(seed: int = 4, n: int = 64, prefix: int = 2048, steps: int = 0) -> dict:
    """64 sequences sharing a 2048-token prefix, private suffixes U[16, 512], fp16.
    ``steps``: decode steps beyond the first few the pool must also hold."""
    rng = np.random.default_rng(seed)
    shape = Shape(1, 16, 32, 8, 128, "f16",
                  num_blocks=prefix // 16 + n * ((512 + 16 + 15) // 16 + 1 + -(-steps // 16)) + 64,
                  kv_scale=1.0 / math.sqrt(128.0))
    suffix = rng.integers(16, 512 + 1, size=n)
    order = rng.permutation(shape.num_blocks).astype(np.int32)
    return dict(name="prefix_sharing", seed=seed, shape=shape, prefix=prefix,
                suffix=suffix, order=order)


def lognormal_lengths(n: int, seed: int, median: float = 1500.0, sigma: float = 0.75,
                      cap: int = 16384) -> np.ndarray:
    rng = np.random.default_rng(seed)
    z = rng.standard_normal(n)
    lens = np.rint(np.exp(math.log(median) + sigma * z))
    return np.clip(lens, 1, cap).astype(np.int64)


def large_pool(seed: int = 5, block_size: int = 16, n: int = 384, num_layers: int = 32, steps: int = 0) -> dict:
    """384 sequences, lognormal lengths (median 1500, sigma 0.75, cap 16384), 32 layers, fp16.
    ``steps``: decode steps the pool must also hold (one token per sequence each)."""
    lens = lognormal_lengths(n, seed)
    # pool: every sequence's blocks after one appended token, plus two blocks of headroom each
    # (and room for ``steps`` more tokens per sequence)
    nb = int(sum(-(-(int(l) + 1 + steps) // block_size) for l in lens)) + 2 * n
    shape = Shape(num_layers, block_size, 32, 8, 128, "f16", nb, kv_scale=1.0 / math.sqrt(128.0))
    order = np.random.default_rng(seed + 1000 * block_size).permutation(nb).astype(np.int32)
    return dict(name=f"large_pool_b{block_size}", seed=seed, shape=shape, lens=lens, order=order)


SYSTEM_UID = (1 << 22) - 1   # writer uid of the shared system prompt's keys and values


def shared_prompt_batch(seed: int = 6, n: int = 256, steps: int = 64, system: int = 1024,
                        p_stop: float = 1.0 / 200.0) -> dict:
    """Continuous batch whose prompts all start with the same `system`-token prompt:
    prompt lengths U[system + 128, 4096]; positions < system are written by
    SYSTEM_UID (identical in every request), later ones by the request's own uid.
    Block 16, 32 q / 8 KV heads, d128, bf16."""
    shape = Shape(1, 16, 32, 8, 128, "bf16",
                  num_blocks=n * ((4096 + max(steps, 64) + 15) // 16), kv_scale=1.0 / math.sqrt(128.0))
    order = np.random.default_rng(seed + 1000).permutation(shape.num_blocks).astype(np.int32)
    return dict(name="shared_prompt", seed=seed, shape=shape, order=order, system=system,
                system_uid=SYSTEM_UID,
                schedule=continuous_schedule(n, steps, seed, system + 128, 4096, p_stop))


def prompt_rows(uid: int, plen: int, system: int = 0, system_uid: int = SYSTEM_UID, start: int = 0):
    """(writer uid, token) of prompt positions start..plen-1: the shared system prompt
    for positions < system, the request itself after."""
    pos = np.arange(start, plen)
    return np.where(pos < system, system_uid, uid), pos


def system_block_keys(n_blocks: int, system_uid: int = SYSTEM_UID):
    """Cache keys of the shared system prompt's full blocks (stand-in for a hash chain)."""
    return [(system_uid << 32) | i for i in range(n_blocks)]


def chunked_prefill(seed: int = 7, n: int = 32, lo: int = 1024, hi: int = 4096, chunk: int = 512,
                    dtype: str = "bf16") -> dict:
    """Chunked prefill: n sequences with total lengths U[lo, hi]; the last `chunk` tokens
    of each are the queries (their keys and values are already cached).  Block 16,
    32 q / 8 KV heads, d128, bf16 (or fp16), 1 layer."""
    rng = np.random.default_rng(seed)
    lens = rng.integers(lo, hi + 1, size=n)
    chunks = np.minimum(lens, chunk)
    shape = Shape(1, 16, 32, 8, 128, dtype, int(sum(-(-int(L) // 16) for L in lens)) + 16,
                  kv_scale=1.0 / math.sqrt(128.0))
    order = rng.permutation(shape.num_blocks).astype(np.int32)
    return dict(name="chunked_prefill", seed=seed, shape=shape, lens=lens, chunks=chunks, order=order)
