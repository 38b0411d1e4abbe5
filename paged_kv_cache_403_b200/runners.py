"""Drivers that run the five synthetic decode workloads through the library.

Inputs come from the seeded generators in ``synthetic`` (device-side fill for
keys, values and queries; host-side draws for lengths, pool order and stops).
Each driver records what it did (sequence ids, uids, slots, copy pairs, tables,
lengths, outputs) so tests can replay the same schedule on the oracle.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

from synthetic import gpu as sgpu
from synthetic import values as sv

from .engine import TORCH_DTYPES, PagedCache, max_blocks_for


class DeviceGen:
    """Synthetic K/V/q rows on the device for (uid, token) lists."""

    def __init__(self, seed, shape, device="cuda"):
        self.seed, self.shape, self.device = seed, shape, device

    def _fill(self, kind, layer, uids, toks, heads, scale):
        u = torch.as_tensor(np.asarray(uids, np.int32)).to(self.device)
        t = torch.as_tensor(np.asarray(toks, np.int32)).to(self.device)
        out = torch.empty((len(u), heads, self.shape.head_dim), dtype=TORCH_DTYPES[self.shape.dtype],
                          device=self.device)
        return sgpu.fill_rows(out, kind, self.seed, layer, u, t, scale, self.shape.dtype)

    def kv(self, layer, uids, toks):
        s = self.shape
        return (self._fill(sv.KIND_K, layer, uids, toks, s.num_kv_heads, s.kv_scale),
                self._fill(sv.KIND_V, layer, uids, toks, s.num_kv_heads, s.kv_scale))

    def q(self, layer, uids, toks):
        s = self.shape
        return self._fill(sv.KIND_Q, layer, uids, toks, s.num_q_heads, s.q_scale)


def prefill(cache: PagedCache, gen: DeviceGen, sids, uids, lens, chunk_rows=1 << 16):
    """Append prompt tokens 0..lens[i]-1 of uid uids[i] to sequence sids[i], all layers."""
    slots, cow = cache.reserve(sids, lens)
    assert len(cow) == 0
    row_uid = np.repeat(np.asarray(uids, np.int64), np.asarray(lens, np.int64))
    row_tok = np.concatenate([np.arange(int(L)) for L in lens]) if len(lens) else np.zeros(0, np.int64)
    slots_dev = torch.from_numpy(np.ascontiguousarray(slots)).to(cache.device)
    for lo in range(0, len(slots), chunk_rows):
        hi = min(len(slots), lo + chunk_rows)
        for layer in range(cache.num_layers):
            k, v = gen.kv(layer, row_uid[lo:hi], row_tok[lo:hi])
            cache.append(layer, k, v, slots_dev[lo:hi])
    return slots


@dataclass
class StepRecord:
    sids: list
    uids: list
    positions: np.ndarray           # position of the new token per sequence
    slots: np.ndarray
    cow: np.ndarray
    tables: np.ndarray
    lens: np.ndarray
    outputs: dict = field(default_factory=dict)   # layer -> out tensor (device)


def decode_step(cache: PagedCache, gen: DeviceGen, sids, uids, num_q_heads, max_blocks,
                split_tokens=0, out_dtype=None, keep_layers=None, workspace=None):
    """One decode iteration for every sequence in the batch, every layer."""
    positions = np.array([cache.info(s)[0] for s in sids], np.int64)
    slots, cow = cache.reserve(sids, [1] * len(sids))
    cache.copy_blocks(cow)
    tables, lens = cache.tables(sids, max_blocks)
    dev = cache.device
    slots_dev = torch.from_numpy(np.ascontiguousarray(slots)).to(dev)
    tables_dev = torch.from_numpy(tables).to(dev)
    lens_dev = torch.from_numpy(lens).to(dev)
    out_dtype = out_dtype or TORCH_DTYPES[cache.act_dtype]
    if workspace is None:
        workspace = cache.workspace(len(sids), num_q_heads, max_blocks, split_tokens)
    rec = StepRecord(list(sids), list(uids), positions, slots.copy(), cow.copy(), tables.copy(), lens.copy())
    for layer in range(cache.num_layers):
        k, v = gen.kv(layer, uids, positions)
        cache.append(layer, k, v, slots_dev)
        q = gen.q(layer, uids, positions)
        out = torch.empty((len(sids), num_q_heads, cache.head_dim), dtype=out_dtype, device=dev)
        cache.decode(layer, q, out, tables_dev, lens_dev, 1.0 / math.sqrt(cache.head_dim), split_tokens,
                     workspace)
        if keep_layers is None or layer in keep_layers:
            rec.outputs[layer] = out
    return rec


def make_cache(shape, order, device="cuda", kv_fp8=False):
    """The workload's cache: its own 16-bit type, or an FP8 cache whose queries and
    appended rows keep that type."""
    if kv_fp8:
        return PagedCache(shape.num_layers, shape.num_blocks, shape.block_size, shape.num_kv_heads, shape.head_dim,
                          "fp8", order, device, act_dtype=shape.dtype)
    return PagedCache.from_shape(shape, order, device)


def run_static(recipe, split_tokens=0, out_dtype=None, keep_layers=None, device="cuda", kv_fp8=False):
    """tiny / worked_example / large_pool: prefill every sequence, then one decode step."""
    shape = recipe["shape"]
    cache = make_cache(shape, recipe["order"], device, kv_fp8)
    gen = DeviceGen(recipe["seed"], shape, device)
    lens = [int(L) for L in recipe["lens"]]
    sids = [cache.add() for _ in lens]
    uids = list(range(len(lens)))
    prefill(cache, gen, sids, uids, lens)
    mb = max_blocks_for(lens, shape.block_size, extra_tokens=1)
    rec = decode_step(cache, gen, sids, uids, shape.num_q_heads, mb, split_tokens, out_dtype, keep_layers)
    return cache, gen, rec


def run_prefix_sharing(recipe, split_tokens=0, out_dtype=None, device="cuda"):
    """64 sequences share a prefix (root uid 0, forks uid 1..63) plus private suffixes;
    one decode step for all; then the copy-on-write event: fork the first sequence whose
    length is not a multiple of the block size, append one token to the fork, decode all."""
    shape = recipe["shape"]
    cache = PagedCache.from_shape(shape, recipe["order"], device)
    gen = DeviceGen(recipe["seed"], shape, device)
    n, prefix = len(recipe["suffix"]), recipe["prefix"]
    root = cache.add()
    prefill(cache, gen, [root], [0], [prefix])
    sids = [root] + [cache.fork(root) for _ in range(n - 1)]
    uids = list(range(n))
    # private suffix tokens prefix..prefix+suffix-1, written by each sequence's own uid
    suffix = [int(x) for x in recipe["suffix"]]
    slots, cow = cache.reserve(sids, suffix)
    assert len(cow) == 0
    row_uid = np.repeat(np.asarray(uids, np.int64), suffix)
    row_tok = np.concatenate([prefix + np.arange(x) for x in suffix])
    k, v = gen.kv(0, row_uid, row_tok)
    cache.append(0, k, v, torch.from_numpy(slots).to(device))
    mb = max_blocks_for([prefix + x for x in suffix], shape.block_size, extra_tokens=2)
    step1 = decode_step(cache, gen, sids, uids, shape.num_q_heads, mb, split_tokens, out_dtype)
    # copy-on-write event
    lens_now = [cache.info(s)[0] for s in sids]
    victim = next(i for i, L in enumerate(lens_now) if L % shape.block_size != 0)
    child = cache.fork(sids[victim])
    child_uid = n
    sids2 = sids + [child]
    uids2 = uids + [child_uid]
    step2 = decode_step(cache, gen, sids2, uids2, shape.num_q_heads, mb, split_tokens, out_dtype)
    return cache, gen, dict(step1=step1, step2=step2, victim=victim, child=child)


class ContinuousBatch:
    """Continuous-batch workload: fixed batch slots, stops drawn per step, replacements
    admitted (prefilled) at the start of the next step."""

    def __init__(self, recipe, device="cuda", max_blocks=None, kv_fp8=False):
        self.recipe = recipe
        self.shape = shape = recipe["shape"]
        self.sched = recipe["schedule"]
        self.cache = make_cache(shape, recipe["order"], device, kv_fp8)
        self.gen = DeviceGen(recipe["seed"], shape, device)
        self.device = device
        n = len(self.sched.initial)
        self.sids = [self.cache.add() for _ in range(n)]
        self.uids = list(range(n))
        self.next_uid = n
        prefill(self.cache, self.gen, self.sids, self.uids, [int(L) for L in self.sched.initial])
        self.max_blocks = max_blocks or -(-(4096 + len(self.sched.events) + 1) // shape.block_size)
        self.pending = []          # (slot, prompt_len) admitted at the next step
        self.t = 0

    def admit(self):
        """Retired sequences' slots get new sequences (uid order = slot order)."""
        if not self.pending:
            return []
        new_sids, new_uids, lens = [], [], []
        for slot, plen in self.pending:
            sid = self.cache.add()
            self.sids[slot] = sid
            self.uids[slot] = self.next_uid
            new_sids.append(sid)
            new_uids.append(self.next_uid)
            lens.append(plen)
            self.next_uid += 1
        prefill(self.cache, self.gen, new_sids, new_uids, lens)
        self.pending = []
        return list(zip(new_sids, new_uids, lens))

    def retire(self, t):
        for slot, plen in self.sched.events[t]:
            self.cache.free(self.sids[slot])
            self.pending.append((slot, plen))

    def step(self, split_tokens=0, out_dtype=None, workspace=None):
        admitted = self.admit()
        rec = decode_step(self.cache, self.gen, self.sids, self.uids, self.shape.num_q_heads,
                          self.max_blocks, split_tokens, out_dtype, workspace=workspace)
        rec.outputs["admitted"] = admitted
        self.retire(self.t)
        self.t += 1
        return rec


class SharedPromptBatch(ContinuousBatch):
    """Continuous batch whose prompts share a system prompt; with ``cache`` the system
    prompt's full blocks are registered once and every later admission shares them
    (pa_seq_add_cached) and appends only its own suffix."""

    def __init__(self, recipe, device="cuda", max_blocks=None, cache=True):
        from synthetic.workloads import prompt_rows, system_block_keys
        self._rows, self.cache_on = prompt_rows, cache
        self.recipe = recipe
        self.shape = shape = recipe["shape"]
        self.sched = recipe["schedule"]
        self.system, self.system_uid = recipe["system"], recipe["system_uid"]
        self.keys = system_block_keys(self.system // shape.block_size, self.system_uid)
        self.cache = PagedCache.from_shape(shape, recipe["order"], device)
        self.gen = DeviceGen(recipe["seed"], shape, device)
        self.device = device
        n = len(self.sched.initial)
        self.sids, self.uids = [None] * n, list(range(n))
        self.appended_rows = 0
        init = [int(L) for L in self.sched.initial]
        # the first request writes (and registers) the system prompt; the rest can share it
        self._admit_many([0], [0], init[:1])
        if n > 1:
            self._admit_many(list(range(1, n)), list(range(1, n)), init[1:])
        self.next_uid = n
        self.max_blocks = max_blocks or -(-(4096 + len(self.sched.events) + 1) // shape.block_size)
        self.pending = []
        self.t = 0

    def _admit_many(self, slots, uids, lens):
        from paged_kv_cache_403_b200 import pa_prefix_register, pa_seq_add_cached
        pool = self.cache.pool
        starts = []
        for slot, uid, plen in zip(slots, uids, lens):
            if self.cache_on:
                sid, hit = pa_seq_add_cached(pool, self.keys)
            else:
                sid, hit = self.cache.add(), 0
            self.sids[slot] = sid
            starts.append(hit * self.shape.block_size)
        sids = [self.sids[s] for s in slots]
        ntok = [plen - st for plen, st in zip(lens, starts)]
        slots_host, cow = self.cache.reserve(sids, ntok)
        assert len(cow) == 0
        ru, rt = zip(*[self._rows(u, p, self.system, self.system_uid, st) for u, p, st in zip(uids, lens, starts)])
        ru, rt = np.concatenate(ru), np.concatenate(rt)
        dev = torch.from_numpy(np.ascontiguousarray(slots_host)).to(self.device)
        for lo in range(0, len(ru), 1 << 16):
            hi = min(len(ru), lo + (1 << 16))
            for layer in range(self.cache.num_layers):
                k, v = self.gen.kv(layer, ru[lo:hi], rt[lo:hi])
                self.cache.append(layer, k, v, dev[lo:hi])
        self.appended_rows += len(ru)
        if self.cache_on:
            for sid, st in zip(sids, starts):
                if st == 0:                      # first writer of the system prompt registers it
                    pa_prefix_register(pool, sid, self.keys)

    def admit(self):
        if not self.pending:
            return []
        slots = [s for s, _ in self.pending]
        uids = list(range(self.next_uid, self.next_uid + len(slots)))
        lens = [p for _, p in self.pending]
        for s, u in zip(slots, uids):
            self.uids[s] = u
        self.next_uid += len(slots)
        self._admit_many(slots, uids, lens)
        self.pending = []
        return list(zip([self.sids[s] for s in slots], uids, lens))
