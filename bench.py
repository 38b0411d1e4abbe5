#!/usr/bin/env python
"""Benchmark: paged decode attention over a paged KV cache, one decode step at a time.

Default workload (one replica per GPU), the one the stated target is quoted on:
continuous batch -- 256 sequences, prompt lengths uniform in [128, 4096], block 16,
32 query / 8 KV heads, head_dim 128, bf16 cache, 1 layer; every step each sequence
appends one token and attends over its whole cache; after each step every sequence
stops with probability 1/200 and a new one (prompt uniform in [128, 4096]) takes its
slot at the next step.  ``--workload`` selects the other synthetic workloads (the
pages' worked example, prefix sharing, the ~100 GB 32-layer large pool with block
16 or 32).

A timed step runs the whole path: admissions, one-slot reservations with the
copy-on-write check (host, native), metadata upload, then for every layer one append
of the step's K/V rows and the admitted prompts' rows, and decode attention (split
ranges merged in the kernel), and retirements (host).  Host bookkeeping of step t+1 overlaps the GPU work of step
t: metadata is staged in pinned buffers and uploaded on a side stream into
NSETS rotating device buffer sets.

Prints one JSON line (rank 0).  ``value`` = KV bytes read by decode attention per
second of step time, whole job (all ranks); decode tokens/s beside it.
``--impl reference`` times the CPU oracle on a bounded sample instead.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged decode attention KV-read HBM GB/s (fraction of ~8 TB/s) and decode tokens/s"
UNIT = "GB/s"
NOMINAL_HBM_GBS = 8000.0
WORKLOADS = ("continuous_batch", "large_pool_b16", "large_pool_b32", "worked_example", "prefix_sharing",
             "shared_prompt", "swap", "prefill")
# Longest split-K range per workload, in tokens (0: never split).  With ranges of nearly
# equal length per sequence, 4096 (a split only for sequences past 4096 tokens) measured
# best on the continuous batch and the large pool, for 16-bit and FP8 caches alike.
DEFAULT_SPLIT = {"continuous_batch": 4096, "large_pool_b16": 4096, "large_pool_b32": 4096,
                 "worked_example": 128, "prefix_sharing": 1024, "shared_prompt": 2048, "swap": 0, "prefill": 0}
NSETS = 4           # device input/metadata buffer sets: the host may run this many steps ahead


def default_split(workload):
    """Tokens per split-K range the benchmark uses for a workload (0: never split)."""
    return DEFAULT_SPLIT[workload]


def parse(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None, help="timed steps (default 64; 8 for large_pool)")
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--repeats", type=int, default=None,
                    help="timed passes of --steps steps each, over a longer schedule; the median pass is "
                         "reported (default 7 on the continuous batches, 3 on the fixed batches)")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="continuous_batch", choices=WORKLOADS)
    ap.add_argument("--split", type=int, default=None, help="tokens per split-K range (0: never split)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-sample-seqs", type=int, default=24)
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="oracle time for the CPU baseline")
    ap.add_argument("--dtype", default="bf16", choices=["bf16", "f16"],
                    help="prefill workload: cache / query type (bf16 P enters P.V as two products, fp16 P once)")
    ap.add_argument("--kv-dtype", default="native", choices=["native", "fp8"],
                    help="native: the workload's 16-bit cache; fp8: E4M3 codes + per-row scale bytes "
                         "(queries and appended rows keep the workload's type)")
    ap.add_argument("--prefix-cache", default="on", choices=["on", "off"],
                    help="shared_prompt workload: share the cached system-prompt blocks at admission")
    a = ap.parse_args(argv)
    if a.steps is None:
        a.steps = 8 if a.workload.startswith("large_pool") or a.workload in ("swap", "prefill") else 64
    if a.split is None:
        a.split = default_split(a.workload)
    if a.repeats is None:
        # 3 passes where one step is long (large pool) or sequences only grow (fixed batches)
        a.repeats = 7 if a.workload in ("continuous_batch", "shared_prompt") else 3
    a.repeats = max(1, a.repeats)
    if a.kv_dtype == "fp8" and a.workload not in ("continuous_batch", "large_pool_b16", "large_pool_b32",
                                                    "worked_example"):
        ap.error("--kv-dtype fp8 runs the continuous_batch, large_pool and worked_example workloads")
    return a


def captured_traffic(fp8=False):
    """DRAM bytes per launch of the decode kernel from profiles/traffic.json (one ncu
    capture), if every kernel source it lists still has the hash it was captured at
    (else None)."""
    import hashlib
    csrc = os.path.join(ROOT, "paged_kv_cache_403_b200", "csrc")
    try:
        entry = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))["decode_fp8" if fp8 else "decode_bf16"]
        for src, sha in entry["sources"].items():
            if not hashlib.sha256(open(os.path.join(csrc, src), "rb").read()).hexdigest().startswith(sha):
                return None
        return int(entry["traffic_bytes_per_launch"])
    except (OSError, KeyError, ValueError, TypeError):
        return None


# ---------------------------------------------------------------------------- schedules
def simulate(sched, n, steps):
    """Continuous batch: per step the uids, token positions, admissions and retirements."""
    lens = np.array(sched.initial, np.int64)
    uids = np.arange(n, dtype=np.int64)
    next_uid, pending = n, []
    plan = []
    for t in range(steps):
        admitted = []
        for slot, plen in pending:
            uids[slot] = next_uid
            lens[slot] = plen
            admitted.append((slot, next_uid, plen))
            next_uid += 1
        plan.append(dict(uids=uids.copy(), pos=lens.copy(), admitted=admitted, retire=list(sched.events[t])))
        lens += 1
        pending = list(sched.events[t])
    return plan


def static_plan(uids, lens, steps):
    """Fixed batch: every sequence grows by one token per step."""
    uids = np.asarray(uids, np.int64)
    lens = np.asarray(lens, np.int64)
    return [dict(uids=uids.copy(), pos=lens + t, admitted=[], retire=[]) for t in range(steps)]


def make_recipe(workload, seed_offset, steps):
    from synthetic import workloads as wl
    if workload == "continuous_batch":
        return wl.continuous_batch(seed=3 + seed_offset, steps=steps)
    # the fixed-batch workloads grow by one token per sequence and step: their pools get
    # room for every step the run takes
    if workload.startswith("large_pool"):
        return wl.large_pool(seed=5 + seed_offset, block_size=int(workload[-2:]), steps=steps)
    if workload == "worked_example":
        return wl.worked_example(seed=2 + seed_offset, steps=steps)
    if workload == "shared_prompt":
        return wl.shared_prompt_batch(seed=6 + seed_offset, steps=steps)
    return wl.prefix_sharing(seed=4 + seed_offset, steps=steps)


# Workloads whose KV (or unique KV) per step fits in the 126 MB L2: each step starts by
# overwriting a buffer twice the L2's size, so no step finds the previous step's blocks
# in L2.  Reuse inside one launch (a shared prefix read by many sequences) stays.
L2_RESIDENT = ("worked_example", "prefix_sharing", "shared_prompt")
FLUSH_BYTES = 256 << 20


def describe(workload):
    return {
        "continuous_batch": "continuous_batch: 256 seqs, lengths U[128,4096], block 16, 32 q / 8 KV heads, d128, "
                            "bf16, p_stop 1/200, 1 layer",
        "large_pool_b16": "large_pool: 384 seqs, lognormal lengths (median 1500, sigma 0.75, cap 16384), "
                          "block 16, 32 layers, 32 q / 8 KV heads, d128, fp16, ~100 GB pool",
        "large_pool_b32": "large_pool: 384 seqs, lognormal lengths (median 1500, sigma 0.75, cap 16384), "
                          "block 32, 32 layers, 32 q / 8 KV heads, d128, fp16, ~100 GB pool",
        "worked_example": "worked_example: 4 seqs of 3900/420/2100/70 tokens, block 16, 32 q / 8 KV heads, "
                          "d128, fp16, 1 layer",
        "prefix_sharing": "prefix_sharing: 64 seqs sharing a 2048-token prefix + private suffixes U[16,512], "
                          "block 16, 32 q / 8 KV heads, d128, fp16, 1 layer",
        "shared_prompt": "shared_prompt: continuous batch of 256 seqs whose prompts (U[1152,4096] tokens) start "
                         "with one 1024-token system prompt, block 16, 32 q / 8 KV heads, d128, bf16, "
                         "p_stop 1/200, 1 layer",
    }[workload]


def arm_config(args, sh, n, world):
    """The JSON line's config: the workload and its sizes (the same dict on both arms)."""
    fp8 = args.kv_dtype == "fp8"
    return {"workload": describe(args.workload), "n_seqs": n, "num_layers": sh.num_layers,
            "block_size": sh.block_size, "num_q_heads": sh.num_q_heads, "num_kv_heads": sh.num_kv_heads,
            "head_dim": sh.head_dim, "split_tokens": args.split, "parallelism": f"replicas x{world}",
            "kv_cache": "E4M3 codes + one power-of-two scale byte per (token, KV head) row" if fp8 else sh.dtype,
            "l2": (f"flushed: every step first writes {FLUSH_BYTES >> 20} MiB on the compute stream "
                   "(inside the step time, outside the attention events)"
                   if args.workload in L2_RESIDENT else
                   "no flush: the KV read per step exceeds the 126 MB L2")}


# ---------------------------------------------------------------------------- clocks
class ClockSampler:
    """SM clock and throttle reasons sampled through NVML every ~2 ms while timing runs."""

    REASONS = [("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake", "nvmlClocksEventReasonHwPowerBrakeSlowdown")]

    def __init__(self, cuda_index):
        self.samples, self.thread, self.stop_flag, self.h = [], None, False, None
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(cuda_index).uuid)
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.h = None

    def _run(self):
        nv = self.nv
        while not self.stop_flag:
            try:
                self.samples.append((nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM),
                                     nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)))
            except Exception:
                pass
            time.sleep(0.002)

    def start(self):
        if self.h is None:
            return
        import threading
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()

    def stop(self):
        if self.thread is None:
            return None
        self.stop_flag = True
        self.thread.join()
        if not self.samples:
            return None
        reasons = set()
        for _, mask in self.samples:
            for name, attr in self.REASONS:
                if mask & getattr(self.nv, attr, 0):
                    reasons.add(name)
        return {"sm_mhz": float(np.median([c for c, _ in self.samples])), "sm_max_mhz": float(self.max_mhz),
                "samples": len(self.samples), "reasons": sorted(reasons), "source": "nvml"}


# ---------------------------------------------------------------------------- ranks
def combine_ranks(dist, times_ms, byte_counts, device):
    """Whole-job figures over ranks: each time is the max over ranks (the slowest
    replica bounds the job), each byte count the sum over ranks."""
    import torch
    t = torch.tensor(times_ms, dtype=torch.float64, device=device)
    b = torch.tensor(byte_counts, dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(b, op=dist.ReduceOp.SUM)
    return t.tolist(), b.tolist()


def replica_seed(rank: int) -> int:
    """Seed offset of each rank's replica: every rank draws its own workload."""
    return 100 * rank


# ---------------------------------------------------------------------------- staging
class Packed:
    """Byte layout of several arrays in one buffer, each starting on a 256-byte
    boundary, so that one copy moves them all.  parts: (name, torch dtype, shape)."""

    ALIGN = 256

    def __init__(self, parts):
        self.parts, off = [], 0
        for name, dtype, shape in parts:
            count = int(np.prod(shape)) if len(shape) else 1
            nbytes = count * dtype.itemsize
            self.parts.append((name, dtype, tuple(shape), off, nbytes))
            off = -(-(off + nbytes) // self.ALIGN) * self.ALIGN
        self.nbytes = max(off, self.ALIGN)
        self.off = {name: o for name, _, _, o, _ in self.parts}
        self.end = {name: o + nb for name, _, _, o, nb in self.parts}

    def views(self, buf):
        """name -> view of buf (a uint8 tensor of at least nbytes) with the part's dtype and shape."""
        return {name: buf[o:o + nb].view(dt).view(shape) for name, dt, shape, o, nb in self.parts}


# ---------------------------------------------------------------------------- our path
class Replica:
    """One GPU's decode state: pools, block manager, sequences, and every step's inputs
    generated in HBM before timing starts."""

    def __init__(self, torch, workload, recipe, total_steps, split, device, e2e_from, prefix_cache=True,
                 kv_fp8=False):
        from paged_kv_cache_403_b200.engine import PagedCache
        from paged_kv_cache_403_b200.runners import DeviceGen, prefill
        import paged_kv_cache_403_b200 as pa
        self.torch, self.pa = torch, pa
        self.workload, self.recipe, self.shape = workload, recipe, recipe["shape"]
        sh = self.shape
        self.NL = sh.num_layers
        self.split, self.device = split, device
        self.kv_fp8 = kv_fp8
        if kv_fp8:
            self.cache = PagedCache(sh.num_layers, sh.num_blocks, sh.block_size, sh.num_kv_heads, sh.head_dim,
                                    "fp8", recipe["order"], device, act_dtype=sh.dtype)
        else:
            self.cache = PagedCache.from_shape(sh, recipe["order"], device)
        gen = DeviceGen(recipe["seed"], sh, device)
        self.prompt_start = lambda plen: 0          # first prompt position an admission appends
        self.system_keys = None
        if workload == "continuous_batch":
            n = len(recipe["schedule"].initial)
            self.plan = simulate(recipe["schedule"], n, total_steps)
            self.sids = [self.cache.add() for _ in range(n)]
            prefill(self.cache, gen, self.sids, list(range(n)), [int(x) for x in recipe["schedule"].initial])
            self.max_blocks = -(-(4096 + total_steps + 1) // sh.block_size)
        elif workload == "shared_prompt":
            from paged_kv_cache_403_b200.runners import SharedPromptBatch
            n = len(recipe["schedule"].initial)
            self.max_blocks = -(-(4096 + total_steps + 1) // sh.block_size)
            sb = SharedPromptBatch(recipe, device, self.max_blocks, cache=prefix_cache)
            self.cache.close()
            self.cache, self.sids = sb.cache, sb.sids
            self.plan = simulate(recipe["schedule"], n, total_steps)
            if prefix_cache:
                self.system_keys = sb.keys
                self.prompt_start = lambda plen: recipe["system"]
            self.prompt_rows = lambda uid, plen: sb._rows(uid, plen, recipe["system"], recipe["system_uid"],
                                                          self.prompt_start(plen))
        elif workload == "prefix_sharing":
            n = len(recipe["suffix"])
            prefix, suffix = recipe["prefix"], [int(x) for x in recipe["suffix"]]
            root = self.cache.add()
            prefill(self.cache, gen, [root], [0], [prefix])
            self.sids = [root] + [self.cache.fork(root) for _ in range(n - 1)]
            slots, _ = self.cache.reserve(self.sids, suffix)
            u = np.repeat(np.arange(n), suffix)
            tk = np.concatenate([prefix + np.arange(x) for x in suffix])
            k, v = gen.kv(0, u, tk)
            self.cache.append(0, k, v, torch.from_numpy(np.ascontiguousarray(slots)).to(device))
            lens = [prefix + x for x in suffix]
            self.plan = static_plan(range(n), lens, total_steps)
            self.max_blocks = -(-(max(lens) + total_steps + 1) // sh.block_size)
        else:
            lens = [int(x) for x in recipe["lens"]]
            n = len(lens)
            self.sids = [self.cache.add() for _ in range(n)]
            prefill(self.cache, gen, self.sids, list(range(n)), lens)
            self.plan = static_plan(range(n), lens, total_steps)
            self.max_blocks = -(-(max(lens) + total_steps + 1) // sh.block_size)
        self.n = n
        # sequence ids as a ready int32 array (and the one-token counts): the per-step
        # reservation and table calls then pass pointers without converting lists
        self.sid_arr = np.asarray(self.sids, np.int32)
        self.ones = np.ones(n, np.int32)
        # every step's inputs (all layers), generated on the device before any timing: q, and
        # the K / V rows to append -- the step's token rows with the admitted prompts' rows
        # right after them, so that one append launch writes both
        self.inputs = []
        for st in self.plan:
            per_layer = []
            for layer in range(self.NL):
                k, v = gen.kv(layer, st["uids"], st["pos"])
                q = gen.q(layer, st["uids"], st["pos"])
                if st["admitted"]:
                    if workload == "shared_prompt":
                        u, tk = map(np.concatenate, zip(*[self.prompt_rows(uid, p) for _, uid, p in st["admitted"]]))
                    else:
                        u = np.concatenate([np.full(p, uid) for _, uid, p in st["admitted"]])
                        tk = np.concatenate([np.arange(p) for _, _, p in st["admitted"]])
                    pk, pv = gen.kv(layer, u, tk)
                    k, v = torch.cat([k, pk]), torch.cat([v, pv])
                per_layer.append((q, k, v))
            self.inputs.append(per_layer)
        torch.cuda.synchronize()
        # end-to-end leg: each (step, layer)'s q and K / V rows (token rows, then the admitted
        # prompts' rows) packed in one pinned host buffer; one copy per layer uploads them
        # into a device buffer of the same layout (sized per step, so only the rows of this
        # step's admissions cross the bus)
        self.host, self.e2e_views, self.e2e_bytes = {}, {}, {}
        dt = self.inputs[0][0][0].dtype
        row_shape = lambda rows: (rows, sh.num_kv_heads, sh.head_dim)  # noqa: E731
        self.e2e_layout = {}
        if e2e_from is not None:
            for t in range(e2e_from, total_steps):
                rows_t = self.inputs[t][0][1].shape[0]
                lay = Packed([("q", dt, (n, sh.num_q_heads, sh.head_dim)), ("k", dt, row_shape(rows_t)),
                              ("v", dt, row_shape(rows_t))])
                self.e2e_layout[t] = lay
                self.host[t] = []
                for src in self.inputs[t]:
                    buf = torch.empty(lay.nbytes, dtype=torch.uint8).pin_memory()
                    views = lay.views(buf)
                    for name, x in zip(("q", "k", "v"), src):
                        views[name].copy_(x)
                    self.host[t].append(buf)
                self.e2e_bytes[t] = lay.end["v"]
        mb = self.max_blocks
        pin = lambda shape, dt: torch.empty(shape, dtype=dt).pin_memory()  # noqa: E731
        max_prompt = max([sum(p - self.prompt_start(p) for _, _, p in st["admitted"]) for st in self.plan] + [1])
        H, D2 = NSETS + 1, NSETS
        # one step's metadata, packed so that one copy uploads it; the slots come last --
        # the step's n token slots, then the admitted prompts' slots, matching the order of
        # the rows to append -- and only the used ones are copied
        self.meta = Packed([("tables", torch.int32, (n, mb)), ("lens", torch.int32, (n,)),
                            ("cow", torch.int32, (n, 2)), ("slots", torch.int64, (n + max_prompt,))])
        self.h_meta = [pin((self.meta.nbytes,), torch.uint8) for _ in range(H)]
        self.d_meta = [torch.empty(self.meta.nbytes, dtype=torch.uint8, device=device) for _ in range(D2)]
        hv = [self.meta.views(b) for b in self.h_meta]
        dv = [self.meta.views(b) for b in self.d_meta]
        self.h_tables, self.h_lens, self.h_cow, self.h_all_slots = (
            [v[k] for v in hv] for k in ("tables", "lens", "cow", "slots"))
        self.d_tables, self.d_lens, self.d_cow, self.d_slots = (
            [v[k] for v in dv] for k in ("tables", "lens", "cow", "slots"))
        self.h_slots = [x[:n] for x in self.h_all_slots]      # token slots
        self.h_pslots = [x[n:] for x in self.h_all_slots]     # admitted prompts' slots
        self.h_done = [None] * H
        self.d_free = [None] * D2
        if e2e_from is not None:
            big = max(lay.nbytes for lay in self.e2e_layout.values())
            self.d_in = [[torch.empty(big, dtype=torch.uint8, device=device) for _ in range(self.NL)]
                         for _ in range(D2)]
            for t, lay in self.e2e_layout.items():
                self.e2e_views[t] = [lay.views(b) for b in self.d_in[t % NSETS]]
        self.out = [torch.empty((self.NL, n, sh.num_q_heads, sh.head_dim), dtype=dt, device=device)
                    for _ in range(D2)]
        self.h_out = [pin(tuple(self.out[0].shape), dt) for _ in range(D2)] if e2e_from is not None else None
        self.out_read = [None] * D2
        self.ws = self.cache.workspace(n, sh.num_q_heads, mb, split)
        self.compute = torch.cuda.current_stream(device)
        self.copy = torch.cuda.Stream(device)
        self.readback = torch.cuda.Stream(device)
        self.scale = 1.0 / math.sqrt(sh.head_dim)
        self.attn_events = []
        self._kv_bytes, self._alg_bytes, self.h2d, self.d2h, self.prompt_rows_appended = [], [], [], [], []
        self._pending_lens = []   # each step's lengths, turned into byte counts off the step's path
        # events are made once and re-recorded: per staging set the upload's, per device set
        # the compute's and the read-back's, and a pair around each timed attention call
        self.up_ev = [torch.cuda.Event() for _ in range(H)]
        self.free_ev = [torch.cuda.Event() for _ in range(D2)]
        self.rd_ev = [torch.cuda.Event() for _ in range(D2)]
        self.attn_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                        for _ in range(total_steps * self.NL)]
        self.host_s = []
        self.flush = (torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=device) if workload in L2_RESIDENT
                      else None)

    def step(self, t, e2e=False, time_attention=True):
        torch, pa, sh, plan = self.torch, self.pa, self.shape, self.plan[t]
        n, hs, ds = self.n, t % (NSETS + 1), t % NSETS
        if self.h_done[hs] is not None:      # staging set hs: its uploads (NSETS + 1 steps ago) are done
            self.h_done[hs].synchronize()
        h0 = time.perf_counter()             # host work of this step, not counting that wait
        # 1. admissions: new sequences take the retired slots; their prompts are appended below
        ptot = 0
        if plan["admitted"]:
            new = []
            for slot, _, plen in plan["admitted"]:
                if self.system_keys is not None:       # share the cached system-prompt blocks
                    sid, hit = pa.pa_seq_add_cached(self.cache.pool, self.system_keys)
                    assert hit * sh.block_size == self.prompt_start(plen)
                else:
                    sid = self.cache.add()
                self.sids[slot] = sid
                self.sid_arr[slot] = sid
                new.append((sid, plen - self.prompt_start(plen)))
            pslots, _ = pa.pa_reserve_slots(self.cache.pool, [s for s, _ in new], [p for _, p in new],
                                            slot_out=self.h_pslots[hs])
            ptot = len(pslots)
        self.prompt_rows_appended.append(ptot)
        # 2. one slot per sequence for this step's token (new block, or copy-on-write of a shared tail)
        _, cow = pa.pa_reserve_slots(self.cache.pool, self.sid_arr, self.ones, slot_out=self.h_slots[hs],
                                     cow_out=self.h_cow[hs])
        ncow = len(cow)
        _, lens = pa.pa_build_block_tables(self.cache.pool, self.sid_arr, self.max_blocks, self.h_tables[hs],
                                           self.h_lens[hs])
        # 3. uploads (metadata; end to end also the step's inputs) on the copy stream
        if self.d_free[ds] is not None:
            self.copy.wait_event(self.d_free[ds])
        mbytes = self.meta.off["slots"] + (n + ptot) * 8     # everything through the used slots
        h2d = mbytes
        with torch.cuda.stream(self.copy):
            self.d_meta[ds][:mbytes].copy_(self.h_meta[hs][:mbytes], non_blocking=True)
            if e2e:
                layers = []
                nb = self.e2e_bytes[t]
                for layer, host in enumerate(self.host[t]):
                    self.d_in[ds][layer][:nb].copy_(host[:nb], non_blocking=True)
                    h2d += nb
                    v = self.e2e_views[t][layer]
                    layers.append((v["q"], v["k"], v["v"]))
            else:
                layers = self.inputs[t]
            up = self.up_ev[hs]
            up.record(self.copy)
        self.h_done[hs] = up
        self.compute.wait_event(up)
        if self.out_read[ds] is not None:    # the read-back of out[ds] (NSETS steps ago) is done
            self.compute.wait_event(self.out_read[ds])
        # 4. device work
        if self.flush is not None:           # evict the previous step's blocks from L2
            self.flush.fill_(t & 0xFF)
        if ncow:
            pa.pa_copy_blocks(self.cache.pool, self.d_cow[ds], ncow, stream=self.compute)
        for layer, (q, k, v) in enumerate(layers):
            # one launch appends the token rows and the admitted prompts' rows
            assert k.shape[0] == n + ptot
            pa.pa_append_kv(self.cache.pool, layer, k, v, self.d_slots[ds], n + ptot, stream=self.compute)
            if time_attention:
                e0, e1 = self.attn_ev[len(self.attn_events)]
                e0.record(self.compute)
            pa.pa_decode_attention(self.cache.pool, layer, q, self.out[ds][layer], self.d_tables[ds],
                                   self.d_lens[ds], self.scale, self.split, self.ws, stream=self.compute)
            if time_attention:
                e1.record(self.compute)
                self.attn_events.append((e0, e1))
        free = self.free_ev[ds]
        free.record(self.compute)
        self.d_free[ds] = free
        d2h = 0
        if e2e:                              # result read back on its own stream
            self.readback.wait_event(free)
            with torch.cuda.stream(self.readback):
                self.h_out[ds].copy_(self.out[ds], non_blocking=True)
                rd = self.rd_ev[ds]
                rd.record(self.readback)
            self.out_read[ds] = rd
            d2h = self.out[ds].numel() * self.out[ds].element_size()
        # 5. retirements: blocks go back to the free list at once
        for slot, _ in plan["retire"]:
            self.cache.free(self.sids[slot])
        self._pending_lens.append(lens.numpy().copy())   # counted in _settle, off this path
        self.host_s.append(time.perf_counter() - h0)
        self.h2d.append(h2d)
        self.d2h.append(d2h)

    def _settle(self):
        """Bytes decode attention read / wrote in each step recorded since the last call
        (all layers), from that step's sequence lengths."""
        sh, n = self.shape, self.n
        e = 2                                                  # bytes of a query / output element
        row = sh.head_dim + 1 if self.kv_fp8 else sh.head_dim * e   # cached bytes of one (token, head) row
        for lens in self._pending_lens:
            L = lens.astype(np.int64)
            kv = self.NL * int((2 * L * sh.num_kv_heads * row).sum())
            alg = kv + self.NL * (2 * n * sh.num_q_heads * sh.head_dim * e +
                                  int((4 * -(-L // sh.block_size)).sum()) + 4 * n)
            self._kv_bytes.append(kv)
            self._alg_bytes.append(alg)
        self._pending_lens.clear()

    @property
    def kv_bytes(self):
        """KV bytes decode attention read, per step so far."""
        self._settle()
        return self._kv_bytes

    @property
    def alg_bytes(self):
        """Algorithmic bytes of decode attention (KV, q, out, tables, lengths), per step."""
        self._settle()
        return self._alg_bytes

    def drain(self):
        """Make the compute stream wait for outstanding read-backs (end of a timed leg)."""
        for ev in self.out_read:
            if ev is not None:
                self.compute.wait_event(ev)


def run_ours(args):
    import torch
    import torch.distributed as dist
    import paged_kv_cache_403_b200 as pa

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the path has no CPU fallback)")
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=device)

    K, W, R = args.steps, args.warmup, args.repeats
    e2e = not args.no_e2e
    RE = min(R, 3) if e2e else 0          # end-to-end passes
    total = W + R * K + RE * K
    recipe = make_recipe(args.workload, replica_seed(rank), total)
    rep = Replica(torch, args.workload, recipe, total, args.split, device, W + R * K if e2e else None,
                  prefix_cache=args.prefix_cache == "on", kv_fp8=args.kv_dtype == "fp8")

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for t in range(W):
        rep.step(t, time_attention=False)
    rep.kv_bytes.clear()
    rep.alg_bytes.clear()
    rep.host_s.clear()
    rep.prompt_rows_appended.clear()
    barrier()
    clocks = ClockSampler(local)
    clocks.start()
    lc0 = pa.pa_launch_count()
    # R passes of K steps each over one continuing schedule; every pass is bracketed by a
    # barrier and a device synchronisation, and the median pass is reported
    pass_ms, pass_kv = [], []
    for r in range(R):
        barrier()
        kv0 = len(rep.kv_bytes)
        ev0 = torch.cuda.Event(enable_timing=True)
        ev1 = torch.cuda.Event(enable_timing=True)
        ev0.record(rep.compute)
        for t in range(W + r * K, W + (r + 1) * K):
            rep.step(t)
        ev1.record(rep.compute)
        barrier()
        pass_ms.append(ev0.elapsed_time(ev1))
        pass_kv.append(sum(rep.kv_bytes[kv0:]))
    launches = (pa.pa_launch_count() - lc0) / R
    prompt_rows = sum(rep.prompt_rows_appended) / R
    attn_ms = [a.elapsed_time(b) for a, b in rep.attn_events]
    alg_per_launch = sum(rep.alg_bytes) / (R * K * rep.NL)
    host_ms = 1e3 * sum(rep.host_s) / (R * K)

    e2e_ms, e2e_kv = [], []
    e2e_io = (0, 0)
    if e2e:
        rep.host_s.clear()
        rep.h2d.clear()
        rep.d2h.clear()
        for r in range(RE):
            barrier()
            kv0 = len(rep.kv_bytes)
            t0 = torch.cuda.Event(enable_timing=True)
            t1 = torch.cuda.Event(enable_timing=True)
            t0.record(rep.compute)
            base = W + R * K + r * K
            for t in range(base, base + K):
                rep.step(t, e2e=True, time_attention=False)
            rep.drain()
            t1.record(rep.compute)
            barrier()
            e2e_ms.append(t0.elapsed_time(t1))
            e2e_kv.append(sum(rep.kv_bytes[kv0:]))
        e2e_host_ms = 1e3 * sum(rep.host_s) / (RE * K)
        e2e_io = (sum(rep.h2d) / (RE * K), sum(rep.d2h) / (RE * K))
    clk = clocks.stop()

    if world > 1:   # per pass: the slowest rank's time, every rank's bytes
        times, byts = combine_ranks(dist, pass_ms + e2e_ms, pass_kv + e2e_kv, device)
        pass_ms, e2e_ms = times[:R], times[R:]
        pass_kv, e2e_kv = byts[:R], byts[R:]

    def median_pass(ms_list, kv_list):
        i = int(np.argsort(ms_list)[len(ms_list) // 2])
        return ms_list[i], kv_list[i]

    ms, kv_tot = median_pass(pass_ms, pass_kv)
    if e2e:
        e2e_ms_med, e2e_kv_med = median_pass(e2e_ms, e2e_kv)

    if rank == 0:
        peaks = {}
        pk_path = os.path.join(ROOT, "MEASURED_PEAKS.json")
        if os.path.exists(pk_path):
            peaks = json.load(open(pk_path))
        peak = float(peaks.get("hbm_gbs", 6650.0))
        peak_src = "measured" if "hbm_gbs" in peaks else "fallback"
        attn_mean_ms = float(np.mean(attn_ms))
        achieved = alg_per_launch / (attn_mean_ms * 1e-3) / 1e9
        value = kv_tot / (ms * 1e-3) / 1e9
        sh = rep.shape
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": W, "ms_per_step": round(ms / K, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "fp8_e4m3 cache, " + sh.dtype if rep.kv_fp8 else sh.dtype,
            "data": "synthetic (seeded counter-based K/V/q values; seeded lengths, pool order and stops)",
            "config": arm_config(args, sh, rep.n, world),
            "passes": {"n": R, "ms_per_step": [round(x / K, 4) for x in pass_ms],
                       "reported": "median pass; each pass is --steps steps of one continuing schedule"},
            "decode_tokens_per_s": round(world * rep.n * K / (ms * 1e-3), 1),
            "kv_gb_per_step": round(kv_tot / K / 1e9 / world, 4),
            "hbm_fraction_of_8tbs": round(value / world / NOMINAL_HBM_GBS, 4),
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(achieved / peak, 4),
                         "traffic": (captured_traffic(rep.kv_fp8) if args.workload == "continuous_batch"
                                     else None),
                         "kernel": ("fp8::decode_kernel" if rep.kv_fp8 else "paged_decode_mma_kernel")
                                   + " (+ plan_kernel; split partials merged in the kernel)",
                         "attn_ms_mean": round(attn_mean_ms, 4), "alg_bytes_per_launch": int(alg_per_launch),
                         "launches_timed": len(attn_ms), "peak_source": peak_src},
            "gpu_launches": int(round(launches)),   # per timed pass (mean over the passes)
            "host_ms_per_step": round(host_ms, 4),
            "device_error": pa.pa_device_error(),
            "clocks": clk,
        }
        stats = rep.pa.pa_pool_stats(rep.cache.pool)
        line["pool"] = {"peak_blocks_used": stats["peak_used"], "num_blocks": stats["num_blocks"],
                        "cache_hits": stats["cache_hits"], "cached_blocks": stats["num_cached"],
                        "prompt_rows_appended_per_step": round(prompt_rows / K, 1),
                        "prompt_bytes_appended_per_step": int(prompt_rows / K * 2 * sh.num_kv_heads
                                                              * sh.head_dim * 2 * rep.NL)}
        if args.workload == "shared_prompt":
            line["config"]["prefix_cache"] = args.prefix_cache
        if e2e:
            line["e2e"] = {"value": round(e2e_kv_med / (e2e_ms_med * 1e-3) / 1e9, 1), "unit": UNIT,
                           "h2d_bytes_per_step": int(e2e_io[0]), "d2h_bytes_per_step": int(e2e_io[1]),
                           "ms_per_step": round(e2e_ms_med / K, 4), "host_ms_per_step": round(e2e_host_ms, 4),
                           "passes": {"n": RE, "ms_per_step": [round(x / K, 4) for x in e2e_ms]}}
        if not args.no_cpu_baseline and args.workload not in ("prefix_sharing", "shared_prompt") and not rep.kv_fp8:
            line["cpu_baseline"] = cpu_baseline(rep, args.cpu_sample_seqs, W, args.cpu_seconds)
        print(json.dumps(line), flush=True)
        if line["device_error"]:
            print(f"bench.py: the kernels reported device error word {line['device_error']:#x}; "
                  "the figures above are not of a valid run", file=sys.stderr)
    bad = rank == 0 and bool(line["device_error"])
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if bad:
        raise SystemExit(1)


# ---------------------------------------------------------------------------- oracle (CPU)
def oracle_sample(recipe, plan_step, picks, layer=0):
    """Host inputs for the sampled sequences of one step, regenerated from the seeded
    generator (never read from the GPU): each sequence's history laid contiguously."""
    from synthetic import values as sv
    sh = recipe["shape"]
    B, hkv, d = sh.block_size, sh.num_kv_heads, sh.head_dim
    ks, vs, tabs, lens, qs = [], [], [], [], []
    nb = 0
    for i in picks:
        uid, L = int(plan_step["uids"][i]), int(plan_step["pos"][i]) + 1
        pos = np.arange(L)
        k = sv.rows(sv.KIND_K, recipe["seed"], layer, np.full(L, uid), pos, hkv, d, sh.kv_scale, sh.dtype)
        v = sv.rows(sv.KIND_V, recipe["seed"], layer, np.full(L, uid), pos, hkv, d, sh.kv_scale, sh.dtype)
        nblk = -(-L // B)
        pad = nblk * B - L
        k = np.concatenate([k, np.zeros((pad, hkv, d), k.dtype)]).reshape(nblk, B, hkv, d).transpose(0, 2, 1, 3)
        v = np.concatenate([v, np.zeros((pad, hkv, d), v.dtype)]).reshape(nblk, B, hkv, d).transpose(0, 2, 1, 3)
        ks.append(k)
        vs.append(v)
        tabs.append(np.arange(nb, nb + nblk))
        nb += nblk
        lens.append(L)
        qs.append(sv.rows(sv.KIND_Q, recipe["seed"], layer, [uid], [L - 1], sh.num_q_heads, d, sh.q_scale,
                          sh.dtype)[0])
    mb = max(len(t) for t in tabs)
    tables = np.full((len(picks), mb), -1, np.int32)
    for j, t in enumerate(tabs):
        tables[j, :len(t)] = t
    return (np.ascontiguousarray(np.concatenate(ks)), np.ascontiguousarray(np.concatenate(vs)), tables,
            np.array(lens, np.int32), np.stack(qs))


def time_oracle(recipe, plan_step, picks, min_seconds=0.0, max_reps=1000, n_threads=0):
    """Runs the oracle (as it stands) on the sample, repeated until min_seconds have passed
    (n_threads 0: every host core)."""
    import oracle
    sh = recipe["shape"]
    k, v, tables, lens, q = oracle_sample(recipe, plan_step, picks)
    kv1 = int((2 * lens.astype(np.int64) * sh.num_kv_heads * sh.head_dim * 2).sum())
    reps, dt = 0, 0.0
    while reps < max_reps and (reps == 0 or dt < min_seconds):
        t0 = time.perf_counter()
        oracle.paged_decode(k, v, sh.dtype, tables, lens, q, 1.0 / math.sqrt(sh.head_dim), n_threads)
        dt += time.perf_counter() - t0
        reps += 1
    return kv1 * reps, dt, reps, kv1


def cpu_baseline(rep, nseq, step, seconds):
    import oracle
    picks = list(range(0, rep.n, max(1, rep.n // nseq)))[:nseq]
    kv, dt, reps, kv1 = time_oracle(rep.recipe, rep.plan[step], picks, min_seconds=seconds)
    kv_1, dt_1, _, _ = time_oracle(rep.recipe, rep.plan[step], picks, min_seconds=seconds / 4, n_threads=1)
    layers = f"; 1 of {rep.NL} layers" if rep.NL > 1 else ""
    return {"value": round(kv / dt / 1e9, 4), "unit": UNIT, "cores": oracle.max_threads(), "kind": "oracle",
            "value_1_thread": round(kv_1 / dt_1 / 1e9, 4),
            "sample": f"fp64 oracle attention for {len(picks)} of {rep.n} sequences of one decode step "
                      f"({kv1 / 1e6:.1f} MB of KV{layers}), repeated {reps}x for {dt:.1f} s; "
                      f"OpenMP over (sequence, head); value_1_thread: the same sample on one thread "
                      f"for {dt_1:.1f} s"}


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    from synthetic import workloads as wl
    if args.workload != "continuous_batch" or args.kv_dtype != "native":
        raise SystemExit("bench.py --impl reference times the oracle on the continuous batch (bf16 cache) only")
    K, W = args.steps, args.warmup
    recipe = wl.continuous_batch(seed=3, steps=W + K)
    plan = simulate(recipe["schedule"], len(recipe["schedule"].initial), W + K)
    nseq = 4
    for t in range(W):
        time_oracle(recipe, plan[t], list(range(t * nseq % 256, t * nseq % 256 + nseq)))
    kv_tot, dt_tot = 0, 0.0
    for t in range(W, W + K):
        kv, dt, _, _ = time_oracle(recipe, plan[t], list(range(t * nseq % 256, t * nseq % 256 + nseq)))
        kv_tot += kv
        dt_tot += dt
    value = kv_tot / dt_tot / 1e9
    sample = (f"each step: fp64 oracle attention for {nseq} of the 256 sequences of that step (KV bytes of "
              "those sequences / oracle wall time), OpenMP over (sequence, head)")
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": world,
            "steps": K, "warmup": W, "ms_per_step": round(dt_tot / K * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": arm_config(args, recipe["shape"], len(recipe["schedule"].initial), world),
            "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": oracle.max_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_swap(args):
    """Preemption with swap: 64 sequences of the continuous batch (~0.5 GB of cache) moved to
    page-locked host memory and back, timed with CUDA events, next to a plain pinned
    cudaMemcpy of the same size (the PCIe roofline of this box)."""
    import torch
    import paged_kv_cache_403_b200 as pa
    from paged_kv_cache_403_b200.engine import PagedCache
    from paged_kv_cache_403_b200.runners import DeviceGen, prefill
    from synthetic import workloads as wl
    torch.cuda.set_device(0)
    r = wl.continuous_batch(seed=3, steps=1)
    sh = r["shape"]
    cache = PagedCache.from_shape(sh, r["order"], "cuda")
    gen = DeviceGen(r["seed"], sh, "cuda")
    lens = [int(x) for x in r["schedule"].initial]
    sids = [cache.add() for _ in lens]
    prefill(cache, gen, sids, list(range(len(lens))), lens)
    victims = sids[:64]
    sizes = [pa.pa_swap_bytes(cache.pool, s) for s in victims]
    bufs = [torch.empty(n, dtype=torch.uint8).pin_memory() for n in sizes]
    total = sum(sizes)
    st = torch.cuda.current_stream()

    def timed(fn):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(st)
        fn()
        e1.record(st)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1)

    def out_all():
        for s, b in zip(victims, bufs):
            pa.pa_swap_out(cache.pool, s, b)

    def in_all():
        for s, b in zip(victims, bufs):
            pa.pa_swap_in(cache.pool, s, b)

    results = {"out": [], "in": []}
    for rep in range(args.warmup + args.steps):
        t_out = timed(out_all)
        t_in = timed(in_all)
        if rep >= args.warmup:
            results["out"].append(t_out)
            results["in"].append(t_in)
    dev = torch.empty(total, dtype=torch.uint8, device="cuda")
    host = torch.empty(total, dtype=torch.uint8).pin_memory()
    d2h = min(timed(lambda: host.copy_(dev, non_blocking=True)) for _ in range(5))
    h2d = min(timed(lambda: dev.copy_(host, non_blocking=True)) for _ in range(5))
    gbs = lambda ms: total / (ms * 1e-3) / 1e9  # noqa: E731
    out_ms, in_ms = float(np.median(results["out"])), float(np.median(results["in"]))
    line = {"metric": "swap GB/s (device->host and host->device of a sequence's KV blocks)",
            "value": round(gbs(out_ms + in_ms) * 2, 1), "unit": "GB/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "higher_is_better": True, "dtype": sh.dtype, "data": "synthetic",
            "config": {"workload": f"swap 64 of 256 continuous-batch sequences, {total / 1e6:.0f} MB of KV"},
            "swap_out": {"ms": round(out_ms, 3), "GB/s": round(gbs(out_ms), 1)},
            "swap_in": {"ms": round(in_ms, 3), "GB/s": round(gbs(in_ms), 1)},
            "roofline": {"bound": "pcie", "d2h_memcpy_GB/s": round(gbs(d2h), 1), "h2d_memcpy_GB/s": round(gbs(h2d), 1),
                         "frac_out": round(gbs(out_ms) / gbs(d2h), 3), "frac_in": round(gbs(in_ms) / gbs(h2d), 3)},
            "device_error": pa.pa_device_error()}
    print(json.dumps(line), flush=True)


def prefill_setup(torch, recipe, device="cuda"):
    """Cache holding every sequence's tokens, the chunk queries and the launch metadata."""
    from paged_kv_cache_403_b200.engine import PagedCache
    from paged_kv_cache_403_b200.runners import DeviceGen, prefill
    sh = recipe["shape"]
    cache = PagedCache.from_shape(sh, recipe["order"], device)
    gen = DeviceGen(recipe["seed"], sh, device)
    lens = [int(x) for x in recipe["lens"]]
    chunks = [int(x) for x in recipe["chunks"]]
    sids = [cache.add() for _ in lens]
    prefill(cache, gen, sids, list(range(len(lens))), lens)
    uids = np.concatenate([np.full(c, s) for s, c in enumerate(chunks)])
    pos = np.concatenate([np.arange(L - c, L) for L, c in zip(lens, chunks)])
    q = gen.q(0, uids, pos)
    max_blocks = max(-(-L // sh.block_size) for L in lens)
    tables, ln = cache.tables(sids, max_blocks)
    q_start = np.concatenate([[0], np.cumsum(chunks)]).astype(np.int32)
    flops = sum(4.0 * (L - c + i + 1) * sh.num_q_heads * sh.head_dim for L, c in zip(lens, chunks) for i in range(c))
    return dict(cache=cache, q=q, tables=torch.from_numpy(tables).to(device), lens=torch.from_numpy(ln).to(device),
                q_start=torch.from_numpy(q_start).to(device), max_q=max(chunks), flops=flops, rows=int(q_start[-1]),
                lens_list=lens, chunks=chunks, uids=uids, pos=pos, tables_np=tables)


def run_prefill(args):
    """Chunked-prefill attention (tcgen05) on the synthetic chunked-prefill workload."""
    import torch
    import paged_kv_cache_403_b200 as pa
    from synthetic import workloads as wl
    torch.cuda.set_device(0)
    r = wl.chunked_prefill(dtype=args.dtype)
    sh = r["shape"]
    c = prefill_setup(torch, r)
    out = torch.empty((c["rows"], sh.num_q_heads, sh.head_dim),
                      dtype=torch.bfloat16 if args.dtype == "bf16" else torch.float16, device="cuda")
    st = torch.cuda.current_stream()
    scale = 1.0 / math.sqrt(sh.head_dim)

    def call():
        pa.pa_prefill_attention(c["cache"].pool, 0, c["q"], out, c["tables"], c["lens"], c["q_start"], c["max_q"],
                                scale)
    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    clocks = ClockSampler(0)
    clocks.start()
    lc0 = pa.pa_launch_count()
    evs = []
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(st)
    for _ in range(args.steps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(st)
        call()
        b.record(st)
        evs.append((a, b))
    t1.record(st)
    torch.cuda.synchronize()
    clk = clocks.stop()
    ms = t0.elapsed_time(t1)
    kern_ms = float(np.mean([a.elapsed_time(b) for a, b in evs]))
    peaks = {}
    pk_path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(pk_path):
        peaks = json.load(open(pk_path))
    peak = float(peaks.get("bf16_tflops", 1590.0))
    achieved = c["flops"] / (kern_ms * 1e-3) / 1e12
    line = {"metric": "paged chunked-prefill attention TFLOP/s and prefill tokens/s", "impl": "ours",
            "value": round(c["flops"] * args.steps / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 4),
            "higher_is_better": True, "dtype": args.dtype, "data": "synthetic",
            "config": {"workload": "chunked_prefill: 32 seqs, lengths U[1024,4096], last 512 tokens as queries, "
                                   "block 16, 32 q / 8 KV heads, d128, " + args.dtype},
            "prefill_tokens_per_s": round(c["rows"] * args.steps / (ms * 1e-3), 1),
            "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
                         "frac": round(achieved / peak, 4), "traffic": None, "kernel": "paged_prefill_kernel",
                         "kernel_ms": round(kern_ms, 4), "flops_per_launch": c["flops"],
                         "peak_source": "measured" if "bf16_tflops" in peaks else "fallback"},
            "gpu_launches": pa.pa_launch_count() - lc0, "clocks": clk, "device_error": pa.pa_device_error()}
    if not args.no_cpu_baseline:
        import oracle
        import time as _t
        from synthetic import values as sv
        s0 = 0
        L, C = c["lens_list"][s0], c["chunks"][s0]
        k = sv.rows(sv.KIND_K, r["seed"], 0, np.zeros(L, np.int64), np.arange(L), sh.num_kv_heads, sh.head_dim,
                    sh.kv_scale, sh.dtype)
        v = sv.rows(sv.KIND_V, r["seed"], 0, np.zeros(L, np.int64), np.arange(L), sh.num_kv_heads, sh.head_dim,
                    sh.kv_scale, sh.dtype)
        nblk = -(-L // sh.block_size)
        pad = nblk * sh.block_size - L
        shp = (nblk, sh.block_size, sh.num_kv_heads, sh.head_dim)
        kp = np.concatenate([k, np.zeros((pad,) + k.shape[1:], k.dtype)]).reshape(shp).transpose(0, 2, 1, 3)
        vp = np.concatenate([v, np.zeros((pad,) + v.shape[1:], v.dtype)]).reshape(shp).transpose(0, 2, 1, 3)
        qq = sv.rows(sv.KIND_Q, r["seed"], 0, np.zeros(C, np.int64), np.arange(L - C, L), sh.num_q_heads,
                     sh.head_dim, sh.q_scale, sh.dtype)
        fl = sum(4.0 * (L - C + i + 1) * sh.num_q_heads * sh.head_dim for i in range(C))
        reps, dt = 0, 0.0
        while reps == 0 or dt < args.cpu_seconds:
            t = _t.perf_counter()
            oracle.paged_prefill(np.ascontiguousarray(kp), np.ascontiguousarray(vp), sh.dtype,
                                 np.arange(nblk, dtype=np.int32)[None], [L], [0, C], qq, scale)
            dt += _t.perf_counter() - t
            reps += 1
        line["cpu_baseline"] = {"value": round(fl * reps / dt / 1e12, 6), "unit": "TFLOP/s",
                                "cores": oracle.max_threads(), "kind": "oracle",
                                "sample": f"fp64 oracle prefill of sequence 0 ({C} queries over {L} keys), "
                                          f"repeated {reps}x for {dt:.1f} s"}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.workload == "swap":
        run_swap(args)
        return
    if args.workload == "prefill":
        run_prefill(args)
        return
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
