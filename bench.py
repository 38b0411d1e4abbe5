#!/usr/bin/env python
"""Benchmark: paged decode attention on the continuous-batch workload.

Workload (one replica per GPU): 256 sequences, prompt lengths uniform in
[128, 4096], block 16, 32 query / 8 KV heads, head_dim 128, bf16 cache; every step
each sequence appends one token and attends over its whole cache; after each step
every sequence stops with probability 1/200 and a new one (prompt length uniform
in [128, 4096]) takes its slot at the next step.  A timed step runs the whole
path: admissions (prompt K/V appended), one-slot reservations (host), metadata
upload, append of the step's K/V, decode attention (+ split-K reduce),
retirements (host).

Prints one JSON line (rank 0).  ``value`` is KV bytes read by decode attention per
second over the timed steps (whole-job, all ranks); decode tokens/s is reported
beside it.  ``--impl reference`` times the CPU oracle instead on a bounded sample.
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


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=64)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--split", type=int, default=2048, help="tokens per split-K range (0: never split)")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-sample-seqs", type=int, default=24)
    return ap.parse_args()


def captured_traffic():
    """DRAM bytes per launch of the decode kernel from the committed ncu summary, if the
    kernel source is still the one that was captured (else None)."""
    import hashlib
    import re
    prof = os.path.join(ROOT, "profiles", "decode_mma_continuous_batch.md")
    src = os.path.join(ROOT, "paged_kv_cache_403_b200", "csrc", "kernels.cu")
    try:
        text = open(prof).read()
        sha = re.search(r"kernels.cu sha256 prefix at capture: ([0-9a-f]+)", text).group(1)
        gb = float(re.search(r"traffic per launch \(read \+ write\) \| ([0-9.]+) GB", text).group(1))
    except (OSError, AttributeError):
        return None
    if not hashlib.sha256(open(src, "rb").read()).hexdigest().startswith(sha):
        return None
    return int(gb * 1e9)


# ---------------------------------------------------------------------------- schedule
def simulate(sched, n, steps):
    """Host-side replay of the schedule: per step the uids, token positions and admissions."""
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
        pending = []
        plan.append(dict(uids=uids.copy(), pos=lens.copy(), admitted=admitted,
                         retire=list(sched.events[t])))
        lens += 1
        pending = list(sched.events[t])
    return plan


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
    """Each rank runs an independent replica of the workload with its own draws."""
    return 3 + 100 * rank


# ---------------------------------------------------------------------------- our path
class Replica:
    """One GPU's continuous-batch state, inputs pre-generated in HBM."""

    def __init__(self, torch, recipe, total_steps, split, device, e2e_from):
        from paged_kv_cache_403_b200.engine import PagedCache
        from paged_kv_cache_403_b200.runners import DeviceGen, prefill
        import paged_kv_cache_403_b200 as pa
        self.torch, self.pa = torch, pa
        self.recipe, self.shape = recipe, recipe["shape"]
        sh = self.shape
        self.n = n = len(recipe["schedule"].initial)
        self.split = split
        self.device = device
        self.plan = simulate(recipe["schedule"], n, total_steps)
        self.cache = PagedCache.from_shape(sh, recipe["order"], device)
        gen = DeviceGen(recipe["seed"], sh, device)
        self.sids = [self.cache.add() for _ in range(n)]
        prefill(self.cache, gen, self.sids, list(range(n)), [int(x) for x in recipe["schedule"].initial])
        self.max_blocks = -(-(4096 + total_steps + 1) // sh.block_size)
        # per-step inputs, generated on the device before any timing
        self.q, self.kn, self.vn, self.pk, self.pv = [], [], [], [], []
        for t, st in enumerate(self.plan):
            k, v = gen.kv(0, st["uids"], st["pos"])
            self.kn.append(k)
            self.vn.append(v)
            self.q.append(gen.q(0, st["uids"], st["pos"]))
            if st["admitted"]:
                u = np.concatenate([np.full(p, uid) for _, uid, p in st["admitted"]])
                tk = np.concatenate([np.arange(p) for _, _, p in st["admitted"]])
                pk, pv = gen.kv(0, u, tk)
            else:
                pk = pv = None
            self.pk.append(pk)
            self.pv.append(pv)
        # host copies for the end-to-end variant (pinned)
        self.host = {}
        if e2e_from is not None:
            for t in range(e2e_from, total_steps):
                self.host[t] = [None if x is None else x.cpu().pin_memory()
                                for x in (self.q[t], self.kn[t], self.vn[t], self.pk[t], self.pv[t])]
        # metadata: pinned host staging (3 sets) and device buffers (2 sets)
        mb = self.max_blocks
        pin = lambda shape, dt: torch.empty(shape, dtype=dt).pin_memory()  # noqa: E731
        self.h_tables = [pin((n, mb), torch.int32) for _ in range(3)]
        self.h_lens = [pin((n,), torch.int32) for _ in range(3)]
        self.h_slots = [pin((n,), torch.int64) for _ in range(3)]
        max_prompt = max([sum(p for _, _, p in st["admitted"]) for st in self.plan] + [1])
        self.h_pslots = [pin((max_prompt,), torch.int64) for _ in range(3)]
        self.h_cow = [pin((n, 2), torch.int32) for _ in range(3)]
        self.h_done = [None, None, None]
        self.d_tables = [torch.empty((n, mb), dtype=torch.int32, device=device) for _ in range(2)]
        self.d_lens = [torch.empty((n,), dtype=torch.int32, device=device) for _ in range(2)]
        self.d_slots = [torch.empty((n,), dtype=torch.int64, device=device) for _ in range(2)]
        self.d_pslots = [torch.empty((max_prompt,), dtype=torch.int64, device=device) for _ in range(2)]
        self.d_free = [None, None]
        self.d_in = [[torch.empty_like(x) for x in (self.q[0], self.kn[0], self.vn[0])] for _ in range(2)]
        self.d_pk = [torch.empty((max_prompt, sh.num_kv_heads, sh.head_dim), dtype=self.q[0].dtype,
                                 device=device) for _ in range(2)]
        self.d_pv = [torch.empty_like(self.d_pk[0]) for _ in range(2)]
        self.out = torch.empty((n, sh.num_q_heads, sh.head_dim), dtype=self.q[0].dtype, device=device)
        self.h_out = [pin(tuple(self.out.shape), self.out.dtype) for _ in range(2)]
        self.ws = self.cache.workspace(n, sh.num_q_heads, mb, split)
        self.compute = torch.cuda.current_stream(device)
        self.copy = torch.cuda.Stream(device)
        self.scale = 1.0 / math.sqrt(sh.head_dim)
        self.attn_events = []
        self.kv_bytes = []
        self.alg_bytes = []
        self.launches_before = 0

    def step(self, t, e2e=False, time_attention=True):
        torch, pa, sh, plan = self.torch, self.pa, self.shape, self.plan[t]
        n, hs, ds = self.n, t % 3, t % 2
        # host staging set hs is free once the copies that used it (3 steps ago) are done
        if self.h_done[hs] is not None:
            self.h_done[hs].synchronize()
        # 1. admissions: new sequences take the retired slots, their prompts are appended
        ptot = 0
        if plan["admitted"]:
            new = []
            for slot, _, plen in plan["admitted"]:
                self.sids[slot] = self.cache.add()
                new.append((self.sids[slot], plen))
            pslots, cow = pa.pa_reserve_slots(self.cache.pool, [s for s, _ in new], [p for _, p in new],
                                              slot_out=self.h_pslots[hs])
            ptot = len(pslots)
        # 2. one slot per sequence for this step's token (new block or copy-on-write)
        slots, cow = pa.pa_reserve_slots(self.cache.pool, self.sids, [1] * n, slot_out=self.h_slots[hs],
                                         cow_out=self.h_cow[hs])
        assert len(cow) == 0          # no sharing in this workload
        tables, lens = pa.pa_build_block_tables(self.cache.pool, self.sids, self.max_blocks,
                                                self.h_tables[hs], self.h_lens[hs])
        # 3. upload metadata (and, end to end, the step's inputs) on the copy stream
        if self.d_free[ds] is not None:
            self.copy.wait_event(self.d_free[ds])
        with torch.cuda.stream(self.copy):
            self.d_tables[ds].copy_(self.h_tables[hs], non_blocking=True)
            self.d_lens[ds].copy_(self.h_lens[hs], non_blocking=True)
            self.d_slots[ds].copy_(self.h_slots[hs], non_blocking=True)
            if ptot:
                self.d_pslots[ds][:ptot].copy_(self.h_pslots[hs][:ptot], non_blocking=True)
            if e2e:
                hq, hk, hv, hpk, hpv = self.host[t]
                q, kn, vn = self.d_in[ds]
                q.copy_(hq, non_blocking=True)
                kn.copy_(hk, non_blocking=True)
                vn.copy_(hv, non_blocking=True)
                if ptot:
                    self.d_pk[ds][:ptot].copy_(hpk, non_blocking=True)
                    self.d_pv[ds][:ptot].copy_(hpv, non_blocking=True)
                pk, pv = self.d_pk[ds][:ptot], self.d_pv[ds][:ptot]
            else:
                q, kn, vn, pk, pv = self.q[t], self.kn[t], self.vn[t], self.pk[t], self.pv[t]
            up = torch.cuda.Event()
            up.record(self.copy)
        self.h_done[hs] = up
        self.compute.wait_event(up)
        # 4. device work on the compute stream
        if ptot:
            pa.pa_append_kv(self.cache.pool, 0, pk, pv, self.d_pslots[ds], ptot, stream=self.compute)
        pa.pa_append_kv(self.cache.pool, 0, kn, vn, self.d_slots[ds], n, stream=self.compute)
        if time_attention:
            e0 = torch.cuda.Event(enable_timing=True)
            e0.record(self.compute)
        pa.pa_decode_attention(self.cache.pool, 0, q, self.out, self.d_tables[ds], self.d_lens[ds], self.scale,
                               self.split, self.ws, stream=self.compute)
        if time_attention:
            e1 = torch.cuda.Event(enable_timing=True)
            e1.record(self.compute)
            self.attn_events.append((e0, e1))
        free = torch.cuda.Event()
        free.record(self.compute)
        self.d_free[ds] = free
        if e2e:
            self.h_out[ds].copy_(self.out, non_blocking=True)
        # 5. retirements: blocks go back to the free list at once
        for slot, _ in plan["retire"]:
            self.cache.free(self.sids[slot])
        # accounting (host): KV bytes the attention reads this step
        L = lens.numpy().astype(np.int64)
        e = 2
        kv = int((2 * L * sh.num_kv_heads * sh.head_dim * e).sum())
        alg = kv + 2 * n * sh.num_q_heads * sh.head_dim * e + int((4 * -(-L // sh.block_size)).sum()) + 4 * n
        self.kv_bytes.append(kv)
        self.alg_bytes.append(alg)
        return ptot


def run_ours(args):
    import torch
    import torch.distributed as dist
    from synthetic import workloads as wl
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

    K, W = args.steps, args.warmup
    e2e = not args.no_e2e
    total = W + K + (K if e2e else 0)
    recipe = wl.continuous_batch(seed=replica_seed(rank), steps=total)
    rep = Replica(torch, recipe, total, args.split, device, W + K if e2e else None)
    torch.cuda.synchronize()

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for t in range(W):
        rep.step(t, time_attention=False)
    rep.kv_bytes.clear()
    rep.alg_bytes.clear()
    barrier()
    clocks = ClockSampler(local)
    clocks.start()
    lc0 = pa.pa_launch_count()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    ev0.record(rep.compute)
    for t in range(W, W + K):
        rep.step(t)
    ev1.record(rep.compute)
    barrier()
    launches = pa.pa_launch_count() - lc0
    ms = ev0.elapsed_time(ev1)
    kv_bytes = sum(rep.kv_bytes)
    attn_ms = [a.elapsed_time(b) for a, b in rep.attn_events]
    alg_bytes = list(rep.alg_bytes)

    e2e_res = None
    if e2e:
        rep.kv_bytes.clear()
        rep.alg_bytes.clear()
        barrier()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(rep.compute)
        h2d = d2h = 0
        for t in range(W + K, W + 2 * K):
            ptot = rep.step(t, e2e=True, time_attention=False)
            sh = rep.shape
            h2d += (rep.q[t].numel() + rep.kn[t].numel() + rep.vn[t].numel() + 2 * ptot * sh.num_kv_heads
                    * sh.head_dim) * 2
            h2d += rep.n * rep.max_blocks * 4 + rep.n * 4 + rep.n * 8 + ptot * 8
            d2h += rep.out.numel() * 2
        t1.record(rep.compute)
        barrier()
        e_ms = t0.elapsed_time(t1)
        e_kv = sum(rep.kv_bytes)
        e2e_res = (e_ms, e_kv, h2d / K, d2h / K)
    clk = clocks.stop()

    # whole-job numbers: bytes summed over ranks, time = max over ranks
    if world > 1:
        (ms, e2e_ms), (kv_tot, e2e_kv) = combine_ranks(
            dist, [ms, e2e_res[0] if e2e_res else 0.0], [kv_bytes, e2e_res[1] if e2e_res else 0], device)
    else:
        kv_tot = kv_bytes
        e2e_ms, e2e_kv = (e2e_res[0], e2e_res[1]) if e2e_res else (0.0, 0)

    if rank == 0:
        import json as _json
        peaks = {}
        pk_path = os.path.join(ROOT, "MEASURED_PEAKS.json")
        if os.path.exists(pk_path):
            peaks = _json.load(open(pk_path))
        peak = float(peaks.get("hbm_gbs", 6650.0))
        peak_src = "measured" if "hbm_gbs" in peaks else "fallback"
        attn_mean_ms = float(np.mean(attn_ms))
        alg_mean = float(np.mean(alg_bytes))
        achieved = alg_mean / (attn_mean_ms * 1e-3) / 1e9
        value = kv_tot / (ms * 1e-3) / 1e9
        tokens_per_s = world * rep.n * K / (ms * 1e-3)
        line = {
            "metric": METRIC, "value": round(value, 1), "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": W, "ms_per_step": round(ms / K, 4), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded counter-based K/V/q, "
            "seeded lengths and stops)",
            "config": {"workload": "continuous_batch: 256 seqs, lengths U[128,4096], block 16, "
                       "32 q / 8 KV heads, d128, bf16, p_stop 1/200, 1 layer", "n_seqs": rep.n,
                       "block_size": 16, "num_q_heads": 32, "num_kv_heads": 8, "head_dim": 128,
                       "split_tokens": args.split, "parallelism": f"replicas x{world}",
                       "l2": "inputs larger than L2 (KV read per step ~2.2 GB > 126 MB)"},
            "decode_tokens_per_s": round(tokens_per_s, 1),
            "kv_gb_per_step": round(kv_tot / K / 1e9 / world, 4),
            "hbm_fraction_of_8tbs": round(value / world / NOMINAL_HBM_GBS, 4),
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(achieved / peak, 4), "traffic": captured_traffic(),
                         "kernel": "paged_decode_mma_kernel (+ split_reduce_kernel)",
                         "attn_ms_mean": round(attn_mean_ms, 4),
                         "alg_bytes_per_launch": int(alg_mean), "peak_source": peak_src},
            "gpu_launches": int(launches),
            "clocks": clk,
        }
        if e2e_res:
            line["e2e"] = {"value": round(e2e_kv / (e2e_ms * 1e-3) / 1e9, 1), "unit": UNIT,
                           "h2d_bytes_per_step": int(e2e_res[2]), "d2h_bytes_per_step": int(e2e_res[3]),
                           "ms_per_step": round(e2e_ms / K, 4)}
        if not args.no_cpu_baseline and world == 1:
            line["cpu_baseline"] = cpu_baseline(recipe, rep, args.cpu_sample_seqs, W)
        elif not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline(recipe, rep, args.cpu_sample_seqs, W)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


# ---------------------------------------------------------------------------- oracle (CPU)
def oracle_sample(recipe, plan_step, picks):
    """Host inputs (regenerated) for the sampled sequences of one step: contiguous pools."""
    from synthetic import values as sv
    sh = recipe["shape"]
    B, hkv, d = sh.block_size, sh.num_kv_heads, sh.head_dim
    ks, vs, tabs, lens, qs = [], [], [], [], []
    nb = 0
    for i in picks:
        uid, L = int(plan_step["uids"][i]), int(plan_step["pos"][i]) + 1
        pos = np.arange(L)
        k = sv.rows(sv.KIND_K, recipe["seed"], 0, np.full(L, uid), pos, hkv, d, sh.kv_scale, sh.dtype)
        v = sv.rows(sv.KIND_V, recipe["seed"], 0, np.full(L, uid), pos, hkv, d, sh.kv_scale, sh.dtype)
        nblk = -(-L // B)
        pad = nblk * B - L
        k = np.concatenate([k, np.zeros((pad, hkv, d), k.dtype)]).reshape(nblk, B, hkv, d).transpose(0, 2, 1, 3)
        v = np.concatenate([v, np.zeros((pad, hkv, d), v.dtype)]).reshape(nblk, B, hkv, d).transpose(0, 2, 1, 3)
        ks.append(k)
        vs.append(v)
        tabs.append(np.arange(nb, nb + nblk))
        nb += nblk
        lens.append(L)
        qs.append(sv.rows(sv.KIND_Q, recipe["seed"], 0, [uid], [L - 1], sh.num_q_heads, d, sh.q_scale,
                          sh.dtype)[0])
    mb = max(len(t) for t in tabs)
    tables = np.full((len(picks), mb), -1, np.int32)
    for j, t in enumerate(tabs):
        tables[j, :len(t)] = t
    return (np.ascontiguousarray(np.concatenate(ks)), np.ascontiguousarray(np.concatenate(vs)), tables,
            np.array(lens, np.int32), np.stack(qs))


def time_oracle(recipe, plan_step, picks):
    import oracle
    sh = recipe["shape"]
    k, v, tables, lens, q = oracle_sample(recipe, plan_step, picks)
    t0 = time.perf_counter()
    oracle.paged_decode(k, v, sh.dtype, tables, lens, q, 1.0 / math.sqrt(sh.head_dim))
    dt = time.perf_counter() - t0
    kv = int((2 * lens.astype(np.int64) * sh.num_kv_heads * sh.head_dim * 2).sum())
    return kv, dt


def cpu_baseline(recipe, rep, nseq, step):
    import oracle
    picks = list(range(0, rep.n, max(1, rep.n // nseq)))[:nseq]
    kv, dt = time_oracle(recipe, rep.plan[step], picks)
    return {"value": round(kv / dt / 1e9, 4), "unit": UNIT, "cores": oracle.max_threads(), "kind": "oracle",
            "sample": f"fp64 oracle attention for {len(picks)} of {rep.n} sequences of one decode step "
                      f"({kv / 1e6:.1f} MB of KV), OpenMP over (sequence, head)", "seconds": round(dt, 3)}


def run_reference(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    from synthetic import workloads as wl
    K, W = args.steps, args.warmup
    recipe = wl.continuous_batch(seed=3, steps=W + K)
    plan = simulate(recipe["schedule"], len(recipe["schedule"].initial), W + K)
    nseq = 4
    for t in range(W):
        time_oracle(recipe, plan[t], list(range(t * nseq % 256, t * nseq % 256 + nseq)))
    kv_tot, dt_tot = 0, 0.0
    for t in range(W, W + K):
        kv, dt = time_oracle(recipe, plan[t], list(range(t * nseq % 256, t * nseq % 256 + nseq)))
        kv_tot += kv
        dt_tot += dt
    value = kv_tot / dt_tot / 1e9
    sample = (f"each step: fp64 oracle attention for {nseq} of 256 sequences (KV bytes of those "
              f"sequences / oracle wall time), OpenMP over (sequence, head)")
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": UNIT, "n_gpus": world,
            "steps": K, "warmup": W, "ms_per_step": round(dt_tot / K * 1e3, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "continuous_batch: 256 seqs, lengths U[128,4096], block 16, 32 q / 8 KV "
                       "heads, d128, bf16, p_stop 1/200, 1 layer", "parallelism": "cpu"},
            "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": oracle.max_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
