"""The seeded input generator (CPU): published SplitMix64 outputs, determinism,
moments, rounding rules and the workload recipes' sizes."""
import math

import numpy as np
import torch

from synthetic import values as sv
from synthetic import workloads as wl


def test_splitmix64_published_outputs():
    # seed 0: first three outputs of the SplitMix64 stream (Steele, Lea & Flood 2014)
    got = [int(x) for x in sv.splitmix64(0, np.arange(3))]
    assert got == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_counter_fields_are_distinct():
    c = sv.counters(sv.KIND_V, 5, 3, 77, 2, 9)
    assert int(c) == (1 << 62) | (5 << 40) | (3 << 34) | (77 << 14) | (2 << 8) | 9


def test_values_deterministic_and_standardised():
    r1 = sv.rows(sv.KIND_K, 11, 0, np.arange(2000), np.arange(2000), 4, 64, 1.0, "f32")
    r2 = sv.rows(sv.KIND_K, 11, 0, np.arange(2000), np.arange(2000), 4, 64, 1.0, "f32")
    assert np.array_equal(r1, r2)
    assert abs(r1.mean()) < 0.01 and abs(r1.std() - 1.0) < 0.01
    assert np.abs(r1).max() <= 131070 * float(sv.unit_scale_f32(1.0)) + 1e-6
    r3 = sv.rows(sv.KIND_V, 11, 0, np.arange(2000), np.arange(2000), 4, 64, 1.0, "f32")
    assert not np.array_equal(r1, r3)


def test_bf16_rounding_matches_torch():
    x = np.random.default_rng(0).standard_normal(100000).astype(np.float32) * 100
    ours = sv.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)


def test_workload_sizes():
    t = wl.tiny()
    assert t["shape"].num_blocks == 64 and sorted(t["order"]) == list(range(64))
    c = wl.continuous_batch()
    assert c["shape"].num_blocks == 66560 and len(c["schedule"].events) == 64
    assert c["schedule"].initial.min() >= 128 and c["schedule"].initial.max() <= 4096
    lp = wl.large_pool()
    assert lp["lens"].max() <= 16384 and lp["lens"].min() >= 1
    tokens = int(lp["lens"].sum())
    # about 100 GB of fp16 cache at 128 KiB per token
    assert 80e9 < tokens * 131072 < 130e9
    assert abs(math.log(np.median(lp["lens"])) - math.log(1500)) < 0.15


def test_continuous_schedule_stop_rate_and_replacements():
    """Stops are independent Bernoulli(1/200) per sequence and step; replacements draw
    U[128, 4096]: over 64 steps x 256 slots the stop count sits within 4 sigma of 81.92."""
    s = wl.continuous_schedule(256, 64, seed=3)
    stops = [e for ev in s.events for e in ev]
    mean, sd = 256 * 64 / 200, math.sqrt(256 * 64 * (1 / 200) * (199 / 200))
    assert abs(len(stops) - mean) < 4 * sd
    assert all(0 <= slot < 256 and 128 <= plen <= 4096 for slot, plen in stops)
    for ev in s.events:                   # ascending slot order, each slot at most once per step
        slots = [slot for slot, _ in ev]
        assert slots == sorted(set(slots))
    big = wl.continuous_schedule(256, 2000, seed=11)
    rate = sum(len(ev) for ev in big.events) / (256 * 2000)
    assert abs(rate - 1 / 200) < 4 * math.sqrt((1 / 200) * (199 / 200) / (256 * 2000))


def test_benchmark_plan_follows_the_schedule():
    """The benchmark's step plan: batch size fixed, continuing sequences grow by one token
    a step, a retired slot is taken at the next step by a new uid at its prompt length."""
    import bench
    r = wl.continuous_batch(seed=3, steps=40, p_stop=0.05)
    sched = r["schedule"]
    plan = bench.simulate(sched, 256, 40)
    assert np.array_equal(plan[0]["pos"], sched.initial) and np.array_equal(plan[0]["uids"], np.arange(256))
    next_uid = 256
    for t in range(1, 40):
        prev, cur = plan[t - 1], plan[t]
        retired = {slot: plen for slot, plen in sched.events[t - 1]}
        assert [a[0] for a in cur["admitted"]] == sorted(retired)
        for slot, uid, plen in cur["admitted"]:
            assert uid == next_uid and plen == retired[slot] and cur["pos"][slot] == plen
            next_uid += 1
        keep = np.array([i not in retired for i in range(256)])
        assert np.array_equal(cur["pos"][keep], prev["pos"][keep] + 1)
        assert np.array_equal(cur["uids"][keep], prev["uids"][keep])
        assert cur["retire"] == list(sched.events[t])
