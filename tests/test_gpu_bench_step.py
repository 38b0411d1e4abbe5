"""bench.py's timed step checked against the oracle.

The benchmark drives the library through its own step: packed metadata uploads on a
side copy stream, four rotating device buffer sets, host bookkeeping running ahead of
the GPU, and an end-to-end leg whose inputs come from pinned host memory in one packed
copy per layer and whose output is read back on a third stream.  These tests run that
step on the continuous-batch workload (bf16 and FP8 caches, at the splits it times) and
compare sampled outputs of both legs with the fp64 oracle over regenerated histories.
"""
import numpy as np
import pytest
import torch

import bench
import paged_kv_cache_403_b200 as pa

from oracle_replay import check_close, sequence_attention, sequence_attention_fp8

pytestmark = pytest.mark.gpu


def _picks(lens, rng):
    return sorted(set(rng.choice(len(lens), size=4, replace=False).tolist())
                  | {int(np.argmax(lens)), int(np.argmin(lens))})


@pytest.mark.slow
@pytest.mark.parametrize("kv_fp8", [False, True])
def test_bench_step_matches_oracle(kv_fp8):
    W, K = 3, 5
    total = W + 2 * K
    torch.cuda.set_device(0)
    pa.pa_device_error(clear=True)
    recipe = bench.make_recipe("continuous_batch", bench.replica_seed(0), total)
    sh = recipe["shape"]
    split = bench.default_split("continuous_batch")
    rep = bench.Replica(torch, "continuous_batch", recipe, total, split, torch.device("cuda", 0), W + K,
                        kv_fp8=kv_fp8)
    for t in range(W + K):
        rep.step(t)
    torch.cuda.synchronize()
    t_dev = W + K - 1
    dev_out = rep.out[t_dev % bench.NSETS][0].float().cpu().numpy()
    for t in range(W + K, total):
        rep.step(t, e2e=True, time_attention=False)
    rep.drain()
    torch.cuda.synchronize()
    t_e2e = total - 1
    e2e_out = rep.h_out[t_e2e % bench.NSETS][0].float().numpy()
    assert pa.pa_device_error(clear=True) == 0
    ref_fn = sequence_attention_fp8 if kv_fp8 else sequence_attention
    rng = np.random.default_rng(7)
    for t, out in ((t_dev, dev_out), (t_e2e, e2e_out)):
        plan = rep.plan[t]
        lens = np.asarray(plan["pos"]) + 1
        for i in _picks(lens, rng):
            uid, pos = int(plan["uids"][i]), int(plan["pos"][i])
            ref = ref_fn(sh, recipe["seed"], 0, uid, pos + 1, uid, pos)
            check_close(out[i], ref, "bf16", "bf16", f"{'fp8' if kv_fp8 else 'bf16'} step {t} seq {i}")
    # the e2e leg moved what it says it moved: the packed inputs of one layer per step
    assert rep.h2d and all(b > 0 for b in rep.h2d)
