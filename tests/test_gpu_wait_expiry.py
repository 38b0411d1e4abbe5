"""Failure detection on the GPU without a GPU fault (pytest -m gpu).

Every device-side wait of the decode kernels is bounded (a running copy that never
lands must not stall the launch -- the failure has to come back to the host as a
status it can act on, as "Continuous Batching & Paged Attention -- LLM Inference
Optimization & Serving", section "Decisions leaders and practitioners actually
face", asks of a server: reject cleanly rather than stall).  Here a test hook
lowers the bound to 1 ms and makes one decode CTA's producer issue no copies at all,
so nothing is ever in flight for it and its consumers' waits run out.  The kernel
must record device error bit 4 and return; every other CTA's output must be exactly
the normal one; once the hook is switched off the same call gives the normal bits
again, and they match the fp64 oracle.
"""
import numpy as np
import pytest
import torch

import paged_kv_cache_403_b200 as pa
from paged_kv_cache_403_b200.runners import run_static
from synthetic import workloads as wl

from oracle_replay import check_close, sequence_attention, sequence_attention_fp8

pytestmark = pytest.mark.gpu
ERR_TIMEOUT = 4


@pytest.fixture(autouse=True)
def hook_off():
    pa.pa_debug_wait_test(0, -1)
    pa.pa_device_error(clear=True)
    yield
    pa.pa_debug_wait_test(0, -1)
    assert pa.pa_device_error(clear=True) == 0


@pytest.mark.parametrize("kv_fp8", [False, True], ids=["fp16_cache", "fp8_cache"])
@pytest.mark.parametrize("split", [0, 1024])
def test_withheld_copies_time_out_and_report(kv_fp8, split):
    r = wl.worked_example()                  # 4 sequences, 32 q / 8 KV heads, fp16 activations
    sh = r["shape"]
    cache, gen, rec = run_static(r, split_tokens=0, out_dtype=torch.float32, kv_fp8=kv_fp8)
    n, hq, d = len(rec.lens), sh.num_q_heads, sh.head_dim
    tables = torch.from_numpy(rec.tables).cuda()
    lens = torch.from_numpy(rec.lens).cuda()
    q = gen.q(0, rec.uids, rec.positions)
    ws = cache.workspace(n, hq, tables.shape[1], split)

    def decode():
        out = torch.full((n, hq, d), 7.0, dtype=torch.float32, device="cuda")
        cache.decode(0, q, out, tables, lens, d ** -0.5, split, ws)
        torch.cuda.synchronize()
        return out

    normal = decode()
    assert pa.pa_device_error(clear=True) == 0

    pa.pa_debug_wait_test(1_000_000, 0)      # 1 ms bound; CTA 0 gets no copies
    try:
        failed = decode()
        code = pa.pa_device_error(clear=True)
    finally:
        pa.pa_debug_wait_test(0, -1)
    assert code & ERR_TIMEOUT, f"device error word {code:#x}: the withheld CTA's waits did not report"
    # CTA 0 serves one (range, KV-head group) of one sequence; without a split and with
    # fewer than two CTAs per SM there is no longest-first order, so it is sequence 0's
    # first KV-head group.  Everything outside the sequence it serves is untouched.
    differs = ~torch.eq(failed, normal).all(dim=2).cpu().numpy()      # [n][hq]
    assert differs.any(), "the withheld CTA's outputs look normal"
    bad_seqs = np.nonzero(differs.any(axis=1))[0]
    assert len(bad_seqs) == 1, f"outputs of sequences {bad_seqs} changed"
    heads_per_group = hq // sh.num_kv_heads * (2 if kv_fp8 else 1)
    assert differs.sum() <= heads_per_group

    again = decode()
    assert pa.pa_device_error(clear=True) == 0
    assert torch.equal(again, normal)
    out = again.cpu().numpy()
    for i in range(n):
        L = int(rec.lens[i])
        if kv_fp8:
            ref = sequence_attention_fp8(sh, r["seed"], 0, rec.uids[i], L, rec.uids[i], int(rec.positions[i]))
        else:
            ref = sequence_attention(sh, r["seed"], 0, rec.uids[i], L, rec.uids[i], int(rec.positions[i]))
        check_close(out[i], ref, "f32", "f16", f"sequence {i} after the hook is off")


def test_hook_rejects_bad_arguments():
    with pytest.raises(pa.PaError) as e:
        pa.pa_debug_wait_test(0, -2)
    assert e.value.status == pa.PA_ERR_INVALID_ARG


def test_prefill_withheld_copies_time_out_and_report():
    """The same on the tcgen05 chunked-prefill kernel, whose TMA, tensor-core and softmax
    roles hand tiles to each other through mbarriers: with CTA 0's copies withheld its
    tensor-core warp's wait for the first key tile runs out, the shared abort flag
    releases the softmax warps, the CTA frees its tensor memory and ends; its output rows
    are left untouched and every other CTA's rows are exactly the normal ones."""
    from test_gpu_prefill import prefill_case, run
    c = prefill_case([600, 300], [200, 129], seed=21)   # group 4: 64 tokens x 4 heads per CTA
    normal = run(c)
    assert pa.pa_device_error(clear=True) == 0
    pa.pa_debug_wait_test(1_000_000, 0)
    try:
        failed = run(c)                                  # outputs start as NaN
        code = pa.pa_device_error(clear=True)
    finally:
        pa.pa_debug_wait_test(0, -1)
    assert code & ERR_TIMEOUT, f"device error word {code:#x}: the withheld CTA's waits did not report"
    # CTA 0 = sequence 0, KV head 0 (query heads 0-3), the chunk's first 64 tokens (rows 0-63)
    mine = np.zeros(failed.shape[:2], bool)
    mine[0:64, 0:4] = True
    assert np.isnan(failed[mine]).all()
    assert np.array_equal(failed[~mine], normal[~mine])
    again = run(c)
    assert pa.pa_device_error(clear=True) == 0
    assert np.array_equal(again, normal)
    check_close(again, c["ref"], "f32", "bf16", "prefill after the hook is off")
