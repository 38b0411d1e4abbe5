"""The allocation-free decode entry point (pytest -m gpu; collected last on purpose).

pa_decode_attention_static serves callers that cannot allocate device memory: a
serving process that has already given nearly all of the GPU to its KV pool, a
host whose allocator must not run on the decode path (cudaMalloc can synchronise
the device), or a plain C embedding without an allocator.  It keeps its split-K
partials in a fixed array inside the library instead of a caller workspace.

Checked here through the C ABI, on batches that split (so the built-in array is
really used):
  * two calls in a row each give exactly the bits of the workspace-taking
    pa_decode_attention -- the same kernels with the same merge order -- so the
    second call also shows that stale contents left by the first do not leak;
  * the result matches the fp64 oracle within the parity tolerance of the other GPU
    tests (2e-3 max-abs for a 16-bit or FP8 cache, fp32 output), for a fp16 cache and
    for an FP8 cache;
  * a batch whose partials would not fit is refused before anything is launched.
Works run alone in a fresh process or after the rest of the suite.
"""
import numpy as np
import pytest
import torch

import paged_kv_cache_403_b200 as pa
from paged_kv_cache_403_b200.runners import run_static
from synthetic import workloads as wl

from oracle_replay import OracleRun, check_close, sequence_attention_fp8

pytestmark = pytest.mark.gpu


def oracle_outputs(r, kv_fp8):
    """fp64 oracle of the worked example's decode step, from regenerated host inputs."""
    sh = r["shape"]
    lens = [int(L) for L in r["lens"]]
    if kv_fp8:
        return np.stack([sequence_attention_fp8(sh, r["seed"], 0, i, L + 1, i, L) for i, L in enumerate(lens)])
    o = OracleRun(sh, r["order"], r["seed"])
    sids = [o.bm.seq_add() for _ in lens]
    o.prefill(sids, list(range(len(lens))), lens)
    mb = max(-(-(L + 1) // sh.block_size) for L in lens)
    return o.decode_step(sids, list(range(len(lens))), mb)["outputs"][0]


@pytest.mark.parametrize("kv_fp8", [False, True], ids=["fp16_cache", "fp8_cache"])
def test_static_scratch_matches_workspace_entry_and_oracle_two_calls(kv_fp8):
    torch.cuda.set_device(0)
    pa.pa_device_error(clear=True)
    r = wl.worked_example()                      # 3900/420/2100/70 tokens, fp16, 32 q / 8 KV heads
    cache, gen, rec = run_static(r, split_tokens=0, out_dtype=torch.float32, kv_fp8=kv_fp8)
    tables = torch.from_numpy(rec.tables).cuda()
    lens = torch.from_numpy(rec.lens).cuda()
    n, hq, d = len(rec.lens), r["shape"].num_q_heads, r["shape"].head_dim
    q = gen.q(0, rec.uids, rec.positions)
    split = 256                                  # 3901 tokens -> 16 splits: the scratch is used
    ms = pa.pa_decode_max_splits(16, tables.shape[1], split)
    need = pa.pa_decode_workspace_bytes(n, hq, d, ms)
    assert ms > 1 and 0 < need <= pa.PA_STATIC_WORKSPACE_BYTES

    ws = torch.empty(need // 4, dtype=torch.float32, device="cuda")
    ref = torch.empty((n, hq, d), dtype=torch.float32, device="cuda")
    pa.pa_decode_attention(cache.pool, 0, q, ref, tables, lens, d ** -0.5, split, ws)
    outs = []
    for _ in range(2):
        out = torch.full((n, hq, d), float("nan"), dtype=torch.float32, device="cuda")
        pa.pa_decode_attention_static(cache.pool, 0, q, out, tables, lens, d ** -0.5, split)
        outs.append(out)
    torch.cuda.synchronize()
    assert pa.pa_device_error(clear=True) == 0
    for out in outs:
        assert torch.equal(out, ref)             # same kernels, same merge order: the same bits
    expect = oracle_outputs(r, kv_fp8)
    err = check_close(outs[1].cpu().numpy(), expect, "f32", "f16", "static entry vs oracle")
    print(f"{'fp8' if kv_fp8 else 'fp16'} cache: static entry bit-identical, max err vs oracle {err:.3g}")


def test_static_scratch_refuses_batches_that_do_not_fit():
    torch.cuda.set_device(0)
    pool = pa.pa_pool_create(1, 4, 16, 8, 128, "f16",
                             torch.zeros(1, 4, 8, 16, 128, dtype=torch.float16, device="cuda"),
                             torch.zeros(1, 4, 8, 16, 128, dtype=torch.float16, device="cuda"))
    n, hq, d, max_blocks = 4096, 32, 128, 1024  # 4096 sequences x 64 splits of 16 tokens
    need = pa.pa_decode_workspace_bytes(n, hq, d, pa.pa_decode_max_splits(16, max_blocks, 16))
    assert need > pa.PA_STATIC_WORKSPACE_BYTES
    q = torch.zeros((n, hq, d), dtype=torch.float16, device="cuda")
    out = torch.zeros((n, hq, d), dtype=torch.float32, device="cuda")
    tables = torch.zeros((n, max_blocks), dtype=torch.int32, device="cuda")
    lens = torch.ones(n, dtype=torch.int32, device="cuda")
    before = pa.pa_launch_count()
    with pytest.raises(pa.PaError) as e:
        pa.pa_decode_attention_static(pool, 0, q, out, tables, lens, 0.1, 16)
    assert e.value.status == pa.PA_ERR_INVALID_ARG and "bytes of split scratch" in str(e.value)
    assert pa.pa_launch_count() == before
    pa.pa_pool_destroy(pool)
