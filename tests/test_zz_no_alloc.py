"""The allocation-free decode entry point (pytest -m gpu; collected last on purpose).

pa_decode_attention_static serves callers that cannot allocate device memory: a
serving process that has already given nearly all of the GPU to its KV pool, a
host whose allocator must not run on the decode path (cudaMalloc can synchronise
the device), or a plain C embedding without an allocator.  It keeps its split-K
partials in a fixed array inside the library instead of a caller workspace.

Checked here through the C ABI: on a batch that splits (so the built-in array is
really used), two calls in a row each match the workspace-taking
pa_decode_attention within the parity tolerance of the other GPU tests (2e-3
max-abs for a fp16 cache, fp32 output) -- the second call also shows that stale
contents left by the first do not leak into the result; a batch whose partials
would not fit is refused before anything is launched.  Works run alone in a fresh
process or after the rest of the suite.
"""
import numpy as np
import pytest
import torch

import paged_kv_cache_403_b200 as pa
from paged_kv_cache_403_b200.runners import run_static
from synthetic import workloads as wl

pytestmark = pytest.mark.gpu


def test_static_scratch_matches_workspace_entry_two_calls():
    torch.cuda.set_device(0)
    r = wl.worked_example()                      # 3900/420/2100/70 tokens, fp16, 32 q / 8 KV heads
    cache, gen, rec = run_static(r, split_tokens=0, out_dtype=torch.float32)
    tables = torch.from_numpy(rec.tables).cuda()
    lens = torch.from_numpy(rec.lens).cuda()
    n, hq, d = len(rec.lens), r["shape"].num_q_heads, r["shape"].head_dim
    positions = rec.positions
    q = gen.q(0, rec.uids, positions)
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
        err = (out - ref).abs().max().item()
        assert np.isfinite(err) and err <= 2e-3, err
    # the unsplit result (no scratch at all) agrees too
    plain = torch.empty_like(ref)
    pa.pa_decode_attention(cache.pool, 0, q, plain, tables, lens, d ** -0.5, 0)
    assert (outs[1] - plain).abs().max().item() <= 2e-3


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
