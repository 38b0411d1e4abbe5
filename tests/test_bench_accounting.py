"""bench.py's byte accounting on CPU: the bytes decode attention reads per step (the
metric's numerator) and the algorithmic bytes behind the roofline, counted from each
step's sequence lengths after the timed pass.  Expected values are worked by hand."""
from types import SimpleNamespace

import numpy as np

import bench
from synthetic.workloads import Shape


def _rep(kv_fp8, lens_per_step):
    # a stand-in carrying only what the accounting reads: 2 layers, 4 q / 2 KV heads, d8,
    # block 16, a 16-bit activation type
    sh = Shape(num_layers=2, block_size=16, num_q_heads=4, num_kv_heads=2, head_dim=8, dtype="bf16",
               num_blocks=64, kv_scale=1.0)
    r = SimpleNamespace(shape=sh, n=2, NL=2, kv_fp8=kv_fp8, _kv_bytes=[], _alg_bytes=[],
                        _pending_lens=[np.asarray(x, np.int32) for x in lens_per_step])
    bench.Replica._settle(r)
    return r


def test_16bit_cache_bytes():
    # lengths 17 and 32: K and V rows of 2 heads x 8 elements x 2 bytes = 16 bytes each
    #   KV: 2 layers x 2 (K, V) x (17 + 32) tokens x 2 heads x 16 B = 6272
    #   q and out: 2 layers x 2 x 2 seqs x 4 heads x 8 x 2 B = 512; tables: 2 layers x 4 B x
    #   (2 + 2) blocks = 32; lengths: 2 layers x 4 B x 2 = 16  ->  6272 + 560 = 6832
    r = _rep(False, [[17, 32]])
    assert r._kv_bytes == [6272] and r._alg_bytes == [6832]
    assert r._pending_lens == []


def test_fp8_cache_bytes():
    # an FP8 row is 8 code bytes and 1 scale byte: 2 x 2 x 49 x 2 x 9 = 3528; + 560 = 4088
    r = _rep(True, [[17, 32]])
    assert r._kv_bytes == [3528] and r._alg_bytes == [4088]


def test_steps_counted_in_order_and_once():
    r = _rep(False, [[1, 16], [17, 32]])
    # step 1: 2 x 2 x 17 x 2 x 16 = 2176; tables 2 x 4 x (1 + 1) = 16
    assert r._kv_bytes == [2176, 6272]
    assert r._alg_bytes == [2176 + 512 + 16 + 16, 6832]
    bench.Replica._settle(r)                 # nothing pending: nothing added
    assert len(r._kv_bytes) == 2
