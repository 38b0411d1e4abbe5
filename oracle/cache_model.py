"""Oracle model of the cache contents -- TEST INFRASTRUCTURE ONLY.

Host numpy pools laid out [num_layers][num_blocks][num_kv_heads][block_size][head_dim]
(storage dtype: float32 / float16 / uint16 bit patterns for bf16), written the
way the pages describe:

* "What problem does PagedAttention solve, and what is continuous batching?",
  section "Why the KV cache becomes the problem": each decode step reads the
  cache and appends a small amount of new data -- the new token's key and value
  rows go into the slot the block manager handed out (slot = block * B + offset).
* same page, section "How PagedAttention works": copy-on-write gives a diverging
  sequence a private copy of the shared block; the copy here is the whole block,
  every layer, keys and values (a reading: the pages do not say how much is
  copied, and copying the whole block keeps every earlier slot valid).

Writes are bit copies, so the GPU pools must match these arrays exactly.

FP8 pools (``dtype == "fp8"``) hold E4M3 codes and, beside them, one scale byte per
(token, KV head) row of K and of V, in one array [num_layers][num_blocks][num_kv_heads]
[2][block_size] (index 0 = K, 1 = V; a layout reading: a block's scales for one head
sit together, next to those of the neighbouring heads); an appended row is quantised
by ``oracle.fp8.quantize_rows`` (the format and the scale rule are stated there), and
block copies and swaps carry the scales with the codes.
"""
from __future__ import annotations

import numpy as np

from synthetic.values import ELEM_BYTES

from .fp8 import quantize_rows

_NP = {"f32": np.float32, "f16": np.float16, "bf16": np.uint16}


def empty_pools(num_layers, num_blocks, num_kv_heads, block_size, head_dim, dtype):
    shape = (num_layers, num_blocks, num_kv_heads, block_size, head_dim)
    if dtype == "fp8":
        return np.zeros(shape, np.uint8), np.zeros(shape, np.uint8)
    assert ELEM_BYTES[dtype] == np.dtype(_NP[dtype]).itemsize
    return np.zeros(shape, _NP[dtype]), np.zeros(shape, _NP[dtype])


def empty_scales(num_layers, num_blocks, num_kv_heads, block_size):
    """Scale bytes of an FP8 pool, [layers][blocks][kv heads][K, V][block_size]."""
    return np.zeros((num_layers, num_blocks, num_kv_heads, 2, block_size), np.uint8)


def append_rows_fp8(k_pool, v_pool, scales, layer, slots, k_rows, v_rows, act_dtype):
    """Quantise row i of k_rows / v_rows ([n][Hkv][d], storage of ``act_dtype``) and
    write its codes and scale bytes into slot slots[i] of ``layer``."""
    from . import widen                      # the oracle's own exact decoders
    kc, ks = quantize_rows(widen(k_rows, act_dtype).astype(np.float32))
    vc, vs = quantize_rows(widen(v_rows, act_dtype).astype(np.float32))
    block_size = k_pool.shape[3]
    for i, slot in enumerate(slots):
        slot = int(slot)
        if slot < 0:
            continue
        blk, off = divmod(slot, block_size)
        k_pool[layer, blk, :, off, :] = kc[i]
        v_pool[layer, blk, :, off, :] = vc[i]
        scales[layer, blk, :, 0, off] = ks[i]
        scales[layer, blk, :, 1, off] = vs[i]


def append_rows(k_pool, v_pool, layer, slots, k_rows, v_rows):
    """Write row i of k_rows / v_rows ([n][Hkv][d]) into slot slots[i] of ``layer``."""
    block_size = k_pool.shape[3]
    for i, slot in enumerate(slots):
        slot = int(slot)
        if slot < 0:
            continue                       # padding row: nothing is written
        blk, off = divmod(slot, block_size)
        k_pool[layer, blk, :, off, :] = k_rows[i]
        v_pool[layer, blk, :, off, :] = v_rows[i]


def copy_blocks(k_pool, v_pool, pairs):
    """Copy-on-write: physical block dst becomes a copy of src in every layer, K and V."""
    for src, dst in pairs:
        k_pool[:, int(dst)] = k_pool[:, int(src)]
        v_pool[:, int(dst)] = v_pool[:, int(src)]


def copy_scales(scales, pairs):
    """The scale bytes travel with a copied FP8 block, every layer."""
    for src, dst in pairs:
        scales[:, int(dst)] = scales[:, int(src)]


def swap_buffer_fp8(k_pool, v_pool, scales, blocks):
    """Host copy of a swapped-out sequence of an FP8 pool, as bytes: for block i in
    logical order and each layer, the K codes [heads][block_size][dim], the V codes,
    then the block's scale bytes [heads][K, V][block_size] (reading: the scales ride in
    the same block-major record as their codes)."""
    out = []
    for b in blocks:
        for layer in range(k_pool.shape[0]):
            out += [k_pool[layer, int(b)].ravel(), v_pool[layer, int(b)].ravel(), scales[layer, int(b)].ravel()]
    return np.concatenate(out) if out else np.zeros(0, np.uint8)


def swap_restore_fp8(k_pool, v_pool, scales, blocks, buf):
    nl, _, h, bs, d = k_pool.shape
    pos = 0
    for b in blocks:
        for layer in range(nl):
            for arr, n, shape in ((k_pool, h * bs * d, (h, bs, d)), (v_pool, h * bs * d, (h, bs, d)),
                                  (scales, 2 * h * bs, (h, 2, bs))):
                arr[layer, int(b)] = buf[pos:pos + n].reshape(shape)
                pos += n


def swap_buffer(k_pool, v_pool, blocks):
    """Host copy of a swapped-out sequence: [block i][layer][K, V][heads][block_size][dim]
    (reading: block-major so one block's data is contiguous and can be restored into
    any free block)."""
    parts = [np.stack([k_pool[:, int(b)], v_pool[:, int(b)]], axis=1) for b in blocks]
    return np.ascontiguousarray(np.stack(parts)) if parts else np.zeros((0,) + k_pool.shape[:1] + (2,)
                                                                          + k_pool.shape[2:], k_pool.dtype)


def swap_restore(k_pool, v_pool, blocks, buf):
    """Write a swap buffer back into the given (new) blocks, logical order."""
    for i, b in enumerate(blocks):
        k_pool[:, int(b)] = buf[i, :, 0]
        v_pool[:, int(b)] = buf[i, :, 1]
