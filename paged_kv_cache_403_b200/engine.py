"""Device pools plus the native block manager, and the per-step call sequence.

``PagedCache`` owns the key/value pools (torch device memory, zero-filled) and a
libpa pool handle.  ``decode_step`` is one iteration of the serving loop of "What
problem does PagedAttention solve, and what is continuous batching?", section
"How the two fit together in production" (every active sequence generates one
token): reserve one slot per sequence (new block or copy-on-write), copy blocks,
upload tables and slots, then per layer append the new key/value rows and run
decode attention.  All arithmetic and bookkeeping happen in libpa; this module
only sequences the calls and moves metadata to the device.
"""
from __future__ import annotations

import math

import numpy as np
import torch

from . import (pa_append_kv, pa_build_block_tables, pa_copy_blocks, pa_decode_attention,
               pa_decode_max_splits, pa_decode_workspace_bytes, pa_pool_create, pa_pool_destroy,
               pa_pool_set_scales, pa_pool_stats, pa_reserve_slots, pa_seq_add, pa_seq_fork, pa_seq_free,
               pa_seq_info)

TORCH_DTYPES = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16, "fp8": torch.uint8}


class PagedCache:
    def __init__(self, num_layers, num_blocks, block_size, num_kv_heads, head_dim, dtype,
                 free_order=None, device="cuda", act_dtype=None):
        """``dtype`` "fp8" stores E4M3 codes plus per-row scale bytes; ``act_dtype`` ("f16" or
        "bf16") is then the type of queries, appended rows and 16-bit outputs."""
        self.num_layers, self.num_blocks, self.block_size = num_layers, num_blocks, block_size
        self.num_kv_heads, self.head_dim, self.dtype = num_kv_heads, head_dim, dtype
        self.act_dtype = act_dtype if dtype == "fp8" else dtype
        self.device = device
        self.scales = None
        if device is not None:
            shape = (num_layers, num_blocks, num_kv_heads, block_size, head_dim)
            self.k_pool = torch.zeros(shape, dtype=TORCH_DTYPES[dtype], device=device)
            self.v_pool = torch.zeros(shape, dtype=TORCH_DTYPES[dtype], device=device)
            if dtype == "fp8":
                self.scales = torch.zeros((num_layers, num_blocks, num_kv_heads, 2, block_size), dtype=torch.uint8,
                                          device=device)
        else:
            self.k_pool = self.v_pool = None
        self.pool = pa_pool_create(num_layers, num_blocks, block_size, num_kv_heads, head_dim, dtype,
                                   self.k_pool, self.v_pool, free_order, self.act_dtype)
        if self.scales is not None:
            pa_pool_set_scales(self.pool, self.scales)

    @classmethod
    def from_shape(cls, shape, free_order=None, device="cuda"):
        return cls(shape.num_layers, shape.num_blocks, shape.block_size, shape.num_kv_heads,
                   shape.head_dim, shape.dtype, free_order, device, getattr(shape, "act_dtype", None))

    def close(self):
        if self.pool is not None:
            pa_pool_destroy(self.pool)
            self.pool = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # host bookkeeping
    def add(self) -> int:
        return pa_seq_add(self.pool)

    def fork(self, parent: int) -> int:
        return pa_seq_fork(self.pool, parent)

    def free(self, sid: int) -> None:
        pa_seq_free(self.pool, sid)

    def info(self, sid: int):
        return pa_seq_info(self.pool, sid)

    def stats(self) -> dict:
        return pa_pool_stats(self.pool)

    def reserve(self, sids, ntok):
        return pa_reserve_slots(self.pool, sids, ntok)

    def tables(self, sids, max_blocks):
        return pa_build_block_tables(self.pool, sids, max_blocks)

    # device work
    def copy_blocks(self, pairs: np.ndarray, stream=None):
        if len(pairs):
            dev = torch.from_numpy(np.ascontiguousarray(pairs, np.int32)).to(self.device, non_blocking=False)
            pa_copy_blocks(self.pool, dev, stream=stream)

    def append(self, layer, k_new, v_new, slots_dev, stream=None):
        pa_append_kv(self.pool, layer, k_new, v_new, slots_dev, stream=stream)

    def decode(self, layer, q, out, tables_dev, lens_dev, scale=None, split_tokens=0, workspace=None,
               stream=None):
        scale = 1.0 / math.sqrt(self.head_dim) if scale is None else scale
        pa_decode_attention(self.pool, layer, q, out, tables_dev, lens_dev, scale, split_tokens,
                            workspace, stream=stream)

    def workspace(self, n_seqs, num_q_heads, max_blocks, split_tokens):
        ms = pa_decode_max_splits(self.block_size, max_blocks, split_tokens)
        nbytes = pa_decode_workspace_bytes(n_seqs, num_q_heads, self.head_dim, ms)
        if nbytes == 0:
            return None
        return torch.empty(nbytes // 4, dtype=torch.float32, device=self.device)


def max_blocks_for(lens, block_size, extra_tokens=0) -> int:
    return max(1, max(-(-(int(L) + extra_tokens) // block_size) for L in lens))
