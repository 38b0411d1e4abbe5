"""Python binding of libpa.so, the paged KV-cache decode library for B200 (sm_100a).

Each function has the name of the C entry point it calls (include/pa.h) and does
argument marshalling only: torch tensors become device pointers, numpy arrays
become host pointers, a non-OK status becomes PaError.  Every step of the path --
the host block manager and all device work -- runs in the native library.
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import _native
from ._native import PoolConfig, PoolStats

(PA_OK, PA_ERR_INVALID_ARG, PA_ERR_OUT_OF_BLOCKS, PA_ERR_DOUBLE_FREE, PA_ERR_CUDA, PA_ERR_UNSUPPORTED,
 PA_ERR_HOST_MEMORY) = range(7)
PA_F32, PA_F16, PA_BF16, PA_FP8_E4M3 = 0, 1, 2, 3
DTYPE_CODES = {"f32": PA_F32, "f16": PA_F16, "bf16": PA_BF16, "fp8": PA_FP8_E4M3}


class PaError(RuntimeError):
    def __init__(self, status: int, message: str):
        self.status = status
        names = {1: "PA_ERR_INVALID_ARG", 2: "PA_ERR_OUT_OF_BLOCKS", 3: "PA_ERR_DOUBLE_FREE",
                 4: "PA_ERR_CUDA", 5: "PA_ERR_UNSUPPORTED", 6: "PA_ERR_HOST_MEMORY"}
        super().__init__(f"{names.get(status, status)}: {message}")


def _lib():
    return _native.lib()


def _check(status: int) -> None:
    if status != PA_OK:
        raise PaError(status, _lib().pa_last_error().decode())


def _dtype_code(dtype) -> int:
    if isinstance(dtype, int):
        return dtype
    if isinstance(dtype, str):
        return DTYPE_CODES[dtype]
    import torch
    return {torch.float32: PA_F32, torch.float16: PA_F16, torch.bfloat16: PA_BF16}[dtype]


def _host_ptr(a):
    """Pointer to a contiguous host buffer (numpy array or CPU torch tensor)."""
    if a is None:
        return None
    if isinstance(a, np.ndarray):
        assert a.flags.c_contiguous
        return a.ctypes.data
    assert not a.is_cuda and a.is_contiguous()
    return a.data_ptr()


def _dev_ptr(t):
    if t is None:
        return None
    assert t.is_cuda and t.is_contiguous(), "expected a contiguous CUDA tensor"
    return t.data_ptr()


def _stream(stream):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


# ------------------------------------------------------------------ pool
def pa_pool_create(num_layers, num_blocks, block_size, num_kv_heads, head_dim, dtype,
                   k_pool=None, v_pool=None, free_order=None, act_dtype=None):
    """Host block manager over caller-owned device pools (None for host-only use).
    ``act_dtype`` is the query / appended-row type of an "fp8" pool."""
    act = _dtype_code(act_dtype) if act_dtype is not None else _dtype_code(dtype)
    cfg = PoolConfig(num_layers, num_blocks, block_size, num_kv_heads, head_dim, _dtype_code(dtype), act)
    order = None
    if free_order is not None:
        order = np.ascontiguousarray(free_order, dtype=np.int32)
    out = ctypes.c_void_p()
    _check(_lib().pa_pool_create(ctypes.byref(cfg), _dev_ptr(k_pool), _dev_ptr(v_pool),
                                 _host_ptr(order), ctypes.byref(out)))
    return out


def pa_pool_set_scales(pool, scales) -> None:
    """Attach the uint8 scale array [layers][blocks][kv heads][K, V][block_size] of an FP8 pool."""
    _check(_lib().pa_pool_set_scales(pool, _dev_ptr(scales)))


def pa_pool_destroy(pool) -> None:
    _check(_lib().pa_pool_destroy(pool))


def pa_pool_stats(pool) -> dict:
    s = PoolStats()
    _check(_lib().pa_pool_stats(pool, ctypes.byref(s)))
    return {f: getattr(s, f) for f, _ in PoolStats._fields_}


# ------------------------------------------------------------------ blocks
def pa_alloc_block(pool) -> int:
    b = ctypes.c_int32()
    _check(_lib().pa_alloc_block(pool, ctypes.byref(b)))
    return b.value


def pa_free_block(pool, block: int) -> None:
    _check(_lib().pa_free_block(pool, block))


def pa_incref_block(pool, block: int) -> None:
    _check(_lib().pa_incref_block(pool, block))


def pa_block_refcount(pool, block: int) -> int:
    r = ctypes.c_int32()
    _check(_lib().pa_block_refcount(pool, block, ctypes.byref(r)))
    return r.value


def pa_num_free_blocks(pool) -> int:
    n = ctypes.c_int32()
    _check(_lib().pa_num_free_blocks(pool, ctypes.byref(n)))
    return n.value


def pa_free_list(pool) -> np.ndarray:
    """Free stack bottom first: the last entry is handed out next."""
    got = ctypes.c_int32()
    _check(_lib().pa_free_list(pool, None, 0, ctypes.byref(got)))
    out = np.empty(got.value, np.int32)
    _check(_lib().pa_free_list(pool, out.ctypes.data, got.value, ctypes.byref(got)))
    return out


def pa_debug_fail_alloc_after(pool, n: int) -> None:
    _check(_lib().pa_debug_fail_alloc_after(pool, n))


# ------------------------------------------------------------------ sequences
def pa_seq_add(pool) -> int:
    s = ctypes.c_int32()
    _check(_lib().pa_seq_add(pool, ctypes.byref(s)))
    return s.value


def pa_seq_fork(pool, parent: int) -> int:
    c = ctypes.c_int32()
    _check(_lib().pa_seq_fork(pool, parent, ctypes.byref(c)))
    return c.value


def pa_seq_free(pool, seq_id: int) -> None:
    _check(_lib().pa_seq_free(pool, seq_id))


def pa_seq_info(pool, seq_id: int):
    """(length, block table as int32 array)."""
    ln, nb = ctypes.c_int32(), ctypes.c_int32()
    _check(_lib().pa_seq_info(pool, seq_id, ctypes.byref(ln), None, 0, ctypes.byref(nb)))
    table = np.empty(nb.value, np.int32)
    _check(_lib().pa_seq_info(pool, seq_id, ctypes.byref(ln), table.ctypes.data, nb.value, ctypes.byref(nb)))
    return ln.value, table


def pa_reserve_slots(pool, seq_ids, ntok, slot_out=None, cow_out=None):
    """Reserve slots for ntok[i] tokens of seq_ids[i].

    Returns (slot_mapping int64[sum(ntok)], cow_pairs int32[k][2]); when slot_out /
    cow_out (host buffers, e.g. pinned torch tensors) are given they are filled
    in place and views of them are returned.
    """
    ids = np.ascontiguousarray(seq_ids, dtype=np.int32)
    nt = np.ascontiguousarray(ntok, dtype=np.int32)
    n = ids.shape[0]
    total = int(nt.sum()) if n else 0
    slots = slot_out if slot_out is not None else np.empty(max(total, 1), np.int64)
    cow = cow_out if cow_out is not None else np.empty((max(n, 1), 2), np.int32)
    ncow = ctypes.c_int32(0)
    _check(_lib().pa_reserve_slots(pool, ids.ctypes.data, nt.ctypes.data, n, _host_ptr(slots),
                                   _host_ptr(cow), ctypes.byref(ncow)))
    return slots[:total], cow[:ncow.value]


def pa_build_block_tables(pool, seq_ids, max_blocks: int, tables_out=None, lens_out=None):
    """Dense tables [n][max_blocks] (pad -1) and lengths [n] into host buffers."""
    ids = np.ascontiguousarray(seq_ids, dtype=np.int32)
    n = ids.shape[0]
    tables = tables_out if tables_out is not None else np.empty((n, max_blocks), np.int32)
    lens = lens_out if lens_out is not None else np.empty(n, np.int32)
    _check(_lib().pa_build_block_tables(pool, ids.ctypes.data, n, max_blocks, _host_ptr(tables),
                                        _host_ptr(lens)))
    return tables, lens


# ------------------------------------------------------------------ prefix caching
def pa_prefix_register(pool, seq_id: int, keys) -> int:
    """Register the first len(keys) (full) blocks of seq_id under keys; returns how many were new."""
    k = np.ascontiguousarray(keys, dtype=np.uint64)
    n = ctypes.c_int32()
    _check(_lib().pa_prefix_register(pool, seq_id, k.ctypes.data, k.shape[0], ctypes.byref(n)))
    return n.value


def pa_seq_add_cached(pool, keys):
    """New sequence sharing the registered blocks of its leading keys: (seq_id, hits)."""
    k = np.ascontiguousarray(keys, dtype=np.uint64)
    sid, hit = ctypes.c_int32(), ctypes.c_int32()
    _check(_lib().pa_seq_add_cached(pool, k.ctypes.data, k.shape[0], ctypes.byref(sid), ctypes.byref(hit)))
    return sid.value, hit.value


def pa_prefix_evictable(pool) -> np.ndarray:
    """Evictable cached blocks, next to be evicted first."""
    n = ctypes.c_int32()
    _check(_lib().pa_prefix_evictable(pool, None, 0, ctypes.byref(n)))
    out = np.empty(n.value, np.int32)
    _check(_lib().pa_prefix_evictable(pool, out.ctypes.data, n.value, ctypes.byref(n)))
    return out


# ------------------------------------------------------------------ preemption with swap
def pa_swap_bytes(pool, seq_id: int) -> int:
    n = ctypes.c_size_t()
    _check(_lib().pa_swap_bytes(pool, seq_id, ctypes.byref(n)))
    return n.value


def _swap_buf(host_buf):
    if host_buf is None:
        return None, 0
    assert not host_buf.is_cuda and host_buf.is_pinned() and host_buf.is_contiguous()
    return host_buf.data_ptr(), host_buf.numel() * host_buf.element_size()


def pa_swap_out(pool, seq_id: int, host_buf=None, stream=None) -> None:
    """Copy seq_id's blocks to the pinned CPU tensor host_buf and release them."""
    ptr, nbytes = _swap_buf(host_buf)
    _check(_lib().pa_swap_out(pool, seq_id, ptr, nbytes, _stream(stream) if ptr else None))


def pa_swap_in(pool, seq_id: int, host_buf=None, stream=None) -> None:
    """Give seq_id new blocks and copy host_buf back into them."""
    ptr, nbytes = _swap_buf(host_buf)
    _check(_lib().pa_swap_in(pool, seq_id, ptr, nbytes, _stream(stream) if ptr else None))


# ------------------------------------------------------------------ device work
def pa_copy_blocks(pool, pairs_dev, n_pairs=None, stream=None) -> None:
    n = pairs_dev.shape[0] if n_pairs is None else n_pairs
    _check(_lib().pa_copy_blocks(pool, _dev_ptr(pairs_dev), n, _stream(stream)))


def pa_append_kv(pool, layer: int, k_new, v_new, slot_mapping_dev, n_tokens=None, stream=None) -> None:
    n = slot_mapping_dev.shape[0] if n_tokens is None else n_tokens
    _check(_lib().pa_append_kv(pool, layer, _dev_ptr(k_new), _dev_ptr(v_new), _dev_ptr(slot_mapping_dev),
                               n, _stream(stream)))


def pa_decode_max_splits(block_size: int, max_blocks: int, split_tokens: int) -> int:
    return int(_lib().pa_decode_max_splits(block_size, max_blocks, split_tokens))


def pa_decode_workspace_bytes(n_seqs: int, num_q_heads: int, head_dim: int, max_splits: int) -> int:
    return int(_lib().pa_decode_workspace_bytes(n_seqs, num_q_heads, head_dim, max_splits))


def pa_decode_attention(pool, layer: int, q, out, block_tables_dev, seq_lens_dev, scale: float,
                        split_tokens: int = 0, workspace=None, n_seqs=None, stream=None) -> None:
    """q [n][Hq][D] (pool dtype), out [n][Hq][D] (fp32 or pool dtype), tables [n][max_blocks],
    lens [n]; all CUDA tensors."""
    n = q.shape[0] if n_seqs is None else n_seqs
    hq = q.shape[1]
    max_blocks = block_tables_dev.shape[1]
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib().pa_decode_attention(pool, layer, _dev_ptr(q), _dev_ptr(out), _dtype_code(out.dtype),
                                      _dev_ptr(block_tables_dev), max_blocks, _dev_ptr(seq_lens_dev), n, hq,
                                      float(scale), split_tokens, _dev_ptr(workspace), ws_bytes,
                                      _stream(stream)))


def pa_prefill_attention(pool, layer: int, q, out, block_tables_dev, seq_lens_dev, q_start_dev,
                         max_q_len: int, scale: float, stream=None) -> None:
    """Causal chunked-prefill attention: q / out [total][Hq][128], q_start [n + 1] (CUDA tensors)."""
    n = seq_lens_dev.shape[0]
    _check(_lib().pa_prefill_attention(pool, layer, _dev_ptr(q), _dev_ptr(out), _dtype_code(out.dtype),
                                       _dev_ptr(block_tables_dev), block_tables_dev.shape[1],
                                       _dev_ptr(seq_lens_dev), _dev_ptr(q_start_dev), n, max_q_len, q.shape[1],
                                       float(scale), _stream(stream)))


PA_STATIC_WORKSPACE_BYTES = 16 << 20


def pa_decode_attention_static(pool, layer: int, q, out, block_tables_dev, seq_lens_dev, scale: float,
                               split_tokens: int = 0, n_seqs=None, stream=None) -> None:
    """pa_decode_attention without a caller workspace: the split partials live in a
    fixed array inside the library, so the call allocates no device memory."""
    n = q.shape[0] if n_seqs is None else n_seqs
    _check(_lib().pa_decode_attention_static(pool, layer, _dev_ptr(q), _dev_ptr(out), _dtype_code(out.dtype),
                                             _dev_ptr(block_tables_dev), block_tables_dev.shape[1],
                                             _dev_ptr(seq_lens_dev), n, q.shape[1], float(scale), split_tokens,
                                             _stream(stream)))


# ------------------------------------------------------------------ diagnostics
def pa_device_error(clear: bool = False) -> int:
    code = ctypes.c_int32()
    _check(_lib().pa_device_error(ctypes.byref(code), 1 if clear else 0))
    return code.value


def pa_debug_wait_test(wait_limit_ns: int = 0, withhold_cta: int = -1) -> None:
    """Failure-detection test hook: bound of every device-side wait (0: the 2 s
    default) and the decode CTA whose copies are withheld (-1: none)."""
    _check(_lib().pa_debug_wait_test(int(wait_limit_ns), int(withhold_cta)))


def pa_launch_count() -> int:
    return int(_lib().pa_launch_count())


def pa_last_error() -> str:
    return _lib().pa_last_error().decode()
