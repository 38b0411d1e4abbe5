"""Oracle for the paged decode path -- TEST INFRASTRUCTURE ONLY.

Plain CPU implementations, fp64 for the attention arithmetic, written from the
pages and independent of the GPU library (no shared code, headers, constants or
helpers; neither imports the other).  Only tests/, __graft_entry__.smoke() and
bench.py's CPU-baseline leg may import it.

* ``paged_decode``          -- gather K/V through the block table, textbook softmax
                               attention in double precision (oracle.c).
* ``block_manager``         -- free stack, refcounts, tables, copy-on-write (Python).
* ``cache_model``           -- where appended rows and copied blocks land (numpy).
* ``fp8``                   -- E4M3 codes with per-row power-of-two scales: encode,
                               decode, row quantisation (numpy).
* ``paged_decode_fp8``      -- decode attention over an FP8 cache: dequantise exactly,
                               then the same fp64 attention.

Parity status of each function is recorded with its tests: all are pinned
(closed forms and page figures, exhaustive decoder checks, brute force, a library
routine, planted-mistake checks).
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import block_manager, cache_model, fp8  # noqa: F401
from .build import build as _build

_CODES = {"f32": 0, "f16": 1, "bf16": 2, "f64": 3}
_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build()
        L = ctypes.CDLL(path)
        L.oracle_paged_decode.restype = ctypes.c_int
        L.oracle_paged_decode.argtypes = [
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p,
            ctypes.c_int, ctypes.c_void_p, ctypes.c_int, ctypes.c_double, ctypes.c_void_p,
            ctypes.c_int]
        L.oracle_paged_prefill.restype = ctypes.c_int
        L.oracle_paged_prefill.argtypes = [
            ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_int,
            ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p,
            ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_int, ctypes.c_double,
            ctypes.c_void_p, ctypes.c_int]
        L.oracle_widen.restype = None
        L.oracle_widen.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p]
        L.oracle_max_threads.restype = ctypes.c_int
        _lib = L
    return _lib


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def widen(stored: np.ndarray, dtype: str) -> np.ndarray:
    """Decode stored fp32 / fp16 / bf16-bit values to float64 with the oracle's decoders."""
    a = np.ascontiguousarray(stored)
    out = np.empty(a.shape, np.float64)
    lib().oracle_widen(_ptr(a), _CODES[dtype], a.size, _ptr(out))
    return out


def paged_decode(k_layer: np.ndarray, v_layer: np.ndarray, dtype: str, tables, lens,
                 q: np.ndarray, scale: float, n_threads: int = 0) -> np.ndarray:
    """fp64 paged decode attention.

    k_layer, v_layer: [num_blocks][num_kv_heads][block_size][head_dim] storage arrays.
    tables [n][max_blocks] int32, lens [n] int32, q [n][num_q_heads][head_dim] storage.
    Returns [n][num_q_heads][head_dim] float64.
    """
    k = np.ascontiguousarray(k_layer)
    v = np.ascontiguousarray(v_layer)
    nb, hkv, bs, d = k.shape
    t = np.ascontiguousarray(tables, dtype=np.int32)
    ln = np.ascontiguousarray(lens, dtype=np.int32)
    qq = np.ascontiguousarray(q)
    n, hq, dq = qq.shape
    assert dq == d and t.shape[0] == n and ln.shape[0] == n
    out = np.empty((n, hq, d), np.float64)
    rc = lib().oracle_paged_decode(_ptr(k), _ptr(v), _CODES[dtype], nb, bs, hkv, d, _ptr(t),
                                   t.shape[1] if t.ndim == 2 else 0, _ptr(ln), n, _ptr(qq), hq,
                                   float(scale), _ptr(out), int(n_threads))
    if rc != 0:
        raise ValueError("oracle_paged_decode rejected its arguments")
    return out


def paged_prefill(k_layer: np.ndarray, v_layer: np.ndarray, dtype: str, tables, lens, q_start,
                  q: np.ndarray, scale: float, n_threads: int = 0) -> np.ndarray:
    """fp64 causal chunked-prefill attention over the paged cache.

    q_start [n+1]: sequence s owns query rows q_start[s]..q_start[s+1]-1, the last
    tokens of its length lens[s].  Returns [total_q][num_q_heads][head_dim] float64.
    """
    k = np.ascontiguousarray(k_layer)
    v = np.ascontiguousarray(v_layer)
    nb, hkv, bs, d = k.shape
    t = np.ascontiguousarray(tables, dtype=np.int32)
    ln = np.ascontiguousarray(lens, dtype=np.int32)
    qs = np.ascontiguousarray(q_start, dtype=np.int32)
    qq = np.ascontiguousarray(q)
    rows, hq, dq = qq.shape
    assert dq == d and qs[-1] == rows and t.shape[0] == ln.shape[0] == qs.shape[0] - 1
    out = np.empty((rows, hq, d), np.float64)
    rc = lib().oracle_paged_prefill(_ptr(k), _ptr(v), _CODES[dtype], nb, bs, hkv, d, _ptr(t), t.shape[1],
                                    _ptr(ln), _ptr(qs), ln.shape[0], _ptr(qq), hq, float(scale), _ptr(out),
                                    int(n_threads))
    if rc != 0:
        raise ValueError("oracle_paged_prefill rejected its arguments")
    return out


def paged_decode_fp8(k_codes: np.ndarray, v_codes: np.ndarray, k_scales: np.ndarray, v_scales: np.ndarray,
                     tables, lens, q: np.ndarray, q_dtype: str, scale: float, n_threads: int = 0) -> np.ndarray:
    """fp64 paged decode attention over an FP8 cache (one layer).

    k_codes, v_codes: [num_blocks][num_kv_heads][block_size][head_dim] E4M3 codes;
    k_scales, v_scales: [num_blocks][num_kv_heads][block_size] scale bytes; q in its
    own storage type ``q_dtype``.  Every cached value is dequantised exactly
    (fp8.dequantize), then attention runs as in ``paged_decode``.
    """
    k = np.ascontiguousarray(fp8.dequantize(k_codes, k_scales))
    v = np.ascontiguousarray(fp8.dequantize(v_codes, v_scales))
    q64 = np.ascontiguousarray(widen(q, q_dtype))
    return paged_decode(k, v, "f64", tables, lens, q64, scale, n_threads)


def max_threads() -> int:
    return lib().oracle_max_threads()
