"""ctypes binding of the device-side input generator (synthetic/libpa_synth.so).

Fills device tensors with the same values synthetic.values produces on the host,
so large workloads need no host-side generation or copies.
"""
from __future__ import annotations

import ctypes
import os

import torch

from .values import unit_scale_f32

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB = os.path.join(_HERE, "libpa_synth.so")
_CODES = {"f32": 0, "f16": 1, "bf16": 2}
_TORCH = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}
_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB):
            raise RuntimeError(f"{LIB} is missing: run __graft_entry__.build()")
        L = ctypes.CDLL(LIB)
        L.synth_fill_rows.restype = ctypes.c_int
        L.synth_fill_rows.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_int, ctypes.c_uint64,
                                      ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int64,
                                      ctypes.c_int, ctypes.c_int, ctypes.c_float, ctypes.c_void_p]
        _lib = L
    return _lib


def fill_rows(out: torch.Tensor, kind: int, seed: int, layer: int, uids: torch.Tensor,
              tokens: torch.Tensor, scale: float, dtype: str, stream=None) -> torch.Tensor:
    """out: device tensor [n][heads][dim] of ``dtype``; uids, tokens: device int32 [n]."""
    assert out.is_cuda and out.dtype == _TORCH[dtype] and out.dim() == 3 and out.is_contiguous()
    assert uids.dtype == torch.int32 and tokens.dtype == torch.int32
    n, heads, dim = out.shape
    s = (stream or torch.cuda.current_stream()).cuda_stream
    rc = lib().synth_fill_rows(out.data_ptr(), _CODES[dtype], kind, seed, layer, uids.data_ptr(),
                               tokens.data_ptr(), n, heads, dim, float(unit_scale_f32(scale)), s)
    if rc != 0:
        raise RuntimeError("synth_fill_rows launch failed")
    return out
