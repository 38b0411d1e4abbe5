"""The C ABI library loads without a GPU and exports every symbol include/pa.h declares."""
import ctypes
import os
import re

import pytest

import paged_kv_cache_403_b200 as pa
from paged_kv_cache_403_b200 import _native

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    text = open(os.path.join(ROOT, "include", "pa.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_path():
    names = declared_functions()
    for required in ["pa_pool_create", "pa_alloc_block", "pa_free_block", "pa_append_kv",
                     "pa_copy_blocks", "pa_decode_attention", "pa_reserve_slots"]:
        assert required in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(_native.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert missing == []


def test_binding_covers_every_declared_symbol():
    assert sorted(_native.SIGNATURES) == declared_functions()
    for n in declared_functions():
        assert hasattr(pa, n) or n in ("pa_status_string",)


def test_status_strings_and_sizes():
    lib = _native.lib()
    assert lib.pa_status_string(2) == b"PA_ERR_OUT_OF_BLOCKS"
    assert pa.pa_decode_max_splits(16, 260, 0) == 1
    assert pa.pa_decode_max_splits(16, 260, 512) == 9
    assert pa.pa_decode_max_splits(16, 260, 8) == 0          # smaller than a block
    # split partials and merge counters (only with more than one split) + the
    # longest-first range order, each rounded up to 16 bytes
    assert pa.pa_decode_workspace_bytes(4, 32, 128, 1) == 16
    assert pa.pa_decode_workspace_bytes(4, 32, 128, 3) == 4 * 3 * 32 * (128 + 2) * 4 + 48 + 4 * 32 * 4


def test_device_calls_without_device_memory_fail_cleanly():
    pool = pa.pa_pool_create(1, 8, 16, 2, 64, "f32")
    with pytest.raises(pa.PaError) as e:
        pa._check(pa._lib().pa_append_kv(pool, 0, None, None, None, 1, None))
    assert e.value.status == pa.PA_ERR_INVALID_ARG
    with pytest.raises(pa.PaError):
        pa._check(pa._lib().pa_decode_attention(pool, 0, None, None, 0, None, 1, None, 1, 2, 1.0, 0,
                                                None, 0, None))
    pa.pa_pool_destroy(pool)
