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


def test_fp8_pool_configuration_rules():
    """FP8 pools: a 16-bit activation type is required, block sizes are multiples of 16,
    the scale array attaches to FP8 pools only, and host bookkeeping works without device
    memory; the swap record of a block carries its codes and its scale bytes."""
    with pytest.raises(pa.PaError) as e:                    # no activation type given
        pa.pa_pool_create(1, 8, 16, 2, 128, "fp8")
    assert e.value.status == pa.PA_ERR_INVALID_ARG
    with pytest.raises(pa.PaError) as e:
        pa.pa_pool_create(1, 8, 16, 2, 128, "fp8", act_dtype="f32")
    assert e.value.status == pa.PA_ERR_INVALID_ARG
    with pytest.raises(pa.PaError) as e:
        pa.pa_pool_create(1, 8, 8, 2, 128, "fp8", act_dtype="bf16")
    assert e.value.status == pa.PA_ERR_UNSUPPORTED
    bf = pa.pa_pool_create(1, 8, 16, 2, 128, "bf16")
    with pytest.raises(pa.PaError) as e:                    # scales on a 16-bit pool
        pa._check(pa._lib().pa_pool_set_scales(bf, 16))
    assert e.value.status == pa.PA_ERR_INVALID_ARG
    pa.pa_pool_destroy(bf)
    p = pa.pa_pool_create(3, 40, 16, 2, 128, "fp8", act_dtype="bf16")
    with pytest.raises(pa.PaError) as e:                    # misaligned scale array
        pa._check(pa._lib().pa_pool_set_scales(p, 8))
    assert e.value.status == pa.PA_ERR_INVALID_ARG
    s = pa.pa_seq_add(p)
    pa.pa_reserve_slots(p, [s], [50])                       # 4 blocks
    # per block and layer: K and V codes (2 * 2 heads * 16 * 128) + scale bytes (2 heads * 2 * 16)
    assert pa.pa_swap_bytes(p, s) == 4 * 3 * (2 * 2 * 16 * 128 + 2 * 2 * 16)
    pa.pa_swap_out(p, s)                                    # bookkeeping only (no device pools)
    pa.pa_swap_in(p, s)
    assert pa.pa_seq_info(p, s)[0] == 50
    pa.pa_pool_destroy(p)


def test_decode_workspace_sizes_cover_every_part():
    # n * max_splits range ids; with splits also partials (acc + (m, l)) and one counter
    # per (sequence, query head); each part rounded up to 16 bytes
    for n, hq, d, ms in [(1, 1, 64, 1), (7, 8, 128, 1), (7, 8, 128, 5), (256, 32, 128, 3)]:
        parts = n * ms * hq
        partials = -(-(parts * d * 4 + parts * 8) // 16) * 16 if ms > 1 else 0
        order = -(-(n * ms * 4) // 16) * 16
        counters = -(-(n * hq * 4) // 16) * 16 if ms > 1 else 0
        assert pa.pa_decode_workspace_bytes(n, hq, d, ms) == partials + order + counters


def test_static_entry_limit_matches_header_and_refuses_oversize_batches_before_any_device_call():
    text = open(os.path.join(ROOT, "include", "pa.h")).read()
    m = re.search(r"#define PA_STATIC_WORKSPACE_BYTES \((\d+)u << (\d+)\)", text)
    assert m and int(m.group(1)) << int(m.group(2)) == pa.PA_STATIC_WORKSPACE_BYTES
    # 4096 sequences of 32 q heads, 17 split ranges each: partials far beyond the array
    pool = pa.pa_pool_create(1, 8, 16, 8, 128, "bf16")
    ms = pa.pa_decode_max_splits(16, 4096 // 16 + 1, 256)
    assert pa.pa_decode_workspace_bytes(4096, 32, 128, ms) > pa.PA_STATIC_WORKSPACE_BYTES
    st = pa._lib().pa_decode_attention_static(pool, 0, None, None, 2, None, 4096 // 16 + 1, None, 4096, 32,
                                             0.1, 256, None)
    assert st == pa.PA_ERR_INVALID_ARG
    assert "split scratch" in pa.pa_last_error() and str(pa.PA_STATIC_WORKSPACE_BYTES) in pa.pa_last_error()
    pa.pa_pool_destroy(pool)
