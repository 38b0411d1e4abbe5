"""Oracle for the FP8 KV cache -- TEST INFRASTRUCTURE ONLY.

Plain numpy, written from the format definitions; shares nothing with the GPU
library.  Only tests/, __graft_entry__.smoke() and bench.py's CPU legs may use it.

Why a quantised cache at all: "What problem does PagedAttention solve, and what is
continuous batching?", section "Common misconception" (and the FAQ answer on whether
PagedAttention shrinks the cache): paging changes layout and allocation, not the
bytes each cached token needs; KV-cache quantisation is one of the things that do
reduce them.  The pages name the idea and fix no format, so everything below is a
reading, stated once here and listed with the other readings of the pages:

* Element format: 8-bit floating point E4M3 in the "fn" variant of the OCP 8-bit
  floating point specification -- 1 sign bit, 4 exponent bits with bias 7, 3
  mantissa bits, no infinities, the all-ones exponent and mantissa (0x7F / 0xFF)
  is NaN, so the largest finite magnitude is 1.75 * 2^8 = 448.  Exponent field 0
  holds the subnormals m/8 * 2^-6.
* Scale: one per (token, KV head) row of head_dim elements, a power of two
  2^X stored as the byte X + 127 (the E8M0 encoding of the OCP Microscaling
  formats).  X is the smallest integer with max|row| <= 448 * 2^X, clamped to
  [-127, 127] (an all-zero row gets X = -127).  A power of two keeps x / 2^X
  exact, and a per-row scale makes a row's codes depend on that row alone, so an
  append never has to re-encode earlier rows of the block.
* Encoding of one element x of the row (taken in fp32, exactly as stored in the
  activation type): y = fp32(x * 2^-X), then y rounded to the nearest E4M3 value,
  ties to even mantissa, magnitudes above 448 saturating to 448 (none occur for a
  finite row, because |y| <= 448 by the choice of X).  The sign is kept, so a
  negative value that rounds to zero is -0 (code 0x80).
* Decoding: value = E4M3(code) * 2^(e - 127), exact in double precision.

Parity status: every function here is pinned in tests/test_oracle_fp8.py
(exhaustive decode against torch.float8_e4m3fn, encode against torch on all ties
and their neighbours, brute-force nearest-value search, the scale rule checked by
its defining inequalities, planted-mistake checks).
"""
from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0
SCALE_BIAS = 127


def e4m3_decode(codes) -> np.ndarray:
    """E4M3 ("fn") codes -> float64 values, from the bit-field definition."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    field = (c >> 3) & 0xF
    mant = c & 0x7
    subnormal = np.ldexp(mant.astype(np.float64) / 8.0, -6)
    normal = np.ldexp(1.0 + mant.astype(np.float64) / 8.0, (field - 7).astype(np.int64))
    mag = np.where(field == 0, subnormal, normal)
    mag = np.where((c & 0x7F) == 0x7F, np.nan, mag)
    return sign * mag


def e4m3_encode(y) -> np.ndarray:
    """Round float values to E4M3 codes: nearest, ties to even, saturate at 448.

    Works on the exact double value of each input (fp32 inputs widen exactly).
    NaN becomes 0x7F (with the input's sign bit).
    """
    y = np.asarray(y, dtype=np.float64)
    neg = np.signbit(y)
    a = np.abs(y)
    # exponent of the leading bit: a = f * 2^k with f in [0.5, 1)  ->  a in [2^(k-1), 2^k)
    _, k = np.frexp(np.where(a > 0, a, 1.0))
    unb = k - 1                                         # a in [2^unb, 2^(unb+1))
    # Quantum (distance between neighbouring codes) at this magnitude: 2^(unb-3) for
    # normals (unb >= -6), the subnormal step 2^-9 below that.
    step_exp = np.where(unb >= -6, unb - 3, -9)
    r = np.rint(np.ldexp(a, -step_exp))                 # multiples of the quantum; rint ties to even
    # Code of r quanta: normals are (unb + 7) << 3 | (r - 8), subnormals just r; a
    # carry (r == 16) rolls into the next exponent by plain addition.
    code = np.where(unb >= -6, ((unb + 7) << 3) + (r - 8), r)
    code = np.where(a == 0, 0, code)
    code = np.minimum(code, 0x7E)                       # saturate at 448
    code = np.where(np.isnan(y), 0x7F, code).astype(np.int64)
    return (code | np.where(neg, 0x80, 0)).astype(np.uint8)


def row_exponent(amax) -> np.ndarray:
    """Smallest integer X with amax <= 448 * 2^X, clamped to [-127, 127] (0 -> -127).

    Decided from the fp32 value's bits, exactly: amax = 1.M * 2^(E - 127) for a
    biased exponent E in 1..254, and amax <= 1.75 * 2^(8 + X) holds first at
    X = E - 135 when 1.M <= 1.75 (M <= 0x600000), else at X = E - 134.
    """
    a = np.asarray(amax, dtype=np.float32)
    bits = a.view(np.uint32).astype(np.int64) & 0x7FFFFFFF
    E = bits >> 23
    M = bits & 0x7FFFFF
    X = np.where(M <= 0x600000, E - 135, E - 134)
    X = np.where(E == 0, -127, X)                       # zero and fp32 subnormals
    return np.clip(X, -127, 127)


def quantize_rows(x) -> tuple[np.ndarray, np.ndarray]:
    """Quantise rows (last axis = one row of head_dim) to (codes uint8, scale bytes uint8)."""
    x = np.asarray(x, dtype=np.float32)
    amax = np.max(np.abs(x), axis=-1)
    X = row_exponent(amax)
    factor = np.ldexp(np.float32(1.0), (-X).astype(np.int32)).astype(np.float32)   # 2^-X, exact
    y = (x * factor[..., None]).astype(np.float32)      # one fp32 multiply per element
    return e4m3_encode(y), (X + SCALE_BIAS).astype(np.uint8)


def dequantize(codes, scale_bytes) -> np.ndarray:
    """codes [..., d] with scale bytes [...] -> float64 values, exactly."""
    e = np.asarray(scale_bytes, dtype=np.int64) - SCALE_BIAS
    return np.ldexp(e4m3_decode(codes), e[..., None])
