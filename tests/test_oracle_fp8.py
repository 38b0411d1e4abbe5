"""Pins for the FP8 (E4M3, per-row power-of-two scale) oracle, CPU only.

The oracle's codec is written from the bit-field definition; here it is held to
things outside itself: torch's independent float8_e4m3fn conversions (all 256
codes decoded, every rounding tie and its fp32 neighbours encoded), a brute-force
nearest-value search over the 254 finite codes, the scale rule's defining
inequalities at every power-of-two boundary, exact round trips of representable
rows, the half-quantum error bound, and decode attention checked against the
pinned fp64 attention oracle fed with torch-decoded values.  Planted mistakes in
the oracle's source must each fail at least one of these checks.
"""
import inspect
import types

import numpy as np
import pytest
import torch

import oracle
from oracle import fp8 as FP8

FINITE = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], np.uint8)


def torch_decode(codes):
    t = torch.from_numpy(np.asarray(codes, np.uint8).copy()).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def torch_encode(y):
    return torch.from_numpy(np.asarray(y, np.float32).copy()).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def tie_points():
    """fp32 values at every midpoint between neighbouring positive codes, and one fp32
    ulp either side of it, with both signs."""
    v = np.sort(torch_decode(FINITE[FINITE < 0x80]))
    mids = ((v[:-1] + v[1:]) / 2).astype(np.float32)     # exact in fp32
    pts = np.concatenate([mids, np.nextafter(mids, np.float32(np.inf)), np.nextafter(mids, np.float32(0)),
                          v.astype(np.float32)])
    return np.concatenate([pts, -pts]).astype(np.float32)


# ------------------------------------------------------------------ checks (module under test F)
def check_decode(F):
    ours, ref = F.e4m3_decode(np.arange(256)), torch_decode(np.arange(256))
    return bool(np.array_equal(np.isnan(ours), np.isnan(ref)) and
                np.array_equal(ours[~np.isnan(ref)], ref[~np.isnan(ref)]) and
                np.array_equal(np.signbit(ours[~np.isnan(ref)]), np.signbit(ref[~np.isnan(ref)])))


def check_encode_vs_torch(F):
    rng = np.random.default_rng(0)
    y = np.concatenate([tie_points(),
                        rng.uniform(-464, 464, 20000).astype(np.float32),
                        (np.exp2(rng.uniform(-14, np.log2(464.0), 20000)) * rng.choice([-1, 1], 20000)).astype(np.float32),
                        np.array([0.0, -0.0, 464.0, -464.0, 2.0 ** -10, -2.0 ** -10, 1e-30, -1e-30], np.float32)])
    return bool(np.array_equal(F.e4m3_encode(y), torch_encode(y)))


def check_encode_saturates(F):
    big = np.array([448.0001, 465, 500, 1e4, 3e38, np.inf], np.float32)
    return bool((F.e4m3_encode(big) == 0x7E).all() and (F.e4m3_encode(-big) == 0xFE).all() and
                (F.e4m3_encode(np.array([np.nan], np.float32)) & 0x7F == 0x7F).all())


def check_encode_is_nearest(F):
    rng = np.random.default_rng(1)
    y = np.concatenate([rng.uniform(-448, 448, 3000), np.exp2(rng.uniform(-12, 8.8, 3000)),
                        -np.exp2(rng.uniform(-12, 8.8, 3000))]).astype(np.float32).astype(np.float64)
    vals = torch_decode(FINITE)
    codes = F.e4m3_encode(y)
    got = torch_decode(codes)
    dist = np.abs(y[:, None] - vals[None, :])
    best = dist.min(axis=1)
    if not np.array_equal(np.abs(y - got), best):
        return False
    ties = (dist == best[:, None]).sum(axis=1) > 1
    nonzero = got != 0
    return bool(((codes[ties & nonzero] & 1) == 0).all())     # ties go to the even mantissa


def check_row_exponent(F):
    ks = np.arange(-150, 120)              # 448 * 2^119 is the last finite fp32 one
    base = (448.0 * np.exp2(ks.astype(np.float64))).astype(np.float32)
    a = np.concatenate([base, np.nextafter(base, np.float32(np.inf)), np.nextafter(base, np.float32(0)),
                        np.array([0.0, 1e-45, 1e-40, 2.0 ** -126, 1.0, 3.4e38], np.float32),
                        np.abs(np.random.default_rng(2).standard_normal(5000)).astype(np.float32) * 10])
    a = a[np.isfinite(a)]
    X = F.row_exponent(a).astype(np.int64)
    a64 = a.astype(np.float64)
    fits = a64 <= 448.0 * np.exp2(X.astype(np.float64))
    minimal = (X == -127) | (a64 > 448.0 * np.exp2((X - 1).astype(np.float64)))
    return bool(fits.all() and minimal.all() and (X >= -127).all() and (X <= 127).all() and
                F.row_exponent(np.float32(0.0)) == -127)


def representable_rows(rng, n, d):
    """Rows code * 2^X whose largest |code| has exponent field 15 (values 256..448), so
    the scale rule must give back exactly X."""
    codes = rng.choice(FINITE, size=(n, d)).astype(np.uint8)
    lead = rng.integers(0, d, n)
    codes[np.arange(n), lead] = (0x78 + rng.integers(0, 7, n)) | (rng.integers(0, 2, n) << 7)
    X = rng.integers(-20, 20, n)
    x = (torch_decode(codes) * np.exp2(X.astype(np.float64))[:, None]).astype(np.float32)
    return x, codes, X


def check_round_trip(F):
    rng = np.random.default_rng(3)
    x, codes, X = representable_rows(rng, 400, 64)
    qc, qs = F.quantize_rows(x)
    return bool(np.array_equal(qc, codes) and np.array_equal(qs.astype(np.int64) - 127, X))


def check_error_bound(F):
    rng = np.random.default_rng(4)
    ok = True
    for sigma in (1e-6, 1e-2, 1.0, 37.0, 1e5):
        x = (rng.standard_normal((300, 128)) * sigma).astype(np.float32)
        qc, qs = F.quantize_rows(x)
        X = qs.astype(np.int64) - 127
        deq = F.dequantize(qc, qs)
        bound = np.abs(x.astype(np.float64)) * 2.0 ** -4 + np.exp2(X - 10.0)[:, None]
        ok &= bool((np.abs(x - deq) <= bound).all())
        ok &= bool((np.abs(x).max(axis=1) > 448 * np.exp2(X - 1.0)).all())   # the scale uses the range
    return ok


def fp8_case(rng, lens, hq, hkv, d, B, nb):
    order = rng.permutation(nb)
    nblk = [-(-L // B) for L in lens]
    tables = np.full((len(lens), max(nblk)), -1, np.int32)
    it = iter(order)
    for s, n in enumerate(nblk):
        for b in range(n):
            tables[s, b] = next(it)
    kc = rng.choice(FINITE, size=(nb, hkv, B, d)).astype(np.uint8)
    vc = rng.choice(FINITE, size=(nb, hkv, B, d)).astype(np.uint8)
    ks = rng.integers(118, 124, (nb, hkv, B)).astype(np.uint8)
    vs = rng.integers(118, 124, (nb, hkv, B)).astype(np.uint8)
    q = rng.standard_normal((len(lens), hq, d)).astype(np.float32)
    return kc, vc, ks, vs, tables, np.array(lens, np.int32), q


def check_attention(F):
    """Attention over the FP8 cache equals the pinned fp32 attention oracle over the
    same values decoded by torch (exact in fp32: 4 significant bits times 2^X)."""
    rng = np.random.default_rng(5)
    kc, vc, ks, vs, tables, lens, q = fp8_case(rng, [1, 15, 16, 17, 70, 33], 8, 2, 64, 16, 40)
    kf = (torch_decode(kc) * np.exp2(ks.astype(np.float64) - 127)[..., None]).astype(np.float32)
    vf = (torch_decode(vc) * np.exp2(vs.astype(np.float64) - 127)[..., None]).astype(np.float32)
    ref = oracle.paged_decode(kf, vf, "f32", tables, lens, q, 0.125)
    got = oracle.paged_decode(np.ascontiguousarray(F.dequantize(kc, ks)), np.ascontiguousarray(F.dequantize(vc, vs)),
                              "f64", tables, lens, q.astype(np.float64), 0.125)
    return bool(np.array_equal(got, ref))


CHECKS = [check_decode, check_encode_vs_torch, check_encode_saturates, check_encode_is_nearest, check_row_exponent,
          check_round_trip, check_error_bound, check_attention]


@pytest.mark.parametrize("check", CHECKS, ids=lambda c: c.__name__)
def test_oracle_passes(check):
    assert check(FP8)


def test_format_facts():
    v = FP8.e4m3_decode(np.array([0x7E, 0x01, 0x08, 0x80, 0x38, 0xFE], np.uint8))
    assert list(v[:3]) == [448.0, 2.0 ** -9, 2.0 ** -6]
    assert v[3] == 0 and np.signbit(v[3])
    assert v[4] == 1.0 and v[5] == -448.0


def test_paged_decode_fp8_is_dequantise_then_attend():
    rng = np.random.default_rng(6)
    kc, vc, ks, vs, tables, lens, q = fp8_case(rng, [5, 40, 16], 4, 2, 64, 16, 12)
    qb = oracle.cache_model  # noqa: F841  (module import check)
    from synthetic import values as sv
    qh = sv.narrow(q, "bf16")
    got = oracle.paged_decode_fp8(kc, vc, ks, vs, tables, lens, qh, "bf16", 0.3)
    kf = (torch_decode(kc) * np.exp2(ks.astype(np.float64) - 127)[..., None]).astype(np.float32)
    vf = (torch_decode(vc) * np.exp2(vs.astype(np.float64) - 127)[..., None]).astype(np.float32)
    ref = oracle.paged_decode(kf, vf, "f32", tables, lens, oracle.widen(qh, "bf16").astype(np.float32), 0.3)
    assert np.array_equal(got, ref)


def test_cache_model_append_and_copy_fp8():
    from oracle import cache_model as cm
    rng = np.random.default_rng(7)
    kp, vp = cm.empty_pools(2, 6, 2, 16, 64, "fp8")
    sc = cm.empty_scales(2, 6, 2, 16)
    rows_k = rng.standard_normal((3, 2, 64)).astype(np.float16)
    rows_v = rng.standard_normal((3, 2, 64)).astype(np.float16)
    cm.append_rows_fp8(kp, vp, sc, 1, [5 * 16 + 3, -1, 2 * 16], rows_k, rows_v, "f16")
    codes, ks = FP8.quantize_rows(rows_k.astype(np.float32))
    _, vs = FP8.quantize_rows(rows_v.astype(np.float32))
    assert np.array_equal(kp[1, 5, :, 3], codes[0]) and np.array_equal(sc[1, 5, :, 0, 3], ks[0])
    assert np.array_equal(sc[1, 5, :, 1, 3], vs[0]) and np.array_equal(kp[1, 2, :, 0], codes[2])
    assert kp[0].sum() == 0 and np.count_nonzero(sc) == 8       # 2 rows x 2 heads x K, V; layer 1 only
    cm.copy_blocks(kp, vp, [(5, 1)])
    cm.copy_scales(sc, [(5, 1)])
    assert np.array_equal(kp[:, 1], kp[:, 5]) and np.array_equal(sc[:, 1], sc[:, 5])
    buf = cm.swap_buffer_fp8(kp, vp, sc, [5, 2])
    assert buf.size == 2 * 2 * (2 * 2 * 16 * 64 + 2 * 2 * 16)
    k2, v2 = cm.empty_pools(2, 6, 2, 16, 64, "fp8")
    sc2 = cm.empty_scales(2, 6, 2, 16)
    cm.swap_restore_fp8(k2, v2, sc2, [0, 4], buf)
    assert np.array_equal(k2[:, 0], kp[:, 5]) and np.array_equal(sc2[:, 4], sc[:, 2])


def test_bytes_per_token_halved_for_the_pages_model():
    # "What problem does PagedAttention solve...", "A concrete memory example": 32 layers x
    # 8 KV heads x head_dim 128 in fp16 is 128 KiB per token.  E4M3 codes plus one scale
    # byte per (token, head) row, for K and V.
    fp16 = 32 * 8 * 128 * 2 * 2
    fp8 = 32 * 8 * (128 + 1) * 2
    assert fp16 == 128 * 1024 and fp8 == 66048 and fp8 / fp16 == pytest.approx(0.50390625)


# ------------------------------------------------------------------ planted mistakes
MUTANTS = {
    "exponent_bias": ("(field - 7)", "(field - 8)"),
    "subnormal_scale": ("/ 8.0, -6)", "/ 8.0, -7)"),
    "round_half_up": ("r = np.rint(np.ldexp(a, -step_exp))", "r = np.floor(np.ldexp(a, -step_exp) + 0.5)"),
    "truncate": ("r = np.rint(np.ldexp(a, -step_exp))", "r = np.floor(np.ldexp(a, -step_exp))"),
    "no_saturation": ("np.minimum(code, 0x7E)", "np.minimum(code, 0x7F)"),
    "negative_zero_lost": ("np.where(neg, 0x80, 0)", "np.where(y < 0, 0x80, 0)"),
    "subnormal_step": ("unb - 3, -9)", "unb - 3, -10)"),
    "scale_boundary": ("np.where(M <= 0x600000,", "np.where(M < 0x600000,"),
    "scale_too_large": ("E - 135, E - 134", "E - 134, E - 134"),
    "dequantize_bias": ("e = np.asarray(scale_bytes, dtype=np.int64) - SCALE_BIAS",
                        "e = np.asarray(scale_bytes, dtype=np.int64) - SCALE_BIAS + 1"),
}


def mutant_module(name):
    src = inspect.getsource(FP8)
    old, new = MUTANTS[name]
    assert src.count(old) == 1, name
    mod = types.ModuleType("fp8_" + name)
    exec(compile(src.replace(old, new), "fp8_" + name, "exec"), mod.__dict__)
    return mod


def battery(F):
    for c in CHECKS:
        try:
            if not c(F):
                return False
        except Exception:
            return False
    return True


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_battery_rejects_planted_mistake(name):
    assert not battery(mutant_module(name)), f"mutant {name} passed every pin"
