"""Pins for the CPU oracle: each test ties it to something other than itself.

Sources of the pins: the hand-derived fixtures under tests/golden (each names
the page passage it follows), exact rational arithmetic, library decoders
(ml_dtypes, torch), Python's own IEEE half packing, and a brute-force
nearest-level characterisation of the quantiser.
"""

import math
import struct
from fractions import Fraction

import numpy as np
import pytest

from oracle import int4, lut3, matmul


# ----------------------------------------------------------------------------- INT4 fixtures

def test_sym_4x4_golden(golden):
    g = golden("int4_sym_4x4.json")
    W = np.array(g["W"], dtype=np.float32)
    q, s = int4.quantize_sym(W, g["group"])
    assert q.tolist() == g["q"]
    assert s.astype(np.float64).tolist() == g["scale"]
    packed = int4.pack_nibbles(q)
    assert packed.tolist() == g["packed"]
    assert [[int(h, 16) for h in row] for row in g["packed_hex"]] == g["packed"]
    deq = int4.dequant(q, s, g["group"])
    assert deq.tolist() == g["dequant"]
    Y = matmul.matmul_f64(np.array(g["X"]), deq)
    assert Y.tolist() == g["Y"]


def test_asym_4x2_golden(golden):
    g = golden("int4_asym_4x2.json")
    W = np.array(g["W"], dtype=np.float32)
    q, s, zp = int4.quantize_asym(W, g["group"])
    assert q.tolist() == g["q"]
    assert s.astype(np.float64).tolist() == g["scale"]
    assert zp.tolist() == g["zp"]
    assert int4.pack_nibbles(q).tolist() == g["packed"]
    assert [[int(h, 16) for h in row] for row in g["packed_hex"]] == g["packed"]
    assert int4.dequant(q, s, g["group"], zp).tolist() == g["dequant"]


def test_metal_listing_byte_example():
    """The INT4 listing: low nibble 15 -> (15-8)*s = 7s; high nibble 9 -> (9-8)*s = s,
    and the low nibble belongs to the even k."""
    packed = np.array([[0x9F]], dtype=np.uint8)
    q = int4.unpack_nibbles(packed)
    assert q[:, 0].tolist() == [15, 9]
    s = np.array([[0.375]], dtype=np.float16)
    assert int4.dequant(q, s, 2)[:, 0].tolist() == [7 * 0.375, 0.375]


def test_low_nibble_is_even_k():
    q = np.zeros((4, 1), np.uint8)
    q[0, 0] = 1
    q[3, 0] = 2
    assert int4.pack_nibbles(q)[:, 0].tolist() == [0x01, 0x20]


def test_pack_roundtrip_random():
    rng = np.random.default_rng(7)
    q = rng.integers(0, 16, size=(64, 24), dtype=np.uint8)
    assert np.array_equal(int4.unpack_nibbles(int4.pack_nibbles(q)), q)
    b = rng.integers(0, 256, size=(32, 24), dtype=np.uint8)
    assert np.array_equal(int4.pack_nibbles(int4.unpack_nibbles(b)), b)


# ----------------------------------------------------------------------------- quantiser

def _half_via_struct(x):
    """Python's own IEEE binary16 packing (round to nearest even)."""
    return struct.unpack("<e", struct.pack("<e", x))[0]


def _f32_div(a, b):
    """Correctly rounded FP32 quotient via FP64 (53 >= 2*24+2 bits makes this exact)."""
    return float(np.float32(float(a) / float(b)))


@pytest.mark.parametrize("group", [32, 64, 128])
def test_sym_scale_is_fp16_of_fp32_quotient(group):
    rng = np.random.default_rng(group)
    W = (rng.standard_normal((4 * group, 16)) * 0.02).astype(np.float32)
    _, s = int4.quantize_sym(W, group)
    for gi in range(4):
        for n in range(16):
            amax = max(abs(float(v)) for v in W[gi * group:(gi + 1) * group, n])
            assert float(s[gi, n]) == _half_via_struct(_f32_div(amax, 7.0))


def test_asym_scale_is_fp16_of_fp32_quotient():
    rng = np.random.default_rng(11)
    W = (rng.standard_normal((64, 16)) * 0.02).astype(np.float32)
    _, s, _ = int4.quantize_asym(W, 32)
    for gi in range(2):
        for n in range(16):
            col = W[gi * 32:(gi + 1) * 32, n]
            span = float(np.float32(float(col.max()) - float(col.min())))
            assert float(s[gi, n]) == _half_via_struct(_f32_div(span, 15.0))


def _not_a_tie(v):
    return abs(v - math.floor(v) - 0.5) > 1e-4


@pytest.mark.parametrize("group", [32, 128])
def test_sym_codes_are_nearest_levels(group):
    """Independent characterisation: each code is the level (c-8)*s, c in 0..15,
    nearest to w (ties excluded), i.e. no other code would reconstruct w better."""
    rng = np.random.default_rng(100 + group)
    W = (rng.standard_normal((2 * group, 40)) * 0.02).astype(np.float32)
    W[3, 5] *= 20.0  # an outlier group
    q, s = int4.quantize_sym(W, group)
    levels = np.arange(16) - 8.0
    checked = 0
    for k in range(W.shape[0]):
        for n in range(W.shape[1]):
            sc = float(s[k // group, n])
            w = float(W[k, n])
            if not _not_a_tie(float(np.float32(w) / np.float32(sc))):
                continue
            best = int(np.argmin(np.abs(w - levels * sc)))
            assert q[k, n] == best
            checked += 1
    assert checked > 0.99 * W.size


def test_asym_codes_are_nearest_levels():
    rng = np.random.default_rng(5)
    W = (rng.standard_normal((128, 32)) * 0.02).astype(np.float32)
    W[:32, 0] = np.abs(W[:32, 0]) + 0.05     # an all-positive group
    W[32:64, 1] = -np.abs(W[32:64, 1]) - 0.05  # an all-negative group
    q, s, zp = int4.quantize_asym(W, 32)
    for gi in range(4):
        for n in range(32):
            sc = float(s[gi, n])
            lo = float(W[gi * 32:(gi + 1) * 32, n].min())
            t = float(np.float32(-lo) / np.float32(sc))
            if _not_a_tie(t):
                assert zp[gi, n] == int(np.clip(round(t), -128, 127))
            for k in range(gi * 32, (gi + 1) * 32):
                w = float(W[k, n])
                if not _not_a_tie(float(np.float32(w) / np.float32(sc))):
                    continue
                levels = (np.arange(16) - float(zp[gi, n])) * sc
                assert q[k, n] == int(np.argmin(np.abs(w - levels)))


def test_quantisation_error_within_half_step():
    rng = np.random.default_rng(9)
    W = (rng.standard_normal((256, 64)) * 0.02).astype(np.float32)
    for mode in ("sym", "asym"):
        q, s, zp = int4.quantize(W, 32, mode)
        deq = int4.dequant(q, s, 32, zp)
        step = np.repeat(s.astype(np.float64), 32, axis=0)
        # the fp16 rounding of the scale can push the extreme code by < 1/14 step
        assert np.all(np.abs(W - deq) <= 0.5 * step * (1 + 1 / 7) + 1e-12)


def test_sym_range_and_extremes():
    rng = np.random.default_rng(3)
    W = (rng.standard_normal((128, 64)) * 0.02).astype(np.float32)
    q, s = int4.quantize_sym(W, 32)
    assert q.min() >= 1 and q.max() <= 15          # code 0 (-8) is never produced
    Wg = W.reshape(4, 32, 64)
    arg = np.abs(Wg).argmax(axis=1)
    for gi in range(4):
        for n in range(64):
            k = gi * 32 + arg[gi, n]
            assert q[k, n] == (15 if W[k, n] > 0 else 1)


def test_degenerate_groups():
    W = np.zeros((64, 3), np.float32)
    W[32:, 1] = 0.5          # constant non-zero group: hi == lo
    W[:32, 2] = 1e-9         # max/7 underflows FP16 to 0
    q, s = int4.quantize_sym(W, 32)
    assert float(s[0, 0]) == 0.0 and np.all(q[:32, 0] == 8)
    assert np.all(int4.dequant(q, s, 32)[:32, 0] == 0.0)
    assert float(s[0, 2]) == 0.0 and np.all(q[:32, 2] == 8)
    qa, sa, za = int4.quantize_asym(W, 32)
    assert float(sa[1, 1]) == 0.0 and za[1, 1] == 0 and np.all(qa[32:, 1] == 0)
    assert np.all(int4.dequant(qa, sa, 32, za) == 0.0)


def test_dequant_is_exact_rational():
    rng = np.random.default_rng(21)
    W = (rng.standard_normal((64, 8)) * 0.02).astype(np.float32)
    q, s, zp = int4.quantize_asym(W, 32)
    deq = int4.dequant(q, s, 32, zp)
    for k in range(64):
        for n in range(8):
            exact = (int(q[k, n]) - int(zp[k // 32, n])) * Fraction(float(s[k // 32, n]))
            assert Fraction(float(deq[k, n])) == exact


# ----------------------------------------------------------------------------- matmul + tolerance

def test_matmul_matches_exact_rational_brute_force():
    rng = np.random.default_rng(13)
    M, K, N = 3, 64, 8
    X = rng.standard_normal((M, K)).astype(np.float16).astype(np.float64)
    W = (rng.standard_normal((K, N)) * 0.02).astype(np.float32)
    q, s, zp = int4.quantize_asym(W, 32)
    deq = int4.dequant(q, s, 32, zp)
    Y = matmul.matmul_f64(X, deq)
    S = matmul.abs_scale(X, deq)
    for m in range(M):
        for n in range(N):
            exact = sum(Fraction(float(X[m, k])) * Fraction(float(deq[k, n])) for k in range(K))
            assert abs(Fraction(float(Y[m, n])) - exact) <= Fraction(1e-14) * Fraction(float(S[m, n]))


def test_ulp16_values():
    u = matmul.ulp16(np.array([1.0, 1.5, 2.0, 1000.0, 2.0 ** -14, 1e-6, 0.0, -3.0]))
    assert u.tolist() == [2.0 ** -10, 2.0 ** -10, 2.0 ** -9, 0.5, 2.0 ** -24, 2.0 ** -24, 2.0 ** -24, 2.0 ** -9]


def test_abs_scale_hand_values(golden):
    """S = sum_k |x_k w_kn| against hand sums: a mixed-sign 2x3 . 3x2 case with
    cancelling terms, and the sym 4x4 fixture (S far above |y| in column 0)."""
    g = golden("acceptance_2x3x2.json")
    X, W = np.array(g["X"]), np.array(g["W"])
    assert matmul.matmul_f64(X, W).tolist() == g["Y"]
    assert matmul.abs_scale(X, W).tolist() == g["S"]
    assert matmul.ulp16(np.array(g["Y"])).tolist() == g["ulp16"]
    g4 = golden("int4_sym_4x4.json")
    assert matmul.abs_scale(np.array(g4["X"]), np.array(g4["dequant"])).tolist() == g4["S"]


@pytest.mark.parametrize("factor,accepted", [(1.5, False), (1.05, False), (0.9, True), (0.5, True)])
def test_acceptance_bound_is_tight(golden, factor, accepted):
    """An output off by `factor` hand-derived bounds is rejected above 1 and
    accepted below it, element by element, and error_ratio reports the factor:
    a 2x change in the 4e-3 factor or in S moves 1.5 or 0.9 across 1."""
    g = golden("acceptance_2x3x2.json")
    X, W = np.array(g["X"]), np.array(g["W"])
    Y_ref = np.array(g["Y"])
    bound = np.array(g["bound"])
    S = matmul.abs_scale(X, W)
    for sign in (1.0, -1.0):
        for m in range(2):
            for n in range(2):
                Y = Y_ref.copy()
                Y[m, n] += sign * factor * bound[m, n]
                r = matmul.error_ratio(Y, Y_ref, S)
                assert r[m, n] == pytest.approx(factor, rel=1e-12)
                assert matmul.check(Y, Y_ref, S)[0] is accepted


def test_tolerance_accepts_fp32_accumulation_and_rejects_mistakes():
    rng = np.random.default_rng(17)
    M, K, N = 2, 512, 64
    X = rng.standard_normal((M, K)).astype(np.float16)
    W = (rng.standard_normal((K, N)) * 0.02).astype(np.float32)
    q, s = int4.quantize_sym(W, 32)
    deq = int4.dequant(q, s, 32)
    Y_ref = matmul.matmul_f64(X, deq)
    S = matmul.abs_scale(X, deq)
    # FP32 accumulation, rounded to fp16 output: accepted
    Y32 = (X.astype(np.float32) @ deq.astype(np.float32)).astype(np.float16)
    ok, _ = matmul.check(Y32, Y_ref, S)
    assert ok
    # nibble order swapped (high nibble taken as the even k): rejected
    packed = int4.pack_nibbles(q)
    swapped = np.empty_like(q)
    swapped[0::2] = packed >> 4
    swapped[1::2] = packed & 0xF
    ok, _ = matmul.check(matmul.matmul_f64(X, int4.dequant(swapped, s, 32)), Y_ref, S)
    assert not ok
    # scale of the neighbouring group: rejected
    s_shift = np.roll(s, 1, axis=0)
    ok, _ = matmul.check(matmul.matmul_f64(X, int4.dequant(q, s_shift, 32)), Y_ref, S)
    assert not ok
    # zero point off by one (7 instead of 8): rejected
    ok, _ = matmul.check(matmul.matmul_f64(X, int4.dequant(q, s, 32, np.full(s.shape, 7, np.int8))), Y_ref, S)
    assert not ok
    # a NaN output is never accepted
    Ybad = Y32.astype(np.float64)
    Ybad[0, 0] = np.nan
    assert not matmul.check(Ybad, Y_ref, S)[0]


# ----------------------------------------------------------------------------- LUT3

def test_e4m3_table_matches_ml_dtypes_and_torch():
    import ml_dtypes
    import torch
    raw = np.arange(256, dtype=np.uint8)
    lib = raw.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    tor = torch.from_numpy(raw.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for ref in (lib, tor):
        nan = np.isnan(ref)
        assert np.array_equal(nan, np.isnan(lut3.E4M3_TABLE))
        assert np.array_equal(ref[~nan], lut3.E4M3_TABLE[~nan])
    assert sorted(np.flatnonzero(np.isnan(lut3.E4M3_TABLE)).tolist()) == [0x7F, 0xFF]
    assert lut3.e4m3_value(0x7E) == 448.0 and lut3.e4m3_value(0x01) == 2.0 ** -9


def test_ue8m0_values():
    import ml_dtypes
    raw = np.arange(255, dtype=np.uint8)
    if hasattr(ml_dtypes, "float8_e8m0fnu"):
        lib = raw.view(ml_dtypes.float8_e8m0fnu).astype(np.float64)
        assert [lut3.ue8m0_value(b) for b in range(255)] == lib.tolist()
    assert [lut3.ue8m0_value(b) for b in (0, 127, 130, 254)] == [2.0 ** -127, 1.0, 8.0, 2.0 ** 127]
    assert math.isnan(lut3.ue8m0_value(255))


def test_lut3_tile_golden(golden):
    g = golden("lut3_tile_64x8.json")
    K, N = g["K"], g["N"]
    idx = ((np.arange(K)[:, None] + np.arange(N)[None, :]) % 8).astype(np.uint8)
    cb = np.array(g["codebook"], np.uint8).reshape(1, 1, 8)
    ex = np.array([[g["exponent"]]], np.uint8)
    assert [lut3.e4m3_value(b) for b in g["codebook"]] == g["codebook_values"]
    W = lut3.dequant(idx, cb, ex)
    for k, n, v in g["W_samples"]:
        assert W[k, n] == v
    p = lut3.pack_indices(idx)
    assert p.shape == (1, 1, 8, 24)
    assert p[0, 0, 0].tolist() == g["stream_ch0"] * 8
    assert p[0, 0, 1].tolist() == g["stream_ch1"] * 8
    ones = lut3.pack_indices(np.ones((K, N), np.uint8))
    assert np.all(ones[0, 0] == np.array(g["stream_all_ones"] * 8, np.uint8))
    Y = matmul.matmul_f64(np.ones((1, K)), W)
    assert np.all(Y == g["Y_ones"])


def test_lut3_pack_roundtrip_random():
    rng = np.random.default_rng(31)
    idx = rng.integers(0, 8, size=(128, 24), dtype=np.uint8)
    assert np.array_equal(lut3.unpack_indices(lut3.pack_indices(idx)), idx)


def test_lut3_sizes_match_the_page():
    # "about 3.14 bits per weight" and 6144 index bytes per 128N x 128K block
    assert lut3.algorithmic_bytes(64, 8) * 8 / (64 * 8) == 3.140625
    assert 128 * 128 * 3 // 8 == lut3.pack_indices(np.zeros((128, 128), np.uint8)).size
    assert lut3.algorithmic_bytes(4096, 14336) == 23052288


def test_lut3_rejects_nan_entries():
    idx = np.zeros((64, 8), np.uint8)
    with pytest.raises(ValueError):
        lut3.dequant(idx, np.full((1, 1, 8), 0x7F, np.uint8), np.array([[127]], np.uint8))
    with pytest.raises(ValueError):
        lut3.dequant(idx, np.zeros((1, 1, 8), np.uint8), np.array([[255]], np.uint8))


def test_int4_algorithmic_bytes():
    # bits per weight: 4 + 16/g (sym), 4 + 24/g (asym)
    assert int4.algorithmic_bytes(4096, 4096, 32, "sym") == 4096 * 4096 * 4.5 / 8
    assert int4.algorithmic_bytes(4096, 14336, 128, "asym") == 4096 * 14336 * (4 + 24 / 128) / 8


# ----------------------------------------------------------------------------- MXFP8 activations

def _e4m3_neighbours_midpoints():
    vals = sorted({v for v in lut3.E4M3_TABLE.tolist() if not math.isnan(v) and v >= 0})
    return [(a + b) / 2 for a, b in zip(vals, vals[1:])]


def test_e4m3_rounding_matches_torch_and_ml_dtypes_in_range():
    """Round-to-nearest-even into E4M3 equals the libraries' casts for every
    value the libraries convert without saturation (|v| <= 448): random
    values across all binades, every midpoint between neighbours (ties), and
    values that underflow."""
    import ml_dtypes
    import torch
    from oracle import mxfp8
    rng = np.random.default_rng(17)
    mags = np.ldexp(rng.uniform(1.0, 2.0, 4000), rng.integers(-14, 9, 4000))
    mids = np.array(_e4m3_neighbours_midpoints())
    v = np.concatenate([mags, mids, [2.0 ** -10, 2.0 ** -11, 3 * 2.0 ** -11, 1e-9, 448.0]])
    v = v[v <= 448.0]
    v = np.concatenate([v, -v]).astype(np.float32)  # values exact in FP32 (midpoints included)
    ours = np.array([mxfp8.e4m3_byte(mxfp8.round_e4m3(float(x))) for x in v], dtype=np.uint8)
    tor = torch.from_numpy(v).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    lib = v.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    assert np.array_equal(ours, tor)
    assert np.array_equal(ours, lib)


def test_e4m3_rounding_saturates_above_448():
    from oracle import mxfp8
    assert [mxfp8.round_e4m3(x) for x in (448.0, 463.9, 464.0, 511.9, -500.0)] == [448.0] * 4 + [-448.0]


def test_mx_scale_rule_hand_examples():
    """Scale byte = floor(log2 amax) - 8 + 127 and elements x / 2^(that - 127):
    amax 1 -> scale 2^-8 and x = 1 becomes 256; amax 448 -> scale 1; amax 500
    -> scale 1 and 500 saturates to 448; amax 0.75 -> scale 2^-9 and 0.75
    becomes 384; amax 2^-130 -> the smallest scale 2^-127 (clamped), so it
    becomes 2^-3; a zero block stores scale 1."""
    from oracle import mxfp8
    def block(first, rest=0.0):
        return np.array([[first] + [rest] * 31])
    cases = [
        (1.0, 119, 256.0), (448.0, 127, 448.0), (500.0, 127, 448.0), (0.75, 118, 384.0),
        (2.0 ** -130, 0, 2.0 ** -3), (0.0, 127, 0.0),
    ]
    for amax, sbyte, elem in cases:
        codes, scales = mxfp8.quantize(block(amax))
        assert scales[0, 0] == sbyte
        assert lut3.E4M3_TABLE[codes[0, 0]] == elem
        assert mxfp8.dequant(codes, scales)[0, 0] == elem * 2.0 ** (sbyte - 127)
    # a second element is scaled by the same power of two: 0.3 * 256 = 76.8 -> 80 (quantum 8)
    codes, scales = mxfp8.quantize(block(1.0, 0.3))
    assert lut3.E4M3_TABLE[codes[0, 1]] == 80.0


def test_mx_block_maximum_lands_in_the_top_binade_and_error_is_bounded():
    """Every block's largest element is in [256, 448] after scaling, and each
    element's error is at most half an E4M3 step: 2^-4 relative in the normal
    range, 2^-10 of the scale in the subnormal range."""
    from oracle import mxfp8
    rng = np.random.default_rng(5)
    X = (rng.standard_normal((4, 256)) * np.ldexp(1.0, rng.integers(-20, 20, (4, 1)))).astype(np.float32)
    codes, scales = mxfp8.quantize(X)
    Xq = mxfp8.dequant(codes, scales)
    elems = np.abs(lut3.E4M3_TABLE[codes]).reshape(4, 8, 32)
    assert np.all(elems.max(axis=2) >= 256.0) and np.all(elems.max(axis=2) <= 448.0)
    scale = np.ldexp(1.0, scales.astype(np.int64) - 127)[:, np.arange(256) // 32]
    x = X.astype(np.float64)
    scaled = np.abs(x) / scale
    normal = (scaled >= 2.0 ** -6) & (scaled < 448.0)
    assert np.all(np.abs(Xq - x)[normal] <= 2.0 ** -4 * np.abs(x)[normal])
    assert np.all(np.abs(Xq - x)[scaled < 2.0 ** -6] <= 2.0 ** -10 * scale[scaled < 2.0 ** -6])


def test_mx_representable_blocks_round_trip_exactly():
    """A block that already is E4M3 values times one power of two, with its
    largest element in [256, 448], comes back bit for bit."""
    from oracle import mxfp8
    rng = np.random.default_rng(9)
    finite = [b for b in range(256) if not math.isnan(lut3.E4M3_TABLE[b])]
    top = [b for b in finite if 256.0 <= abs(lut3.E4M3_TABLE[b]) <= 448.0]
    for s in (-20, 0, 7):
        bytes_ = rng.choice(finite, size=(3, 64))
        bytes_[:, 0] = rng.choice(top, size=3)
        bytes_[:, 32] = rng.choice(top, size=3)
        vals = np.abs(lut3.E4M3_TABLE[bytes_]).reshape(3, 2, 32)
        assert np.all(vals.max(axis=2) <= 448.0)
        X = lut3.E4M3_TABLE[bytes_] * 2.0 ** s
        codes, scales = mxfp8.quantize(X)
        assert np.array_equal(mxfp8.dequant(codes, scales), X)
        assert np.all(scales == 127 + s)


def test_lut3_mxfp8_product_matches_exact_rational_brute_force():
    """The LUT3 x MXFP8 product equals the exact rational sum of the exact
    products of the dequantised operands (one 64 x 8 tile, two rows)."""
    from fractions import Fraction
    from oracle import mxfp8
    rng = np.random.default_rng(21)
    K, N, M = 64, 8, 2
    idx = rng.integers(0, 8, size=(K, N)).astype(np.uint8)
    cb = np.array([[[0x38, 0xB8, 0x40, 0x30, 0x7E, 0x01, 0x00, 0xC4]]], dtype=np.uint8)
    ex = np.array([[120]], dtype=np.uint8)
    X = rng.standard_normal((M, K)).astype(np.float32)
    Y = mxfp8.lut3_matmul(X, idx, cb, ex)
    codes, scales = mxfp8.quantize(X)
    Xq = mxfp8.dequant(codes, scales)
    W = lut3.dequant(idx, cb, ex)
    for m in range(M):
        for n in range(N):
            exact = sum(Fraction(float(Xq[m, k])) * Fraction(float(W[k, n])) for k in range(K))
            assert abs(Fraction(float(Y[m, n])) - exact) <= abs(exact) * Fraction(1, 2 ** 50) + Fraction(1, 2 ** 200)


# ----------------------------------------------------------------------------- generic b-bit affine

from oracle import affine  # noqa: E402


def test_affine_b3_golden(golden):
    g = golden("affine_b3_8x2.json")
    W = np.array(g["W"], dtype=np.float32)
    q, s, zp = affine.quantize(W, g["group"], g["bits"])
    assert q.tolist() == g["q"]
    assert s.astype(np.float64).tolist() == g["scale"]
    assert zp.tolist() == g["zp"]
    assert affine.pack(q, g["bits"]).tolist() == g["packed"]
    assert affine.unpack(np.array(g["packed"], dtype=np.uint8), g["bits"], g["K"]).tolist() == g["q"]
    assert affine.dequant(q, s, g["group"], zp).tolist() == g["dequant"]


def test_affine_4_bit_is_the_asymmetric_int4_form():
    """b = 4 reduces to the (separately pinned) asymmetric INT4 quantiser and
    its canonical two-nibbles-per-byte packing."""
    W = (np.random.default_rng(21).standard_normal((256, 40)) * 0.02).astype(np.float32)
    q, s, zp = affine.quantize(W, 32, 4)
    q4, s4, zp4 = int4.quantize_asym(W, 32)
    assert np.array_equal(q, q4) and np.array_equal(s.view(np.int16), s4.view(np.int16)) and np.array_equal(zp, zp4)
    assert np.array_equal(affine.pack(q, 4), int4.pack_nibbles(q4))


@pytest.mark.parametrize("bits", [1, 2, 3, 5, 6, 7, 8])
def test_affine_codes_are_nearest_levels_and_round_trip(bits):
    """Every code is the nearest of the L + 1 levels (q - zp) s to w, clamped
    to the range; packing round-trips; the bit stream holds exactly b bits per
    code (brute force over the stream)."""
    rng = np.random.default_rng(30 + bits)
    K, N, group = 64, 12, 32
    W = (rng.standard_normal((K, N)) * 0.02).astype(np.float32)
    q, s, zp = affine.quantize(W, group, bits)
    L = (1 << bits) - 1
    assert q.max() <= L
    deq = affine.dequant(q, s, group, zp)
    s_k = np.repeat(s.astype(np.float64), group, axis=0)
    z_k = np.repeat(zp.astype(np.float64), group, axis=0)
    lv = (np.arange(L + 1)[None, None, :] - z_k[:, :, None]) * s_k[:, :, None]     # [K, N, L+1]
    best = np.min(np.abs(lv - W[:, :, None].astype(np.float64)), axis=2)
    # the chosen level is a nearest one, up to the FP32 rounding of w / s
    assert np.all(np.abs(deq - W) <= best + 1e-6 * s_k + 1e-12)
    packed = affine.pack(q, bits)
    assert packed.shape == (K * bits // 8, N)
    assert np.array_equal(affine.unpack(packed, bits, K), q)
    stream = np.unpackbits(packed, axis=0, bitorder="little")   # [K*bits, N]
    for k in (0, 1, K - 1):
        val = sum(int(stream[bits * k + i, 0]) << i for i in range(bits))
        assert val == int(q[k, 0])


def test_affine_algorithmic_bytes():
    assert affine.algorithmic_bytes(4096, 4096, 32, 3) == 4096 * 4096 * 3 // 8 + 128 * 4096 * 3
    assert affine.algorithmic_bytes(4096, 14336, 64, 4) == int4.algorithmic_bytes(4096, 14336, 64, "asym")


# ----------------------------------------------------------------------------- W4A8

from oracle import w4a8  # noqa: E402


def _w4a8_golden_inputs(g):
    K, group = g["K"], g["group"]
    q = np.full((K, 2), 8, dtype=np.uint8)
    q[:, 0] = g["q_col0"]
    q[:, 1] = g["q_col1_default"]
    q[0, 1] = g["q_col1_k0"]
    sw = np.array(g["sw"], dtype=np.float16)
    return q, sw, group


def test_w4a8_activation_golden(golden):
    g = golden("w4a8_block_1x64.json")
    X = np.array(g["x"], dtype=np.float16).astype(np.float32)
    assert np.array_equal(X, np.array(g["x"], dtype=np.float64))   # every value is exact in FP16
    xq, s = w4a8.quantize_activations(X)
    assert xq.tolist() == g["xq"]
    assert s.tolist() == g["s"]


@pytest.mark.parametrize("mode", ["sym", "asym"])
def test_w4a8_product_golden(golden, mode):
    g = golden("w4a8_block_1x64.json")
    q, sw, group = _w4a8_golden_inputs(g)
    xq = np.array(g["xq"], dtype=np.int8)
    sx = np.array(g["s"], dtype=np.float32)
    zp = None if mode == "sym" else np.array(g["zp_asym"], dtype=np.int8)
    y = w4a8.matmul(xq, sx, q, sw, zp, group)
    assert y.tolist() == g["y_" + mode]


def test_w4a8_activation_invariants():
    rng = np.random.default_rng(21)
    X = (rng.standard_normal((5, 256)) * np.exp(rng.uniform(-6, 4, (5, 1)))).astype(np.float16).astype(np.float32)
    X[0, 32:64] = 0.0                        # zero block
    X[1, 64:96] = np.float32(np.float16(6e-8))  # FP16 subnormals only
    xq, s = w4a8.quantize_activations(X)
    Xb = X.reshape(5, 8, 32)
    qb = xq.reshape(5, 8, 32).astype(np.int64)
    assert np.all(np.abs(qb) <= 127)
    assert np.all(qb[0, 1] == 0) and s[0, 1] == 0
    amax_pos = np.abs(Xb).argmax(axis=2)
    for m in range(5):
        for b in range(8):
            if s[m, b] == 0:
                continue
            i = amax_pos[m, b]
            assert abs(qb[m, b, i]) == 127                     # the block maximum takes the extreme code
            err = np.abs(Xb[m, b].astype(np.float64) - qb[m, b] * np.float64(s[m, b]))
            assert np.all(err <= np.float64(s[m, b]) * (0.5 + 1e-6))   # nearest level
    # odd symmetry and exact power-of-two scaling
    xqn, sn = w4a8.quantize_activations(-X)
    assert np.array_equal(xqn, -xq) and np.array_equal(sn, s)
    xq2, s2 = w4a8.quantize_activations(X * np.float32(4.0))
    assert np.array_equal(xq2, xq) and np.array_equal(s2, s * np.float32(4.0))


def test_w4a8_scale_is_fp32_quotient_and_codes_are_fp32_rint():
    """Against a scalar restatement with Python floats rounded through struct:
    s = f32(amax / 127); xq = rint(f32(x / s)) with ties to even."""
    rng = np.random.default_rng(22)
    X = rng.standard_normal((3, 96)).astype(np.float16).astype(np.float32)
    xq, s = w4a8.quantize_activations(X)

    def f32(v):
        return struct.unpack("<f", struct.pack("<f", v))[0]

    for m in range(3):
        for b in range(3):
            blk = [float(v) for v in X[m, 32 * b:32 * b + 32]]
            amax = max(abs(v) for v in blk)
            sb = f32(amax / 127.0)
            assert float(s[m, b]) == sb
            for i, v in enumerate(blk):
                r = round(f32(v / sb))          # Python's round() is half-to-even
                assert int(xq[m, 32 * b + i]) == max(-127, min(127, r))


def test_w4a8_product_matches_exact_rational_brute_force():
    rng = np.random.default_rng(23)
    M, K, N, group = 2, 64, 3, 32
    xq = rng.integers(-127, 128, (M, K)).astype(np.int8)
    sx = rng.uniform(0.001, 0.1, (M, K // 32)).astype(np.float32)
    q = rng.integers(0, 16, (K, N)).astype(np.uint8)
    sw = rng.uniform(0.001, 0.1, (K // group, N)).astype(np.float16)
    zp = rng.integers(-128, 128, (K // group, N)).astype(np.int8)
    for z in (None, zp):
        y = w4a8.matmul(xq, sx, q, sw, z, group)
        for m in range(M):
            for n in range(N):
                exact = Fraction(0)
                for k in range(K):
                    zz = 8 if z is None else int(z[k // group, n])
                    exact += (Fraction(int(xq[m, k])) * Fraction(float(sx[m, k // 32]))
                              * (int(q[k, n]) - zz) * Fraction(float(sw[k // group, n])))
                assert abs(Fraction(float(y[m, n])) - exact) <= abs(exact) * Fraction(1, 2 ** 50) + Fraction(1, 2 ** 80)


def test_w4a8_product_is_the_product_of_the_dequantised_operands():
    """The integer-block form equals the FP64 product of the dequantised
    activations with the INT4 oracle's dequantised weight (both paths)."""
    rng = np.random.default_rng(24)
    X = rng.standard_normal((3, 256)).astype(np.float16).astype(np.float32)
    W = (rng.standard_normal((256, 40)) * 0.02).astype(np.float32)
    xq, sx = w4a8.quantize_activations(X)
    for group, mode in ((32, "sym"), (64, "asym"), (128, "asym")):
        q, s, zp = int4.quantize(W, group, mode)
        y = w4a8.matmul(xq, sx, q, s, zp if mode == "asym" else None, group)
        ref = matmul.matmul_f64(w4a8.dequant_activations(xq, sx), int4.dequant(q, s, group, zp))
        assert np.allclose(y, ref, rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------------------- MoE grouped GEMM

from oracle import moe  # noqa: E402


def test_moe_align_golden(golden):
    g = golden("moe_align_6x2.json")
    s, e, total = moe.align(np.array(g["topk_ids"]), g["num_experts"], g["block"])
    assert s.tolist() == g["sorted_ids"] and e.tolist() == g["expert_ids"] and total == g["total"]
    P = np.array(g["topk_ids"]).size
    assert moe.max_padded(P, g["num_experts"], g["block"]) == g["max_padded"]


def test_moe_align_invariants_and_bound():
    rng = np.random.default_rng(31)
    for T, top_k, E, block in ((1, 8, 256, 128), (37, 2, 8, 16), (300, 4, 16, 128), (5, 1, 3, 4)):
        ids = rng.integers(0, E, size=(T, top_k))
        s, e, total = moe.align(ids, E, block)
        P = T * top_k
        assert total % block == 0 and total <= moe.max_padded(P, E, block)
        valid = s[s < P]
        assert sorted(valid.tolist()) == list(range(P))          # every pair exactly once
        assert np.all(s[s >= P] == P)                            # padding carries the one id
        flat = ids.reshape(-1)
        for b in range(total // block):
            blk = s[b * block:(b + 1) * block]
            assert np.all(flat[blk[blk < P]] == e[b])            # one expert per block
            assert blk[0] < P                                    # no block is all padding
        assert np.all(np.diff(e) >= 0)                           # experts in ascending order
    # the bound is reached: every expert gets one pair
    s, e, total = moe.align(np.arange(8).reshape(8, 1), 8, 4)
    assert total == moe.max_padded(8, 8, 4) == 32


def _tiny_experts(rng, E, K, N):
    out = []
    for _ in range(E):
        idx = rng.integers(0, 8, size=(K, N), dtype=np.uint8)
        cb = rng.integers(0, 0x7F, size=(K // 64, N // 8, 8), dtype=np.uint8)   # finite E4M3 bytes
        ex = rng.integers(117, 128, size=(K // 64, N // 8), dtype=np.uint8)
        out.append((idx, cb, ex))
    return out


def test_moe_gathered_product_equals_the_routed_definition():
    """The aligned, gathered, padded form reproduces the pair-by-pair routing
    definition (an independent loop without sorting), also with a map that
    takes some experts off this rank."""
    rng = np.random.default_rng(32)
    T, top_k, E, K, N, block = 7, 3, 5, 64, 16, 4
    codes = rng.integers(0, 256, size=(T, K), dtype=np.uint8)
    codes[(codes & 0x7F) == 0x7F] -= 1
    scales = rng.integers(120, 130, size=(T, K // 32), dtype=np.uint8)
    ids = rng.integers(0, E, size=(T, top_k))
    experts = _tiny_experts(rng, E, K, N)
    s, e, total = moe.align(ids, E, block)
    Y = moe.grouped_matmul(codes, scales, top_k, s, e, total, block, experts)
    assert not np.any(np.isnan(Y))                              # every pair written
    assert np.array_equal(Y, moe.routed_matmul(codes, scales, ids, experts))
    emap = np.array([0, -1, 1, -1, 2])                           # experts 1 and 3 are remote
    local = [experts[0], experts[2], experts[4]]
    Ym = moe.grouped_matmul(codes, scales, top_k, s, e, total, block, local, emap)
    assert np.array_equal(Ym, moe.routed_matmul(codes, scales, ids, local, emap))
    remote = np.isin(ids.reshape(-1), [1, 3])
    assert np.all(Ym[remote] == 0) and np.array_equal(Ym[~remote], Y[~remote])
