"""Pins for the oracle's FP8 E4M3 codec and per-group quantizer (CPU only).

The codec is pinned to the format definition (fixed points from the specification, a brute
force nearest-value search, ties-to-even at every midpoint); the quantizer to the IEEE fp32
rounding of its scale (numpy float32 arithmetic) and to the half-spacing error bound.
"""
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _all_finite_codes():
    return np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)


def test_spec_points():
    for line in open(os.path.join(GOLDEN, "e4m3_spec_points.txt")):
        line = line.split("#")[0].strip()
        if not line:
            continue
        code, val = line.split()
        got = float(oracle.e4m3_decode(np.uint8(int(code, 16))))
        if val == "nan":
            assert math.isnan(got)
        else:
            assert got == float(val), (code, got, val)
            if val.startswith("-"):
                assert math.copysign(1.0, got) < 0


def test_decode_table_structure():
    codes = _all_finite_codes()
    assert len(codes) == 254
    vals = oracle.e4m3_decode(codes)
    pos = oracle.e4m3_decode(np.arange(0, 0x7F, dtype=np.uint8))
    # strictly increasing in the code for the positive half, sign bit mirrors
    assert np.all(np.diff(pos) > 0)
    neg = oracle.e4m3_decode(np.arange(0x80, 0xFF, dtype=np.uint8))
    assert np.array_equal(neg, -pos)
    assert vals.max() == 448.0 and vals.min() == -448.0
    # 3 mantissa bits: every positive normal value times 8 / 2^floor(log2 v) is an integer in [8, 16)
    for v in pos[8:]:
        e = math.floor(math.log2(v))
        m = v / 2.0 ** e * 8
        assert m == int(m) and 8 <= m < 16


def _brute_encode(x: float, table_codes, table_vals) -> int:
    """Nearest finite E4M3 value by exhaustive search; a tie goes to the even code; values beyond
    the largest finite magnitude saturate."""
    if x > 448.0:
        x = 448.0
    if x < -448.0:
        x = -448.0
    d = np.abs(table_vals - x)
    best = d.min()
    cands = [int(c) for c, dd in zip(table_codes, d) if dd == best]
    if len(cands) > 1:
        cands = [c for c in cands if c % 2 == 0] or cands
        # +0 / -0 tie: follow the sign of x
        if set(cands) == {0x00, 0x80}:
            return 0x80 if math.copysign(1.0, x) < 0 else 0x00
    if len(cands) == 2 and set(cands) == {0x00, 0x80}:
        return 0x80 if math.copysign(1.0, x) < 0 else 0x00
    return cands[0]


def test_encode_matches_exhaustive_search():
    codes = _all_finite_codes()
    vals = oracle.e4m3_decode(codes)
    rng = np.random.default_rng(123)
    xs = np.concatenate([
        rng.standard_normal(3000).astype(np.float32) * np.float32(50),
        rng.standard_normal(2000).astype(np.float32) * np.float32(0.01),
        rng.uniform(-500, 500, 1000).astype(np.float32),
    ])
    enc = oracle.e4m3_encode(xs)
    for x, c in zip(xs, enc):
        assert int(c) == _brute_encode(float(x), codes, vals), (x, c)


def test_round_trip_and_midpoints_ties_to_even():
    codes = np.arange(0, 0x7F, dtype=np.uint8)
    vals = oracle.e4m3_decode(codes)
    assert np.array_equal(oracle.e4m3_encode(vals.astype(np.float32)), codes)
    mids = ((vals[:-1] + vals[1:]) / 2).astype(np.float32)
    assert np.array_equal(mids.astype(np.float64), (vals[:-1] + vals[1:]) / 2)  # exact in fp32
    enc = oracle.e4m3_encode(mids).astype(int)
    lo, hi = codes[:-1].astype(int), codes[1:].astype(int)
    expect = np.where(lo % 2 == 0, lo, hi)
    assert np.array_equal(enc, expect)
    # negative side mirrors
    assert np.array_equal(oracle.e4m3_encode(-mids).astype(int), expect | 0x80)
    # saturation just above the largest finite value, and far above
    for x in (448.0 * (1 + 2 ** -10), 464.0, 479.0, 480.0, 1e6):
        assert int(oracle.e4m3_encode(np.float32(x))) == 0x7E
        assert int(oracle.e4m3_encode(np.float32(-x))) == 0xFE


def test_quantize_scale_rule_and_error_bound():
    rng = np.random.default_rng(7)
    x = rng.standard_normal((64, 128)).astype(np.float32)
    x[3] = 0.0
    x[5, :] = np.float32(1e-30)
    codes, scales = oracle.quantize_rows(x, 128)
    amax = np.abs(x).max(axis=1)
    with np.errstate(divide="ignore"):
        exp_scale = np.where(amax == 0, np.float32(1), amax / np.float32(448))
    assert np.array_equal(scales[:, 0], exp_scale.astype(np.float32))
    assert np.all(codes[3] == 0) and scales[3, 0] == 1.0
    # the amax element maps to the largest code magnitude
    for r in range(64):
        if amax[r] > 0:
            j = int(np.abs(x[r]).argmax())
            assert (int(codes[r, j]) & 0x7F) == 0x7E
    # dequantization error <= half the E4M3 spacing at the scaled value, times the scale
    deq = oracle.dequantize_rows(codes, scales, 128)
    with np.errstate(divide="ignore"):
        inv = np.where(amax == 0, 0, (np.float32(448) / amax).astype(np.float32))
    y = np.abs(x.astype(np.float64) * inv[:, None].astype(np.float64))
    spacing = np.where(y < 2.0 ** -6, 2.0 ** -9, 2.0 ** (np.floor(np.log2(np.maximum(y, 1e-300))) - 3))
    bound = 0.5 * spacing * scales[:, :1].astype(np.float64) * (1 + 1e-6) + 1e-45
    assert np.all(np.abs(deq - x) <= bound + np.abs(x) * 1e-6)


@pytest.mark.parametrize("amax", [1e-37, 1e-40, 2.0 ** -64, 2.0 ** -65, 2.0 ** -140])
def test_quantize_tiny_group_maximum(amax):
    """A group whose maximum is so small that 448 / amax overflows float32 (below about
    1.3e-36): no NaN or saturated code appears, the group's zeros stay code 0, its maximum
    takes the top code, and every value dequantizes within half a spacing (times the scale)."""
    amax = np.float32(amax)
    x = np.zeros((2, 32), dtype=np.float32)
    x[0, 3] = amax
    x[0, 9] = -amax / np.float32(2)
    x[0, 17] = amax * np.float32(0.3)
    x[1] = x[0] * np.float32(-1)
    codes, scales = oracle.quantize_rows(x, 32)
    assert not np.any((codes & 0x7F) == 0x7F)                 # no NaN code
    for r in range(2):
        zero = x[r] == 0
        assert np.all((codes[r][zero] & 0x7F) == 0)                # +0 or -0
        assert (int(codes[r, 3]) & 0x7F) == 0x7E                # the maximum -> 448
        assert int(codes[r, 9]) & 0x7F == 0x76                   # half of it -> 224 = 1.75 * 2^7
        assert scales[r, 0] == np.float32(np.float64(amax) / 448.0)
    deq = oracle.dequantize_rows(codes, scales, 32)
    # half the top binade's spacing (16) times the scale, plus what the stored scale lost by
    # rounding (it is subnormal, or 0, for the smallest maxima) times the largest code
    s_exact = np.float64(amax) / 448.0
    s = np.float64(scales[0, 0])
    assert np.all(np.abs(deq - x) <= 16 * s * (1 + 1e-6) + 448 * abs(s - s_exact) * (1 + 1e-6))


def test_quantize_lift_changes_no_code_where_the_reciprocal_is_finite():
    """Groups above and below the 2^-64 lift threshold but with a finite 448 / amax get exactly
    the codes of the same group scaled up by a power of two (the scale rule is homogeneous
    under exact power-of-two scaling)."""
    rng = np.random.default_rng(11)
    base = rng.standard_normal((16, 32)).astype(np.float32)
    c_ref, s_ref = oracle.quantize_rows(base, 32)
    for k in (-60, -64, -66, -90, -110):
        c, s = oracle.quantize_rows(base * np.float32(2.0 ** k), 32)
        assert np.array_equal(c, c_ref), k
        assert np.array_equal(s.astype(np.float64), s_ref.astype(np.float64) * 2.0 ** k), k


def test_group_32_variant_shares_scales_per_group():
    rng = np.random.default_rng(8)
    x = rng.standard_normal((4, 128)).astype(np.float32)
    x[:, 32:64] *= 100
    codes, scales = oracle.quantize_rows(x, 32)
    assert scales.shape == (4, 4)
    for g in range(4):
        sub_c, sub_s = oracle.quantize_rows(np.ascontiguousarray(x[:, 32 * g:32 * (g + 1)]), 32)
        assert np.array_equal(sub_c, codes[:, 32 * g:32 * (g + 1)])
        assert np.array_equal(sub_s[:, 0], scales[:, g])


def test_pages_quantization_table_and_storage_claim():
    rows = {}
    claim = None
    for line in open(os.path.join(GOLDEN, "tiered_quantization.txt")):
        line = line.split("#")[0].strip()
        if not line:
            continue
        parts = line.split()
        if parts[0] == "index_storage_ratio_claim":
            claim = float(parts[1])
        else:
            rows[parts[0]] = (parts[1], int(parts[2]))
    assert rows["index_qk"] == ("fp8", 32) and rows["kv_cache"] == ("fp8", 128)
    # FP8 key of 128 dims: one byte per element plus the fp32 scales, against two bytes per
    # element in bf16.  Per-key scale (this build's index cache) and group-32 scales both land
    # near the pages' "about half".
    D = 128
    for group in (D, rows["index_qk"][1]):
        ratio = (D + 4 * (D // group)) / (2 * D)
        assert abs(ratio - claim) < 0.07, ratio


# ------------------------------------------------------------------------------ MXFP8 blocks
def _golden_mx_blocks():
    blocks = {}
    for line in open(os.path.join(GOLDEN, "mxfp8_blocks.txt")):
        line = line.split("#")[0].strip()
        if not line:
            continue
        name, E, i, x, code = line.split()
        if x.lstrip("-").startswith("2^"):
            v = math.ldexp(1.0, int(x.lstrip("-")[2:])) * (-1.0 if x.startswith("-") else 1.0)
        else:
            v = float(x)
        b = blocks.setdefault(name, {"E": int(E), "x": np.zeros(32), "code": np.zeros(32, np.uint8)})
        assert b["E"] == int(E)
        b["x"][int(i)] = v
        b["code"][int(i)] = int(code, 16)
    return blocks


def test_mx_golden_blocks():
    """Blocks worked by hand from the MX definition, one per case: plain rounding, ties to even
    at subnormal and normal midpoints, saturation, a negative shared exponent, an all-zero
    block, the lower clamp of the shared exponent and a block near the float32 maximum."""
    blocks = _golden_mx_blocks()
    assert len(blocks) == 6
    x = np.stack([b["x"] for b in blocks.values()]).astype(np.float32)
    assert np.array_equal(x.astype(np.float64), np.stack([b["x"] for b in blocks.values()]))
    codes, scales = oracle.mx_quantize_rows(x)
    for r, (name, b) in enumerate(blocks.items()):
        assert scales[r, 0] == b["E"], name
        assert np.array_equal(codes[r], b["code"]), (name, codes[r], b["code"])


def _mx_data(n, D, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((n, D)) * np.exp2(rng.integers(-20, 20, (n, 1)))
    x[0, :32] = 0.0                                   # an all-zero block
    x[1, 32:64] *= 1e-30                              # a block near the bottom of float32
    return x.astype(np.float32)


def test_mx_scale_rule_and_error_bound():
    """For every block: the block maximum lies in [256, 512) after the division by 2^X (the top
    E4M3 binade and the range above it that saturates to 448), its code decodes into
    [256, 448], and every element is within half an E4M3 spacing of x / 2^X, or saturated at
    +-448 when it rounds past it."""
    x = _mx_data(64, 128, 5)
    codes, scales = oracle.mx_quantize_rows(x)
    deq = oracle.mx_dequantize_rows(codes, scales)
    for r in range(x.shape[0]):
        for blk in range(4):
            xs = x[r, 32 * blk:32 * blk + 32].astype(np.float64)
            E = int(scales[r, blk])
            amax = np.abs(xs).max()
            if amax == 0:
                assert E == 0 and not codes[r, 32 * blk:32 * blk + 32].any()
                continue
            X = E - 127
            y = xs / 2.0 ** X
            top = np.abs(oracle.e4m3_decode(codes[r, 32 * blk + np.argmax(np.abs(xs))]))
            if X > -127:
                assert 256 <= np.abs(y).max() < 512 and 256 <= top <= 448
            else:
                assert np.abs(y).max() < 512
            d = deq[r, 32 * blk:32 * blk + 32] / 2.0 ** X
            for yi, di in zip(y, d):
                a = abs(yi)
                if a >= 2.0 ** -6:
                    spacing = 2.0 ** (math.floor(math.log2(a)) - 3)
                else:
                    spacing = 2.0 ** -9
                assert abs(di - yi) <= spacing / 2 or (abs(di) == 448 and a > 448), (r, blk, yi, di)


def test_mx_power_of_two_rescaling_moves_only_the_scale():
    """Multiplying a block by 2^k leaves its codes unchanged and adds k to the scale byte (away
    from the exponent clamps): the shared exponent carries the whole magnitude."""
    x = _mx_data(32, 64, 6)[2:]
    c0, s0 = oracle.mx_quantize_rows(x)
    for k in (-9, -1, 1, 13):
        c1, s1 = oracle.mx_quantize_rows(x * np.float32(2.0 ** k))
        assert np.array_equal(c0, c1)
        assert np.array_equal(s0.astype(int) + k, s1.astype(int))


def test_mx_values_on_the_grid_are_fixed_points():
    """A block whose values already are E4M3 codes times 2^X, with one code in the top binade,
    quantizes back to exactly those codes and E = X + 127."""
    rng = np.random.default_rng(7)
    finite = _all_finite_codes()
    top = finite[(oracle.e4m3_decode(finite) >= 256)]
    for X in (-30, -8, 0, 17):
        codes = rng.choice(finite, (8, 32))
        codes[:, 5] = rng.choice(top, 8)
        vals = oracle.e4m3_decode(codes) * 2.0 ** X
        got_c, got_s = oracle.mx_quantize_rows(vals.astype(np.float32))
        assert np.all(got_s == X + 127)
        same = oracle.e4m3_decode(got_c) == oracle.e4m3_decode(codes)   # +0 and -0 both decode to 0
        assert same.all()
        assert np.array_equal(oracle.mx_dequantize_rows(got_c, got_s), vals)


def test_mx_rejects_non_finite_input():
    x = np.zeros((1, 32), dtype=np.float32)
    x[0, 3] = np.inf
    with pytest.raises(oracle.OracleError):
        oracle.mx_quantize_rows(x)
