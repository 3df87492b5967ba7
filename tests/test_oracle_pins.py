"""Pins of the CPU oracle against facts that do not come from the oracle itself.

What each group of tests ties the oracle to:
  * E4M3 codec -- brute force over all 256 codes; an independent nearest-value
    encoder (sorted-table search, ties to the even code) over every finite bf16 value
    scaled by every power of two the MX rule can apply; the library casts of torch
    and ml_dtypes inside the range where those casts are defined the same way; and
    hand-picked special values.
  * bf16 rounding -- torch's float32 -> bfloat16 cast (RNE) on random and edge bit
    patterns, subnormals included.
  * E8M0 scale byte -- the closed form max(biased_exponent(amax) - 8, 0) read from the
    bf16 bits, for all 32768 non-negative finite bf16 values.
  * MX blocks and per-group columns -- hand-worked fixtures under tests/golden/,
    brute-force Python implementations on tiny inputs, round-trip error bounds,
    idempotence, and layout invariants (transposes, dual-axis == two single calls).
  * Group bounds -- the clamp rule against its closed form (running maximum).
"""
import json
import math
import os

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle
from mxfp8_quantization_moe_mx_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _hex(s):
    return float.fromhex(s)


def _bf16_bits_of(values):
    """bf16 bit patterns of values that are exactly representable in bf16."""
    f = np.asarray(values, dtype=np.float64).astype(np.float32)
    assert np.all(f.astype(np.float64) == np.asarray(values, dtype=np.float64))
    u = f.view(np.uint32)
    assert np.all((u & 0xFFFF) == 0), "value not exactly representable in bf16"
    return (u >> 16).astype(np.uint16)


# ---------------------------------------------------------------------------------------
# Independent brute-force E4M3 encoder: nearest of the 127 non-negative finite values,
# ties to the even code.  Saturation is not special-cased: above 448 the nearest finite
# value simply is 448.
# ---------------------------------------------------------------------------------------

def _e4m3_positive_table():
    vals = []
    for code in range(0x7F):  # 0x00 .. 0x7E
        E, m = code >> 3, code & 7
        vals.append(m * 2.0 ** -9 if E == 0 else (1 + m / 8) * 2.0 ** (E - 7))
    return np.array(vals, dtype=np.float64)


_TABLE = _e4m3_positive_table()


def brute_encode(v):
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    hi = np.clip(np.searchsorted(_TABLE, a, side="left"), 0, len(_TABLE) - 1)
    lo = np.clip(hi - 1, 0, len(_TABLE) - 1)
    d_lo = np.abs(a - _TABLE[lo])
    d_hi = np.abs(_TABLE[hi] - a)
    pick = np.where(d_lo < d_hi, lo, hi)
    tie = d_lo == d_hi
    pick = np.where(tie, np.where(lo % 2 == 0, lo, hi), pick)
    sign = np.where(np.signbit(v), 0x80, 0)
    return (pick | sign).astype(np.uint8)


def test_table_is_monotone_and_has_254_finite_codes():
    assert np.all(np.diff(_TABLE) > 0)
    dec = oracle.e4m3_decode(np.arange(256))
    assert np.sum(np.isnan(dec)) == 2
    assert np.isnan(dec[0x7F]) and np.isnan(dec[0xFF])
    np.testing.assert_array_equal(dec[:0x7F], _TABLE)
    np.testing.assert_array_equal(dec[0x80:0xFF], -_TABLE)
    assert math.copysign(1.0, dec[0x80]) == -1.0


def test_decode_matches_torch_and_ml_dtypes():
    codes = np.arange(256, dtype=np.uint8)
    dec = oracle.e4m3_decode(codes)
    t = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    m = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    for ref in (t, m):
        assert np.array_equal(np.isnan(dec), np.isnan(ref))
        ok = ~np.isnan(dec)
        np.testing.assert_array_equal(dec[ok], ref[ok])
        np.testing.assert_array_equal(np.signbit(dec[ok]), np.signbit(ref[ok]))


def test_encode_decode_roundtrip_all_codes():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    assert codes.size == 254
    np.testing.assert_array_equal(oracle.e4m3_encode(oracle.e4m3_decode(codes)), codes)


def test_encode_midpoints_and_neighbours():
    mids, below, above, lo_code, hi_code = [], [], [], [], []
    for c in range(0x7E):
        a, b = _TABLE[c], _TABLE[c + 1]
        mid = (a + b) / 2
        mids.append(mid)
        below.append(np.nextafter(np.float32(mid), np.float32(0)))
        above.append(np.nextafter(np.float32(mid), np.float32(1e9)))
        lo_code.append(c)
        hi_code.append(c + 1)
    mids = np.array(mids)
    even = np.where(np.array(lo_code) % 2 == 0, lo_code, hi_code)
    np.testing.assert_array_equal(oracle.e4m3_encode(mids), even)
    np.testing.assert_array_equal(oracle.e4m3_encode(-mids), np.array(even) | 0x80)
    np.testing.assert_array_equal(oracle.e4m3_encode(np.array(below, np.float64)), lo_code)
    np.testing.assert_array_equal(oracle.e4m3_encode(np.array(above, np.float64)), hi_code)


@pytest.mark.parametrize("value,code", [
    (448.0, 0x7E), (449.0, 0x7E), (464.0, 0x7E), (1e6, 0x7E), (math.inf, 0x7E),
    (-464.0, 0xFE), (-math.inf, 0xFE), (2.0 ** -9, 0x01), (2.0 ** -10, 0x00),
    (1.5 * 2.0 ** -10, 0x01), (2.0 ** -6, 0x08), (-0.0, 0x80), (0.0, 0x00),
    (-1e-30, 0x80), (1.0, 0x38), (432.0, 0x7E), (416.0, 0x7D), (400.0, 0x7C),
])
def test_encode_special_values(value, code):
    assert int(oracle.e4m3_encode(np.array([value]))[0]) == code


def test_encode_nan_gives_nan_code():
    out = oracle.e4m3_encode(np.array([math.nan, -math.nan]))
    assert (out[0] & 0x7F) == 0x7F and (out[1] & 0x7F) == 0x7F


def test_encode_all_bf16_times_all_scales_vs_brute_force():
    """Every finite bf16 value times 2^-e for every e the MX rule can produce; these
    are exactly the exact products the MX quantizer hands to the encoder."""
    bits = np.arange(0x10000, dtype=np.uint32)
    with np.errstate(invalid="ignore"):
        vals = (bits << 16).view(np.float32).astype(np.float64)
    vals = vals[np.isfinite(vals)]
    for e in range(-127, 128):
        v = np.ldexp(vals, -e)
        np.testing.assert_array_equal(oracle.e4m3_encode(v), brute_encode(v), err_msg=f"e={e}")


def test_encode_random_fp32_vs_brute_force_and_torch():
    rng = np.random.default_rng(7)
    u = rng.integers(0, 2 ** 32, size=2_000_000, dtype=np.uint64).astype(np.uint32)
    f = u.view(np.float32)
    f = f[np.isfinite(f)]
    # fold most of them into the interesting range
    g = (f.astype(np.float64) % 600.0).astype(np.float32)
    for arr in (f, g):
        got = oracle.e4m3_encode_f32(arr)
        np.testing.assert_array_equal(got, brute_encode(arr.astype(np.float64)))
    inrange = g[np.abs(g) < 464.0]
    ref = torch.from_numpy(inrange).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(oracle.e4m3_encode_f32(inrange), ref)
    ref2 = inrange.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    np.testing.assert_array_equal(oracle.e4m3_encode_f32(inrange), ref2)


# ---- bf16 rounding ---------------------------------------------------------------------

def test_double_to_bf16_matches_torch_cast_on_fp32_inputs():
    rng = np.random.default_rng(11)
    u = rng.integers(0, 2 ** 32, size=3_000_000, dtype=np.uint64).astype(np.uint32)
    edge = np.array([0x00000001, 0x00007FFF, 0x00008000, 0x00018000, 0x007FFFFF, 0x00800000,
                     0x7F7F7FFF, 0x7F7F8000, 0x7F7FFFFF, 0x7F800000, 0x80000001,
                     0x3F808000, 0x3F818000, 0xFF7FFFFF], dtype=np.uint32)
    u = np.concatenate([u, edge, np.arange(0, 0x20000, dtype=np.uint32)])
    f = u.view(np.float32)
    f = f[~np.isnan(f)]
    got = oracle.double_to_bf16(f.astype(np.float64))
    ref = torch.from_numpy(f.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(got, ref)


def test_bf16_widening_is_exact():
    bits = np.arange(0x10000, dtype=np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).double().numpy()
    got = oracle.bf16_to_double(bits)
    same = (got == ref) | (np.isnan(got) & np.isnan(ref))
    assert np.all(same)


# ---- E8M0 ----------------------------------------------------------------------------------

def test_scale_byte_closed_form_all_bf16():
    bits = np.arange(0, 0x7F80, dtype=np.uint16)  # every non-negative finite bf16
    vals = oracle.bf16_to_double(bits)
    got = np.array([oracle.mx_scale_byte(v) for v in vals])
    biased = (bits.astype(np.int64) >> 7) & 0xFF
    closed = np.maximum(biased - 8, 0)
    np.testing.assert_array_equal(got, closed)
    assert oracle.mx_scale_byte(math.inf) == 0xFF and oracle.mx_scale_byte(math.nan) == 0xFF


def test_floor_log2_by_halving():
    rng = np.random.default_rng(3)
    for a in np.concatenate([rng.lognormal(0, 30, 2000), [2.0 ** -140, 1.0, 448.0, 2.0 ** 127]]):
        p = 0
        x = float(a)
        while x >= 2.0:
            x /= 2.0
            p += 1
        while x < 1.0:
            x *= 2.0
            p -= 1
        assert oracle.floor_log2(a) == p


def test_e8m0_decode_matches_torch():
    ref = torch.arange(256, dtype=torch.uint8).view(torch.float8_e8m0fnu).double().numpy()
    for b in range(256):
        got = oracle.e8m0_decode(b)
        assert (math.isnan(got) and math.isnan(ref[b])) or got == ref[b]


# ---- hand-worked blocks ----------------------------------------------------------------------

def _expand(spec_fill, spec_set, conv):
    out = [conv(spec_fill)] * 32
    for k, v in spec_set.items():
        out[int(k)] = conv(v)
    return out


def test_golden_mx_blocks_row_and_column():
    data = json.load(open(os.path.join(GOLDEN, "mx_hand_worked.json")))
    for blk in data["blocks"]:
        x = _expand(blk["fill"], blk["set"], _hex)
        codes = _expand(blk["code_fill"], blk["code_set"], int)
        deq = _expand(blk["deq_fill"], blk["deq_set"], _hex)
        bits = _bf16_bits_of(x)
        # one 1x32 row block
        r = oracle.mx_quantize(bits.reshape(1, 32).repeat(32, 0), oracle.ROW)
        assert int(r["s_row"][0, 0]) == blk["scale_byte"], blk["name"]
        np.testing.assert_array_equal(r["q_row"][0], codes, err_msg=blk["name"])
        y = oracle.mx_dequantize(r["q_row"], r["s_row"], 1, 32, 32, oracle.ROW)
        yv = oracle.bf16_to_double(y[0])
        np.testing.assert_array_equal(yv, deq, err_msg=blk["name"])
        np.testing.assert_array_equal(np.signbit(yv), np.signbit(deq), err_msg=blk["name"])
        # the same block as a 32x1 column block
        c = oracle.mx_quantize(bits.reshape(32, 1).repeat(32, 1), oracle.COL)
        assert int(c["s_col"][0, 0]) == blk["scale_byte"], blk["name"]
        np.testing.assert_array_equal(c["q_col"][0], codes, err_msg=blk["name"])
        yc = oracle.mx_dequantize(c["q_col"], c["s_col"], 1, 32, 32, oracle.COL)
        np.testing.assert_array_equal(oracle.bf16_to_double(yc[:, 0]), deq, err_msg=blk["name"])


def test_golden_per_group():
    d = json.load(open(os.path.join(GOLDEN, "per_group_hand_worked.json")))
    M, K = d["M"], d["K"]
    x = np.array([[_hex(v) for v in row] for row in d["x"]])
    bits = _bf16_bits_of(x.ravel()).reshape(M, K)
    q, s = oracle.per_group_quant(bits, d["offs"], oracle.ROW_MAJOR, q_init=np.full((M, K), 0xA5))
    for key, val in d["scale_exact"].items():
        g, k = map(int, key.split(","))
        assert s[g, k] == np.float32(_hex(val))
    for key, code in d["codes_row_major"].items():
        m, k = map(int, key.split(","))
        assert int(q[m, k]) == code, key
    # all-zero column of group 0 and the empty group: 448 / fl32(1e-12), within 1 ulp of 4.48e14
    for g, k in ((0, 1), (1, 0), (1, 1)):
        assert abs(float(s[g, k]) - 4.48e14) <= float(np.spacing(np.float32(4.48e14)))
    np.testing.assert_array_equal(q[6], [0xA5, 0xA5])  # row in no group: untouched


# ---- brute-force implementations on tiny inputs -----------------------------------------------

def _brute_mx_block(vals):
    """Block scale and codes by a Python loop: scale exponent found by halving."""
    amax = max(abs(v) for v in vals)
    if amax == 0:
        e = -127
    else:
        p, x = 0, amax
        while x >= 2.0:
            x /= 2.0
            p += 1
        while x < 1.0:
            x *= 2.0
            p -= 1
        e = min(max(p - 8, -127), 127)
    codes = brute_encode(np.array([math.ldexp(v, -e) for v in vals]))
    return e + 127, codes


def test_mx_quantize_vs_brute_force_tiny():
    t = workloads.tiny(rows=64, cols=96)
    bits = workloads.bf16_bits(t["x"])
    vals = oracle.bf16_to_double(bits)
    r = oracle.mx_quantize(bits, oracle.ROW | oracle.COL)
    for i in range(64):
        for j in range(3):
            b, codes = _brute_mx_block(list(vals[i, 32 * j:32 * j + 32]))
            assert r["s_row"][i, j] == b
            np.testing.assert_array_equal(r["q_row"][i, 32 * j:32 * j + 32], codes)
    for c in range(96):
        for i in range(2):
            b, codes = _brute_mx_block(list(vals[32 * i:32 * i + 32, c]))
            assert r["s_col"][c, i] == b
            np.testing.assert_array_equal(r["q_col"][c, 32 * i:32 * i + 32], codes)


def test_mx_dequantize_vs_brute_force_tiny():
    rng = np.random.default_rng(5)
    q = rng.integers(0, 256, size=(32, 64), dtype=np.uint8)
    s = rng.integers(0, 255, size=(32, 2), dtype=np.uint8)
    s[0, 0], s[1, 1], s[2, 0] = 0, 254, 1
    y = oracle.mx_dequantize(q, s, 1, 32, 64, oracle.ROW)
    tbl = np.concatenate([_TABLE, [np.nan], -_TABLE, [np.nan]])
    for r in range(32):
        for c in range(64):
            v = tbl[q[r, c]] * 2.0 ** (int(s[r, c // 32]) - 127)
            ref = torch.tensor(v, dtype=torch.float64).to(torch.bfloat16)
            if math.isnan(v):
                assert y[r, c] == 0x7FC0
            else:
                # v has at most 4 significant bits, so torch's double -> float -> bf16
                # cast rounds it only once (float overflow gives inf, as bf16 RNE does)
                assert int(ref.view(torch.int16).item()) & 0xFFFF == y[r, c]


def _brute_per_group(vals, offs, M, K):
    prev = 0
    scales = np.zeros((len(offs), K), np.float32)
    q = np.zeros((M, K), np.uint8)
    for g, o in enumerate(offs):
        end = min(max(o, prev), M)
        for k in range(K):
            amax = 0.0
            for m in range(prev, end):
                amax = max(amax, abs(vals[m, k]))
            s = np.float32(448.0) / np.maximum(np.float32(amax), np.float32(1e-12))
            scales[g, k] = s
            for m in range(prev, end):
                q[m, k] = brute_encode(np.array([np.float32(vals[m, k]) * s], np.float64))[0]
        prev = end
    return q, scales


def test_per_group_vs_brute_force_tiny():
    t = workloads.tiny(rows=48, cols=16)
    bits = workloads.bf16_bits(t["x"])
    vals = oracle.bf16_to_double(bits)
    for offs in ([5, 5, 30, 48], [0, 48], [48], [10, 7, 60], [-3, 12, 12, 40]):
        q, s = oracle.per_group_quant(bits, offs, oracle.ROW_MAJOR)
        qb, sb = _brute_per_group(vals, offs, 48, 16)
        np.testing.assert_array_equal(s, sb)
        np.testing.assert_array_equal(q, qb)


# ---- bounds, invariants, layouts -------------------------------------------------------------

def test_mx_roundtrip_error_bounds_and_idempotence():
    t = workloads.tiny()
    bits = workloads.bf16_bits(t["x"])
    x = oracle.bf16_to_double(bits)
    r = oracle.mx_quantize(bits, oracle.ROW)
    y = oracle.bf16_to_double(oracle.mx_dequantize(r["q_row"], r["s_row"], 1, 256, 512))
    e = r["s_row"].astype(np.int64).repeat(32, axis=1) - 127
    scaled = np.abs(np.ldexp(x, -e))
    err = np.abs(y - x)
    normal = (scaled >= 2.0 ** -6) & (scaled <= 448)
    assert np.all(err[normal] <= np.abs(x[normal]) * 2.0 ** -4)
    sat = scaled > 448
    assert np.all(err[sat] <= np.abs(x[sat]) * 64 / 448)
    small = scaled < 2.0 ** -6
    assert np.all(err[small] <= np.ldexp(2.0 ** -10, e[small]))
    # idempotence
    ybits = oracle.mx_dequantize(r["q_row"], r["s_row"], 1, 256, 512)
    r2 = oracle.mx_quantize(ybits, oracle.ROW)
    y2 = oracle.mx_dequantize(r2["q_row"], r2["s_row"], 1, 256, 512)
    np.testing.assert_array_equal(y2, ybits)


def test_mx_col_equals_row_of_transpose_and_dual_equals_single():
    t = workloads.tiny()
    bits = workloads.bf16_bits(t["x"])
    d = oracle.mx_quantize(bits, oracle.ROW | oracle.COL)
    rr = oracle.mx_quantize(bits, oracle.ROW)
    cc = oracle.mx_quantize(bits, oracle.COL)
    tt = oracle.mx_quantize(np.ascontiguousarray(bits.T), oracle.ROW)
    np.testing.assert_array_equal(d["q_row"], rr["q_row"])
    np.testing.assert_array_equal(d["s_row"], rr["s_row"])
    np.testing.assert_array_equal(d["q_col"], cc["q_col"])
    np.testing.assert_array_equal(d["s_col"], cc["s_col"])
    np.testing.assert_array_equal(cc["q_col"], tt["q_row"])
    np.testing.assert_array_equal(cc["s_col"], tt["s_row"])
    # batched == per-matrix
    b3 = np.stack([bits[:128], bits[128:]])
    bb = oracle.mx_quantize(b3, oracle.ROW | oracle.COL)
    for e in range(2):
        one = oracle.mx_quantize(np.ascontiguousarray(b3[e]), oracle.ROW | oracle.COL)
        for k in one:
            np.testing.assert_array_equal(bb[k][e], one[k])
    # column dequant of the column layout == row dequant of the transpose, transposed
    yc = oracle.mx_dequantize(cc["q_col"], cc["s_col"], 1, 256, 512, oracle.COL)
    yt = oracle.mx_dequantize(tt["q_row"], tt["s_row"], 1, 512, 256, oracle.ROW)
    np.testing.assert_array_equal(yc, yt.T)


def test_per_group_layouts_and_amax_maps_to_448():
    t = workloads.tiny()
    bits = workloads.bf16_bits(t["x"])
    offs = t["offs"].numpy()
    qr, sr = oracle.per_group_quant(bits, offs, oracle.ROW_MAJOR)
    qc, sc = oracle.per_group_quant(bits, offs, oracle.COL_MAJOR)
    np.testing.assert_array_equal(qc, qr.T)
    np.testing.assert_array_equal(sc, sr)
    x = oracle.bf16_to_double(bits)
    start, end = oracle.group_bounds(offs, 256)
    dec = oracle.e4m3_decode(qr)
    for g in range(len(offs)):
        if end[g] == start[g]:
            continue
        blk = x[start[g]:end[g]]
        amax = np.abs(blk).max(axis=0)
        arg = np.abs(blk).argmax(axis=0)
        for k in range(512):
            if amax[k] >= 1e-12:
                assert abs(dec[start[g] + arg[k], k]) == 448.0
        # dequantized error within half an E4M3 step of x*s (plus fp32 rounding)
        s = sr[g].astype(np.float64)
        xs = blk * s
        step = np.where(np.abs(xs) < 2.0 ** -6, 2.0 ** -9,
                        2.0 ** (np.floor(np.log2(np.maximum(np.abs(xs), 2.0 ** -6))) - 3))
        assert np.all(np.abs(dec[start[g]:end[g]] - xs) <= step / 2 + np.abs(xs) * 2.0 ** -23)


@pytest.mark.parametrize("offs,M", [
    ([3, 3, 9, 16], 16), ([16], 16), ([0, 0, 0], 16), ([20, 5, 40], 16),
    ([-4, 2, 1, 14], 16), ([7, 3, 10], 16), ([2 ** 31 - 1], 16), ([], 16),
])
def test_group_bounds_clamp_rule_closed_form(offs, M):
    start, end = oracle.group_bounds(np.array(offs, np.int32), M)
    running = 0
    for g, o in enumerate(offs):
        closed_end = min(M, max([0] + list(offs[:g + 1])))
        assert end[g] == closed_end
        assert start[g] == running
        assert start[g] <= end[g] <= M
        running = end[g]


# ---- exact rational checks of the fp32 scale rule ----------------------------------------------

def _f32_round(fr):
    """Round a non-negative Fraction to the nearest float32, ties to even (normal range)."""
    from fractions import Fraction
    if fr == 0:
        return 0.0
    e = fr.numerator.bit_length() - fr.denominator.bit_length()
    if Fraction(2) ** e > fr:
        e -= 1
    while Fraction(2) ** (e + 1) <= fr:
        e += 1
    quantum = Fraction(2) ** (e - 23)
    n = fr / quantum
    fl = n.numerator // n.denominator
    rem = n - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return float(fl * quantum)


def test_per_group_scale_is_correctly_rounded_quotient():
    from fractions import Fraction
    t = workloads.tiny(rows=64, cols=64)
    bits = workloads.bf16_bits(t["x"])
    bits[:, 5] = 0            # an all-zero feature
    bits[:, 6] = 0x0001       # a feature whose amax is below 1e-12
    offs = [20, 20, 64]
    _, s = oracle.per_group_quant(bits, offs, oracle.ROW_MAJOR)
    x = oracle.bf16_to_double(bits)
    eps = Fraction(float(np.float32(1e-12)))
    # the fp32 nearest to 1e-12, found by exact comparison of neighbours
    t12 = Fraction(1, 10 ** 12)
    for c in (np.nextafter(np.float32(1e-12), np.float32(0)),
              np.nextafter(np.float32(1e-12), np.float32(1))):
        assert abs(Fraction(float(c)) - t12) > abs(eps - t12)
    start, end = oracle.group_bounds(offs, 64)
    for g in range(3):
        for k in range(64):
            amax = Fraction(float(np.abs(x[start[g]:end[g], k]).max())) if end[g] > start[g] else Fraction(0)
            want = _f32_round(Fraction(448) / max(amax, eps))
            assert float(s[g, k]) == want, (g, k)
    assert float(s[1, 0]) == float.fromhex("0x1.97742p+48")   # empty group: 448 / fl32(1e-12)


def test_nonfinite_block_reading():
    """A block holding Inf or NaN gets the NaN scale 0xFF and NaN codes with each
    element's sign; dequantizing a NaN scale or a NaN code gives the bf16 NaN 0x7FC0."""
    bits = np.full((32, 32), 0x3F80, np.uint16)       # 1.0
    bits[0, 3] = 0x7F80                               # +inf in row block 0
    bits[1, 0] = 0xBF80                               # -1.0 next to a NaN
    bits[1, 9] = 0x7FC1                               # NaN in row block 1
    r = oracle.mx_quantize(bits, oracle.ROW)
    assert r["s_row"][0, 0] == 0xFF and r["s_row"][1, 0] == 0xFF and r["s_row"][2, 0] == 119
    np.testing.assert_array_equal(r["q_row"][0], 0x7F)
    assert r["q_row"][1, 0] == 0xFF and r["q_row"][1, 1] == 0x7F
    y = oracle.mx_dequantize(r["q_row"], r["s_row"], 1, 32, 32, oracle.ROW)
    np.testing.assert_array_equal(y[0:2], 0x7FC0)
    q = np.zeros((32, 32), np.uint8)
    q[0, 0], q[0, 1] = 0x7F, 0xFF
    s = np.full((32, 1), 127, np.uint8)
    y = oracle.mx_dequantize(q, s, 1, 32, 32, oracle.ROW)
    assert y[0, 0] == 0x7FC0 and y[0, 1] == 0x7FC0 and y[0, 2] == 0


# ---- layouts for the scaled grouped GEMM --------------------------------------------------

def test_transpose_matches_numpy_and_inverts():
    """The byte transpose reduces to numpy's transpose; applying it twice is the
    identity; a batch is transposed matrix by matrix."""
    rng = np.random.default_rng(11)
    for shape in [(1, 1), (3, 7), (64, 48), (33, 129), (2, 17, 5)]:
        x = rng.integers(0, 256, shape, dtype=np.uint8)
        t = oracle.transpose_u8(x)
        np.testing.assert_array_equal(t, np.swapaxes(x, -1, -2))
        np.testing.assert_array_equal(oracle.transpose_u8(t), x)


def _blocked_by_reshape(s2d: np.ndarray) -> np.ndarray:
    """The 128 x 4 tile layout written as a reshape/permute of the zero-padded scale
    matrix (an independent formulation of the oracle's index map): padded row p =
    128 t + 32 a + l and scale column k = 4 j + c go to tile (t, j), byte 16 l + 4 a + c."""
    r, k = s2d.shape
    R, Kp = -(-r // 128) * 128, -(-k // 4) * 4
    p = np.zeros((R, Kp), np.uint8)
    p[:r, :k] = s2d
    v = p.reshape(R // 128, 4, 32, Kp // 4, 4)          # t, a, l, j, c
    return v.transpose(0, 3, 2, 1, 4).reshape(-1)        # t, j, l, a, c


def test_blocked_layout_equals_reshape_formulation():
    rng = np.random.default_rng(12)
    for rows, nk in [(1, 1), (128, 4), (130, 5), (300, 160), (512, 3)]:
        s = rng.integers(0, 256, (rows, nk), dtype=np.uint8)
        np.testing.assert_array_equal(oracle.mx_scales_to_blocked(s), _blocked_by_reshape(s))
    # batched: matrices one after another, each padded on its own
    s = rng.integers(0, 256, (3, 200, 6), dtype=np.uint8)
    ref = np.concatenate([_blocked_by_reshape(s[b]) for b in range(3)])
    np.testing.assert_array_equal(oracle.mx_scales_to_blocked(s), ref)


def test_blocked_layout_per_group_padding():
    """With group offsets every group's rows start a fresh 128-row tile (the clamp rule
    decides the groups); the used part equals the per-group reshape formulation and
    the rest of the capacity keeps its fill."""
    rng = np.random.default_rng(13)
    rows, nk = 700, 10
    s = rng.integers(1, 256, (rows, nk), dtype=np.uint8)
    for offs in ([100, 100, 356, 700], [0, 129, 600], [650, 640, 900], [700]):
        start, end = oracle.group_bounds(offs, rows)
        ref = np.concatenate([_blocked_by_reshape(s[a:b]) if b > a else np.zeros(0, np.uint8)
                              for a, b in zip(start, end)])
        got = oracle.mx_scales_to_blocked(s, offs, fill=0xEE)
        assert got.size == oracle.mx_scales_blocked_bytes(1, rows, nk, len(offs)) >= ref.size
        np.testing.assert_array_equal(got[:ref.size], ref)
        assert np.all(got[ref.size:] == 0xEE)


def test_blocked_layout_is_a_permutation_of_the_padded_scales():
    """Every scale byte appears exactly once and every other used byte is padding."""
    rows, nk = 257, 7
    s = (np.arange(rows * nk) % 251 + 1).astype(np.uint8).reshape(rows, nk)
    got = oracle.mx_scales_to_blocked(s)
    assert np.count_nonzero(got) == rows * nk
    assert np.array_equal(np.sort(got[got != 0]), np.sort(s.reshape(-1)))


# ---- MXFP8 grouped GEMM -----------------------------------------------------------------------

def _decode_e4m3_torch(codes: np.ndarray) -> np.ndarray:
    """E4M3 decode by torch's float8_e4m3fn (independent of the oracle's decoder)."""
    t = torch.from_numpy(np.ascontiguousarray(codes, np.uint8)).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def _gemm_reference(qa, sa, qb, sb, offs):
    """The grouped product from torch's E4M3 decode, ldexp scales and numpy matmul."""
    M, K = qa.shape
    a = _decode_e4m3_torch(qa) * np.ldexp(1.0, np.repeat(sa.astype(np.int64) - 127, 32, axis=1))
    b = _decode_e4m3_torch(qb) * np.ldexp(1.0, np.repeat(sb.astype(np.int64) - 127, 32, axis=2))
    out = np.full((M, qb.shape[1]), np.nan)
    start, end = oracle.group_bounds(offs, M)
    for g, (s0, e0) in enumerate(zip(start, end)):
        out[s0:e0] = a[s0:e0] @ b[g].T
    return out


def test_grouped_gemm_exact_on_integer_operands():
    """Codes whose values are small integers and unit scales: every partial sum is an
    exact integer, so the oracle must equal numpy's matmul of torch-decoded operands
    bit for bit (a dropped term, a wrong expert or a transposed operand changes it)."""
    rng = np.random.default_rng(21)
    ints = np.array([0x00, 0x38, 0x40, 0x44, 0x48, 0x4A, 0x4C, 0x4E, 0x50, 0xB8, 0xC0, 0xC8, 0xD0], np.uint8)
    M, N, K, G = 40, 24, 96, 3
    qa = ints[rng.integers(0, ints.size, (M, K))]
    qb = ints[rng.integers(0, ints.size, (G, N, K))]
    sa = np.full((M, K // 32), 127, np.uint8)
    sb = np.full((G, N, K // 32), 127, np.uint8)
    offs = [10, 10, 37]
    out, mag = oracle.mx_grouped_gemm(qa, sa, qb, sb, offs)
    ref = _gemm_reference(qa, sa, qb, sb, offs)
    np.testing.assert_array_equal(out[:37], ref[:37])
    assert np.all(np.isnan(out[37:]))           # rows in no group untouched
    assert np.all(mag[:37] >= np.abs(out[:37]))


def test_grouped_gemm_random_scales_and_exponent_shift():
    rng = np.random.default_rng(22)
    M, N, K, G = 64, 16, 128, 4
    codes = np.array([c for c in range(256) if c & 0x7F != 0x7F], np.uint8)
    qa = codes[rng.integers(0, codes.size, (M, K))]
    qb = codes[rng.integers(0, codes.size, (G, N, K))]
    sa = rng.integers(110, 140, (M, K // 32)).astype(np.uint8)
    sb = rng.integers(110, 140, (G, N, K // 32)).astype(np.uint8)
    offs = [5, 40, 40, 64]
    out, mag = oracle.mx_grouped_gemm(qa, sa, qb, sb, offs)
    ref = _gemm_reference(qa, sa, qb, sb, offs)
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12 * mag.max())
    # one more unit in every scale of row 7 doubles that row exactly
    sa2 = sa.copy()
    sa2[7] += 1
    out2, _ = oracle.mx_grouped_gemm(qa, sa2, qb, sb, offs)
    np.testing.assert_array_equal(out2[7], 2 * out[7])
    np.testing.assert_array_equal(np.delete(out2, 7, 0), np.delete(out, 7, 0))


def test_grouped_gemm_brute_force_tiny():
    """Python loops over a 3-group case with the E4M3 values from the format's
    definition (sign, exponent, mantissa fields)."""
    def dec(c):
        s, e, m = c >> 7, (c >> 3) & 15, c & 7
        v = m * 2.0 ** -9 if e == 0 else (1 + m / 8) * 2.0 ** (e - 7)
        return -v if s else v
    rng = np.random.default_rng(23)
    M, N, K, G = 7, 3, 64, 3
    codes = np.array([c for c in range(256) if c & 0x7F != 0x7F], np.uint8)
    qa = codes[rng.integers(0, codes.size, (M, K))]
    qb = codes[rng.integers(0, codes.size, (G, N, K))]
    sa = rng.integers(120, 135, (M, 2)).astype(np.uint8)
    sb = rng.integers(120, 135, (G, N, 2)).astype(np.uint8)
    offs = [2, 2, 9]  # the last offset is past M: clamped
    out, _ = oracle.mx_grouped_gemm(qa, sa, qb, sb, offs)
    bounds = [(0, 2), (2, 2), (2, 7)]
    for g, (a0, a1) in enumerate(bounds):
        for m in range(a0, a1):
            for n in range(N):
                acc = 0.0
                for k in range(K):
                    acc += (dec(int(qa[m, k])) * 2.0 ** (int(sa[m, k // 32]) - 127) *
                            dec(int(qb[g, n, k])) * 2.0 ** (int(sb[g, n, k // 32]) - 127))
                assert abs(out[m, n] - acc) <= 1e-12 * max(1.0, abs(acc))


def test_batched_per_group_is_uniform_groups_of_the_flat_tensor():
    """A 3-D tensor's per-matrix groups equal the 2-D call over the flattened rows with
    one group per matrix (row-major codes byte for byte, same scales), and the
    column-major codes are each matrix's transpose."""
    rng = np.random.default_rng(31)
    E, M, K = 3, 40, 24
    x = oracle.double_to_bf16(rng.standard_normal((E, M, K)) * np.exp(rng.standard_normal((E, 1, K))))
    qb, sb = oracle.per_group_quant_batched(x, oracle.ROW_MAJOR)
    q2, s2 = oracle.per_group_quant(x.reshape(E * M, K), np.arange(1, E + 1) * M, oracle.ROW_MAJOR)
    np.testing.assert_array_equal(qb.reshape(E * M, K), q2)
    np.testing.assert_array_equal(sb.view(np.uint32), s2.view(np.uint32))
    qc, sc = oracle.per_group_quant_batched(x, oracle.COL_MAJOR)
    np.testing.assert_array_equal(qc, np.swapaxes(qb, 1, 2))
    np.testing.assert_array_equal(sc.view(np.uint32), sb.view(np.uint32))
