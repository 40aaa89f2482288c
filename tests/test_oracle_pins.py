"""Pins of the CPU oracle against what the pages and the mathematics fix.

None of these re-types the oracle's formulas: each compares it with an
independent library routine (numpy / torch conversions, numpy matmul), an
exact rational brute force, a closed form, an invariant stated on the pages,
or a number the pages print (fixtures under ``tests/golden``).
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16_bits(x) -> np.ndarray:
    """Round float data to bf16 with torch (RNE) and return the bit patterns."""
    t = torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16).copy()


def bits_to_f64(bits: np.ndarray) -> np.ndarray:
    with np.errstate(invalid="ignore"):
        return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f16_to_f64(bits: np.ndarray) -> np.ndarray:
    return np.asarray(bits, np.uint16).view(np.float16).astype(np.float64)


# --------------------------------------------------------------------------
# IEEE conversions vs independent library conversions
# --------------------------------------------------------------------------

def _conversion_inputs():
    rng = np.random.default_rng(1)
    parts = [
        (rng.standard_normal(200_000) * 10.0 ** rng.integers(-9, 6, 200_000)).astype(np.float32),
        np.array([0.0, -0.0, np.inf, -np.inf, 65504.0, 65519.99, 65520.0, 1e-8, 5.96e-8, 2.98e-8,
                  2.9802322e-08, 6.1035156e-05, 6.0975552e-05], np.float32),
    ]
    # every fp16 value and every midpoint between neighbouring fp16 values
    h = np.arange(0, 0x7c00, dtype=np.uint16).view(np.float16).astype(np.float32)
    mids = ((h[:-1].astype(np.float64) + h[1:].astype(np.float64)) / 2).astype(np.float32)
    parts += [h, -h, mids, -mids]
    return np.concatenate(parts).astype(np.float32)


def test_f32_to_f16_matches_numpy():
    x = _conversion_inputs()
    ours = oracle.f32_to_f16_bits_array(x)
    with np.errstate(over="ignore"):
        ref = x.astype(np.float16).view(np.uint16)
    assert np.array_equal(ours, ref)


def test_f16_to_f32_exhaustive_matches_numpy():
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.f16_bits_to_f32_array(h)
    ref = h.view(np.float16).astype(np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def test_f32_to_bf16_matches_torch():
    rng = np.random.default_rng(2)
    x = np.concatenate([
        (rng.standard_normal(200_000) * 10.0 ** rng.integers(-30, 30, 200_000)).astype(np.float32),
        # exact bf16 midpoints (ties) and their neighbours
        ((rng.integers(0, 1 << 15, 50_000).astype(np.uint32) << 16) | 0x8000).view(np.float32),
        ((rng.integers(0, 1 << 15, 50_000).astype(np.uint32) << 16) | 0x7FFF).view(np.float32),
        np.array([3.3895314e38, 3.4028235e38, -3.4028235e38, np.inf, -np.inf, 0.0, -0.0, 1e-45], np.float32),
    ])
    x = x.astype(np.float32)
    ours = oracle.f32_to_bf16_bits_array(x)
    ref = bf16_bits(x)
    nan = np.isnan(x)
    assert np.all((ours[nan] & 0x7F80) == 0x7F80) and np.all((ours[nan] & 0x7F) != 0)
    assert np.array_equal(ours[~nan], ref[~nan])


# --------------------------------------------------------------------------
# Level counts and code ranges (golden: printed by the pages)
# --------------------------------------------------------------------------

def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


@pytest.mark.parametrize("entry", _golden("page_memory_examples.json")["levels"], ids=lambda e: f"b{e['bits']}")
def test_level_count_asymmetric_ramp(entry):
    b = entry["bits"]
    g = 512
    ramp = bf16_bits(np.linspace(-1.0, 3.0, g))
    codes, scales, zeros, flags = oracle.quantize(ramp[None, :], g, bits=b, symmetric=False)
    assert len(np.unique(codes)) == entry["levels"]
    assert codes.min() == 0 and codes.max() == entry["levels"] - 1


@pytest.mark.parametrize("entry", _golden("page_memory_examples.json")["code_ranges"], ids=lambda e: e["format"])
def test_code_ranges(entry):
    rng = np.random.default_rng(3)
    g = 64
    rows = [rng.standard_normal(g) * 0.02 for _ in range(200)]
    # adversarial rows: exact endpoints, one-sided groups, a dominant negative value
    rows += [np.full(g, -1.0), np.full(g, 1.0), np.r_[-1.0, np.full(g - 1, 0.25)],
             np.r_[1.0, np.full(g - 1, -0.999)], np.linspace(-1, 1, g), np.linspace(-1.0, 0.1, g)]
    W = bf16_bits(np.stack(rows))
    codes, _, _, _ = oracle.quantize(W, g, bits=entry["bits"], symmetric=entry["symmetric"],
                                     narrow=entry["narrow"])
    assert codes.min() >= entry["qmin"] and codes.max() <= entry["qmax"]
    # both endpoints are reached on this data
    assert codes.min() == entry["qmin"] or entry["narrow"] or entry["symmetric"]
    assert codes.max() == entry["qmax"]
    if entry["narrow"]:
        assert codes.min() == -127  # the symmetric INT8 range excludes -128 but reaches -127


# --------------------------------------------------------------------------
# Zero exactly representable under asymmetric quantization
# --------------------------------------------------------------------------

def test_zero_exactly_representable():
    rng = np.random.default_rng(4)
    g = 128
    W = rng.standard_normal((300, 512)) * 0.02
    W[:100] = np.abs(W[:100])          # all-positive groups
    W[100:200] = -np.abs(W[100:200])   # all-negative groups
    W[:, ::7] = 0.0                    # exact zeros inside every group
    Wb = bf16_bits(W)
    codes, scales, zeros, _ = oracle.quantize(Wb, g, bits=4, symmetric=False)
    W_hat = oracle.dequantize(codes, scales, zeros, g)
    z_int = f16_to_f64(zeros)
    assert np.all(z_int == np.round(z_int)) and z_int.min() >= 0 and z_int.max() <= 15
    # code z dequantizes to +0 and x = 0 is coded as z
    zero_pos = (Wb == 0)
    assert np.all(W_hat[zero_pos] == 0)
    zr = np.repeat(z_int, g, axis=1)
    assert np.all(codes[zero_pos] == zr[zero_pos])


# --------------------------------------------------------------------------
# |x - x_hat| <= s/2 for values inside the clamp range
# --------------------------------------------------------------------------

@pytest.mark.parametrize("symmetric", [False, True])
def test_rounding_error_bound(symmetric):
    rng = np.random.default_rng(5)
    g = 128
    W = rng.standard_normal((256, 1024)) * 0.02
    W[rng.random(W.shape) < 0.001] = 0.4
    Wb = bf16_bits(W)
    codes, scales, zeros, _ = oracle.quantize(Wb, g, bits=4, symmetric=symmetric)
    x = bits_to_f64(Wb)
    s = np.repeat(f16_to_f64(scales), g, axis=1)
    z = np.zeros_like(s) if symmetric else np.repeat(f16_to_f64(zeros), g, axis=1)
    qmin, qmax = (-8, 7) if symmetric else (0, 15)
    pre = np.rint(x / s) + z
    inside = (pre >= qmin) & (pre <= qmax)
    assert inside.mean() > 0.99
    recon = s * (codes - z)  # exact in fp64: <= 11 + 5 significant bits
    err = np.abs(x - recon)
    # the quotient is rounded to fp32 before rint: allow that one fp32 rounding
    assert np.all(err[inside] <= s[inside] * (0.5 + 2.0 ** -22))
    # after the bf16 rounding of x_hat the bound grows by half a bf16 ulp of x_hat
    W_hat = bits_to_f64(oracle.dequantize(codes, scales, None if symmetric else zeros, g))
    half_ulp = np.abs(W_hat) * 2.0 ** -8  # >= half a bf16 ulp at |W_hat|
    assert np.all(np.abs(x - W_hat)[inside] <= s[inside] * (0.5 + 2.0 ** -22) + half_ulp[inside])


# --------------------------------------------------------------------------
# The one-outlier-at-20 example (golden, hand-derived from the page's setup)
# --------------------------------------------------------------------------

def _outlier_group():
    rng = np.random.default_rng(6)
    vals = np.r_[-1.0, 1.0, 20.0, rng.uniform(-0.999, 0.999, 125)]
    return bf16_bits(vals)[None, :]


def test_outlier20_symmetric():
    gold = _golden("outlier20_example.json")["symmetric_int4"]
    Wb = _outlier_group()
    codes, scales, _, _ = oracle.quantize(Wb, 128, bits=4, symmetric=True)
    assert f16_to_f64(scales)[0, 0] == gold["scale_fp16"]
    assert codes[0, 2] == gold["outlier_code"]
    small = np.delete(codes[0], 2)
    assert sorted(set(small.tolist())) == gold["small_value_codes"]


def test_outlier20_asymmetric_and_clipping():
    gold = _golden("outlier20_example.json")
    ga = gold["asymmetric_uint4"]
    Wb = _outlier_group()
    codes, scales, zeros, _ = oracle.quantize(Wb, 128, bits=4, symmetric=False)
    assert f16_to_f64(scales)[0, 0] == ga["scale_fp16"]
    assert f16_to_f64(zeros)[0, 0] == ga["zero"]
    assert codes[0, 2] == ga["outlier_code"]
    W_hat = bits_to_f64(oracle.dequantize(codes, scales, zeros, 128))
    assert W_hat[0, 2] == ga["outlier_dequant_bf16"]
    small = np.delete(codes[0], 2)
    assert set(small.tolist()) <= set(ga["small_value_codes"])
    # clipping the outlier to the small values' range restores resolution
    clipped = Wb.copy()
    clipped[0, 2] = bf16_bits([1.0])[0]
    c2, _, _, _ = oracle.quantize(clipped, 128, bits=4, symmetric=False)
    n_levels = len(set(np.delete(c2[0], 2).tolist()))
    assert n_levels >= gold["clipped_to_unit_range_asymmetric"]["min_distinct_levels_for_small_values"]
    assert n_levels > len(set(small.tolist()))


# --------------------------------------------------------------------------
# Round-trip fixed point: exactly representable groups come back unchanged
# --------------------------------------------------------------------------

@pytest.mark.parametrize("symmetric", [False, True])
def test_round_trip_fixed_point(symmetric):
    rng = np.random.default_rng(7)
    g, rows, G = 128, 64, 4
    codes = np.empty((rows, G * g), np.int64)
    s = np.empty((rows, G))
    z = np.zeros((rows, G), np.int64)
    for r in range(rows):
        for j in range(G):
            if symmetric:
                c = rng.integers(-7, 8, g)
                c[:2] = [7, -7]
            else:
                c = rng.integers(0, 16, g)
                c[:2] = [0, 15]
                z[r, j] = rng.integers(0, 16)
            rng.shuffle(c)
            codes[r, j * g:(j + 1) * g] = c
            s[r, j] = 2.0 ** -int(rng.integers(2, 14))
    x = np.repeat(s, g, axis=1) * (codes - np.repeat(z, g, axis=1))
    Wb = bf16_bits(x)
    assert np.array_equal(bits_to_f64(Wb), x)  # exact in bf16
    qc, qs, qz, flags = oracle.quantize(Wb, g, bits=4, symmetric=symmetric)
    assert flags == 0
    assert np.array_equal(qc, codes)
    assert np.array_equal(f16_to_f64(qs), s)
    if not symmetric:
        assert np.array_equal(f16_to_f64(qz), z.astype(np.float64))
    # round ties to even on x/s: codes at exact half-integers
    tie = np.zeros((1, 16))
    tie[0, 0] = 3.75          # hi = 3.75 -> s = 0.25, z = 0
    tie[0, 1:4] = [0.625, 0.875, 0.125]  # x/s = 2.5 -> 2, 3.5 -> 4, 0.5 -> 0
    tc, ts, tz, _ = oracle.quantize(bf16_bits(tie), 16, bits=4, symmetric=False)
    assert f16_to_f64(ts)[0, 0] == 0.25 and f16_to_f64(tz)[0, 0] == 0
    assert tc[0, 1:4].tolist() == [2, 4, 0]


# --------------------------------------------------------------------------
# Brute force in exact rational arithmetic on tiny groups
# --------------------------------------------------------------------------

def _all_bf16_in(lo: float, hi: float) -> np.ndarray:
    u = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    v = bits_to_f64(u)
    keep = np.isfinite(v) & (v >= lo) & (v <= hi) & ~((u == 0x8000))
    return u[keep]


@pytest.mark.parametrize("lo,hi,symmetric", [
    (-1.0, 1.5, False), (-0.0625, 0.75, False), (-3.0, -0.5, False), (0.25, 7.0, False),
    (-0.5, 0.5, True), (-2.0, 0.75, True),
])
def test_brute_force_argmin(lo, hi, symmetric):
    g = 8
    pool = _all_bf16_in(lo, hi)
    lo_b, hi_b = bf16_bits([lo, hi])
    n_free = g - 2
    n_grp = math.ceil(len(pool) / n_free)
    free = np.resize(pool, n_grp * n_free).reshape(n_grp, n_free)
    W = np.concatenate([np.full((n_grp, 1), lo_b, np.uint16), np.full((n_grp, 1), hi_b, np.uint16), free], axis=1)
    codes, scales, zeros, _ = oracle.quantize(W, g, bits=4, symmetric=symmetric)

    # scale: fp16 nearest to the fp32 quotient, computed with numpy's IEEE fp32 ops and conversion
    f32 = np.float32
    if symmetric:
        s_expect = np.float16(f32(max(abs(lo), abs(hi))) / f32(7))
        qmin, qmax = -8, 7
    else:
        s_expect = np.float16((f32(max(hi, 0.0)) - f32(min(lo, 0.0))) / f32(15))
        qmin, qmax = 0, 15
    assert np.all(scales == np.uint16(s_expect.view(np.uint16)))
    S = Fraction(float(s_expect))
    if symmetric:
        Z = 0
    else:
        zq = Fraction(0) - Fraction(min(lo, 0.0)) / S
        Z = int(zq.numerator * 2 + zq.denominator) // (2 * zq.denominator)  # nearest (tie -> up)
        if zq - int(zq) == Fraction(1, 2):  # exact tie: even
            Z = int(zq) if int(zq) % 2 == 0 else int(zq) + 1
        Z = min(max(Z, qmin), qmax)
        assert np.all(f16_to_f64(zeros) == Z)

    near_ties = 0
    x_all = bits_to_f64(free.reshape(-1))
    c_all = codes[:, 2:].reshape(-1)
    seen = set()
    for xb, x, c in zip(free.reshape(-1), x_all, c_all):
        if xb in seen:
            continue
        seen.add(xb)
        X = Fraction(float(x))
        best = min(range(qmin, qmax + 1),
                   key=lambda q: (abs(X - S * (q - Z)), (q - Z) % 2))
        if best != c:
            # allowed only where x/s lies within one fp32 ulp of a half-integer
            t = X / S
            frac = t - math.floor(t)
            ulp = Fraction(2) ** (math.frexp(float(t))[1] - 24) if t != 0 else Fraction(0)
            assert abs(frac - Fraction(1, 2)) <= ulp, (float(x), c, best)
            near_ties += 1
    assert near_ties <= max(2, len(seen) // 500)


def test_brute_force_roundtrip_all_code_vectors_g4():
    # every 4-code vector (16^4) with a power-of-two scale and zero z = 3
    q = np.stack(np.meshgrid(*[np.arange(16)] * 4, indexing="ij"), -1).reshape(-1, 4)
    keep = (q.min(1) == 0) & (q.max(1) == 15)  # lo and hi pinned to the code ends
    q = q[keep]
    s, z = 0.125, 3
    x = s * (q - z)
    codes, scales, zeros, _ = oracle.quantize(bf16_bits(x), 4, bits=4, symmetric=False)
    assert np.array_equal(codes, q)
    assert np.all(f16_to_f64(scales) == s) and np.all(f16_to_f64(zeros) == z)


# --------------------------------------------------------------------------
# Degenerate and non-finite groups
# --------------------------------------------------------------------------

def test_degenerate_and_nonfinite_groups():
    g = 32
    W = np.zeros((5, g))
    W[1] = 1e-30            # scale underflows in fp16
    W[2] = np.linspace(-1, 1, g)
    W[2, 5] = np.nan
    W[3] = np.linspace(-1, 1, g)
    W[3, 7] = np.inf
    W[4] = np.linspace(-1, 1, g) * 3e6   # fp16 scale overflow
    Wb = bf16_bits(W)
    codes, scales, zeros, flags = oracle.quantize(Wb[:2], g, bits=4, symmetric=False)
    assert flags == 0
    assert np.all(scales == 0x3C00) and np.all(zeros == 0) and np.all(codes == 0)
    _, _, _, f2 = oracle.quantize(Wb[2:3], g, bits=4, symmetric=False)
    assert f2 == oracle.FLAG_NONFINITE
    c2, s2, z2, _ = oracle.quantize(Wb[2:3], g, bits=4, symmetric=False)
    assert c2[0, 5] == f16_to_f64(z2)[0, 0]   # NaN coded as zero
    _, s3, _, f3 = oracle.quantize(Wb[3:4], g, bits=4, symmetric=False)
    assert f3 & oracle.FLAG_NONFINITE and f3 & oracle.FLAG_RANGE and s3[0, 0] == 0x7BFF
    _, s4, _, f4 = oracle.quantize(Wb[4:5], g, bits=4, symmetric=True)
    assert f4 == oracle.FLAG_RANGE and s4[0, 0] == 0x7BFF


# --------------------------------------------------------------------------
# Packing layout v1
# --------------------------------------------------------------------------

def test_pack8_layout_low_byte_first():
    """W8A16 artifact: 4 codes per word, byte j = column 4c + j, two's complement."""
    codes = np.array([[1, -1, 127, -127, 0, 5, -2, 64]], np.int32)
    q = oracle.pack8(codes)
    assert q.tolist() == [[0x81_7F_FF_01, 0x40_FE_05_00]]
    assert np.array_equal(oracle.unpack8(q, 8), codes)


def test_int8_per_channel_scale_is_amax_over_127():
    """Per-channel INT8 (group = d_in): s = fp16(amax / 127) per row, codes
    rint(x / s) in [-127, 127]; the row's largest magnitude maps to +-127."""
    rng = np.random.default_rng(8)
    W = bf16_bits(rng.standard_normal((16, 96)).astype(np.float32) * 0.05)
    qw, sc, flags, codes = oracle.quantize_pack8(W, 96)
    x = torch.from_numpy(W.view(np.int16)).view(torch.bfloat16).float().numpy()
    amax = np.abs(x).max(axis=1)
    s_ref = np.array([np.float16(np.float32(a) / np.float32(127.0)) for a in amax])
    assert np.array_equal(sc[:, 0], s_ref.view(np.uint16)) and flags == 0
    s32 = s_ref.astype(np.float32)[:, None]
    assert np.array_equal(codes, np.clip(np.rint((x / s32).astype(np.float32)), -127, 127).astype(np.int32))
    assert np.all(np.abs(codes).max(axis=1) == 127)
    assert np.array_equal(oracle.unpack8(qw, 96), codes)

def test_pack_layout_low_nibble_first():
    codes = np.array([[0, 1, 2, 3, 4, 5, 6, 7, 8, 9, 10, 11, 12, 13, 14, 15]], np.int32)
    q = oracle.pack4(codes)
    assert q.tolist() == [[0x76543210, 0xFEDCBA98]]
    sym = np.array([[-8, -1, 0, 7, -2, 3, -5, 1]], np.int32)
    qs = oracle.pack4(sym)
    assert qs[0, 0] == (0x8 | 0xF << 4 | 0x0 << 8 | 0x7 << 12 | 0xE << 16 | 0x3 << 20 | 0xB << 24 | 0x1 << 28)
    assert np.array_equal(oracle.unpack4(qs, 8, True), sym)


# --------------------------------------------------------------------------
# Dequantization: every finite fp16 scale x every (q, z) against numpy/torch
# --------------------------------------------------------------------------

def test_dequant_exhaustive_against_library_rounding():
    h = np.arange(0, 0x7C00, dtype=np.uint16)                 # all finite positive fp16
    qz = np.stack(np.meshgrid(np.arange(16), np.arange(16), indexing="ij"), -1).reshape(-1, 2)
    n_s = len(h)
    codes = np.broadcast_to(qz[:, 0][None, :], (n_s, 256)).astype(np.int32)
    zeros = np.broadcast_to(np.float16(qz[:, 1]).view(np.uint16)[None, :], (n_s, 256)).copy()
    scales = np.broadcast_to(h[:, None], (n_s, 256)).copy()
    ours = oracle.dequantize(codes, scales, zeros, 1)
    prod = h.view(np.float16).astype(np.float32)[:, None] * (qz[:, 0] - qz[:, 1]).astype(np.float32)[None, :]
    ref = bf16_bits(prod)
    assert np.array_equal(ours, ref)


# --------------------------------------------------------------------------
# Linear layer
# --------------------------------------------------------------------------

def test_linear_special_cases_and_matmul():
    rng = np.random.default_rng(8)
    K, N, M = 256, 48, 3
    Wh = bf16_bits(rng.standard_normal((N, K)) * 0.02)
    X = bf16_bits(rng.standard_normal((M, K)))
    Y, A = oracle.linear(X, Wh)
    ref = bits_to_f64(X) @ bits_to_f64(Wh).T
    assert np.all(np.abs(Y - ref) <= 1e-12 * A + 1e-300)
    assert np.all(A >= np.abs(Y))
    # W = 0 gives y = 0
    Y0, A0 = oracle.linear(X, np.zeros_like(Wh))
    assert np.all(Y0 == 0) and np.all(A0 == 0)
    # a one-hot x picks column k of W_hat exactly
    k = 77
    e = np.zeros((1, K))
    e[0, k] = 1.0
    Y1, _ = oracle.linear(bf16_bits(e), Wh)
    assert np.array_equal(Y1[0], bits_to_f64(Wh[:, k]))
    # transposition check: a row-one-hot W picks x
    Wr = np.zeros((N, K), np.uint16)
    Wr[5, 9] = bf16_bits([1.0])[0]
    Y2, _ = oracle.linear(X, Wr)
    assert np.array_equal(Y2[:, 5], bits_to_f64(X[:, 9]))
    assert np.all(np.delete(Y2, 5, axis=1) == 0)


# --------------------------------------------------------------------------
# Byte arithmetic (golden: printed by the pages)
# --------------------------------------------------------------------------

def test_payload_bytes_printed_examples():
    gold = _golden("page_memory_examples.json")
    for e in gold["payload"]:
        payload, _, _ = oracle.artifact_bytes(int(e["params"]), e["bits"], 128, True)
        assert abs(payload - e["printed_bytes"]) <= e["rel_tol"] * e["printed_bytes"] + 1e-6, e
    for e in gold["group_scale_overhead"]:
        _, sb, _ = oracle.artifact_bytes(e["group_size"] * 1000, 4, e["group_size"], True)
        assert sb / (e["group_size"] * 1000) == e["printed_bytes_per_weight"]
    for e in gold["bits_per_weight"]:
        payload, sb, zb = oracle.artifact_bytes(e["group_size"], e["bits"], e["group_size"], True)
        assert (payload + sb + zb) * 8 / e["group_size"] == e["printed_bpw"]


def test_whole_model_artifact_bytes():
    from w4a16_bit_gemm_b200 import synthetic
    P = synthetic.total_params(synthetic.WHOLE_MODEL)
    assert P == 6_476_005_376
    payload, sb, zb = oracle.artifact_bytes(P, 4, 128, False)
    assert payload == 3_238_002_688 and sb + zb == 202_375_168
    assert payload + sb + zb == 3_440_377_856
    assert (payload + sb + zb) * 8 / P == 4.25


# --------------------------------------------------------------------------
# Monotonicity: within a group, a larger weight never gets a smaller code
# --------------------------------------------------------------------------

@pytest.mark.parametrize("bits,symmetric,narrow", [(4, False, False), (4, True, False), (8, True, True)])
def test_codes_are_monotone_within_a_group(bits, symmetric, narrow):
    """[P1] Affine Quantization: q = clamp(round(x/s) + z) is non-decreasing in
    x for s > 0, and so is x_hat = s (q - z)."""
    rng = np.random.default_rng(11)
    g = 128
    x = rng.laplace(0, 0.02, (64, g)).astype(np.float32)
    x[::7, 0] = 0.5  # a few outliers
    W = bf16_bits(x)
    codes, scales, zeros, _ = oracle.quantize(W, g, bits=bits, symmetric=symmetric, narrow=narrow)
    vals = torch.from_numpy(W.view(np.int16)).view(torch.bfloat16).float().numpy()
    W_hat = oracle.dequantize(codes, scales, zeros, g)
    hat = torch.from_numpy(W_hat.view(np.int16)).view(torch.bfloat16).float().numpy()
    for r in range(W.shape[0]):
        order = np.argsort(vals[r], kind="stable")
        assert np.all(np.diff(codes[r][order]) >= 0), r
        assert np.all(np.diff(hat[r][order]) >= 0), r
