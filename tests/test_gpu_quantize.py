"""GPU quantize+pack and dequantize vs the CPU oracle: bit-exact codes,
scales, zeros and dequantized bf16, on edge shapes, every supported group
size, degenerate/non-finite groups, and the exhaustive (s, q, z) table."""
import numpy as np
import pytest
import torch

import oracle
from tests._util import bits16, bits32, bf16_from_bits, fp16_from_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clear_status():
    from w4a16_bit_gemm_b200 import binding
    binding.device_error()
    yield


def _binding():
    from w4a16_bit_gemm_b200 import binding
    return binding


def gpu_quantize(Wb: np.ndarray, g: int, sym: bool):
    b = _binding()
    W = bf16_from_bits(Wb).cuda()
    b.device_error()  # clear
    p = b.quantize_rtn(W, g, sym)
    st, flags = b.device_error()
    return p, bits32(p.qweight), bits16(p.scales), None if sym else bits16(p.zeros), flags


def check_quantize(Wb: np.ndarray, g: int, sym: bool):
    p, q, s, z, flags = gpu_quantize(Wb, g, sym)
    oq, os_, oz, oflags, codes = oracle.quantize_pack4(Wb, g, sym)
    assert np.array_equal(q, oq), "packed codes differ"
    assert np.array_equal(s, os_), "scales differ"
    if not sym:
        assert np.array_equal(z, oz), "zeros differ"
    assert flags == oflags
    return p, codes, os_, oz


def bf16_bits_of(x: np.ndarray) -> np.ndarray:
    return bits16(torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16))


@pytest.mark.parametrize("g", [32, 64, 128, 256, 512, 1024])
@pytest.mark.parametrize("sym", [False, True])
def test_group_sizes(g, sym):
    rng = np.random.default_rng(g + sym)
    d_out, d_in = 37, 2048
    W = rng.standard_normal((d_out, d_in)) * 0.02
    W[rng.random(W.shape) < 0.002] = 0.4
    check_quantize(bf16_bits_of(W), g, sym)


@pytest.mark.parametrize("shape", [(1, 32), (3, 96), (7, 128), (5, 4096), (129, 384)])
def test_ragged_shapes(shape):
    d_out, d_in = shape
    g = 32 if d_in % 128 else 128
    rng = np.random.default_rng(d_out * d_in)
    W = bf16_bits_of(rng.standard_normal(shape) * 0.05)
    check_quantize(W, g, False)
    check_quantize(W, g, True)


def test_degenerate_and_nonfinite():
    g = 32
    W = np.zeros((8, g * 4), np.float64)
    W[1] = 1e-30                     # fp16 scale underflow -> s = 1, z = 0
    W[2] = np.linspace(-1, 1, g * 4)
    W[2, 5] = np.nan                 # NaN coded as z
    W[3] = np.linspace(-3, 2, g * 4)
    W[3, 70] = np.inf                # Inf -> scale saturates
    W[4] = np.linspace(-1, 1, g * 4) * 3e6   # fp16 overflow of the scale
    W[5] = -np.abs(np.linspace(-1, 1, g * 4))  # all-negative groups
    W[6] = np.abs(np.linspace(-1, 1, g * 4))   # all-positive groups
    W[7, ::3] = 0.25                 # exact ties (x/s = k + 0.5 with s = 2^-k)
    for sym in (False, True):
        check_quantize(bf16_bits_of(W), g, sym)


def test_flags_reported():
    b = _binding()
    W = np.zeros((2, 128))
    W[0, 3] = np.nan
    _, _, _, _, flags = gpu_quantize(bf16_bits_of(W), 128, False)
    assert flags & b.WQ_DEVFLAG_NONFINITE
    W = np.linspace(-1, 1, 256).reshape(2, 128) * 3e6
    _, _, _, _, flags = gpu_quantize(bf16_bits_of(W), 128, True)
    assert flags == b.WQ_DEVFLAG_RANGE
    st, flags = b.device_error()
    assert st == b.WQ_OK and flags == 0  # cleared by the previous read


def test_round_trip_codes_exact():
    rng = np.random.default_rng(11)
    g, rows = 128, 64
    q = rng.integers(0, 16, (rows, 4 * g))
    q[:, ::g] = 0
    q[:, 1::g] = 15
    z = rng.integers(0, 16, (rows, 4))
    s = 2.0 ** -rng.integers(2, 12, (rows, 4)).astype(np.float64)
    x = np.repeat(s, g, 1) * (q - np.repeat(z, g, 1))
    p, codes, _, _ = check_quantize(bf16_bits_of(x), g, False)
    assert np.array_equal(codes, q)


@pytest.mark.parametrize("sym", [False, True])
def test_dequantize_matches_oracle(sym):
    rng = np.random.default_rng(12 + sym)
    Wb = bf16_bits_of(rng.standard_normal((300, 1024)) * 0.02)
    p, codes, os_, oz = check_quantize(Wb, 128, sym)
    W_hat = _binding().dequantize(p)
    ref = oracle.dequantize(codes, os_, oz, 128)
    assert np.array_equal(bits16(W_hat), ref)


@pytest.mark.parametrize("sym", [False, True])
def test_dequantize_exhaustive_scale_code_zero(sym):
    """Every finite non-negative fp16 scale x every code x every zero point
    (the quantizer only emits positive scales; a negative scale could differ
    from the oracle in the sign of a zero result)."""
    b = _binding()
    h = np.arange(0, 0x7C00, dtype=np.uint16)
    if sym:
        g, G = 32, 1                    # codes -8..7 twice per row
        qrow = np.tile(np.arange(-8, 8), 2)
        zrow = None
    else:
        g, G = 32, 16                   # group j has zero point j; codes 0..15 twice
        qrow = np.tile(np.arange(16), 2 * 16)
        zrow = np.arange(16)
    d_out, d_in = len(h), g * G
    codes = np.broadcast_to(qrow[None, :], (d_out, d_in)).astype(np.int32)
    qweight = oracle.pack4(codes)
    scales = np.broadcast_to(h[:, None], (d_out, G)).copy()
    zeros = None if sym else np.broadcast_to(np.float16(zrow).view(np.uint16)[None, :], (d_out, G)).copy()
    ref = oracle.dequantize(codes, scales, zeros, g)
    P = b.PackedLinear(torch.from_numpy(qweight.view(np.int32)).cuda(), fp16_from_bits(scales).cuda(),
                       None if sym else fp16_from_bits(zeros).cuda(), d_out, d_in, g, sym)
    out = b.dequantize(P)
    assert np.array_equal(bits16(out), ref)


def _all_bf16_between(lo, hi):
    u = np.arange(0, 1 << 16, dtype=np.uint32).astype(np.uint16)
    with np.errstate(invalid="ignore"):
        v = (u.astype(np.uint32) << 16).view(np.float32)
    keep = np.isfinite(v) & (v >= lo) & (v <= hi)
    return u[keep]


@pytest.mark.parametrize("lo,hi,sym", [
    (-1.0, 1.5, False), (-0.0625, 0.75, False), (-3.0, -0.5, False), (0.25, 7.0, False),
    (-0.5, 0.5, True), (-2.0, 0.75, True), (-1e-3, 2e-2, False), (-65000.0, 1.0, False),
])
def test_every_bf16_in_window(lo, hi, sym):
    """Each group holds the window ends plus 30 values; together the groups
    cover every bf16 value in the window, so every quotient near a
    half-integer (the exact-division fallback) is exercised."""
    g = 32
    pool = _all_bf16_between(lo, hi)
    ends = bf16_bits_of([lo, hi])
    n_grp = -(-len(pool) // (g - 2))
    free = np.resize(pool, n_grp * (g - 2)).reshape(n_grp, g - 2)
    W = np.concatenate([np.repeat(ends[None, :], n_grp, 0), free], axis=1)
    # several groups per row
    rows = -(-n_grp // 8)
    W = np.resize(W, (rows * 8, g)).reshape(rows, 8 * g)
    check_quantize(np.ascontiguousarray(W), g, sym)
