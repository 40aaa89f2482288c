"""W8A16 on the GPU against the oracle: symmetric INT8 quantize, pack and
dequant bit-exact (codes, scales, flags); the linear layer (split-K mma.sync
GEMV for M <= 16, tcgen05 GEMM above) within the stated bound.  Sources: "LLM
Quantization: GPTQ, AWQ, SmoothQuant, FP8, KV Cache (7/10)", "Which tensor is
quantized" and Granularity; "Quantization Algorithms" study notes 1.8."""
import numpy as np
import pytest
import torch

import oracle
from tests._util import bits16, bits32, linear_tolerance_ok
from w4a16_bit_gemm_b200 import synthetic as syn

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clear_status():
    from w4a16_bit_gemm_b200 import binding
    binding.device_error()
    yield


def _b():
    from w4a16_bit_gemm_b200 import binding
    return binding


def weights(d_out, d_in, seed, kind="normal"):
    rng = np.random.default_rng(seed)
    x = rng.normal(0, 0.02, (d_out, d_in))
    if kind == "outlier":
        n = max(1, d_out * d_in // 1000)
        x.flat[rng.choice(d_out * d_in, n, replace=False)] = 0.4 * rng.choice([-1, 1], n)
    return torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16)


def check_quant(W, g):
    b = _b()
    p = b.quantize_w8(W.cuda(), g)
    st, flags = b.device_error()
    oq, osc, of, codes = oracle.quantize_pack8(bits16(W), g)
    assert flags == of
    assert np.array_equal(bits32(p.qweight), oq)
    assert np.array_equal(bits16(p.scales), osc)
    return p, codes, osc


QCASES = [
    (64, 256, 32), (37, 512, 128), (300, 384, 384), (129, 1024, 256), (33, 2048, 512), (1000, 4096, 4096),
    (5, 96, 32),
]


@pytest.mark.parametrize("case", QCASES, ids=lambda c: "%dx%d-g%d" % c)
def test_w8_quantize_and_dequant_match_oracle(case):
    d_out, d_in, g = case
    W = weights(d_out, d_in, d_out + d_in, "outlier")
    p, codes, osc = check_quant(W, g)
    assert np.abs(codes).max() == 127 and codes.min() >= -127
    W_hat = oracle.dequantize(codes, osc, None, g)
    assert np.array_equal(bits16(_b().dequantize_w8(p)), W_hat)


def test_w8_degenerate_and_nonfinite_rows():
    x = np.random.default_rng(3).normal(0, 0.02, (8, 256)).astype(np.float32)
    x[0] = 0.0              # all-zero group: s = 1
    x[1] = 1e-30            # underflowing scale
    x[2, 5] = np.nan        # NaN skipped, coded 0
    x[3, 7] = np.inf        # saturated scale
    x[4, :128] = 3e38       # fp16 overflow of the scale
    x[5, 130] = -np.inf
    W = torch.from_numpy(x).to(torch.bfloat16)
    for g in (128, 256):
        check_quant(W, g)


def check_linear(d_out, d_in, g, M, seed, out_fp32=True):
    b = _b()
    W = weights(d_out, d_in, seed)
    p, codes, osc = check_quant(W, g)
    X = syn.activations(M, d_in, seed, 3, "cpu", channel_outlier_frac=0.001)
    Y = b.linear_w8a16(X.cuda(), p, out_dtype=torch.float32 if out_fp32 else torch.bfloat16)
    st, _ = b.device_error()
    assert st == b.WQ_OK
    y_ref, A = oracle.linear(bits16(X), oracle.dequantize(codes, osc, None, g))
    y = Y.cpu().float().numpy().astype(np.float64)
    ok, ratio = linear_tolerance_ok(y, y_ref, A, out_bf16=not out_fp32)
    assert ok, ratio


@pytest.mark.parametrize("M", [1, 2, 3, 5, 8, 9, 12, 16])
def test_w8_gemv_matches_oracle(M):
    check_linear(1000, 4096, 4096, M, 10 + M)   # ragged rows, per-channel
    check_linear(200, 1056, 32, M, 20 + M)      # d_in not a multiple of 64, small groups


def test_w8_gemv_bf16_output_and_groups():
    check_linear(513, 2048, 128, 4, 31, out_fp32=False)
    check_linear(64, 11008, 11008, 1, 32)


@pytest.mark.parametrize("shape", [(17, 600, 1056, 32), (130, 4096, 4096, 4096), (300, 777, 2048, 128),
                                   (512, 4096, 4096, 128)], ids=lambda s: "M%d-N%d-K%d-g%d" % s)
def test_w8_gemm_matches_oracle(shape):
    M, N, K, g = shape
    check_linear(N, K, g, M, M + N)


def test_w8_gemm_sampled_large():
    """M = 2048 on the 8192 x 8192 shape (the tensor-core path's two-tile
    variant), checked on 64 sampled output rows."""
    b = _b()
    W = weights(8192, 8192, 41)
    p = b.quantize_w8(W.cuda())
    X = syn.activations(2048, 8192, 42, 3, "cpu")
    Y = b.linear_w8a16(X.cuda(), p, out_dtype=torch.float32).cpu().numpy().astype(np.float64)
    rows = np.random.default_rng(5).choice(8192, 64, replace=False)
    oq, osc, _, codes = oracle.quantize_pack8(bits16(W[rows]), 8192)
    y_ref, A = oracle.linear(bits16(X), oracle.dequantize(codes, osc, None, 8192))
    ok, ratio = linear_tolerance_ok(Y[:, rows], y_ref, A, out_bf16=False)
    assert ok, ratio


def test_w8_error_smaller_than_w4():
    """Eight bits: the reconstruction error is far below 4-bit RTN's."""
    b = _b()
    W = weights(512, 4096, 50).cuda()
    e8 = float(((W.double() - b.dequantize_w8(b.quantize_w8(W, 128)).double()) ** 2).sum())
    e4 = float(((W.double() - b.dequantize(b.quantize_rtn(W, 128, True)).double()) ** 2).sum())
    assert e8 < e4 / 50
