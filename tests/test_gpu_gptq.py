"""GPTQ (wq_gptq) on the GPU against the oracle ("Quantization Algorithms"
study notes, GPTQ chapter): both compute in fp64 with the same operation
order, so codes, scales, zeros, the processing order and the flags agree bit
for bit."""
import numpy as np
import pytest
import torch

import oracle
from tests._util import bits16, bits32, f64_from_bf16_bits
from tests.test_oracle_gptq_pins import correlated_layer
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


def tensor(bits):
    return torch.from_numpy(np.ascontiguousarray(bits, np.uint16).view(np.int16)).view(torch.bfloat16)


def check(Wb, Xb, g, sym, act):
    b = _b()
    p, perm = b.gptq(tensor(Wb).cuda(), tensor(Xb).cuda(), g, sym, act)
    st, flags = b.device_error()
    oc, osc, oz, operm, _, of = oracle.gptq(Wb, Xb, g, sym, act)
    assert flags == of
    assert np.array_equal(perm.cpu().numpy(), operm)
    assert np.array_equal(bits16(p.scales), osc)
    if not sym:
        assert np.array_equal(bits16(p.zeros), oz)
    assert np.array_equal(bits32(p.qweight), oracle.pack4(oc))
    return p, st, oc


CASES = [
    # (N, K, T, g, sym, act_order)
    (64, 256, 300, 128, True, True),
    (96, 256, 300, 128, False, False),
    (50, 384, 200, 64, True, False),    # ragged rows
    (33, 320, 500, 64, False, True),    # ragged last column block (64)
    (40, 512, 64, 128, True, True),     # T < K: the dampening carries the inverse
    (130, 1024, 700, 32, False, True),
    (200, 768, 1000, 256, True, False),
    (24, 96, 50, 32, True, True),       # one ragged block, three panels
    (8, 32, 16, 32, False, True),       # a single panel
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "%dx%d-T%d-g%d-%s-%s" % (
    c[0], c[1], c[2], c[3], "sym" if c[4] else "asym", "act" if c[5] else "seq"))
def test_gptq_matches_oracle(case):
    N, K, T, g, sym, act = case
    Wb, Xb = correlated_layer(N, K, T, N + K + T)
    _, st, _ = check(Wb, Xb, g, sym, act)
    assert st == _b().WQ_OK


def test_gptq_2048_with_512_calibration_tokens():
    Wb, Xb = correlated_layer(256, 2048, 512, 9)
    check(Wb, Xb, 128, True, True)


def test_gptq_degenerate_calibration():
    """All-zero activations (H = 0, dampening 1: plain rounding in fp64), and
    a dead channel next to live ones."""
    Wb, Xb = correlated_layer(32, 256, 100, 11)
    check(Wb, np.zeros_like(Xb), 128, False, True)
    X = f64_from_bf16_bits(Xb).astype(np.float32)
    X[:, 7] = 0.0
    check(Wb, bits16(torch.from_numpy(X).to(torch.bfloat16)), 128, True, True)


def test_gptq_nonfinite_calibration_is_flagged():
    b = _b()
    Wb, Xb = correlated_layer(16, 256, 40, 12)
    X = f64_from_bf16_bits(Xb).astype(np.float32)
    X[3, 5] = np.inf
    p, perm = b.gptq(tensor(Wb).cuda(), torch.from_numpy(X).to(torch.bfloat16).cuda(), 128, True, True)
    st, flags = b.device_error()
    _, _, _, _, _, of = oracle.gptq(Wb, bits16(torch.from_numpy(X).to(torch.bfloat16)), 128, True, True)
    assert of & b.WQ_DEVFLAG_RANGE and flags & b.WQ_DEVFLAG_RANGE and st == b.WQ_ERR_RANGE
    assert sorted(perm.cpu().numpy().tolist()) == list(range(256))  # still a permutation


def test_gptq_artifact_feeds_the_linear_layer():
    b = _b()
    from tests._util import linear_tolerance_ok
    Wb, Xb = correlated_layer(256, 1024, 300, 13)
    p, _, oc = check(Wb, Xb, 128, True, True)
    W_hat = oracle.dequantize(oc, bits16(p.scales), None, 128)
    assert np.array_equal(bits16(b.dequantize(p)), W_hat)
    X = syn.activations(3, 1024, 5, 1, "cpu")
    Y = b.linear_w4a16(X.cuda(), p, out_dtype=torch.float32)
    y_ref, A = oracle.linear(bits16(X), W_hat)
    ok, ratio = linear_tolerance_ok(Y.cpu().numpy().astype(np.float64), y_ref, A, out_bf16=False)
    assert ok, ratio


def test_gptq_full_size_attention_projection():
    """4096 x 4096 with 512 calibration tokens (the bench workload): the full
    oracle takes minutes here, so check what holds at any size: the
    processing order (recomputed from sequential fp64 sums), the static RTN
    parameters, determinism, and the objective: the layer-output error on the
    calibration activations is well below RTN's."""
    b = _b()
    W = syn.case_weight(syn.ATTN, 0, "cpu")
    X = syn.activations(512, 4096, 21, 2, "cpu", channel_outlier_frac=0.001)
    Wd, Xd = W.cuda(), X.cuda()
    p, perm = b.gptq(Wd, Xd, 128, True, True)
    st, _ = b.device_error()
    assert st == b.WQ_OK
    Xv = f64_from_bf16_bits(bits16(X))
    d = np.zeros(4096)
    for t in range(Xv.shape[0]):  # sequential in t, as both sides sum
        d = d + Xv[t] * Xv[t]
    d = 2.0 * d
    damp = 0.01 * (np.cumsum(d)[-1] / 4096)
    d = d + damp
    assert np.array_equal(perm.cpu().numpy(), np.argsort(-d, kind="stable"))
    r = b.quantize_rtn(Wd, 128, True)
    assert torch.equal(p.scales, r.scales)
    p2, _ = b.gptq(Wd, Xd, 128, True, True)
    assert torch.equal(p.qweight, p2.qweight)
    Wf = Wd.double()
    e_g = float((((Wf - b.dequantize(p).double()) @ Xd.double().T) ** 2).sum())
    e_r = float((((Wf - b.dequantize(r).double()) @ Xd.double().T) ** 2).sum())
    assert e_g < 0.8 * e_r, e_g / e_r
