"""MSE-optimal clipping search (wq_quantize_clip_mse) on the GPU against the
oracle: packed codes, scales and zeros bit-exact, device flags equal; the
artifact then feeds the unchanged dequant and linear kernels."""
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


def make_weights(d_out, d_in, kind, seed):
    rng = np.random.default_rng(seed)
    if kind == "normal":
        x = rng.normal(0, 0.02, (d_out, d_in))
    elif kind == "laplace":
        x = rng.laplace(0, 0.02, (d_out, d_in))
    elif kind == "uniform":
        x = rng.uniform(-0.05, 0.05, (d_out, d_in))
    else:  # entry outliers
        x = rng.normal(0, 0.02, (d_out, d_in))
        n = max(1, d_out * d_in // 100)
        idx = rng.choice(d_out * d_in, n, replace=False)
        x.flat[idx] = 0.4 * rng.choice([-1, 1], n)
    return torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16)


def check(W, g, sym):
    b = _b()
    Wb = bits16(W)
    p = b.quantize_clip_mse(W.cuda(), g, sym)
    st, flags = b.device_error()
    oq, os_, oz, of, codes, best = oracle.quantize_clip_pack4(Wb, g, sym)
    if of == 0:
        assert st == b.WQ_OK
    else:  # non-finite input or a saturated scale is reported through the status word
        assert st in (b.WQ_ERR_NONFINITE, b.WQ_ERR_RANGE)
    assert np.array_equal(bits32(p.qweight), oq)
    assert np.array_equal(bits16(p.scales), os_)
    if not sym:
        assert np.array_equal(bits16(p.zeros), oz)
    assert flags == of
    return p, codes, os_, oz, best


CASES = [
    # (d_out, d_in, g, sym, kind)
    (64, 256, 128, False, "normal"),
    (37, 512, 128, True, "laplace"),
    (300, 384, 128, False, "outlier"),
    (129, 256, 32, False, "laplace"),
    (65, 512, 64, True, "outlier"),
    (33, 1024, 256, False, "uniform"),
    (1000, 4096, 128, False, "laplace"),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "%dx%d-g%d-%s-%s" % (c[0], c[1], c[2], "sym" if c[3] else "asym", c[4]))
def test_clip_matches_oracle(case):
    d_out, d_in, g, sym, kind = case
    _, _, _, _, best = check(make_weights(d_out, d_in, kind, d_out + d_in), g, sym)
    if kind in ("laplace", "outlier"):
        assert (best > 0).any()  # the search really clips somewhere


def test_clip_degenerate_and_nonfinite_groups():
    rng = np.random.default_rng(3)
    x = rng.normal(0, 0.02, (8, 256)).astype(np.float32)
    x[0, :128] = 0.0                 # all-zero group
    x[1, :128] = 1e-30               # underflowing scale
    x[2, 5] = np.nan                 # NaN skipped by the statistics, coded as zero
    x[3, 7] = np.inf                 # infinite value: saturated scale
    x[4, :128] = 3e38                # fp16 overflow of the scale
    x[5, 130] = -np.inf
    W = torch.from_numpy(x).to(torch.bfloat16)
    for sym in (False, True):
        check(W, 128, sym)


@pytest.mark.parametrize("ci", [0])
def test_clip_config1_tiny(ci):
    check(syn.case_weight(syn.TINY, ci, "cpu"), 128, False)


def test_clip_config2_attention_projection():
    check(syn.case_weight(syn.ATTN, 0, "cpu"), 128, False)


def test_clip_config3_mlp_gate_sym():
    check(syn.case_weight(syn.MLP, 0, "cpu"), 128, True)


def test_clip_artifact_feeds_dequant_and_linear():
    b = _b()
    W = make_weights(512, 1024, "laplace", 11)
    p, codes, os_, oz, _ = check(W, 128, False)
    W_hat_ref = oracle.dequantize(codes, os_, oz, 128)
    assert np.array_equal(bits16(b.dequantize(p)), W_hat_ref)
    X = syn.activations(1, 1024, 5, 1, "cpu")
    Y = b.linear_w4a16(X.cuda(), p, out_dtype=torch.float32)
    y_ref, A = oracle.linear(bits16(X), W_hat_ref)
    ok, ratio = linear_tolerance_ok(Y.cpu().numpy().astype(np.float64), y_ref, A, out_bf16=False)
    assert ok, ratio


def test_clip_error_never_above_rtn_on_device():
    """Squared reconstruction error per group (torch on the GPU, fp64):
    the clipping search never does worse than RTN, and does better in total
    on long-tailed weights."""
    b = _b()
    W = make_weights(2048, 4096, "laplace", 12).cuda()
    pc = b.quantize_clip_mse(W, 128, False)
    pr = b.quantize_rtn(W, 128, False)
    Wf = W.double().view(2048, 32, 128)
    ec = ((Wf - b.dequantize(pc).double().view(2048, 32, 128)) ** 2).sum(-1)
    er = ((Wf - b.dequantize(pr).double().view(2048, 32, 128)) ** 2).sum(-1)
    assert bool((ec <= er * (1 + 1e-12)).all())
    assert float(ec.sum()) < 0.95 * float(er.sum())
