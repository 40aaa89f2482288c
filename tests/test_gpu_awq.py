"""AWQ per-input-channel scaling search (wq_awq_search) on the GPU against the
oracle ("Quantization Algorithms" study notes, AWQ procedure).

What must agree and how:
  - the 11 losses: the oracle sums in fp64 over fp64 outputs, the library over
    fp32 outputs (the tcgen05 GEMM on bf16 W for X W^T, the W4A16 linear for
    X' Q(W')^T), so they agree to a relative 1e-4 (the fp32 output rounding is
    ~1e-7 of |Y| against a quantization error of a few per cent of |Y|);
  - the kept alpha: equal to the oracle's (every case here has a loss gap far
    above that tolerance);
  - s: the oracle's scales for the kept alpha, bit for bit (both sides evaluate
    ln and exp by the same fixed fp64 procedure and sum the mean of ln m in
    channel order);
  - the artifact: bit-exact against the oracle's own search."""
import numpy as np
import pytest
import torch

import oracle
from tests._util import bits16, bits32, f64_from_bf16_bits
from w4a16_bit_gemm_b200 import synthetic as syn

pytestmark = pytest.mark.gpu

LOSS_RTOL = 1e-4


@pytest.fixture(autouse=True)
def _clear_status():
    from w4a16_bit_gemm_b200 import binding
    binding.device_error()
    yield


def _b():
    from w4a16_bit_gemm_b200 import binding
    return binding


def layer(N, K, T, seed, outlier_frac=0.01):
    W = syn.weight(N, K, 0.02, seed, 1)
    X = syn.activations(T, K, seed, 2, "cpu", channel_outlier_frac=outlier_frac)
    return W, X


def scaled_weight_bits(Wb, sb):
    """bf16(fl32(W s)) computed with numpy fp32 (one IEEE multiply)."""
    W32 = f64_from_bf16_bits(Wb).astype(np.float32)
    s32 = f64_from_bf16_bits(sb).astype(np.float32)
    prod = (W32 * s32[None, :]).astype(np.float32)
    return bits16(torch.from_numpy(prod).to(torch.bfloat16))


def check(W, X, g=128, sym=False):
    b = _b()
    Wb, Xb = bits16(W), bits16(X)
    r = b.awq_search(W.cuda(), X.cuda(), g, sym)
    st, flags = b.device_error()
    assert st == b.WQ_OK and flags == 0
    losses = r.losses.cpu().numpy()
    best = int(r.best.cpu().item())
    s_gpu = bits16(r.s)
    oc, osc, oz, os_, olosses, obest = oracle.awq_search(Wb, Xb, g, symmetric=sym)
    # losses
    assert np.all(np.abs(losses - olosses) <= LOSS_RTOL * olosses + 1e-30), (losses, olosses)
    # the kept alpha, and a gap that makes it the only correct answer
    assert best == obest, (best, obest, olosses)
    others = np.delete(olosses, obest)
    assert np.all(others - olosses[obest] > LOSS_RTOL * olosses[obest]) or np.all(olosses == olosses[0])
    # the scales of the kept alpha and the artifact, bit for bit
    assert np.array_equal(s_gpu, os_)
    assert np.array_equal(oracle.unpack4(bits32(r.packed.qweight), W.shape[1], sym), oc)
    assert np.array_equal(bits16(r.packed.scales), osc)
    if not sym:
        assert np.array_equal(bits16(r.packed.zeros), oz)
    return r, losses, best, olosses, obest


CASES = [
    # (N, K, T, g, sym) -- T covers the GEMV (T <= 16), the tensor-memory GEMV
    # (T = 2) and the tcgen05 GEMM (T > 16, ragged) paths of the loss linear
    (96, 256, 48, 128, False),
    (96, 256, 48, 128, True),
    (64, 512, 1, 128, False),
    (130, 256, 2, 128, False),
    (200, 384, 5, 128, True),
    (256, 1024, 37, 64, False),
    (384, 512, 129, 32, False),
    (160, 768, 64, 256, True),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "%dx%d-T%d-g%d-%s" % (c[0], c[1], c[2], c[3],
                                                                           "sym" if c[4] else "asym"))
def test_awq_matches_oracle(case):
    N, K, T, g, sym = case
    W, X = layer(N, K, T, N + K + T)
    check(W, X, g, sym)


def test_awq_salient_channels_config2_shape():
    """Attention-projection width with its 0.1% x50 activation channels and a
    wider 1% set: the search picks alpha > 0 and cuts the loss well below RTN."""
    for frac in (0.001, 0.01):
        W, X = layer(256, 4096, 64, 7, outlier_frac=frac)
        _, losses, best, _, _ = check(W, X)
        assert best > 0 and losses[best] < 0.7 * losses[0]


def test_awq_alpha_zero_equals_rtn_artifact():
    """Uniform activations (no salient channel) with a constant |x| per
    channel: every alpha gives s = 1, so all losses are equal, the kept index
    is 0 and the artifact is plain RTN of W."""
    b = _b()
    K = 256
    W, _ = layer(64, K, 4, 9)
    X = torch.full((16, K), 0.5, dtype=torch.bfloat16)
    X[1::2] = -0.5
    r = b.awq_search(W.cuda(), X.cuda(), 128, False)
    assert int(r.best.item()) == 0
    assert np.all(bits16(r.s) == 0x3F80)
    losses = r.losses.cpu().numpy()
    assert np.all(losses == losses[0])
    p = b.quantize_rtn(W.cuda(), 128, False)
    assert torch.equal(p.qweight, r.packed.qweight) and torch.equal(p.scales, r.packed.scales)
    assert torch.equal(p.zeros, r.packed.zeros)


def test_awq_deterministic():
    b = _b()
    W, X = layer(256, 1024, 96, 10)
    r1 = b.awq_search(W.cuda(), X.cuda())
    r2 = b.awq_search(W.cuda(), X.cuda())
    assert torch.equal(r1.losses, r2.losses) and torch.equal(r1.s, r2.s)
    assert torch.equal(r1.packed.qweight, r2.packed.qweight)


def test_awq_scale_activations_bit_exact():
    b = _b()
    _, X = layer(1, 1024, 33, 11)
    s = torch.from_numpy(oracle.awq_scales(bits16(X), 0.5).view(np.int16)).view(torch.bfloat16)
    Xp = b.awq_scale_activations(X.cuda(), s.cuda())
    X32 = f64_from_bf16_bits(bits16(X)).astype(np.float32)
    s32 = f64_from_bf16_bits(bits16(s)).astype(np.float32)
    want = bits16(torch.from_numpy((X32 / s32[None, :]).astype(np.float32)).to(torch.bfloat16))
    assert np.array_equal(bits16(Xp), want)


def test_awq_layer_output_through_the_linear():
    """The scaled layer (X / s) Q(W')^T through the W4A16 linear matches the
    oracle's fp64 output of the same artifact, and is closer to X W^T than the
    plain RTN layer on salient-channel activations."""
    b = _b()
    from tests._util import linear_tolerance_ok
    W, X = layer(512, 2048, 24, 12)
    r = b.awq_search(W.cuda(), X.cuda())
    Xp = b.awq_scale_activations(X.cuda(), r.s)
    Y = b.linear_w4a16(Xp, r.packed, out_dtype=torch.float32).cpu().numpy().astype(np.float64)
    codes = oracle.unpack4(bits32(r.packed.qweight), 2048, False)
    Wh = oracle.dequantize(codes, bits16(r.packed.scales), bits16(r.packed.zeros), 128)
    y_ref, A = oracle.linear(bits16(Xp), Wh)
    ok, ratio = linear_tolerance_ok(Y, y_ref, A, out_bf16=False)
    assert ok, ratio
    Y_true = X.double().numpy() @ W.double().numpy().T
    p = b.quantize_rtn(W.cuda())
    Y_rtn = b.linear_w4a16(X.cuda(), p, out_dtype=torch.float32).cpu().double().numpy()
    assert ((Y - Y_true) ** 2).sum() < ((Y_rtn - Y_true) ** 2).sum()


def test_awq_full_size_attention_projection():
    """4096 x 4096 with 512 calibration tokens (the bench workload): the
    oracle's whole search is too slow here, so its pieces are used.
    - s equals the oracle's scales for the kept alpha, bit for bit;
    - the artifact equals the oracle's RTN of bf16(W s) with the oracle's s;
    - the losses of alpha = 0 and the kept alpha, recomputed in fp64 from the
      oracle's artifacts (torch fp64 products), agree to LOSS_RTOL;
    - the runner-up loss is more than 3 LOSS_RTOL above the kept one, so any
      loss computation within that tolerance keeps the same alpha."""
    b = _b()
    W = syn.case_weight(syn.ATTN, 0, "cpu")
    X = syn.activations(512, 4096, 21, 2, "cpu", channel_outlier_frac=0.001)
    Wd, Xd = W.cuda(), X.cuda()
    r = b.awq_search(Wd, Xd)
    st, _ = b.device_error()
    assert st == b.WQ_OK
    best = int(r.best.item())
    losses = r.losses.cpu().numpy()
    assert best == int(np.argmin(losses)) and best > 0
    gaps = np.delete(losses, best) - losses[best]
    assert gaps.min() > 3 * LOSS_RTOL * losses[best], (losses, best)
    Wb, Xb = bits16(W), bits16(X)
    s_ref = oracle.awq_scales(Xb, best / 10.0)
    assert np.array_equal(bits16(r.s), s_ref)
    rq, rs, rz, _, _ = oracle.quantize_pack4(scaled_weight_bits(Wb, s_ref), 128, False)
    assert np.array_equal(bits32(r.packed.qweight), rq)
    assert np.array_equal(bits16(r.packed.scales), rs) and np.array_equal(bits16(r.packed.zeros), rz)
    Y = Xd.double() @ Wd.double().T
    X32 = f64_from_bf16_bits(Xb).astype(np.float32)
    for i in (0, best):
        si = oracle.awq_scales(Xb, i / 10.0)
        q, sc, z, _, codes = oracle.quantize_pack4(scaled_weight_bits(Wb, si), 128, False)
        Wh = f64_from_bf16_bits(oracle.dequantize(codes, sc, z, 128))
        s32 = f64_from_bf16_bits(si).astype(np.float32)
        Xi = f64_from_bf16_bits(bits16(torch.from_numpy((X32 / s32[None, :]).astype(np.float32)).to(torch.bfloat16)))
        Yi = torch.from_numpy(Xi).cuda() @ torch.from_numpy(Wh).cuda().T
        li = float(((Y - Yi) ** 2).sum())
        assert abs(losses[i] - li) <= LOSS_RTOL * li, (i, losses[i], li)
