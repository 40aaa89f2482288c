"""Pins of the oracle's AWQ per-input-channel scaling search (CPU only).

Source: "Quantization Algorithms" study notes, AWQ section: salient channels
are found from activation magnitude; scale migration W x = (W s)(x / s);
procedure: per-channel mean |x| on a calibration batch, alpha grid
{0, 0.1, ..., 1.0}, s = mean|x|^alpha / geomean, W' = W diag(s), loss =
||W X - Q(W')(X / s)||, alpha* = argmin; quantization error scales with s,
so larger s protects salient channels.  "LLM Quantization: GPTQ, AWQ,
SmoothQuant, FP8, KV Cache (7/10)", AWQ section: per-channel scaling chosen
from activation statistics protects the salient weights.

Independent references: per-channel means, W', X' and the loss are recomputed
here with numpy / torch (fp32 products rounded to bf16 by torch, fp64
matmul); only the RTN artifact comes from the oracle, whose RTN path is pinned
elsewhere."""
import numpy as np
import torch

import oracle
from w4a16_bit_gemm_b200 import synthetic as syn

G = 128


def to_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def bf16_of(x: np.ndarray) -> np.ndarray:
    return to_bits(torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16))


def vals(bits: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.asarray(bits, np.uint16).view(np.int16)).view(torch.bfloat16).double().numpy()


def layer(N, K, T, seed, outlier_frac=0.01):
    W = syn.weight(N, K, 0.02, seed, 1)
    X = syn.activations(T, K, seed, 2, "cpu", channel_outlier_frac=outlier_frac)
    return to_bits(W), to_bits(X)


def independent_loss(Wb, Xb, sb, symmetric=False):
    """||X W^T - X' Q(W')^T||^2 with W' = bf16(fl32(W s)), X' = bf16(fl32(X / s))."""
    W32 = vals(Wb).astype(np.float32)
    X32 = vals(Xb).astype(np.float32)
    s32 = vals(sb).astype(np.float32)
    Wp = bf16_of((W32 * s32[None, :]).astype(np.float32))
    Xp = bf16_of((X32 / s32[None, :]).astype(np.float32))
    codes, sc, zc, _ = oracle.quantize(Wp, G, symmetric=symmetric)
    Wh = vals(oracle.dequantize(codes, sc, zc, G))
    Y = vals(Xb) @ vals(Wb).T
    Yp = vals(Xp) @ Wh.T
    return float(((Y - Yp) ** 2).sum())


def test_alpha_zero_is_plain_rtn():
    Wb, Xb = layer(64, 256, 32, 1)
    assert np.all(oracle.awq_scales(Xb, 0.0) == 0x3F80)  # bf16 1.0
    codes, sc, zc, s, losses, best = oracle.awq_search(Wb, Xb, G)
    rc, rs, rz, _ = oracle.quantize(Wb, G)
    if best == 0:
        assert np.array_equal(codes, rc) and np.array_equal(sc, rs) and np.array_equal(zc, rz)
    assert abs(losses[0] - independent_loss(Wb, Xb, oracle.awq_scales(Xb, 0.0))) <= 1e-9 * losses[0]


def test_scales_follow_the_page_formula():
    _, Xb = layer(8, 512, 64, 2)
    m = np.maximum(np.abs(vals(Xb)).mean(axis=0), 2.0 ** -30)
    for alpha in (0.3, 0.5, 1.0):
        ref = np.exp(alpha * (np.log(m) - np.log(m).mean()))
        want = bf16_of(ref.astype(np.float32))
        got = oracle.awq_scales(Xb, alpha)
        diff = np.abs(got.astype(np.int32) - want.astype(np.int32))
        assert (diff == 0).mean() >= 0.999 and diff.max() <= 1, alpha
        # normalised by the geometric mean: mean log s ~ 0 (bf16 rounding only)
        assert abs(np.log(vals(got)).mean()) < 2.0 ** -8
        # larger activation magnitude, larger (or equal) scale: salient channels protected
        order = np.argsort(m, kind="stable")
        assert np.all(np.diff(vals(got)[order]) >= 0)


def test_losses_and_choice_recomputed_independently():
    for sym in (False, True):
        Wb, Xb = layer(96, 256, 48, 3 + sym)
        codes, sc, zc, s, losses, best = oracle.awq_search(Wb, Xb, G, symmetric=sym)
        ind = [independent_loss(Wb, Xb, oracle.awq_scales(Xb, i / 10.0), sym) for i in range(oracle.AWQ_ALPHAS)]
        for i in range(oracle.AWQ_ALPHAS):
            assert abs(losses[i] - ind[i]) <= 1e-9 * ind[i], (sym, i)
        assert best == int(np.argmin(ind))
        assert np.array_equal(s, oracle.awq_scales(Xb, best / 10.0))
        # the kept artifact is the RTN artifact of W' for that alpha
        Wp = bf16_of((vals(Wb).astype(np.float32) * vals(s).astype(np.float32)[None, :]).astype(np.float32))
        rc, rs, rz, _ = oracle.quantize(Wp, G, symmetric=sym)
        assert np.array_equal(codes, rc) and np.array_equal(sc, rs)
        if not sym:
            assert np.array_equal(zc, rz)


def test_salient_channels_are_protected():
    """With a few activation channels 50x larger (the salient ones), scaling
    cuts the output error well below plain RTN."""
    Wb, Xb = layer(128, 512, 64, 5, outlier_frac=0.01)
    _, _, _, s, losses, best = oracle.awq_search(Wb, Xb, G)
    assert best > 0
    assert losses[best] < 0.5 * losses[0]
    m = np.abs(vals(Xb)).mean(axis=0)
    sal = m > 10 * np.median(m)
    assert sal.any() and vals(s)[sal].min() > vals(s)[~sal].max()


def test_scale_migration_identity():
    """W x = (W s)(x / s) before quantization (exact arithmetic in fp64)."""
    Wb, Xb = layer(32, 256, 16, 6)
    s = vals(oracle.awq_scales(Xb, 0.5))
    Y = vals(Xb) @ vals(Wb).T
    Y2 = (vals(Xb) / s[None, :]) @ (vals(Wb) * s[None, :]).T
    assert np.allclose(Y, Y2, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------------------
# The fixed fp64 ln / exp of the scales (Cody-Waite reduction; atanh series,
# Taylor polynomial): pinned to the libm functions, to closed forms and to
# their own inverse relation.
# ---------------------------------------------------------------------------

def _ulps(a, b):
    return abs(a - b) / np.spacing(abs(b)) if b != 0 else abs(a) / np.spacing(0.0)


def test_ln_matches_libm_within_two_ulps():
    import math
    rng = np.random.default_rng(31)
    xs = np.concatenate([np.exp(rng.uniform(-30, 30, 5000)), rng.uniform(0.5, 2.0, 2000),
                         [2.0 ** -30, 1.0 - 2 ** -52, 1.0 + 2 ** -52, np.sqrt(2.0), 1e-9, 123456.789]])
    worst = max(_ulps(oracle.ln_f64(x), math.log(x)) for x in xs)
    assert worst <= 2.0, worst


def test_exp_matches_libm_within_two_ulps():
    import math
    rng = np.random.default_rng(32)
    xs = np.concatenate([rng.uniform(-40, 40, 5000), rng.uniform(-0.35, 0.35, 2000),
                         [0.5 * math.log(2.0), -0.5 * math.log(2.0), 1e-12, -20.5]])
    worst = max(_ulps(oracle.exp_f64(x), math.exp(x)) for x in xs)
    assert worst <= 2.0, worst


def test_ln_exp_closed_forms():
    import math
    assert oracle.ln_f64(1.0) == 0.0
    assert oracle.exp_f64(0.0) == 1.0
    for k in range(-30, 31):
        if k:  # ln 2^k = k ln 2 (k ln2_hi is exact, so only the tail rounds)
            assert _ulps(oracle.ln_f64(2.0 ** k), k * math.log(2.0)) <= 1.0
    # e^(ln x) = x to a few ulps, across the range the scales use
    for x in (1e-6, 0.02, 0.8, 1.0, 3.0, 50.0, 1e5):
        assert _ulps(oracle.exp_f64(oracle.ln_f64(x)), x) <= 8.0
