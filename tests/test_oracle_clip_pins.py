"""Pins of the oracle's MSE-optimal clipping search against the pages and
exact arithmetic (CPU only).

Sources: "LLM Quantization: GPTQ, AWQ, SmoothQuant, FP8, KV Cache (7/10)",
section "Clipping Trade-off" (clipping an outlier raises its error and lowers
the error of the rest; choose the threshold that minimises the local
reconstruction error); "Quantization Algorithms" study notes, calibration
section 4 (MSE-optimal: argmin ||x - x_dq||^2, independent per channel or
group, better than min-max for long-tailed data).

Exact references here never call the oracle's arithmetic: reconstruction
errors are rational sums over the bf16 inputs and the bf16-rounded products
s(q - z) (torch rounds the exact fp32 product once)."""
from fractions import Fraction

import numpy as np
import torch

import oracle

G = 128


def bf16_bits(x) -> np.ndarray:
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bf16_values(bits: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.asarray(bits, np.uint16).view(np.int16)).view(torch.bfloat16).float().numpy()


def exact_error(x_bits, codes, s16, z) -> Fraction:
    """sum over finite x of (x - bf16(s (q - z)))^2, exactly."""
    x = bf16_values(x_bits)
    s = np.float32(np.array([s16], np.uint16).view(np.float16)[0])
    prod = (s * (np.asarray(codes, np.int64) - z).astype(np.float32)).astype(np.float32)  # exact
    xh = torch.from_numpy(prod).to(torch.bfloat16).float().numpy()
    tot = Fraction(0)
    for v, h in zip(x, xh):
        if np.isfinite(v):
            d = Fraction(float(v)) - Fraction(float(h))
            tot += d * d
    return tot


def group_range(x_bits, symmetric):
    x = bf16_values(x_bits)
    x = x[~np.isnan(x)]
    lo = float(min(0.0, x.min())) if x.size else 0.0
    hi = float(max(0.0, x.max())) if x.size else 0.0
    amax = float(np.abs(x).max()) if x.size else 0.0
    return lo, hi, amax


def candidates(x_bits, symmetric):
    """(codes, s16, z) of every shrink candidate via the oracle's range step."""
    lo, hi, amax = group_range(x_bits, symmetric)
    out = []
    for i in range(oracle.CLIP_CANDIDATES):
        a = np.float32(oracle.clip_alpha(i))
        c, s16, z, _ = oracle.quantize_group_range(x_bits, float(np.float32(a * np.float32(lo))),
                                                   float(np.float32(a * np.float32(hi))),
                                                   float(np.float32(a * np.float32(amax))), symmetric)
        out.append((c, s16, z))
    return out


def seeded_groups(n, kind, seed):
    rng = np.random.default_rng(seed)
    if kind == "normal":
        x = rng.normal(0, 0.02, (n, G))
    elif kind == "laplace":
        x = rng.laplace(0, 0.02, (n, G))
    elif kind == "uniform":
        x = rng.uniform(-0.05, 0.05, (n, G))
    else:  # normal with one outlier per group
        x = rng.normal(0, 0.02, (n, G))
        x[np.arange(n), rng.integers(0, G, n)] = 0.4 * rng.choice([-1, 1], n)
    return bf16_bits(x.astype(np.float32))


def test_alpha_grid():
    for i in range(oracle.CLIP_CANDIDATES):
        assert oracle.clip_alpha(i) == float(np.float32(20 - i) / np.float32(20))
    assert oracle.clip_alpha(0) == 1.0 and oracle.clip_alpha(10) == 0.5


def test_error_formula_is_the_exact_sum_of_squares():
    W = seeded_groups(40, "outlier", 1)
    for row in W:
        c, s16, z, _ = oracle.quantize_group_range(row, *group_range(row, False), symmetric=False)
        ref = exact_error(row, c, s16, z)
        got = oracle.group_sq_error(row, c, s16, z)
        assert abs(Fraction(got) - ref) <= ref * Fraction(1, 10**13) + Fraction(1, 10**300), (got, float(ref))


def test_alpha_one_candidate_is_rtn():
    for sym in (False, True):
        W = seeded_groups(16, "outlier", 2)
        codes, scales, zeros, _ = oracle.quantize(W, G, symmetric=sym)
        for r, row in enumerate(W):
            c, s16, z = candidates(row, sym)[0]
            assert np.array_equal(c, codes[r]) and s16 == int(scales[r, 0])
            if not sym:
                assert z == int(np.float16(np.array([zeros[r, 0]], np.uint16).view(np.float16)[0]))


def test_choice_is_the_exact_argmin():
    ambiguous = 0
    for sym in (False, True):
        for kind, seed in (("normal", 3), ("laplace", 4), ("outlier", 5)):
            W = seeded_groups(24, kind, seed)
            codes, scales, zeros, _, best = oracle.quantize_clip(W, G, sym)
            for r, row in enumerate(W):
                errs = [exact_error(row, c, s16, z) for (c, s16, z) in candidates(row, sym)]
                m = min(errs)
                exact_best = errs.index(m)
                runner = sorted(errs)[1]
                if runner - m <= m * Fraction(1, 10**12):
                    ambiguous += 1  # fp64 summation order may legitimately pick either
                    assert errs[int(best[r, 0])] - m <= m * Fraction(1, 10**12)
                    continue
                assert int(best[r, 0]) == exact_best, (sym, kind, r, int(best[r, 0]), exact_best)
                c, s16, z = candidates(row, sym)[exact_best]
                assert np.array_equal(codes[r], c) and int(scales[r, 0]) == s16
    assert ambiguous <= 4


def test_never_worse_than_rtn():
    W = seeded_groups(32, "laplace", 6)
    cc, sc, zc, _, best = oracle.quantize_clip(W, G, False)
    cr, sr, zr, _ = oracle.quantize(W, G)
    f16 = lambda b: int(np.array([b], np.uint16).view(np.float16)[0])
    for r, row in enumerate(W):
        e_clip = exact_error(row, cc[r], int(sc[r, 0]), f16(zc[r, 0]))
        e_rtn = exact_error(row, cr[r], int(sr[r, 0]), f16(zr[r, 0]))
        assert e_clip <= e_rtn


def test_outlier_trade_off_of_the_page():
    """Many values in (-1, 1) and one at 20: clipping the range raises the
    outlier's error and lowers the error of the other values."""
    rng = np.random.default_rng(7)
    x = rng.uniform(-1, 1, G).astype(np.float32)
    x[0], x[1], x[2] = -1.0, 1.0, 20.0
    xb = bf16_bits(x)
    cands = candidates(xb, False)
    c0, s0, z0 = cands[0]
    c10, s10, z10 = cands[10]  # alpha = 0.5
    out = np.zeros(G, bool)
    out[2] = True
    e_out0 = exact_error(xb[out], c0[out], s0, z0)
    e_out10 = exact_error(xb[out], c10[out], s10, z10)
    e_rest0 = exact_error(xb[~out], c0[~out], s0, z0)
    e_rest10 = exact_error(xb[~out], c10[~out], s10, z10)
    assert e_out10 > e_out0
    assert e_rest10 < e_rest0
    # the MSE objective weighs both: whatever it picks is no worse than either
    _, _, _, _, best = oracle.quantize_clip(xb[None, :], G, False)
    ch = cands[int(best[0, 0])]
    e_best = exact_error(xb, *ch)
    assert e_best <= exact_error(xb, c0, s0, z0) and e_best <= exact_error(xb, c10, s10, z10)


def test_long_tailed_groups_gain_most():
    """MSE-optimal beats min-max more often on long-tailed data."""
    lap = seeded_groups(64, "laplace", 8)
    uni = seeded_groups(64, "uniform", 9)
    _, _, _, _, b_lap = oracle.quantize_clip(lap, G, False)
    _, _, _, _, b_uni = oracle.quantize_clip(uni, G, False)
    assert (b_lap > 0).mean() > (b_uni > 0).mean()
    assert (b_lap > 0).mean() > 0.5


def test_exactly_representable_group_keeps_rtn():
    """A group whose values sit on the RTN grid has zero error at alpha = 1,
    so the search keeps the RTN artifact (ties go to less clipping)."""
    rng = np.random.default_rng(10)
    codes = rng.integers(0, 16, G)
    codes[:2] = [0, 15]
    z = 3
    x = (np.float32(2.0 ** -6) * (codes - z)).astype(np.float32)
    xb = bf16_bits(x)
    cc, sc, zc, _, best = oracle.quantize_clip(xb[None, :], G, False)
    cr, sr, zr, _ = oracle.quantize(xb[None, :], G)
    assert int(best[0, 0]) == 0
    assert np.array_equal(cc, cr) and np.array_equal(sc, sr) and np.array_equal(zc, zr)
