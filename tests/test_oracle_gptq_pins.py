"""Pins of the oracle's GPTQ (CPU only).

Source: "Quantization Algorithms" study notes, GPTQ chapter: layer-wise
objective ||W X - W_hat X||^2; Hessian 2 X X^T with a 1 % diagonal dampening;
L = Cholesky(H^-1); columns quantized in blocks of 128 with
err = (w_j - q_j) / L[j][j] fed into the later columns; act-order (large
|x|^2 first); the OBQ single-step update it derives from.  "LLM Quantization:
GPTQ, AWQ, SmoothQuant, FP8, KV Cache (7/10)", GPTQ section: quantization
error is corrected through approximate second-order information.

Independent references here: numpy/LAPACK for H, its inverse and the
Cholesky factor; an unblocked column-by-column sweep written with numpy
vector operations (the blocked and unblocked forms are the same algorithm);
the two-column OBQ step in closed form.  Only the static RTN group parameters
come from the oracle's RTN path, which is pinned elsewhere."""
import numpy as np
import pytest
import torch

import oracle
from w4a16_bit_gemm_b200 import synthetic as syn


def to_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def vals(bits: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.asarray(bits, np.uint16).view(np.int16)).view(torch.bfloat16).double().numpy()


def f16(bits: np.ndarray) -> np.ndarray:
    return np.asarray(bits, np.uint16).view(np.float16).astype(np.float64)


def bf16_round(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).double().numpy()


def correlated_layer(N, K, T, seed, outlier_frac=0.01):
    """W ~ N(0, 0.02); X with correlated channels (a random mixing of a
    lower-dimensional source) plus the x50 salient channels."""
    W = syn.weight(N, K, 0.02, seed, 1)
    rng = np.random.default_rng(seed)
    Z = rng.normal(0, 1, (T, K // 4))
    A = rng.normal(0, 1, (K // 4, K)) / np.sqrt(K // 4)
    X = Z @ A + 0.3 * rng.normal(0, 1, (T, K))
    n_ch = max(1, int(round(outlier_frac * K)))
    X[:, rng.choice(K, n_ch, replace=False)] *= 50
    return to_bits(W), to_bits(torch.from_numpy(X.astype(np.float32)).to(torch.bfloat16))


def numpy_hessian(Xb):
    X = vals(Xb)
    H = 2.0 * X.T @ X
    d = 0.01 * np.mean(np.diag(H))
    H[np.diag_indices_from(H)] += d if d != 0 else 1.0
    return H


def numpy_gptq(Wb, Xb, g, sym, act_order):
    """Unblocked GPTQ: after each column, every later column is updated."""
    W = vals(Wb)
    N, K = W.shape
    H = numpy_hessian(Xb)
    perm = np.argsort(-np.diag(H), kind="stable") if act_order else np.arange(K)
    U = np.linalg.cholesky(np.linalg.inv(H[np.ix_(perm, perm)])).T
    _, sc, zc, _ = oracle.quantize(Wb, g, symmetric=sym)
    qmin, qmax = (-8, 7) if sym else (0, 15)
    Wp = W[:, perm].copy()
    codes = np.empty((N, K), np.int32)
    for j in range(K):
        col = perm[j]
        s = f16(sc[:, col // g])
        z = np.zeros(N) if sym else f16(zc[:, col // g])
        q = np.clip(np.rint(Wp[:, j] / s) + z, qmin, qmax)
        wh = bf16_round((s * (q - z)).astype(np.float32))
        err = (Wp[:, j] - wh) / U[j, j]
        Wp[:, j + 1:] -= np.outer(err, U[j, j + 1:])
        codes[:, col] = q.astype(np.int32)
    return codes, perm, U


def test_factor_is_the_upper_cholesky_of_the_damped_inverse_hessian():
    _, Xb = correlated_layer(4, 256, 300, 1)
    for act in (False, True):
        perm, U, flags = oracle.gptq_factor(Xb, act)
        assert flags == 0
        H = numpy_hessian(Xb)
        want_perm = np.argsort(-np.diag(H), kind="stable") if act else np.arange(256)
        assert np.array_equal(perm, want_perm)
        assert np.all(np.tril(U, -1) == 0.0) and np.all(np.diag(U) > 0)
        Hp = H[np.ix_(perm, perm)]
        ref = np.linalg.cholesky(np.linalg.inv(Hp)).T
        assert np.max(np.abs(U - ref)) <= 1e-9 * np.max(np.abs(ref))
        # U^T U H = I
        assert np.max(np.abs(U.T @ U @ Hp - np.eye(256))) < 1e-8


def test_damping_is_one_percent_of_the_mean_diagonal():
    """Rank-deficient X (T < K): only the dampening makes H invertible, and
    the factor's diagonal shows it: for a channel with zero activations,
    (H^-1) of that channel is 1/d exactly, d = 0.01 mean(diag 2 X^T X)."""
    rng = np.random.default_rng(2)
    X = rng.normal(0, 1, (16, 128)).astype(np.float32)
    X[:, 5] = 0.0
    Xb = to_bits(torch.from_numpy(X).to(torch.bfloat16))
    perm, U, _ = oracle.gptq_factor(Xb, act_order=False)
    Xv = vals(Xb)
    d = 0.01 * np.mean(np.diag(2 * Xv.T @ Xv))
    Hinv = U.T @ U
    assert abs(Hinv[5, 5] - 1.0 / d) <= 1e-9 / d
    assert np.max(np.abs(Hinv[5, :5])) < 1e-12 / d


CASES = [
    # (N, K, T, g, sym, act_order)
    (24, 256, 300, 128, True, True),
    (24, 256, 300, 128, False, False),
    (16, 384, 200, 64, True, False),
    (16, 320, 500, 64, False, True),   # ragged last block (64 columns)
    (8, 512, 64, 128, True, True),     # T < K: damping carries the inverse
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "%dx%d-T%d-g%d-%s-%s" % (
    c[0], c[1], c[2], c[3], "sym" if c[4] else "asym", "act" if c[5] else "seq"))
def test_codes_match_an_independent_unblocked_sweep(case):
    N, K, T, g, sym, act = case
    Wb, Xb = correlated_layer(N, K, T, N + K + T)
    codes, sc, zc, perm, U, flags = oracle.gptq(Wb, Xb, g, sym, act, want_factor=True)
    assert flags == 0
    rc, rs, rz, _ = oracle.quantize(Wb, g, symmetric=sym)
    assert np.array_equal(sc, rs) and (sym or np.array_equal(zc, rz))  # static group parameters
    ref, ref_perm, _ = numpy_gptq(Wb, Xb, g, sym, act)
    assert np.array_equal(perm, ref_perm)
    assert np.array_equal(codes, ref)
    lo, hi = (-8, 7) if sym else (0, 15)
    assert codes.min() >= lo and codes.max() <= hi
    assert not np.array_equal(codes, rc)  # the feedback changes codes


def test_obq_two_column_step():
    """With two columns the whole algorithm is one OBQ step: quantize w0,
    then w1 <- w1 - (w0 - q0) [H^-1]_01 / [H^-1]_00."""
    rng = np.random.default_rng(4)
    x0 = rng.normal(0, 1, 64)
    X = np.stack([x0, 0.8 * x0 + 0.6 * rng.normal(0, 1, 64)], 1).astype(np.float32)
    Xb = to_bits(torch.from_numpy(X).to(torch.bfloat16))
    H = numpy_hessian(Xb)
    Hinv = np.linalg.inv(H)
    n_diff = 0
    for trial in range(200):
        W = rng.normal(0, 0.02, (1, 2)).astype(np.float32)
        Wb = to_bits(torch.from_numpy(W).to(torch.bfloat16))
        codes, sc, zc, _, _, _ = oracle.gptq(Wb, Xb, 2, symmetric=False, act_order=False)
        s, z = f16(sc[0, 0]), f16(zc[0, 0])
        w0, w1 = vals(Wb)[0]
        q0 = np.clip(np.rint(w0 / s) + z, 0, 15)
        wh0 = bf16_round(np.float32(s * (q0 - z)))
        w1u = w1 - (w0 - wh0) * Hinv[0, 1] / Hinv[0, 0]
        q1 = np.clip(np.rint(w1u / s) + z, 0, 15)
        assert codes[0, 0] == q0 and codes[0, 1] == q1, trial
        n_diff += int(q1 != np.clip(np.rint(w1 / s) + z, 0, 15))
    assert n_diff > 10  # the step really moves codes


def test_diagonal_hessian_reduces_to_rounding():
    """Orthogonal calibration channels give a diagonal H, hence a diagonal
    factor and no feedback: every code is clamp(rint(w / s) + z)."""
    K = 256
    X = np.zeros((K, K), np.float32)
    X[np.arange(K), np.arange(K)] = np.linspace(0.5, 4.0, K)
    Xb = to_bits(torch.from_numpy(X).to(torch.bfloat16))
    Wb, _ = correlated_layer(16, K, 8, 5)
    for act in (False, True):
        codes, sc, zc, perm, _, _ = oracle.gptq(Wb, Xb, 128, symmetric=False, act_order=act)
        W = vals(Wb)
        s = np.repeat(f16(sc), 128, axis=1)
        z = np.repeat(f16(zc), 128, axis=1)
        assert np.array_equal(codes, np.clip(np.rint(W / s) + z, 0, 15).astype(np.int32))
        if act:  # decreasing diagonal; equal bf16 values keep index order
            d = np.diag(numpy_hessian(Xb))
            assert np.array_equal(perm, np.argsort(-d, kind="stable"))
            assert np.all(np.diff(d[perm]) <= 0) and perm[0] == K - 1


def test_gptq_lowers_the_layer_output_error():
    """The objective of the page: ||(W - W_hat) X^T||^2 below plain RTN's on
    correlated calibration activations, with and without act-order."""
    N, K, T, g = 64, 512, 400, 128
    Wb, Xb = correlated_layer(N, K, T, 6)
    X = vals(Xb)
    W = vals(Wb)
    rc, rs, rz, _ = oracle.quantize(Wb, g, symmetric=True)
    e_rtn = np.sum(((W - vals(oracle.dequantize(rc, rs, None, g))) @ X.T) ** 2)
    for act in (False, True):
        codes, sc, _, _, _, _ = oracle.gptq(Wb, Xb, g, symmetric=True, act_order=act)
        e = np.sum(((W - vals(oracle.dequantize(codes, sc, None, g))) @ X.T) ** 2)
        assert e < 0.75 * e_rtn, (act, e / e_rtn)
