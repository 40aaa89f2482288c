"""W4A16 linear layer (GEMV for M <= 16, tcgen05 GEMM above) vs the oracle's
fp64 accumulation over the same dequantized bf16 weights:
|y - y_ref| <= 1e-3 * sum_k |w_hat x| + 1e-6 for every output element."""
import numpy as np
import pytest
import torch

import oracle
from tests._util import bits16, bf16_from_bits, f64_from_bf16_bits, linear_tolerance_ok

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _clear_status():
    from w4a16_bit_gemm_b200 import binding
    binding.device_error()
    yield


def _b():
    from w4a16_bit_gemm_b200 import binding
    return binding


def bf16_bits_of(x) -> np.ndarray:
    return bits16(torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16))


def run_case(Wb, Xb, g, sym, out_dtype=torch.bfloat16, rows=None, cols=None):
    """Quantize on both sides, run the GPU linear, compare (optionally on a
    sample of token rows / output columns)."""
    b = _b()
    W = bf16_from_bits(Wb).cuda()
    X = bf16_from_bits(Xb).cuda()
    p = b.quantize_rtn(W, g, sym)
    Y = b.linear_w4a16(X, p, out_dtype=out_dtype)
    st, flags = b.device_error()
    assert st == b.WQ_OK, (st, flags)
    y = Y.float().cpu().numpy().astype(np.float64)
    Wsel = Wb if cols is None else Wb[cols]
    Xsel = Xb if rows is None else Xb[rows]
    _, _, W_hat, _ = oracle.reference_linear_w4a16(Xsel[:1], Wsel, g, sym)
    y_ref, A = oracle.linear(Xsel, W_hat)
    ysel = y if rows is None else y[rows]
    ysel = ysel if cols is None else ysel[:, cols]
    ok, ratio = linear_tolerance_ok(ysel, y_ref, A, out_bf16=out_dtype == torch.bfloat16)
    assert ok, f"worst error/bound = {ratio:.3f}"
    return y, y_ref, A


GEMV_CASES = [
    # (N, K, g, sym, M)
    (64, 256, 128, False, 1),
    (300, 384, 128, False, 3),
    (1000, 4096, 128, True, 16),
    (130, 96, 32, False, 5),        # K not a multiple of 128
    (17, 1024, 64, False, 8),
    (260, 512, 512, False, 9),      # one group per row (per-channel scale)
    (5000, 1024, 128, False, 2),    # several rows per CTA
    (40, 11008, 128, True, 4),      # long K, shared-memory ring (slots reused)
    (20000, 2944, 128, False, 1),   # several passes per CTA, ring, 23 k blocks per pass
    (4096, 11008, 128, True, 16),   # ring with two n-tiles
    # k-split ring kernel: leading chunks dequantized into tensor memory before
    # the wait, the rest streamed; ragged k-unit sets and row counts
    (11008, 4096, 128, False, 1),
    (12288, 4096, 128, True, 1),
    (4096, 11008, 128, False, 1),   # 86 k-units: the last set of 8 is partial
    (3000, 5120, 64, False, 3),
    (2050, 9216, 128, False, 8),
    # k-major kernel (M = 9..16, and M <= 8 where the k-split kernels do not
    # fit; K >= 2048): partial last chunk and k-unit, several passes, g from
    # 32 to 2048
    (3000, 2048, 64, False, 12),
    (900, 2080, 32, True, 9),       # 2080 = one chunk + one 32-k slice
    (20000, 2048, 128, False, 16),  # nine 16-row blocks per CTA: three passes
    (16, 4096, 1024, False, 13),    # one block, one group per chunk
    (530, 4096, 2048, True, 10),    # a group spans two chunks
    (1500, 11008, 128, False, 8),   # x too large for the k-split kernels
    (700, 16384, 128, True, 5),
    # activations too long for the k-split kernels' shared memory: M = 1, 2 on
    # the k-major kernel
    (64, 131072, 128, False, 1),
    (512, 65536, 128, True, 2),
    # tensor-memory GEMV (M = 2, or M = 1 with K >= 8192; K % 256 == 0): ragged
    # row counts per CTA, several 32-row MMA tiles per CTA, every group size
    (333, 2048, 32, False, 2),
    (10360, 1024, 64, True, 2),     # 70 rows per CTA: three tiles of 24/23/23
    (2000, 512, 256, False, 2),
    (29600, 256, 128, False, 2),    # 200 rows per CTA, capped at 128: more CTAs than SMs
    (40000, 256, 128, True, 2),
    (700, 8192, 128, False, 1),     # M = 1, long rows: tensor-memory kernel
]


@pytest.mark.parametrize("case", GEMV_CASES, ids=lambda c: "N%d-K%d-g%d-%s-M%d" % (c[0], c[1], c[2], "sym" if c[3] else "asym", c[4]))
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32], ids=["bf16", "fp32"])
def test_gemv(case, out_dtype):
    N, K, g, sym, M = case
    rng = np.random.default_rng(N * 7 + K + M)
    W = rng.standard_normal((N, K)) * 0.02
    W[rng.random(W.shape) < 0.001] = 0.4
    X = rng.standard_normal((M, K))
    run_case(bf16_bits_of(W), bf16_bits_of(X), g, sym, out_dtype)


GEMM_CASES = [
    (256, 512, 128, False, 17),
    (300, 1024, 128, True, 200),     # ragged N and M
    (512, 4096, 128, False, 512),
    (1000, 160, 32, False, 130),     # K tail inside a 64-wide k block
    (264, 768, 256, False, 129),
]


@pytest.mark.parametrize("case", GEMM_CASES, ids=lambda c: "N%d-K%d-g%d-%s-M%d" % (c[0], c[1], c[2], "sym" if c[3] else "asym", c[4]))
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32], ids=["bf16", "fp32"])
def test_gemm(case, out_dtype):
    N, K, g, sym, M = case
    rng = np.random.default_rng(N * 13 + K + M)
    W = rng.standard_normal((N, K)) * 0.02
    X = rng.standard_normal((M, K))
    run_case(bf16_bits_of(W), bf16_bits_of(X), g, sym, out_dtype)


def test_gemm_two_accumulator_tiles_sampled():
    """Enough tiles for the 256-token x 256-channel tile shape; outputs
    compared on a sample of rows and columns."""
    N, K, M = 19000, 256, 512
    rng = np.random.default_rng(5)
    W = bf16_bits_of(rng.standard_normal((N, K)) * 0.02)
    X = bf16_bits_of(rng.standard_normal((M, K)))
    rows = np.sort(rng.choice(M, 64, replace=False))
    cols = np.sort(np.r_[rng.choice(N, 200, replace=False), [0, 255, 256, N - 1]])
    run_case(W, X, 128, False, torch.float32, rows=rows, cols=cols)


@pytest.mark.parametrize("M", [1, 8, 16, 64, 300])
def test_zero_weight_and_one_hot(M):
    b = _b()
    N, K = 96, 512
    W = torch.zeros(N, K, dtype=torch.bfloat16, device="cuda")
    X = torch.randn(M, K, device="cuda").to(torch.bfloat16)
    Y = b.linear_w4a16(X, b.quantize_rtn(W, 128, False), out_dtype=torch.float32)
    assert torch.count_nonzero(Y) == 0
    # a one-hot x picks out one column of x_hat exactly (fp32 output)
    rng = np.random.default_rng(M)
    Wn = bf16_bits_of(rng.standard_normal((N, K)) * 0.02)
    p = b.quantize_rtn(bf16_from_bits(Wn).cuda(), 128, False)
    W_hat = f64_from_bf16_bits(bits16(b.dequantize(p)))
    ks = rng.integers(0, K, M)
    Xo = torch.zeros(M, K, dtype=torch.bfloat16)
    Xo[torch.arange(M), torch.from_numpy(ks)] = 1.0
    Y = b.linear_w4a16(Xo.cuda(), p, out_dtype=torch.float32).cpu().numpy()
    assert np.array_equal(Y.astype(np.float64), W_hat[:, ks].T)


@pytest.mark.parametrize("M", [1, 16, 128])
def test_adversarial_same_sign_products(M):
    """All products positive: |y| = sum |w_hat x|, the tightest case for the
    bound (fp32 output)."""
    rng = np.random.default_rng(99 + M)
    N, K = 256, 4096
    W = np.abs(rng.standard_normal((N, K))) * 0.02 + 0.001
    X = np.abs(rng.standard_normal((M, K))) + 0.01
    run_case(bf16_bits_of(W), bf16_bits_of(X), 128, False, torch.float32)


def test_path_b_cross_check():
    """Cross-check (not the oracle): torch.matmul on the dequantized weights."""
    b = _b()
    rng = np.random.default_rng(3)
    W = bf16_from_bits(bf16_bits_of(rng.standard_normal((512, 2048)) * 0.02)).cuda()
    X = torch.randn(8, 2048, device="cuda").to(torch.bfloat16)
    p = b.quantize_rtn(W, 128, False)
    Y = b.linear_w4a16(X, p, out_dtype=torch.float32)
    Yb = X.float() @ b.dequantize(p).float().T
    A = X.float().abs() @ b.dequantize(p).float().abs().T
    assert torch.all((Y - Yb).abs() <= 1e-3 * A + 1e-6)


def test_bounded_wait_selftest_sets_timeout():
    b = _b()
    b.device_error()
    assert b.wq_selftest_bounded_wait(2000) == b.WQ_OK
    st, flags = b.device_error()
    assert st == b.WQ_ERR_TIMEOUT and flags & b.WQ_DEVFLAG_TIMEOUT
    # the context is still usable afterwards
    W = torch.randn(64, 256, device="cuda").to(torch.bfloat16)
    p = b.quantize_rtn(W, 128, False)
    b.linear_w4a16(torch.randn(1, 256, device="cuda").to(torch.bfloat16), p)
    st, flags = b.device_error()
    assert st == b.WQ_OK and flags == 0


def test_gemv_m1_large_rows_fallback():
    """A single-token GEMV whose per-CTA constants exceed the resident plan
    (many rows per SM) takes the MMA kernel; still within the bound."""
    rng = np.random.default_rng(21)
    N, K = 28672, 1024
    W = bf16_bits_of(rng.standard_normal((N, K)) * 0.02)
    X = bf16_bits_of(rng.standard_normal((1, K)))
    cols = np.sort(rng.choice(N, 300, replace=False))
    run_case(W, X, 128, False, torch.float32, cols=cols)


def test_injected_launch_failure_leaves_outputs_untouched():
    """WQ_FAULT_INJECT=launch in a child process on the GPU: the linear layer
    returns WQ_ERR_CUDA, its output buffer keeps the caller's sentinel and the
    device status stays clean (nothing was enqueued)."""
    import os
    import subprocess
    import sys
    script = r'''
import sys, torch
sys.path.insert(0, sys.argv[1])
from w4a16_bit_gemm_b200 import binding as b
W = torch.randn(256, 512, device="cuda").to(torch.bfloat16)
q = torch.zeros(256, 64, dtype=torch.int32, device="cuda")
s = torch.ones(256, 4, dtype=torch.float16, device="cuda")
z = torch.zeros(256, 4, dtype=torch.float16, device="cuda")
X = torch.randn(1, 512, device="cuda").to(torch.bfloat16)
Y = torch.full((1, 256), 7.0, device="cuda")
st = b.lib.wq_linear_w4a16(X.data_ptr(), 1, q.data_ptr(), s.data_ptr(), z.data_ptr(), 256, 512, 128, 0,
                           Y.data_ptr(), 1, None, 0, torch.cuda.current_stream().cuda_stream)
torch.cuda.synchronize()
print(st, int(b.lib.wq_fault_injections()), bool(torch.all(Y == 7.0)))
'''
    env = dict(os.environ, WQ_FAULT_INJECT="launch")
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", script, root], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    st, n, untouched = r.stdout.split()[-3:]
    assert st == "3" and n == "1" and untouched == "True"
