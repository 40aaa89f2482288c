"""CPU oracle for group-wise RTN weight quantization and the W4A16 linear layer.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The product path
(``w4a16_bit_gemm_b200``) never imports it and shares no code with it.

The arithmetic lives in ``wq_oracle.c`` (plain C, fp32/fp64 with explicit
IEEE 754 conversions written from the standard); this module only builds the
shared object with gcc and marshals numpy arrays through ctypes.

Source pages (title, section):
  * "LLM Quantization: GPTQ, AWQ, SmoothQuant, FP8, KV Cache (7/10)",
    blog.ruahverce.com: "Affine Quantization", "Symmetric and Asymmetric",
    "Per-group", "Memory arithmetic", "Group scale overhead".
  * "Quantization Algorithms" (V10 study notes), brianyu43.github.io:
    section 1.8 "Signed vs Unsigned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "wq_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

FLAG_NONFINITE = 1
FLAG_RANGE = 2


def _compile(out: str, mutant: int = 0) -> None:
    tmp = out + ".tmp%d" % os.getpid()
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
           "-fno-fast-math", "-pthread", "-DWQO_MUTANT=%d" % mutant, _SRC, "-o", tmp, "-lm"]
    subprocess.check_call(cmd)
    os.replace(tmp, out)


def build(force: bool = False) -> str:
    """Compile ``wq_oracle.c`` into ``liboracle.so`` next to it (gcc, -O2,
    strict IEEE: no -ffast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        _compile(_LIB, 0)
    return _LIB


def build_mutant(mutant: int, out_dir: str) -> str:
    """Build a copy of the oracle with one planted mistake (test use only)."""
    out = os.path.join(out_dir, "liboracle_mutant%d.so" % mutant)
    _compile(out, mutant)
    return out


class use_library:
    """Context manager that routes this module's calls to another build of
    the oracle (a planted-mistake variant) and restores the real one."""

    def __init__(self, path: str):
        self.path = path
        self.saved = None

    def __enter__(self):
        global _lib
        _load()
        self.saved = _lib
        _lib = None
        _load(self.path)
        return self

    def __exit__(self, *exc):
        global _lib
        _lib = self.saved
        return False


def _load(path: str | None = None):
    global _lib
    with _lock:
        if _lib is None:
            if path is None:
                build()
            lib = ctypes.CDLL(path or _LIB)
            P = ctypes.c_void_p
            i64 = ctypes.c_int64
            i32 = ctypes.c_int
            lib.wqo_quantize.argtypes = [P, i64, i64, i64, i32, i32, i32, P, P, P, P, i32]
            lib.wqo_quantize.restype = i32
            lib.wqo_pack4.argtypes = [P, i64, i64, P]
            lib.wqo_pack4.restype = i32
            lib.wqo_unpack4.argtypes = [P, i64, i64, i32, P]
            lib.wqo_unpack4.restype = i32
            lib.wqo_dequantize.argtypes = [P, P, P, i64, i64, i64, P, i32]
            lib.wqo_dequantize.restype = i32
            lib.wqo_linear.argtypes = [P, i64, P, i64, i64, P, P, i32]
            lib.wqo_linear.restype = i32
            lib.wqo_artifact_bytes.argtypes = [i64, i32, i64, i32, P, P, P]
            lib.wqo_artifact_bytes.restype = i32
            lib.wqo_f32_to_bf16.argtypes = [ctypes.c_float]
            lib.wqo_f32_to_bf16.restype = ctypes.c_uint16
            lib.wqo_f32_to_f16.argtypes = [ctypes.c_float]
            lib.wqo_f32_to_f16.restype = ctypes.c_uint16
            lib.wqo_f16_to_f32.argtypes = [ctypes.c_uint16]
            lib.wqo_f16_to_f32.restype = ctypes.c_float
            lib.wqo_bf16_to_f32.argtypes = [ctypes.c_uint16]
            lib.wqo_bf16_to_f32.restype = ctypes.c_float
            lib.wqo_dequant_one.argtypes = [ctypes.c_uint16, ctypes.c_int32, ctypes.c_int32]
            lib.wqo_dequant_one.restype = ctypes.c_uint16
            lib.wqo_quantize_clip.argtypes = [P, i64, i64, i64, i32, i32, P, P, P, P, P, i32]
            lib.wqo_quantize_clip.restype = i32
            lib.wqo_quantize_group_range.argtypes = [P, i64, i32, i32, ctypes.c_float, ctypes.c_float,
                                                     ctypes.c_float, P, P, P]
            lib.wqo_quantize_group_range.restype = ctypes.c_uint32
            lib.wqo_group_sq_error.argtypes = [P, i64, P, ctypes.c_uint16, ctypes.c_int32]
            lib.wqo_group_sq_error.restype = ctypes.c_double
            lib.wqo_awq_search.argtypes = [P, i64, i64, P, i64, i64, i32, P, P, P, P, P, P, i32]
            lib.wqo_awq_search.restype = i32
            lib.wqo_awq_scales.argtypes = [P, i64, i64, ctypes.c_double, P]
            lib.wqo_awq_scales.restype = None
            lib.wqo_ln_f64.argtypes = [ctypes.c_double]
            lib.wqo_ln_f64.restype = ctypes.c_double
            lib.wqo_exp_f64.argtypes = [ctypes.c_double]
            lib.wqo_exp_f64.restype = ctypes.c_double
            lib.wqo_pack8.argtypes = [P, i64, i64, P]
            lib.wqo_pack8.restype = i32
            lib.wqo_unpack8.argtypes = [P, i64, i64, P]
            lib.wqo_unpack8.restype = i32
            lib.wqo_gptq.argtypes = [P, i64, i64, P, i64, i64, i32, i32, P, P, P, P, P, P, i32]
            lib.wqo_gptq.restype = i32
            lib.wqo_gptq_factor.argtypes = [P, i64, i64, i32, P, P, i32]
            lib.wqo_gptq_factor.restype = ctypes.c_uint32
            lib.wqo_clip_alpha.argtypes = [i32]
            lib.wqo_clip_alpha.restype = ctypes.c_float
            for nm in ("wqo_f32_to_f16_array", "wqo_f32_to_bf16_array", "wqo_f16_to_f32_array"):
                getattr(lib, nm).argtypes = [P, i64, P]
                getattr(lib, nm).restype = None
            _lib = lib
    return _lib


def _ptr(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def default_threads() -> int:
    return os.cpu_count() or 1


# --------------------------------------------------------------------------
# scalar conversions (exposed for pins)
# --------------------------------------------------------------------------

def f32_to_bf16_bits(x: float) -> int:
    return int(_load().wqo_f32_to_bf16(float(x)))


def f32_to_f16_bits(x: float) -> int:
    return int(_load().wqo_f32_to_f16(float(x)))


def f16_bits_to_f32(h: int) -> float:
    return float(_load().wqo_f16_to_f32(int(h)))


def bf16_bits_to_f32(h: int) -> float:
    return float(_load().wqo_bf16_to_f32(int(h)))


def dequant_one(s16: int, q: int, z: int) -> int:
    return int(_load().wqo_dequant_one(int(s16), int(q), int(z)))


def f32_to_f16_bits_array(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, np.uint16)
    _load().wqo_f32_to_f16_array(_ptr(x), x.size, _ptr(out))
    return out


def f32_to_bf16_bits_array(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    out = np.empty(x.shape, np.uint16)
    _load().wqo_f32_to_bf16_array(_ptr(x), x.size, _ptr(out))
    return out


def f16_bits_to_f32_array(h: np.ndarray) -> np.ndarray:
    h = np.ascontiguousarray(h, dtype=np.uint16)
    out = np.empty(h.shape, np.float32)
    _load().wqo_f16_to_f32_array(_ptr(h), h.size, _ptr(out))
    return out


# --------------------------------------------------------------------------
# array operations; bf16/fp16 tensors are carried as uint16 bit patterns
# --------------------------------------------------------------------------

def quantize(W_bits: np.ndarray, group_size: int, bits: int = 4, symmetric: bool = False,
             narrow: bool = False, nthreads: int | None = None):
    """Group-wise RTN quantization of bf16 weights ``W_bits`` (uint16 [d_out, d_in]).

    Returns ``(codes int32 [d_out,d_in], scales uint16 [d_out,G], zeros uint16
    [d_out,G] or None, flags)``.
    """
    W_bits = np.ascontiguousarray(W_bits, dtype=np.uint16)
    d_out, d_in = W_bits.shape
    G = d_in // group_size
    codes = np.empty((d_out, d_in), np.int32)
    scales = np.empty((d_out, G), np.uint16)
    zeros = None if symmetric else np.empty((d_out, G), np.uint16)
    flags = ctypes.c_uint32(0)
    rc = _load().wqo_quantize(_ptr(W_bits), d_out, d_in, group_size, bits, int(symmetric),
                              int(narrow), _ptr(codes), _ptr(scales),
                              _ptr(zeros) if zeros is not None else None,
                              ctypes.cast(ctypes.pointer(flags), ctypes.c_void_p),
                              nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle quantize rejected its arguments")
    return codes, scales, zeros, int(flags.value)


CLIP_CANDIDATES = 11


def quantize_clip(W_bits: np.ndarray, group_size: int, symmetric: bool = False, bits: int = 4,
                  nthreads: int | None = None):
    """Group-wise quantization with the MSE-optimal clipping search
    ([P1 Clipping Trade-off]; [P2 calibration 4, MSE-optimal]).

    Returns ``(codes, scales, zeros or None, flags, best)`` with ``best`` the
    chosen candidate index per group (uint8 [d_out, G]; alpha = clip_alpha(i)).
    """
    W_bits = np.ascontiguousarray(W_bits, dtype=np.uint16)
    d_out, d_in = W_bits.shape
    G = d_in // group_size
    codes = np.empty((d_out, d_in), np.int32)
    scales = np.empty((d_out, G), np.uint16)
    zeros = None if symmetric else np.empty((d_out, G), np.uint16)
    best = np.empty((d_out, G), np.uint8)
    flags = ctypes.c_uint32(0)
    rc = _load().wqo_quantize_clip(_ptr(W_bits), d_out, d_in, group_size, bits, int(symmetric), _ptr(codes),
                                   _ptr(scales), _ptr(zeros) if zeros is not None else None, _ptr(best),
                                   ctypes.cast(ctypes.pointer(flags), ctypes.c_void_p),
                                   nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle clip quantize rejected its arguments")
    return codes, scales, zeros, int(flags.value), best


def quantize_clip_pack4(W_bits: np.ndarray, group_size: int = 128, symmetric: bool = False,
                        nthreads: int | None = None):
    """quantize_clip + pack4: (qweight, scales, zeros, flags, codes, best)."""
    codes, scales, zeros, flags, best = quantize_clip(W_bits, group_size, symmetric, nthreads=nthreads)
    return pack4(codes), scales, zeros, flags, codes, best


def clip_alpha(i: int) -> float:
    return float(_load().wqo_clip_alpha(int(i)))


def quantize_group_range(x_bits: np.ndarray, lo: float, hi: float, amax: float, symmetric: bool = False,
                         bits: int = 4):
    """One group quantized on a given range: (codes int32, s16, z, flags)."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    codes = np.empty(x_bits.shape[0], np.int32)
    s16 = ctypes.c_uint16(0)
    z = ctypes.c_int32(0)
    f = _load().wqo_quantize_group_range(_ptr(x_bits), x_bits.shape[0], bits, int(symmetric), lo, hi, amax,
                                         _ptr(codes), ctypes.cast(ctypes.pointer(s16), ctypes.c_void_p),
                                         ctypes.cast(ctypes.pointer(z), ctypes.c_void_p))
    return codes, int(s16.value), int(z.value), int(f)


def group_sq_error(x_bits: np.ndarray, codes: np.ndarray, s16: int, z: int) -> float:
    """The oracle's fp64 squared reconstruction error of one group."""
    x_bits = np.ascontiguousarray(x_bits, dtype=np.uint16)
    codes = np.ascontiguousarray(codes, dtype=np.int32)
    return float(_load().wqo_group_sq_error(_ptr(x_bits), x_bits.shape[0], _ptr(codes), s16, z))


AWQ_ALPHAS = 11


def awq_search(W_bits: np.ndarray, X_bits: np.ndarray, group_size: int = 128, symmetric: bool = False,
               nthreads: int | None = None):
    """AWQ per-input-channel scaling search ([P2] AWQ procedure).

    W_bits bf16 [N, K], X_bits bf16 calibration [T, K].  Returns ``(codes,
    scales, zeros or None, s_bf16 [K], losses [11], best)``: the RTN artifact
    of W diag(s) for the best alpha = best / 10, its per-channel scales s
    (bf16 bits; the linear layer then takes x / s) and every alpha's loss.
    """
    W_bits = np.ascontiguousarray(W_bits, dtype=np.uint16)
    X_bits = np.ascontiguousarray(X_bits, dtype=np.uint16)
    N, K = W_bits.shape
    T = X_bits.shape[0]
    G = K // group_size
    codes = np.empty((N, K), np.int32)
    scales = np.empty((N, G), np.uint16)
    zeros = None if symmetric else np.empty((N, G), np.uint16)
    s = np.empty(K, np.uint16)
    losses = np.empty(AWQ_ALPHAS, np.float64)
    best = ctypes.c_int32(-1)
    rc = _load().wqo_awq_search(_ptr(W_bits), N, K, _ptr(X_bits), T, group_size, int(symmetric), _ptr(codes),
                                _ptr(scales), _ptr(zeros) if zeros is not None else None, _ptr(s), _ptr(losses),
                                ctypes.cast(ctypes.pointer(best), ctypes.c_void_p), nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle AWQ search rejected its arguments")
    return codes, scales, zeros, s, losses, int(best.value)


def ln_f64(x: float) -> float:
    """ln x by the fixed fp64 procedure of the AWQ scales (x positive, normal)."""
    return _load().wqo_ln_f64(float(x))


def exp_f64(x: float) -> float:
    """e^x by the fixed fp64 procedure of the AWQ scales (|x| < 700)."""
    return _load().wqo_exp_f64(float(x))


def awq_scales(X_bits: np.ndarray, alpha: float) -> np.ndarray:
    """Per-channel AWQ scales (bf16 bits [K]) for one alpha."""
    X_bits = np.ascontiguousarray(X_bits, dtype=np.uint16)
    T, K = X_bits.shape
    s = np.empty(K, np.uint16)
    _load().wqo_awq_scales(_ptr(X_bits), T, K, float(alpha), _ptr(s))
    return s


GPTQ_BLOCK = 128


def gptq(W_bits: np.ndarray, X_bits: np.ndarray, group_size: int = 128, symmetric: bool = True,
         act_order: bool = True, want_factor: bool = False, nthreads: int | None = None):
    """GPTQ error feedback ([P2] GPTQ chapter and its algorithm; settings
    default to the page's: 4-bit, group 128, symmetric, act-order on).

    W_bits bf16 [N, K], X_bits bf16 calibration [T, K].  Returns ``(codes
    [N, K] original column order, scales, zeros or None, perm [K], U [K, K] or
    None, flags)``; scales/zeros are plain RTN's (static group parameters)."""
    W_bits = np.ascontiguousarray(W_bits, dtype=np.uint16)
    X_bits = np.ascontiguousarray(X_bits, dtype=np.uint16)
    N, K = W_bits.shape
    T = X_bits.shape[0]
    G = K // group_size
    codes = np.empty((N, K), np.int32)
    scales = np.empty((N, G), np.uint16)
    zeros = None if symmetric else np.empty((N, G), np.uint16)
    perm = np.empty(K, np.int32)
    U = np.empty((K, K), np.float64) if want_factor else None
    flags = ctypes.c_uint32(0)
    rc = _load().wqo_gptq(_ptr(W_bits), N, K, _ptr(X_bits), T, group_size, int(symmetric), int(act_order),
                          _ptr(codes), _ptr(scales), _ptr(zeros) if zeros is not None else None, _ptr(perm),
                          _ptr(U) if U is not None else None, ctypes.cast(ctypes.pointer(flags), ctypes.c_void_p),
                          nthreads or default_threads())
    if rc != 0:
        raise ValueError("oracle GPTQ rejected its arguments")
    return codes, scales, zeros, perm, U, int(flags.value)


def gptq_factor(X_bits: np.ndarray, act_order: bool = True, nthreads: int | None = None):
    """(perm [K], U [K, K], flags): processing order and the upper factor of
    the inverse of the permuted damped Hessian 2 X^T X."""
    X_bits = np.ascontiguousarray(X_bits, dtype=np.uint16)
    T, K = X_bits.shape
    perm = np.empty(K, np.int32)
    U = np.empty((K, K), np.float64)
    f = _load().wqo_gptq_factor(_ptr(X_bits), T, K, int(act_order), _ptr(perm), _ptr(U),
                                nthreads or default_threads())
    return perm, U, int(f)


def pack4(codes: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.int32)
    d_out, d_in = codes.shape
    q = np.empty((d_out, d_in // 8), np.uint32)
    if _load().wqo_pack4(_ptr(codes), d_out, d_in, _ptr(q)) != 0:
        raise ValueError("oracle pack4 rejected its arguments")
    return q


def unpack4(qweight: np.ndarray, d_in: int, symmetric: bool) -> np.ndarray:
    qweight = np.ascontiguousarray(qweight, dtype=np.uint32)
    d_out = qweight.shape[0]
    codes = np.empty((d_out, d_in), np.int32)
    if _load().wqo_unpack4(_ptr(qweight), d_out, d_in, int(symmetric), _ptr(codes)) != 0:
        raise ValueError("oracle unpack4 rejected its arguments")
    return codes


def pack8(codes: np.ndarray) -> np.ndarray:
    """4 signed 8-bit codes per uint32, low byte first."""
    codes = np.ascontiguousarray(codes, dtype=np.int32)
    d_out, d_in = codes.shape
    q = np.empty((d_out, d_in // 4), np.uint32)
    if _load().wqo_pack8(_ptr(codes), d_out, d_in, _ptr(q)) != 0:
        raise ValueError("oracle pack8 rejected its arguments")
    return q


def unpack8(qweight: np.ndarray, d_in: int) -> np.ndarray:
    qweight = np.ascontiguousarray(qweight, dtype=np.uint32)
    d_out = qweight.shape[0]
    codes = np.empty((d_out, d_in), np.int32)
    if _load().wqo_unpack8(_ptr(qweight), d_out, d_in, _ptr(codes)) != 0:
        raise ValueError("oracle unpack8 rejected its arguments")
    return codes


def quantize_pack8(W_bits: np.ndarray, group_size: int, nthreads: int | None = None):
    """Symmetric INT8 ([-127, 127]) quantize + pack: ``(qweight uint32
    [d_out, d_in/4], scales, flags, codes)``."""
    codes, scales, _, flags = quantize(W_bits, group_size, 8, True, True, nthreads)
    return pack8(codes), scales, flags, codes


def dequantize(codes: np.ndarray, scales: np.ndarray, zeros, group_size: int,
               nthreads: int | None = None) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.int32)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    d_out, d_in = codes.shape
    out = np.empty((d_out, d_in), np.uint16)
    zp = None
    if zeros is not None:
        zeros = np.ascontiguousarray(zeros, dtype=np.uint16)
        zp = _ptr(zeros)
    if _load().wqo_dequantize(_ptr(codes), _ptr(scales), zp, d_out, d_in, group_size,
                              _ptr(out), nthreads or default_threads()) != 0:
        raise ValueError("oracle dequantize rejected its arguments")
    return out


def linear(X_bits: np.ndarray, W_hat_bits: np.ndarray, nthreads: int | None = None):
    """fp64 ``Y[m,n] = sum_k W_hat[n,k] X[m,k]`` and ``A[m,n] = sum_k |W_hat X|``."""
    X_bits = np.ascontiguousarray(X_bits, dtype=np.uint16)
    W_hat_bits = np.ascontiguousarray(W_hat_bits, dtype=np.uint16)
    M, K = X_bits.shape
    N, K2 = W_hat_bits.shape
    if K != K2:
        raise ValueError("inner dimensions differ")
    Y = np.empty((M, N), np.float64)
    A = np.empty((M, N), np.float64)
    if _load().wqo_linear(_ptr(X_bits), M, _ptr(W_hat_bits), N, K, _ptr(Y), _ptr(A),
                          nthreads or default_threads()) != 0:
        raise ValueError("oracle linear rejected its arguments")
    return Y, A


def artifact_bytes(params: int, bits: int, group_size: int, symmetric: bool):
    """(payload, scale bytes, zero bytes) of a packed artifact."""
    p, s, z = ctypes.c_double(), ctypes.c_double(), ctypes.c_double()
    _load().wqo_artifact_bytes(int(params), int(bits), int(group_size), int(symmetric),
                               ctypes.cast(ctypes.pointer(p), ctypes.c_void_p),
                               ctypes.cast(ctypes.pointer(s), ctypes.c_void_p),
                               ctypes.cast(ctypes.pointer(z), ctypes.c_void_p))
    return p.value, s.value, z.value


def quantize_pack4(W_bits: np.ndarray, group_size: int = 128, symmetric: bool = False,
                   nthreads: int | None = None):
    """4-bit quantize + pack: ``(qweight uint32 [d_out,d_in/8], scales, zeros, flags, codes)``."""
    codes, scales, zeros, flags = quantize(W_bits, group_size, 4, symmetric, False, nthreads)
    return pack4(codes), scales, zeros, flags, codes


def reference_linear_w4a16(X_bits, W_bits, group_size=128, symmetric=False, nthreads=None):
    """Whole path on the CPU: quantize, dequantize, fp64 linear.  Returns
    ``(Y, A, W_hat_bits, (qweight, scales, zeros, flags))``."""
    qweight, scales, zeros, flags, codes = quantize_pack4(W_bits, group_size, symmetric, nthreads)
    W_hat = dequantize(codes, scales, zeros, group_size, nthreads)
    Y, A = linear(X_bits, W_hat, nthreads)
    return Y, A, W_hat, (qweight, scales, zeros, flags)
