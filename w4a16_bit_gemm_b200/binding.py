"""Thin ctypes binding of libwq (include/wq.h).

Argument marshalling only: every step of quantize, dequantize and the W4A16
linear layer runs in the CUDA kernels of libwq.so.  PyTorch supplies device
memory and the current stream.  Importing this module raises if libwq.so is
missing: there is no CPU or PyTorch fallback.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libwq.so")

WQ_OK = 0
WQ_ERR_INVALID_ARG = 1
WQ_ERR_UNSUPPORTED = 2
WQ_ERR_CUDA = 3
WQ_ERR_NONFINITE = 4
WQ_ERR_TIMEOUT = 5
WQ_ERR_RANGE = 6

WQ_DEVFLAG_NONFINITE = 0x1
WQ_DEVFLAG_RANGE = 0x2
WQ_DEVFLAG_TIMEOUT = 0x4

WQ_OUT_BF16 = 0
WQ_OUT_FP32 = 1


class WQError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_string(status)} ({status})")
        self.status = status


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"libwq.so not found at {LIB_PATH}; build it with `python -m w4a16_bit_gemm_b200.build` "
            "(there is no fallback path)")
    lib = ctypes.CDLL(LIB_PATH)
    P, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
    lib.wq_abi_version.argtypes = []
    lib.wq_abi_version.restype = i32
    lib.wq_status_string.argtypes = [ctypes.c_int]
    lib.wq_status_string.restype = ctypes.c_char_p
    lib.wq_quantize_rtn.argtypes = [P, i64, i64, i32, i32, P, P, P, P]
    lib.wq_quantize_rtn.restype = ctypes.c_int
    lib.wq_quantize_clip_mse.argtypes = [P, i64, i64, i32, i32, P, P, P, P]
    lib.wq_quantize_clip_mse.restype = ctypes.c_int
    lib.wq_dequantize.argtypes = [P, P, P, i64, i64, i32, i32, P, P]
    lib.wq_dequantize.restype = ctypes.c_int
    lib.wq_linear_w4a16.argtypes = [P, i64, P, P, P, i64, i64, i32, i32, P, i32, P, sz, P]
    lib.wq_linear_w4a16.restype = ctypes.c_int
    lib.wq_linear_workspace_bytes.argtypes = [i64, i64, i64]
    lib.wq_linear_workspace_bytes.restype = sz
    lib.wq_awq_search.argtypes = [P, i64, i64, P, i64, i32, i32, P, P, P, P, P, P, P, sz, P]
    lib.wq_awq_search.restype = ctypes.c_int
    lib.wq_awq_workspace_bytes.argtypes = [i64, i64, i64, i32]
    lib.wq_awq_workspace_bytes.restype = sz
    lib.wq_awq_search_static.argtypes = [P, i64, i64, P, i64, i32, i32, P, P, P, P, P, P, P]
    lib.wq_awq_search_static.restype = ctypes.c_int
    lib.wq_awq_static_scratch_bytes.argtypes = []
    lib.wq_awq_static_scratch_bytes.restype = sz
    lib.wq_awq_scale_activations.argtypes = [P, i64, i64, P, P, P]
    lib.wq_awq_scale_activations.restype = ctypes.c_int
    lib.wq_quantize_w8.argtypes = [P, i64, i64, i32, P, P, P]
    lib.wq_quantize_w8.restype = ctypes.c_int
    lib.wq_dequantize_w8.argtypes = [P, P, i64, i64, i32, P, P]
    lib.wq_dequantize_w8.restype = ctypes.c_int
    lib.wq_linear_w8a16.argtypes = [P, i64, P, P, i64, i64, i32, P, i32, P]
    lib.wq_linear_w8a16.restype = ctypes.c_int
    lib.wq_gptq.argtypes = [P, i64, i64, P, i64, i32, i32, i32, P, P, P, P, P, sz, P]
    lib.wq_gptq.restype = ctypes.c_int
    lib.wq_gptq_workspace_bytes.argtypes = [i64, i64]
    lib.wq_gptq_workspace_bytes.restype = sz
    lib.wq_get_device_error.argtypes = [P, P]
    lib.wq_get_device_error.restype = ctypes.c_int
    lib.wq_selftest_bounded_wait.argtypes = [ctypes.c_uint32, P]
    lib.wq_selftest_bounded_wait.restype = ctypes.c_int
    lib.wq_fault_injections.argtypes = []
    lib.wq_fault_injections.restype = ctypes.c_uint64
    return lib


lib = _load()


def status_string(status: int) -> str:
    return lib.wq_status_string(int(status)).decode()


def _ptr(t) -> int | None:
    if t is None:
        return None
    return t.data_ptr()


def _stream(stream=None) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _check(status: int, what: str):
    if status != WQ_OK:
        raise WQError(status, what)


def _require_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("libwq takes CUDA tensors only (no CPU fallback)")


# ---------------------------------------------------------------------------
# Raw C-ABI calls (same names as include/wq.h); arguments are tensors or None.
# ---------------------------------------------------------------------------

def wq_quantize_rtn(W, d_out, d_in, group_size, symmetric, qweight, scales, zeros, stream=None) -> int:
    return lib.wq_quantize_rtn(_ptr(W), d_out, d_in, group_size, int(symmetric), _ptr(qweight), _ptr(scales),
                               _ptr(zeros), _stream(stream))


def wq_quantize_clip_mse(W, d_out, d_in, group_size, symmetric, qweight, scales, zeros, stream=None) -> int:
    return lib.wq_quantize_clip_mse(_ptr(W), d_out, d_in, group_size, int(symmetric), _ptr(qweight),
                                    _ptr(scales), _ptr(zeros), _stream(stream))


def wq_dequantize(qweight, scales, zeros, d_out, d_in, group_size, symmetric, W_hat, stream=None) -> int:
    return lib.wq_dequantize(_ptr(qweight), _ptr(scales), _ptr(zeros), d_out, d_in, group_size, int(symmetric),
                             _ptr(W_hat), _stream(stream))


def wq_linear_w4a16(X, M, qweight, scales, zeros, d_out, d_in, group_size, symmetric, Y, y_dtype, workspace=None,
                    workspace_bytes=0, stream=None) -> int:
    return lib.wq_linear_w4a16(_ptr(X), M, _ptr(qweight), _ptr(scales), _ptr(zeros), d_out, d_in, group_size,
                               int(symmetric), _ptr(Y), y_dtype, _ptr(workspace), workspace_bytes, _stream(stream))


def wq_awq_search(W, d_out, d_in, X, T, group_size, symmetric, qweight, scales, zeros, s, losses, best, workspace,
                  workspace_bytes, stream=None) -> int:
    return lib.wq_awq_search(_ptr(W), d_out, d_in, _ptr(X), T, group_size, int(symmetric), _ptr(qweight),
                             _ptr(scales), _ptr(zeros), _ptr(s), _ptr(losses), _ptr(best), _ptr(workspace),
                             workspace_bytes, _stream(stream))


def wq_awq_search_static(W, d_out, d_in, X, T, group_size, symmetric, qweight, scales, zeros, s, losses, best,
                         stream=None) -> int:
    return lib.wq_awq_search_static(_ptr(W), d_out, d_in, _ptr(X), T, group_size, int(symmetric), _ptr(qweight),
                                    _ptr(scales), _ptr(zeros), _ptr(s), _ptr(losses), _ptr(best), _stream(stream))


def wq_awq_workspace_bytes(d_out, d_in, T, group_size) -> int:
    return int(lib.wq_awq_workspace_bytes(d_out, d_in, T, group_size))


def wq_awq_scale_activations(X, T, d_in, s, Xp, stream=None) -> int:
    return lib.wq_awq_scale_activations(_ptr(X), T, d_in, _ptr(s), _ptr(Xp), _stream(stream))


def wq_quantize_w8(W, d_out, d_in, group_size, qweight, scales, stream=None) -> int:
    return lib.wq_quantize_w8(_ptr(W), d_out, d_in, group_size, _ptr(qweight), _ptr(scales), _stream(stream))


def wq_dequantize_w8(qweight, scales, d_out, d_in, group_size, W_hat, stream=None) -> int:
    return lib.wq_dequantize_w8(_ptr(qweight), _ptr(scales), d_out, d_in, group_size, _ptr(W_hat), _stream(stream))


def wq_linear_w8a16(X, M, qweight, scales, d_out, d_in, group_size, Y, y_dtype, stream=None) -> int:
    return lib.wq_linear_w8a16(_ptr(X), M, _ptr(qweight), _ptr(scales), d_out, d_in, group_size, _ptr(Y), y_dtype,
                               _stream(stream))


def wq_gptq(W, d_out, d_in, X, T, group_size, symmetric, act_order, qweight, scales, zeros, perm, workspace,
            workspace_bytes, stream=None) -> int:
    return lib.wq_gptq(_ptr(W), d_out, d_in, _ptr(X), T, group_size, int(symmetric), int(act_order), _ptr(qweight),
                       _ptr(scales), _ptr(zeros), _ptr(perm), _ptr(workspace), workspace_bytes, _stream(stream))


def wq_gptq_workspace_bytes(d_out, d_in) -> int:
    return int(lib.wq_gptq_workspace_bytes(d_out, d_in))


def wq_linear_workspace_bytes(M, d_out, d_in) -> int:
    return int(lib.wq_linear_workspace_bytes(M, d_out, d_in))


def wq_selftest_bounded_wait(limit_us: int, stream=None) -> int:
    return lib.wq_selftest_bounded_wait(int(limit_us), _stream(stream))


def wq_get_device_error(stream=None):
    flags = ctypes.c_uint32(0)
    st = lib.wq_get_device_error(ctypes.addressof(flags), _stream(stream))
    return st, int(flags.value)


# ---------------------------------------------------------------------------
# Tensor-level helpers (allocation with torch, then one C-ABI call)
# ---------------------------------------------------------------------------

class PackedLinear:
    """Packed 4-bit artifact (layout v1) of one weight matrix W[d_out, d_in]."""

    def __init__(self, qweight, scales, zeros, d_out, d_in, group_size, symmetric):
        self.qweight = qweight
        self.scales = scales
        self.zeros = zeros
        self.d_out = d_out
        self.d_in = d_in
        self.group_size = group_size
        self.symmetric = bool(symmetric)

    def nbytes(self) -> int:
        n = self.qweight.numel() * 4 + self.scales.numel() * 2
        if self.zeros is not None:
            n += self.zeros.numel() * 2
        return n


def alloc_packed(d_out: int, d_in: int, group_size: int = 128, symmetric: bool = False, device="cuda"):
    G = d_in // group_size
    qweight = torch.empty(d_out, d_in // 8, dtype=torch.int32, device=device)
    scales = torch.empty(d_out, G, dtype=torch.float16, device=device)
    zeros = None if symmetric else torch.empty(d_out, G, dtype=torch.float16, device=device)
    return PackedLinear(qweight, scales, zeros, d_out, d_in, group_size, symmetric)


def quantize_rtn(W: torch.Tensor, group_size: int = 128, symmetric: bool = False, out: PackedLinear | None = None,
                 stream=None) -> PackedLinear:
    """Group-wise RTN quantization of bf16 W[d_out, d_in] into a packed artifact."""
    _require_cuda(W)
    if W.dtype != torch.bfloat16 or W.dim() != 2 or not W.is_contiguous():
        raise ValueError("W must be a contiguous 2-D bf16 CUDA tensor")
    d_out, d_in = W.shape
    if out is None:
        if d_in % group_size != 0:
            raise ValueError("group_size must divide d_in")
        out = alloc_packed(d_out, d_in, group_size, symmetric, W.device)
    _check(wq_quantize_rtn(W, d_out, d_in, group_size, symmetric, out.qweight, out.scales, out.zeros, stream),
           "wq_quantize_rtn")
    return out


def quantize_clip_mse(W: torch.Tensor, group_size: int = 128, symmetric: bool = False,
                      out: PackedLinear | None = None, stream=None) -> PackedLinear:
    """Group-wise quantization with the per-group MSE-optimal clipping search;
    same artifact format as quantize_rtn."""
    _require_cuda(W)
    if W.dtype != torch.bfloat16 or W.dim() != 2 or not W.is_contiguous():
        raise ValueError("W must be a contiguous 2-D bf16 CUDA tensor")
    d_out, d_in = W.shape
    if out is None:
        if d_in % group_size != 0:
            raise ValueError("group_size must divide d_in")
        out = alloc_packed(d_out, d_in, group_size, symmetric, W.device)
    _check(wq_quantize_clip_mse(W, d_out, d_in, group_size, symmetric, out.qweight, out.scales, out.zeros, stream),
           "wq_quantize_clip_mse")
    return out


class PackedLinearW8:
    """Symmetric INT8 artifact (layout w8 v1) of one weight matrix W[d_out, d_in]."""

    def __init__(self, qweight, scales, d_out, d_in, group_size):
        self.qweight = qweight
        self.scales = scales
        self.d_out = d_out
        self.d_in = d_in
        self.group_size = group_size

    def nbytes(self) -> int:
        return self.qweight.numel() * 4 + self.scales.numel() * 2


def quantize_w8(W: torch.Tensor, group_size: int | None = None, out: PackedLinearW8 | None = None,
                stream=None) -> PackedLinearW8:
    """Symmetric INT8 quantization of bf16 W[d_out, d_in]; group_size None or
    d_in = per-channel (one scale per output row)."""
    _require_cuda(W)
    if W.dtype != torch.bfloat16 or W.dim() != 2 or not W.is_contiguous():
        raise ValueError("W must be a contiguous 2-D bf16 CUDA tensor")
    d_out, d_in = W.shape
    g = d_in if group_size is None else group_size
    if out is None:
        if d_in % g != 0:
            raise ValueError("group_size must divide d_in")
        out = PackedLinearW8(torch.empty(d_out, d_in // 4, dtype=torch.int32, device=W.device),
                             torch.empty(d_out, d_in // g, dtype=torch.float16, device=W.device), d_out, d_in, g)
    _check(wq_quantize_w8(W, d_out, d_in, g, out.qweight, out.scales, stream), "wq_quantize_w8")
    return out


def dequantize_w8(p: PackedLinearW8, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    _require_cuda(p.qweight)
    if out is None:
        out = torch.empty(p.d_out, p.d_in, dtype=torch.bfloat16, device=p.qweight.device)
    _check(wq_dequantize_w8(p.qweight, p.scales, p.d_out, p.d_in, p.group_size, out, stream), "wq_dequantize_w8")
    return out


def linear_w8a16(X: torch.Tensor, p: PackedLinearW8, out_dtype=torch.bfloat16, out: torch.Tensor | None = None,
                 stream=None) -> torch.Tensor:
    """Y[M, d_out] = X[M, d_in] . x_hat^T with fp32 accumulation (INT8 weights)."""
    _require_cuda(X, p.qweight)
    if X.dtype != torch.bfloat16 or X.dim() != 2 or not X.is_contiguous() or X.shape[1] != p.d_in:
        raise ValueError("X must be a contiguous [M, d_in] bf16 CUDA tensor")
    y_dtype = WQ_OUT_FP32 if out_dtype == torch.float32 else WQ_OUT_BF16
    if out is None:
        out = torch.empty(X.shape[0], p.d_out, dtype=torch.float32 if y_dtype == WQ_OUT_FP32 else torch.bfloat16,
                          device=X.device)
    _check(wq_linear_w8a16(X, X.shape[0], p.qweight, p.scales, p.d_out, p.d_in, p.group_size, out, y_dtype, stream),
           "wq_linear_w8a16")
    return out


class AWQResult:
    """Output of awq_search: the artifact of W diag(s), the per-input-channel
    scales s (bf16 [d_in]), the 11 losses (fp64, device) and the kept index
    (int32, device; alpha = index / 10)."""

    def __init__(self, packed, s, losses, best):
        self.packed = packed
        self.s = s
        self.losses = losses
        self.best = best


def awq_search(W: torch.Tensor, X: torch.Tensor, group_size: int = 128, symmetric: bool = False,
               workspace: torch.Tensor | None = None, stream=None) -> AWQResult:
    """AWQ per-input-channel scaling search over alpha = 0, 0.1, ..., 1 on the
    calibration activations X[T, d_in], then RTN of W diag(s)."""
    _require_cuda(W, X)
    if W.dtype != torch.bfloat16 or W.dim() != 2 or not W.is_contiguous():
        raise ValueError("W must be a contiguous 2-D bf16 CUDA tensor")
    if X.dtype != torch.bfloat16 or X.dim() != 2 or not X.is_contiguous() or X.shape[1] != W.shape[1]:
        raise ValueError("X must be a contiguous [T, d_in] bf16 CUDA tensor")
    d_out, d_in = W.shape
    T = X.shape[0]
    if d_in % group_size != 0:
        raise ValueError("group_size must divide d_in")
    out = alloc_packed(d_out, d_in, group_size, symmetric, W.device)
    s = torch.empty(d_in, dtype=torch.bfloat16, device=W.device)
    losses = torch.empty(11, dtype=torch.float64, device=W.device)
    best = torch.empty(1, dtype=torch.int32, device=W.device)
    need = wq_awq_workspace_bytes(d_out, d_in, T, group_size)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=W.device)
    _check(wq_awq_search(W, d_out, d_in, X, T, group_size, symmetric, out.qweight, out.scales, out.zeros, s, losses,
                         best, workspace, workspace.numel() * workspace.element_size(), stream), "wq_awq_search")
    return AWQResult(out, s, losses, best)


def gptq(W: torch.Tensor, X: torch.Tensor, group_size: int = 128, symmetric: bool = True, act_order: bool = True,
         workspace: torch.Tensor | None = None, stream=None):
    """GPTQ of bf16 W[d_out, d_in] with calibration activations X[T, d_in]
    (defaults: the page's symmetric, group 128, act-order).  Returns
    (PackedLinear, perm) with perm the int32 processing order."""
    _require_cuda(W, X)
    if W.dtype != torch.bfloat16 or W.dim() != 2 or not W.is_contiguous():
        raise ValueError("W must be a contiguous 2-D bf16 CUDA tensor")
    if X.dtype != torch.bfloat16 or X.dim() != 2 or not X.is_contiguous() or X.shape[1] != W.shape[1]:
        raise ValueError("X must be a contiguous [T, d_in] bf16 CUDA tensor")
    d_out, d_in = W.shape
    if d_in % group_size != 0:
        raise ValueError("group_size must divide d_in")
    out = alloc_packed(d_out, d_in, group_size, symmetric, W.device)
    perm = torch.empty(d_in, dtype=torch.int32, device=W.device)
    need = wq_gptq_workspace_bytes(d_out, d_in)
    if workspace is None or workspace.numel() * workspace.element_size() < need:
        workspace = torch.empty(need, dtype=torch.uint8, device=W.device)
    _check(wq_gptq(W, d_out, d_in, X, X.shape[0], group_size, symmetric, act_order, out.qweight, out.scales,
                   out.zeros, perm, workspace, workspace.numel() * workspace.element_size(), stream), "wq_gptq")
    return out, perm


def awq_search_static(W: torch.Tensor, X: torch.Tensor, group_size: int = 128, symmetric: bool = False,
                      stream=None) -> AWQResult:
    """awq_search with the library-owned scratch instead of a workspace tensor."""
    _require_cuda(W, X)
    if W.dtype != torch.bfloat16 or W.dim() != 2 or not W.is_contiguous():
        raise ValueError("W must be a contiguous 2-D bf16 CUDA tensor")
    if X.dtype != torch.bfloat16 or X.dim() != 2 or not X.is_contiguous() or X.shape[1] != W.shape[1]:
        raise ValueError("X must be a contiguous [T, d_in] bf16 CUDA tensor")
    d_out, d_in = W.shape
    if d_in % group_size != 0:
        raise ValueError("group_size must divide d_in")
    out = alloc_packed(d_out, d_in, group_size, symmetric, W.device)
    s = torch.empty(d_in, dtype=torch.bfloat16, device=W.device)
    losses = torch.empty(11, dtype=torch.float64, device=W.device)
    best = torch.empty(1, dtype=torch.int32, device=W.device)
    _check(wq_awq_search_static(W, d_out, d_in, X, X.shape[0], group_size, symmetric, out.qweight, out.scales,
                                out.zeros, s, losses, best, stream), "wq_awq_search_static")
    return AWQResult(out, s, losses, best)


def awq_scale_activations(X: torch.Tensor, s: torch.Tensor, out: torch.Tensor | None = None,
                          stream=None) -> torch.Tensor:
    """X' = bf16(X / s) per input channel (the activation side of AWQ)."""
    _require_cuda(X, s)
    if X.dtype != torch.bfloat16 or X.dim() != 2 or not X.is_contiguous() or s.numel() != X.shape[1]:
        raise ValueError("X must be a contiguous [T, d_in] bf16 CUDA tensor and s a [d_in] bf16 tensor")
    if out is None:
        out = torch.empty_like(X)
    _check(wq_awq_scale_activations(X, X.shape[0], X.shape[1], s, out, stream), "wq_awq_scale_activations")
    return out


def dequantize(p: PackedLinear, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """x_hat = bf16_rn(s (q - z)) for every weight of the artifact."""
    _require_cuda(p.qweight)
    if out is None:
        out = torch.empty(p.d_out, p.d_in, dtype=torch.bfloat16, device=p.qweight.device)
    _check(wq_dequantize(p.qweight, p.scales, p.zeros, p.d_out, p.d_in, p.group_size, p.symmetric, out, stream),
           "wq_dequantize")
    return out


def linear_w4a16(X: torch.Tensor, p: PackedLinear, out_dtype=torch.bfloat16, out: torch.Tensor | None = None,
                 workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Y[M, d_out] = X[M, d_in] . x_hat^T with fp32 accumulation."""
    _require_cuda(X, p.qweight)
    if X.dtype != torch.bfloat16 or X.dim() != 2 or not X.is_contiguous() or X.shape[1] != p.d_in:
        raise ValueError("X must be a contiguous [M, d_in] bf16 CUDA tensor")
    M = X.shape[0]
    y_dtype = WQ_OUT_FP32 if out_dtype == torch.float32 else WQ_OUT_BF16
    if out is None:
        out = torch.empty(M, p.d_out, dtype=torch.float32 if y_dtype == WQ_OUT_FP32 else torch.bfloat16,
                          device=X.device)
    need = wq_linear_workspace_bytes(M, p.d_out, p.d_in)
    ws_bytes = 0
    if need > 0:
        if workspace is None or workspace.numel() * workspace.element_size() < need:
            workspace = torch.empty(need, dtype=torch.uint8, device=X.device)
        ws_bytes = workspace.numel() * workspace.element_size()
    _check(wq_linear_w4a16(X, M, p.qweight, p.scales, p.zeros, p.d_out, p.d_in, p.group_size, p.symmetric, out,
                           y_dtype, workspace if need > 0 else None, ws_bytes, stream), "wq_linear_w4a16")
    return out


def device_error(stream=None):
    """Synchronize, read and clear the device status word: (status, flags)."""
    return wq_get_device_error(stream)
