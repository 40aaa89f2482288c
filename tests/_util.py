"""Shared test helpers: bit-pattern views between torch tensors and numpy."""
import numpy as np
import torch


def bits16(t: torch.Tensor) -> np.ndarray:
    """bf16/fp16 tensor (any device) -> numpy uint16 bit patterns."""
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def bits32(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().view(torch.int32).numpy().view(np.uint32)


def f64_from_bf16_bits(b: np.ndarray) -> np.ndarray:
    with np.errstate(invalid="ignore"):
        return (np.asarray(b, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def bf16_from_bits(b: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(b, np.uint16).view(np.int16)).view(torch.bfloat16)


def fp16_from_bits(b: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(b, np.uint16).view(np.int16)).view(torch.float16)


BF16_UNIT_ROUNDOFF = 2.0 ** -8


def linear_tolerance_ok(y: np.ndarray, y_ref: np.ndarray, A: np.ndarray, out_bf16: bool = False):
    """The stated bound |y - y_ref| <= 1e-3 * sum_k |w_hat x| + 1e-6.

    A bf16 output adds its own final rounding, at most the bf16 unit roundoff
    2^-8 times |y_ref|; that term is added only for bf16 outputs (fp32 outputs
    are held to the bound as stated).  Returns (ok, worst error/bound ratio)."""
    err = np.abs(y.astype(np.float64) - y_ref)
    bound = 1e-3 * A + 1e-6
    if out_bf16:
        bound = bound + BF16_UNIT_ROUNDOFF * np.abs(y_ref)
    ratio = float(np.max(err / bound)) if err.size else 0.0
    return bool(np.all(err <= bound)), ratio
