"""Seeded synthetic inputs for the quantization / W4A16 workloads.

This module only draws random tensors; it holds none of the quantization
arithmetic.  Both the CUDA path and the CPU oracle receive the tensors it
returns, so neither side generates its own inputs.

Recipe (shapes and distributions follow the workloads the method targets:
Llama-shaped weight matrices, N(0, sigma) weights, ~0.1% outliers as the
"LLM.int8()" section of the "Quantization Algorithms" study notes describes
for LLM activations/weights):

* weights: ``torch.randn`` (fp32) * sigma, rounded to bf16 by ``Tensor.to``;
* entry outliers: ``round(0.001 * P)`` distinct positions (``torch.randperm``)
  replaced by ``+-20 * sigma`` with a fair-coin sign;
* column outliers: ``round(0.001 * d_in)`` distinct input channels whose
  values are multiplied by a factor (x20 for weights) before bf16 rounding;
* activations: N(0, 1) bf16; channel outliers multiply ``round(0.001 * K)``
  channels by 50.

Every tensor has its own generator seeded from ``(config seed, tensor id)``.
Values depend on the generator's device: CPU and CUDA generators produce
different streams, so a test that compares two implementations passes both
the same tensor rather than regenerating it.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

SEED_BASE = 0x5EED0000


def _gen(seed: int, tensor_id: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((int(seed) * 1_000_003 + int(tensor_id)) & 0x7FFF_FFFF_FFFF_FFFF)
    return g


def normal_bf16(shape, sigma: float, seed: int, tensor_id: int, device="cpu") -> torch.Tensor:
    """N(0, sigma) drawn in fp32 and rounded to bf16."""
    g = _gen(seed, tensor_id, device)
    x = torch.randn(*shape, generator=g, dtype=torch.float32, device=device)
    if sigma != 1.0:
        x.mul_(sigma)
    return x.to(torch.bfloat16)


def weight(d_out: int, d_in: int, sigma: float, seed: int, tensor_id: int, device="cpu",
           entry_outlier_frac: float = 0.0, outlier_mult: float = 20.0,
           column_outlier_frac: float = 0.0, column_mult: float = 20.0) -> torch.Tensor:
    """A bf16 weight matrix W[d_out, d_in] with optional outliers.

    ``entry_outlier_frac``: fraction of entries replaced by +-outlier_mult*sigma.
    ``column_outlier_frac``: fraction of input channels scaled by column_mult
    (the same channels in every row).
    """
    g = _gen(seed, tensor_id, device)
    w = torch.randn(d_out, d_in, generator=g, dtype=torch.float32, device=device)
    w.mul_(sigma)
    if column_outlier_frac > 0.0:
        n_col = int(round(column_outlier_frac * d_in))
        cols = torch.randperm(d_in, generator=g, device=device)[:n_col]
        w[:, cols] *= column_mult
    if entry_outlier_frac > 0.0:
        P = d_out * d_in
        n_out = int(round(entry_outlier_frac * P))
        pos = torch.randperm(P, generator=g, device=device)[:n_out]
        sign = torch.randint(0, 2, (n_out,), generator=g, device=device).to(torch.float32) * 2 - 1
        w.view(-1)[pos] = sign * (outlier_mult * sigma)
    return w.to(torch.bfloat16)


def activations(M: int, K: int, seed: int, tensor_id: int, device="cpu",
                channel_outlier_frac: float = 0.0, channel_mult: float = 50.0) -> torch.Tensor:
    """bf16 activations X[M, K] ~ N(0, 1), optionally with scaled channels."""
    g = _gen(seed, tensor_id, device)
    x = torch.randn(M, K, generator=g, dtype=torch.float32, device=device)
    if channel_outlier_frac > 0.0:
        n_ch = int(round(channel_outlier_frac * K))
        ch = torch.randperm(K, generator=g, device=device)[:n_ch]
        x[:, ch] *= channel_mult
    return x.to(torch.bfloat16)


# --------------------------------------------------------------------------
# The five workloads
# --------------------------------------------------------------------------

@dataclass(frozen=True)
class LinearCase:
    name: str
    d_out: int
    d_in: int
    sigma: float
    symmetric: bool
    Ms: tuple
    entry_outlier_frac: float = 0.0
    column_outlier_frac: float = 0.0
    act_channel_outlier_frac: float = 0.0
    group_size: int = 128


@dataclass(frozen=True)
class Workload:
    index: int
    name: str
    cases: tuple = field(default_factory=tuple)

    @property
    def seed(self) -> int:
        return SEED_BASE + self.index


TINY = Workload(1, "tiny-rtn-512x512", (
    LinearCase("W512", 512, 512, 0.02, False, (1,), entry_outlier_frac=0.001),
))

ATTN = Workload(2, "llama7b-attn-proj-4096x4096", (
    LinearCase("Wqkvo", 4096, 4096, 0.02, False, (1, 8), column_outlier_frac=0.001,
               act_channel_outlier_frac=0.001),
))

MLP = Workload(3, "llama7b-mlp", (
    LinearCase("gate", 11008, 4096, 0.02, True, (1, 4, 16)),
    LinearCase("up", 11008, 4096, 0.02, True, (1, 4, 16)),
    LinearCase("down", 4096, 11008, 0.02, True, (1, 4, 16)),
))

PREFILL = Workload(4, "70b-prefill-gemm", (
    LinearCase("W8192", 8192, 8192, 0.015, False, (512, 2048, 8192)),
    LinearCase("W28672", 28672, 8192, 0.015, False, (512, 2048, 8192)),
))

_LAYER = (("qkv", 12288, 4096), ("o", 4096, 4096), ("gate", 11008, 4096),
          ("up", 11008, 4096), ("down", 4096, 11008))

WHOLE_MODEL = Workload(5, "7b-decoder-32-layers", tuple(
    LinearCase(f"L{l}.{nm}", d_out, d_in, 0.02, False, (1,), entry_outlier_frac=0.001)
    for l in range(32) for (nm, d_out, d_in) in _LAYER
))

WORKLOADS = {w.index: w for w in (TINY, ATTN, MLP, PREFILL, WHOLE_MODEL)}


def case_weight(wl: Workload, case_idx: int, device="cpu") -> torch.Tensor:
    c = wl.cases[case_idx]
    return weight(c.d_out, c.d_in, c.sigma, wl.seed, 2 * case_idx, device,
                  entry_outlier_frac=c.entry_outlier_frac,
                  column_outlier_frac=c.column_outlier_frac)


def case_activations(wl: Workload, case_idx: int, M: int, device="cpu") -> torch.Tensor:
    c = wl.cases[case_idx]
    return activations(M, c.d_in, wl.seed, 2 * case_idx + 1 + 1000 * M, device,
                       channel_outlier_frac=c.act_channel_outlier_frac)


def total_params(wl: Workload) -> int:
    return sum(c.d_out * c.d_in for c in wl.cases)
