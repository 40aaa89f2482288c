"""Seeded synthetic inputs: shapes, determinism, outlier recipe."""
import torch

from w4a16_bit_gemm_b200 import synthetic as syn


def test_deterministic_and_seeded():
    a = syn.case_weight(syn.TINY, 0)
    b = syn.case_weight(syn.TINY, 0)
    assert a.dtype == torch.bfloat16 and a.shape == (512, 512)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    x1 = syn.case_activations(syn.TINY, 0, 1)
    assert x1.shape == (1, 512)


def test_tiny_entry_outliers():
    w = syn.case_weight(syn.TINY, 0).float()
    n = int((w.abs() == torch.tensor(0.4).to(torch.bfloat16).float()).sum())
    assert n == 262  # round(0.001 * 512 * 512) replaced entries


def test_column_outliers_small_shape():
    w = syn.weight(64, 4096, 0.02, 123, 0, column_outlier_frac=0.001)
    col_max = w.float().abs().amax(0)
    assert int((col_max > 0.2).sum()) == 4  # four x20 input channels
    x = syn.activations(2, 4096, 123, 1, channel_outlier_frac=0.001)
    assert int((x.float().abs().amax(0) > 10).sum()) >= 3


def test_workload_table():
    assert syn.total_params(syn.WHOLE_MODEL) == 6_476_005_376
    assert len(syn.WHOLE_MODEL.cases) == 160
    assert [c.symmetric for c in syn.MLP.cases] == [True, True, True]
