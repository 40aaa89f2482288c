"""The AWQ search with library-owned scratch (wq_awq_search_static) gives
bit for bit the results of the same search on a caller workspace."""
import pytest
import torch

from w4a16_bit_gemm_b200 import synthetic as syn

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("shape", [(256, 1024, 96, 128, False), (130, 512, 5, 64, True),
                                   (4096, 4096, 512, 128, False)], ids=lambda s: "%dx%d-T%d" % s[:3])
def test_static_scratch_matches_workspace(shape):
    from w4a16_bit_gemm_b200 import binding as b
    N, K, T, g, sym = shape
    W = syn.weight(N, K, 0.02, N + K, 1).cuda()
    X = syn.activations(T, K, N + K, 2, "cuda", channel_outlier_frac=0.01)
    r1 = b.awq_search(W, X, g, sym)
    r2 = b.awq_search_static(W, X, g, sym)
    st, _ = b.device_error()
    assert st == b.WQ_OK
    assert torch.equal(r1.losses, r2.losses) and torch.equal(r1.best, r2.best) and torch.equal(r1.s, r2.s)
    assert torch.equal(r1.packed.qweight, r2.packed.qweight) and torch.equal(r1.packed.scales, r2.packed.scales)
    if not sym:
        assert torch.equal(r1.packed.zeros, r2.packed.zeros)


def test_static_scratch_too_small_is_unsupported():
    from w4a16_bit_gemm_b200 import binding as b
    W = torch.zeros(8192, 8192, dtype=torch.bfloat16, device="cuda")
    X = torch.zeros(512, 8192, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(b.WQError) as e:
        b.awq_search_static(W, X)
    assert e.value.status == b.WQ_ERR_UNSUPPORTED
