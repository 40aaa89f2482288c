"""The AWQ search on library-owned scratch (wq_awq_search_static), for callers
that cannot allocate device memory, gives bit for bit the results of the same
search on a caller workspace (wq_awq_search), called through the C ABI twice
in a row: the scratch keeps the previous call's contents, and each search
must not depend on them."""
import pytest
import torch

from w4a16_bit_gemm_b200 import synthetic as syn

pytestmark = pytest.mark.gpu


def _same(r1, r2, sym):
    assert torch.equal(r1.losses, r2.losses) and torch.equal(r1.best, r2.best) and torch.equal(r1.s, r2.s)
    assert torch.equal(r1.packed.qweight, r2.packed.qweight) and torch.equal(r1.packed.scales, r2.packed.scales)
    if not sym:
        assert torch.equal(r1.packed.zeros, r2.packed.zeros)


@pytest.mark.parametrize("shape", [(256, 1024, 96, 128, False), (130, 512, 5, 64, True),
                                   (4096, 4096, 512, 128, False)], ids=lambda s: "%dx%d-T%d" % s[:3])
def test_static_scratch_matches_workspace(shape):
    from w4a16_bit_gemm_b200 import binding as b
    N, K, T, g, sym = shape
    W = syn.weight(N, K, 0.02, N + K, 1).cuda()
    X = syn.activations(T, K, N + K, 2, "cuda", channel_outlier_frac=0.01)
    W2 = syn.weight(N, K, 0.03, N + K + 7, 1).cuda()
    X2 = syn.activations(T, K, N + K + 7, 2, "cuda", channel_outlier_frac=0.001)
    ref1 = b.awq_search(W, X, g, sym)
    ref2 = b.awq_search(W2, X2, g, sym)
    # two calls in a row on the shared scratch, different inputs, then the first again
    s1 = b.awq_search_static(W, X, g, sym)
    s2 = b.awq_search_static(W2, X2, g, sym)
    s3 = b.awq_search_static(W, X, g, sym)
    st, _ = b.device_error()
    assert st == b.WQ_OK
    _same(ref1, s1, sym)
    _same(ref2, s2, sym)
    _same(ref1, s3, sym)


def test_static_scratch_too_small_is_unsupported():
    from w4a16_bit_gemm_b200 import binding as b
    W = torch.zeros(8192, 8192, dtype=torch.bfloat16, device="cuda")
    X = torch.zeros(512, 8192, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(b.WQError) as e:
        b.awq_search_static(W, X)
    assert e.value.status == b.WQ_ERR_UNSUPPORTED
