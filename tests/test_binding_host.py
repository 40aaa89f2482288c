"""The Python binding on a host without a GPU: it loads libwq.so, exposes every
operation, and refuses CPU tensors loudly (there is no CPU fallback)."""
import pytest
import torch


@pytest.fixture(scope="module")
def b():
    from w4a16_bit_gemm_b200 import build
    build.build()
    from w4a16_bit_gemm_b200 import binding
    return binding


def test_every_operation_refuses_cpu_tensors(b):
    W = torch.zeros(64, 256, dtype=torch.bfloat16)
    X = torch.zeros(4, 256, dtype=torch.bfloat16)
    calls = [
        lambda: b.quantize_rtn(W),
        lambda: b.quantize_clip_mse(W),
        lambda: b.quantize_w8(W),
        lambda: b.awq_search(W, X),
        lambda: b.awq_search_static(W, X),
        lambda: b.gptq(W, X),
        lambda: b.awq_scale_activations(X, torch.ones(256, dtype=torch.bfloat16)),
    ]
    for call in calls:
        with pytest.raises(ValueError, match="no CPU fallback"):
            call()


def test_status_strings_and_constants(b):
    assert b.status_string(b.WQ_OK) == "WQ_OK"
    assert b.status_string(b.WQ_ERR_UNSUPPORTED) == "WQ_ERR_UNSUPPORTED"
    err = b.WQError(b.WQ_ERR_INVALID_ARG, "x")
    assert err.status == b.WQ_ERR_INVALID_ARG and "WQ_ERR_INVALID_ARG" in str(err)
