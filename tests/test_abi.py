"""C-ABI library: loads, exports every symbol include/wq.h declares, and the
host-side validation rejects bad arguments before any CUDA call (runs without
a GPU: no call here reaches a kernel)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "wq.h")


@pytest.fixture(scope="module")
def lib():
    from w4a16_bit_gemm_b200 import build
    build.build()
    from w4a16_bit_gemm_b200 import binding
    return binding.lib


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(wq_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("wq_quantize_rtn", "wq_quantize_clip_mse", "wq_awq_search", "wq_awq_workspace_bytes",
              "wq_awq_scale_activations", "wq_gptq", "wq_gptq_workspace_bytes", "wq_quantize_w8",
              "wq_dequantize_w8", "wq_linear_w8a16", "wq_dequantize", "wq_linear_w4a16", "wq_linear_workspace_bytes",
              "wq_get_device_error", "wq_status_string", "wq_abi_version"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for n in declared_functions():
        assert hasattr(lib, n), n


def test_abi_version_and_status_strings(lib):
    assert lib.wq_abi_version() == 1
    for code, name in [(0, b"WQ_OK"), (1, b"WQ_ERR_INVALID_ARG"), (3, b"WQ_ERR_CUDA"), (5, b"WQ_ERR_TIMEOUT")]:
        assert lib.wq_status_string(code) == name


FAKE = 0x10000  # 16-byte aligned, never dereferenced: validation fails first


@pytest.mark.parametrize("case", [
    dict(W=None),
    dict(W=FAKE + 2),                        # misaligned input
    dict(q=FAKE + 4),                        # misaligned qweight
    dict(d_out=0),
    dict(d_in=0),
    dict(g=100),                             # not a supported group size
    dict(d_in=1000, g=128),                  # group does not divide d_in
    dict(g=384, d_in=768),                   # > 256 and not a multiple of 256
    dict(zeros=None),                        # asymmetric without zeros
    dict(sym=1),                             # symmetric with zeros
    dict(sym=2),
])
def test_quantize_rejects(lib, case):
    a = dict(W=FAKE, d_out=4, d_in=256, g=128, sym=0, q=FAKE, s=FAKE, zeros=FAKE)
    a.update(case)
    st = lib.wq_quantize_rtn(a["W"], a["d_out"], a["d_in"], a["g"], a["sym"], a["q"], a["s"], a["zeros"], None)
    assert st == 1


@pytest.mark.parametrize("case", [
    dict(X=None), dict(Y=None), dict(X=FAKE + 8), dict(M=0), dict(ydt=2), dict(g=48), dict(sym=1),
])
def test_linear_rejects(lib, case):
    a = dict(X=FAKE, M=1, q=FAKE, s=FAKE, z=FAKE, N=64, K=256, g=128, sym=0, Y=FAKE, ydt=0)
    a.update(case)
    st = lib.wq_linear_w4a16(a["X"], a["M"], a["q"], a["s"], a["z"], a["N"], a["K"], a["g"], a["sym"], a["Y"],
                             a["ydt"], None, 0, None)
    assert st == 1


def test_dequantize_rejects(lib):
    assert lib.wq_dequantize(FAKE, FAKE, FAKE, 4, 256, 128, 0, None, None) == 1
    assert lib.wq_dequantize(None, FAKE, FAKE, 4, 256, 128, 0, FAKE, None) == 1
    assert lib.wq_dequantize(FAKE, FAKE, None, 4, 256, 128, 0, FAKE, None) == 1


def test_workspace_query(lib):
    assert lib.wq_linear_workspace_bytes(1, 4096, 4096) >= 0


@pytest.mark.parametrize("case", [
    dict(W=None), dict(W=FAKE + 8), dict(q=None), dict(d_in=1000, g=128), dict(zeros=None), dict(sym=1),
])
def test_quantize_clip_rejects(lib, case):
    a = dict(W=FAKE, d_out=4, d_in=256, g=128, sym=0, q=FAKE, s=FAKE, zeros=FAKE)
    a.update(case)
    st = lib.wq_quantize_clip_mse(a["W"], a["d_out"], a["d_in"], a["g"], a["sym"], a["q"], a["s"], a["zeros"],
                                  None)
    assert st == 1


def test_quantize_clip_unsupported_group_size(lib):
    # 512 is a valid RTN group size; the clipping search takes 32..256 only
    assert lib.wq_quantize_clip_mse(FAKE, 4, 1024, 512, 0, FAKE, FAKE, FAKE, None) == 2


@pytest.mark.parametrize("case", [
    dict(W=None), dict(X=None), dict(X=FAKE + 8), dict(s=None), dict(T=0), dict(ws=None), dict(wsb=16),
    dict(ws=FAKE + 16), dict(d_in=1000), dict(zeros=None), dict(sym=1), dict(losses=FAKE + 4),
])
def test_awq_search_rejects(lib, case):
    a = dict(W=FAKE, d_out=4, d_in=256, X=FAKE, T=8, g=128, sym=0, q=FAKE, sc=FAKE, zeros=FAKE, s=FAKE,
             losses=None, best=None, ws=FAKE, wsb=1 << 30)
    a.update(case)
    st = lib.wq_awq_search(a["W"], a["d_out"], a["d_in"], a["X"], a["T"], a["g"], a["sym"], a["q"], a["sc"],
                           a["zeros"], a["s"], a["losses"], a["best"], a["ws"], a["wsb"], None)
    assert st == 1


def test_awq_workspace_query(lib):
    n = lib.wq_awq_workspace_bytes(4096, 4096, 512, 128)
    # W' and X' (bf16), the candidate artifact, two fp32 outputs, at least
    assert n >= 4096 * 4096 * 2 + 4096 * 2048 + 512 * 4096 * 2 + 2 * 512 * 4096 * 4
    assert lib.wq_awq_workspace_bytes(4, 1000, 8, 128) == 0
    assert lib.wq_awq_workspace_bytes(0, 256, 8, 128) == 0


def test_awq_scale_activations_rejects(lib):
    assert lib.wq_awq_scale_activations(None, 4, 256, FAKE, FAKE, None) == 1
    assert lib.wq_awq_scale_activations(FAKE, 0, 256, FAKE, FAKE, None) == 1
    assert lib.wq_awq_scale_activations(FAKE, 4, 252, FAKE, FAKE, None) == 1
    assert lib.wq_awq_scale_activations(FAKE + 8, 4, 256, FAKE, FAKE, None) == 1


@pytest.mark.parametrize("case", [
    dict(W=None), dict(X=None), dict(X=FAKE + 2), dict(T=0), dict(act=2), dict(ws=None), dict(wsb=64),
    dict(ws=FAKE + 64), dict(perm=FAKE + 2), dict(zeros=None), dict(g=100),
])
def test_gptq_rejects(lib, case):
    a = dict(W=FAKE, d_out=4, d_in=256, X=FAKE, T=8, g=128, sym=0, act=1, q=FAKE, sc=FAKE, zeros=FAKE, perm=None,
             ws=FAKE, wsb=1 << 30)
    a.update(case)
    st = lib.wq_gptq(a["W"], a["d_out"], a["d_in"], a["X"], a["T"], a["g"], a["sym"], a["act"], a["q"], a["sc"],
                     a["zeros"], a["perm"], a["ws"], a["wsb"], None)
    assert st == 1


def test_gptq_workspace_query(lib):
    n = lib.wq_gptq_workspace_bytes(4096, 4096)
    assert n >= 2 * 4096 * 4096 * 8 + 4096 * 4096 * 8 and n < 2 * 4096 * 4096 * 8 + 4096 * 4096 * 10 + (1 << 24)
    assert lib.wq_gptq_workspace_bytes(0, 256) == 0


@pytest.mark.parametrize("case", [
    dict(W=None), dict(W=FAKE + 8), dict(q=FAKE + 4), dict(s=None), dict(d_in=1000, g=1000), dict(g=48),
    dict(g=16, d_in=256), dict(d_in=96, g=64), dict(d_out=0),
])
def test_w8_quantize_rejects(lib, case):
    a = dict(W=FAKE, d_out=4, d_in=256, g=128, q=FAKE, s=FAKE)
    a.update(case)
    assert lib.wq_quantize_w8(a["W"], a["d_out"], a["d_in"], a["g"], a["q"], a["s"], None) == 1


def test_w8_linear_and_dequant_reject(lib):
    assert lib.wq_linear_w8a16(FAKE, 0, FAKE, FAKE, 64, 256, 256, FAKE, 0, None) == 1
    assert lib.wq_linear_w8a16(FAKE + 8, 1, FAKE, FAKE, 64, 256, 256, FAKE, 0, None) == 1
    assert lib.wq_linear_w8a16(FAKE, 1, FAKE, FAKE, 64, 256, 256, FAKE, 3, None) == 1
    assert lib.wq_dequantize_w8(FAKE, FAKE, 4, 256, 128, None, None) == 1
    assert lib.wq_dequantize_w8(FAKE, None, 4, 256, 128, FAKE, None) == 1


def test_awq_static_rejects_before_any_device_work(lib):
    # a layer whose scratch exceeds the library-owned array
    assert lib.wq_awq_static_scratch_bytes() >= 64 << 20
    st = lib.wq_awq_search_static(FAKE, 8192, 8192, FAKE, 512, 128, 0, FAKE, FAKE, FAKE, FAKE, None, None, None)
    assert st == 2
    assert lib.wq_awq_search_static(None, 64, 256, FAKE, 8, 128, 0, FAKE, FAKE, FAKE, FAKE, None, None, None) == 1


# ---------------------------------------------------------------------------
# Host-side fault injection (WQ_FAULT_INJECT=launch|alloc): every entry point
# that enqueues work fails with WQ_ERR_CUDA after its argument checks and
# before any CUDA call, and each such failure is counted.  Runs in a child
# process per mode (the variable is read once per process).
# ---------------------------------------------------------------------------

_INJECT_SCRIPT = r'''
import ctypes, json, sys
sys.path.insert(0, sys.argv[1])
from w4a16_bit_gemm_b200 import binding
lib = binding.lib
F = 0x10000
out = {}
def call(name, *args):
    before = lib.wq_fault_injections()
    st = getattr(lib, name)(*args)
    out[name] = [st, lib.wq_fault_injections() - before]
call("wq_quantize_rtn", F, 4, 256, 128, 0, F, F, F, None)
call("wq_quantize_clip_mse", F, 4, 256, 128, 0, F, F, F, None)
call("wq_dequantize", F, F, F, 4, 256, 128, 0, F, None)
call("wq_linear_w4a16", F, 1, F, F, F, 64, 256, 128, 0, F, 0, None, 0, None)
call("wq_linear_w4a16", F, 300, F, F, F, 64, 256, 128, 0, F, 1, None, 0, None)
ws = lib.wq_awq_workspace_bytes(64, 256, 8, 128)
call("wq_awq_search", F, 64, 256, F, 8, 128, 0, F, F, F, F, None, None, F, ws, None)
call("wq_awq_search_static", F, 64, 256, F, 8, 128, 0, F, F, F, F, None, None, None)
call("wq_awq_scale_activations", F, 8, 256, F, F, None)
call("wq_quantize_w8", F, 4, 256, 128, F, F, None)
call("wq_dequantize_w8", F, F, 4, 256, 128, F, None)
call("wq_linear_w8a16", F, 1, F, F, 64, 256, 128, F, 0, None)
gws = lib.wq_gptq_workspace_bytes(64, 256)
call("wq_gptq", F, 64, 256, F, 8, 128, 1, 1, F, F, None, None, F, gws, None)
call("wq_get_device_error", None, None)
call("wq_selftest_bounded_wait", 1000, None)
# argument errors are still reported as such, with nothing counted

before = lib.wq_fault_injections()
out["invalid"] = [lib.wq_quantize_rtn(None, 4, 256, 128, 0, F, F, F, None), lib.wq_fault_injections() - before]
print(json.dumps(out))
'''

ENQUEUEING = ["wq_quantize_rtn", "wq_quantize_clip_mse", "wq_dequantize", "wq_linear_w4a16", "wq_awq_search",
              "wq_awq_search_static", "wq_awq_scale_activations", "wq_quantize_w8", "wq_dequantize_w8",
              "wq_linear_w8a16", "wq_gptq", "wq_get_device_error", "wq_selftest_bounded_wait"]


def _run_injected(mode):
    import json
    import subprocess
    import sys
    env = dict(os.environ)
    env.pop("WQ_FAULT_INJECT", None)
    if mode:
        env["WQ_FAULT_INJECT"] = mode
    env["CUDA_VISIBLE_DEVICES"] = ""  # never reach a device, even on a GPU machine
    r = subprocess.run([sys.executable, "-c", _INJECT_SCRIPT, ROOT], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    return json.loads(r.stdout.strip().splitlines()[-1])


def test_fault_injection_covers_every_enqueueing_entry_point(lib):
    declared = set(declared_functions())
    assert set(ENQUEUEING) <= declared
    # the others only compute sizes or strings and never enqueue work
    assert declared - set(ENQUEUEING) == {"wq_abi_version", "wq_status_string", "wq_linear_workspace_bytes",
                                          "wq_awq_workspace_bytes", "wq_awq_static_scratch_bytes",
                                          "wq_gptq_workspace_bytes", "wq_fault_injections"}


@pytest.mark.parametrize("mode", ["launch", "alloc"])
def test_fault_injection_fails_each_call_once(lib, mode):
    out = _run_injected(mode)
    for name in ENQUEUEING:
        st, counted = out[name]
        assert st == 3 and counted == 1, (mode, name, st, counted)  # WQ_ERR_CUDA, one injected failure
    assert out["invalid"] == [1, 0]  # WQ_ERR_INVALID_ARG first, nothing injected


def test_no_injection_without_the_variable(lib):
    out = _run_injected(None)
    for name in ENQUEUEING:
        assert out[name][1] == 0, name
    assert out["invalid"] == [1, 0]
