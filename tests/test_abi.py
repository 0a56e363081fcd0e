"""Host-side contract of the libtc C-ABI (runs without a GPU).

Checks that the library loads, exports every function include/tc.h declares,
and that argument validation returns the documented status codes before any
device work.  On a machine without an sm_100 device, a fully valid call must
return TC_ERR_NO_DEVICE (never fall back to a CPU path).
"""
import ctypes
import os
import re

import pytest
import torch

import sliding_window_attention_tc_b200 as tc

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "tc.h")
HAS_GPU = torch.cuda.is_available()


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(tc_[a-z_0-9]+)\s*\(", src)))


def test_header_functions_are_exported():
    names = _declared_functions()
    assert "tc_prefill" in names and "tc_decode_step" in names
    lib = tc.lib_handle()
    for n in names:
        assert hasattr(lib, n), f"{n} declared in tc.h but not exported"
    assert set(names) == set(tc.EXPORTED)


def test_status_strings_and_version():
    for code in range(8):
        s = tc.status_string(code)
        assert s and s != "unknown status"
    assert tc.status_string(99) == "unknown status"
    assert re.match(r"^\d+\.\d+\.\d+$", tc.version())


def _desc(**kw):
    base = dict(B=2, H=3, T=100, dk=64, dv=64, W=32, C=16, dtype=tc.TC_F32, l1_only=False)
    base.update(kw)
    return tc.make_prefill_desc(**base)


FAKE = ctypes.c_void_p(0x10000)  # non-null, 16-byte aligned, never dereferenced


def _call_prefill(desc, **ptrs):
    p = dict(q=FAKE, k=FAKE, v=FAKE, lam=FAKE, eta=FAKE, g=FAKE, y=FAKE, A=FAKE, ws=FAKE)
    p.update(ptrs)
    return tc.lib_handle().tc_prefill(
        ctypes.byref(desc) if desc is not None else None, p["q"], p["k"], p["v"], p["lam"],
        p["eta"], p["g"], p["y"], p["A"], p["ws"], 1 << 40, None)


@pytest.mark.parametrize("bad", [dict(B=0), dict(H=-1), dict(T=-1), dict(dk=0), dict(dv=0),
                                 dict(W=0), dict(C=0), dict(dtype=7)])
def test_prefill_rejects_invalid_sizes(bad):
    d = _desc(**bad)
    assert _call_prefill(d) == 1
    assert tc.lib_handle().tc_prefill_workspace_size(ctypes.byref(d)) == tc.SIZE_ERROR


def test_prefill_rejects_null_and_misaligned():
    assert _call_prefill(None) == 1
    assert _call_prefill(_desc(), q=None) == 1
    assert _call_prefill(_desc(), y=None) == 1
    assert _call_prefill(_desc(), A=None) == 1  # A_final needed unless L1-only
    assert _call_prefill(_desc(), k=ctypes.c_void_p(0x10004)) == 1
    d = _desc()
    d.flags = 0x80
    assert _call_prefill(d) == 1


def test_prefill_unsupported_head_dim():
    assert _call_prefill(_desc(dk=129)) == 2
    assert _call_prefill(_desc(dv=256)) == 2


@pytest.mark.skipif(HAS_GPU, reason="checks the no-device answer")
def test_valid_prefill_without_device_reports_no_device():
    assert _call_prefill(_desc()) == 3
    assert _call_prefill(_desc(l1_only=True), A=None) == 3
    d = _desc(dtype=tc.TC_BF16, T=0)
    assert _call_prefill(d) == 3


def test_workspace_size_query():
    d = _desc(T=1000, W=100, C=64)
    n = tc.prefill_workspace_size(d)
    assert n >= 0
    d.flags = tc.TC_PREFILL_L1_ONLY
    assert tc.prefill_workspace_size(d) >= 0
    host = tc.prefill_host_workspace_size(_desc(T=1000, W=100, C=64))
    assert host > 2 * 1000 * 64 * 4 * 6  # holds q, k, v, y at least
    # no evictions: the portable path needs no chunk states
    assert tc.prefill_workspace_size(_desc(T=10, W=100, dtype=tc.TC_F32)) == 0


def _state(**kw):
    base = dict(B=2, H=2, dk=64, dv=64, W=16, t=0, kv_dtype=tc.TC_BF16, ring_k=0x10000,
                ring_v=0x10000, A=0x10000, lam=0x10000, eta=0x10000, g=0x10000)
    base.update(kw)
    return tc.DecodeStateC(**base)


def _call_decode(st, q=FAKE):
    return tc.lib_handle().tc_decode_step(ctypes.byref(st), q, FAKE, FAKE, FAKE, None)


@pytest.mark.parametrize("bad", [dict(B=0), dict(W=0), dict(t=-1), dict(kv_dtype=5),
                                 dict(ring_k=None), dict(A=None), dict(A=0x10008)])
def test_decode_rejects_invalid(bad):
    st = _state(**bad)
    assert _call_decode(st) == 1
    assert st.t == bad.get("t", 0)


def test_decode_unsupported_dims():
    assert _call_decode(_state(dk=64, dv=32)) == 2
    assert _call_decode(_state(dk=48, dv=48)) == 2
    assert _call_decode(_state(), q=None) == 1


@pytest.mark.skipif(HAS_GPU, reason="checks the no-device answer")
def test_valid_decode_without_device_reports_no_device():
    st = _state(t=5)
    assert _call_decode(st) == 3
    assert st.t == 5  # the clock only advances on success
    n = tc.lib_handle().tc_decode_step_host_workspace_size(ctypes.byref(st))
    assert n == 4 * 2 * 2 * 64 * 2 + 0 or n >= 4 * 2 * 2 * 64 * 2


def _call_varlen(desc, cu=FAKE, total=300, **ptrs):
    p = dict(q=FAKE, k=FAKE, v=FAKE, lam=FAKE, eta=FAKE, g=FAKE, y=FAKE, A=FAKE, ws=FAKE)
    p.update(ptrs)
    return tc.lib_handle().tc_prefill_varlen(
        ctypes.byref(desc) if desc is not None else None, cu, total, p["q"], p["k"], p["v"],
        p["lam"], p["eta"], p["g"], p["y"], p["A"], p["ws"], 1 << 40, None)


def _varlen_desc(**kw):
    base = dict(B=3, H=2, T=200, dk=64, dv=64, W=128, C=64, dtype=tc.TC_BF16)
    base.update(kw)
    return _desc(**base)


def test_varlen_rejects_invalid_arguments():
    lib = tc.lib_handle()
    assert _call_varlen(None) == 1
    assert _call_varlen(_varlen_desc(), cu=None) == 1
    assert _call_varlen(_varlen_desc(), cu=ctypes.c_void_p(0x10004)) == 1  # not 8-byte aligned
    assert _call_varlen(_varlen_desc(), total=-1) == 1
    assert _call_varlen(_varlen_desc(), total=(1 << 30) + 1) == 1
    assert _call_varlen(_varlen_desc(), q=None) == 1
    assert _call_varlen(_varlen_desc(), A=None) == 1
    assert _call_varlen(_varlen_desc(), k=ctypes.c_void_p(0x10008)) == 1
    # total = 0: the token tensors may be NULL (then only the device is missing)
    st = _call_varlen(_varlen_desc(), total=0, q=None, k=None, v=None, y=None)
    assert st in (0, 3)
    assert lib.tc_prefill_varlen_workspace_size(None) == tc.SIZE_ERROR


@pytest.mark.parametrize("kw", [dict(dtype=tc.TC_F32), dict(dk=32, dv=32), dict(dk=64, dv=128),
                                dict(flags=tc.TC_PREFILL_STATE_ONLY),
                                dict(flags=tc.TC_PREFILL_DELTA_RULE)])
def test_varlen_outside_the_tensor_core_paths_is_unsupported(kw):
    flags = kw.pop("flags", 0)
    d = _varlen_desc(**kw)
    d.flags = flags
    assert _call_varlen(d) == 2
    assert tc.lib_handle().tc_prefill_varlen_workspace_size(ctypes.byref(d)) == tc.SIZE_ERROR


@pytest.mark.skipif(HAS_GPU, reason="checks the no-device answer")
def test_valid_varlen_without_device_reports_no_device():
    assert _call_varlen(_varlen_desc()) == 3
    # the general tensor-core path: W not a multiple of 128, d = 128
    for kw in (dict(W=100), dict(W=64), dict(dk=128, dv=128, W=300)):
        d = _varlen_desc(**kw)
        assert _call_varlen(d) == 3
        assert tc.lib_handle().tc_prefill_varlen_workspace_size(ctypes.byref(d)) > 0
    d = _varlen_desc(l1_only=True)
    assert _call_varlen(d, A=None) == 3
    assert tc.lib_handle().tc_prefill_varlen_workspace_size(ctypes.byref(_varlen_desc())) >= 0
