"""Host-side contract of the libtc entry points beyond tc_prefill and
tc_decode_step (runs without a GPU).

For each call this checks two things.  Invalid arguments return the
documented TC_ERR_* code before any device work: null or misaligned buffers,
negative positions, unsupported flags, and a missing ragged clock array.  On a
machine without an sm_100 device, a fully valid call returns TC_ERR_NO_DEVICE
and never falls back to a CPU path.  Fake device addresses are never
dereferenced: every call here stops at host validation or at the device query.
"""
import ctypes

import pytest
import torch

import sliding_window_attention_tc_b200 as tc

HAS_GPU = torch.cuda.is_available()
OK, INVALID, UNSUPPORTED, NO_DEVICE, WORKSPACE = 0, 1, 2, 3, 7
FAKE = ctypes.c_void_p(0x10000)   # non-null, 16-byte aligned, never dereferenced
SKEW = ctypes.c_void_p(0x10004)   # misaligned by 4 bytes
no_device_only = pytest.mark.skipif(HAS_GPU, reason="checks the no-device answer")


def _desc(**kw):
    base = dict(B=2, H=3, T=100, dk=64, dv=64, W=32, C=16, dtype=tc.TC_F32, l1_only=False)
    flags = kw.pop("flags", None)
    base.update(kw)
    d = tc.make_prefill_desc(**base)
    if flags is not None:
        d.flags = flags
    return d


def _lib():
    return tc.lib_handle()


# ---------------------------------------------------------------- descriptor flags
@pytest.mark.parametrize("flags", [
    tc.TC_PREFILL_CHUNK_MEAN,                                   # chunk mean needs STATE_ONLY
    tc.TC_PREFILL_CHUNK_MEAN | tc.TC_PREFILL_STATE_ONLY | tc.TC_PREFILL_DELTA_RULE,
    tc.TC_PREFILL_L1_ONLY | tc.TC_PREFILL_STATE_ONLY,           # nothing left to compute
    0x100,                                                      # unknown bit
])
def test_flag_combinations_rejected(flags):
    d = _desc(flags=flags)
    assert _lib().tc_prefill_workspace_size(ctypes.byref(d)) == tc.SIZE_ERROR
    assert _lib().tc_prefill_launch_count(ctypes.byref(d)) == -1


def test_launch_counts():
    lm = _desc(B=8, H=12, T=4096, W=512, C=64, dtype=tc.TC_BF16)
    # tensor-core path with several spans per head: summary, prefix, main kernel
    assert _lib().tc_prefill_launch_count(ctypes.byref(lm)) == 3
    lm.flags = tc.TC_PREFILL_L1_ONLY
    assert _lib().tc_prefill_launch_count(ctypes.byref(lm)) == 1
    # portable float32 path: chunk states, then the row kernel
    assert _lib().tc_prefill_launch_count(ctypes.byref(_desc())) == 2
    assert _lib().tc_prefill_launch_count(ctypes.byref(_desc(flags=tc.TC_PREFILL_STATE_ONLY))) == 1


def test_backward_launch_counts():
    """Two window kernels, three for the memory part when something is
    evicted (sums, scan over chunks, per-chunk gradients), one reduction."""
    tcf = ctypes.c_int(-1)
    assert _lib().tc_backward_launch_count(None, None) == -1
    assert _lib().tc_backward_launch_count(ctypes.byref(_desc(flags=tc.TC_PREFILL_L1_ONLY)), None) == -1
    assert _lib().tc_backward_launch_count(ctypes.byref(_desc()), ctypes.byref(tcf)) == 6
    assert tcf.value == 0  # float32: SIMT kernels
    assert _lib().tc_backward_launch_count(ctypes.byref(_desc(T=20, W=32)), None) == 3
    lm = _desc(B=8, H=12, T=4096, W=512, C=64, dtype=tc.TC_BF16)
    assert _lib().tc_backward_launch_count(ctypes.byref(lm), ctypes.byref(tcf)) == 6
    assert tcf.value == (1 if HAS_GPU else 0)


def test_delta_launch_counts():
    """Chunked memory: prep, scan over chunks, reads; plus the window part
    (the tensor-core kernel for bf16, d = 64, W a multiple of 128)."""
    lm = tc.make_prefill_desc(8, 12, 4096, 64, 64, 512, 64, tc.TC_BF16, False)
    lm.flags = tc.TC_PREFILL_DELTA_RULE
    assert tc.prefill_launch_count(lm) == 4
    lm.flags = tc.TC_PREFILL_DELTA_RULE | tc.TC_PREFILL_STATE_ONLY
    assert tc.prefill_launch_count(lm) == 2
    short = tc.make_prefill_desc(1, 1, 100, 64, 64, 128, 64, tc.TC_BF16, False)
    short.flags = tc.TC_PREFILL_DELTA_RULE
    assert tc.prefill_launch_count(short) == 2  # no eviction: the scan (A_final) and the window part


# ---------------------------------------------------------------- tc_prefill_from_state
def _from_state(desc, t0, halo_k=FAKE, halo_v=FAKE, A_init=FAKE, q=FAKE, y=FAKE, A=FAKE):
    return _lib().tc_prefill_from_state(ctypes.byref(desc), t0, halo_k, halo_v, A_init, q, FAKE,
                                        FAKE, FAKE, FAKE, FAKE, y, A, FAKE, 1 << 40, None)


def test_from_state_rejects_invalid():
    d = _desc()
    assert _from_state(d, -1) == INVALID
    assert _lib().tc_prefill_from_state_workspace_size(ctypes.byref(d), -1) == tc.SIZE_ERROR
    # t0 > 0 needs the halo of min(t0, W) tokens
    assert _from_state(d, 10, halo_k=None) == INVALID
    assert _from_state(d, 10, halo_v=None) == INVALID
    assert _from_state(d, 10, A_init=SKEW) == INVALID
    assert _from_state(d, 10, halo_k=SKEW) == INVALID
    assert _from_state(d, 10, q=None) == INVALID
    assert _from_state(d, 10, A=None) == INVALID  # A_final unless L1-only


def test_from_state_state_only_needs_no_queries():
    d = _desc(flags=tc.TC_PREFILL_STATE_ONLY)
    rc = _from_state(d, 10, q=None, y=None)
    assert rc == (NO_DEVICE if not HAS_GPU else INVALID)  # on a GPU the fake pointers fail


@no_device_only
def test_from_state_valid_without_device():
    assert _from_state(_desc(), 0, halo_k=None, halo_v=None, A_init=None) == NO_DEVICE
    assert _from_state(_desc(), 50) == NO_DEVICE


# ---------------------------------------------------------------- tc_backward
def _backward(desc, **ptrs):
    names = ["q", "k", "v", "lam", "eta", "g", "dy", "dq", "dk", "dv", "dlam", "deta", "dg"]
    p = {n: FAKE for n in names}
    p.update(ptrs)
    return _lib().tc_backward(ctypes.byref(desc), *[p[n] for n in names], FAKE, 1 << 40, None)


def test_backward_rejects_invalid():
    d = _desc()
    assert _backward(_desc(flags=tc.TC_PREFILL_DELTA_RULE)) == UNSUPPORTED
    assert _lib().tc_backward_workspace_size(ctypes.byref(_desc(flags=tc.TC_PREFILL_L1_ONLY))) \
        == tc.SIZE_ERROR
    for name in ("q", "dy", "dq", "dv"):
        assert _backward(d, **{name: None}) == INVALID, name
    for name in ("k", "dk"):
        assert _backward(d, **{name: SKEW}) == INVALID, name
    for name in ("lam", "dlam", "dg"):
        assert _backward(d, **{name: None}) == INVALID, name


@no_device_only
def test_backward_valid_without_device():
    assert _backward(_desc()) == NO_DEVICE
    assert _lib().tc_backward_workspace_size(ctypes.byref(_desc())) > 0


# ---------------------------------------------------------------- tc_state_fold
def _fold(B=2, H=3, dk=64, dv=64, n=2, dA=FAKE, E=FAKE, lam=FAKE, out=FAKE):
    return _lib().tc_state_fold(B, H, dk, dv, n, dA, E, lam, out, None)


@pytest.mark.parametrize("bad", [dict(B=0), dict(H=0), dict(dk=0), dict(dv=129), dict(n=-1),
                                 dict(out=None), dict(lam=None), dict(dA=None), dict(E=None),
                                 dict(out=SKEW), dict(dA=SKEW)])
def test_state_fold_rejects_invalid(bad):
    assert _fold(**bad) == INVALID


@no_device_only
def test_state_fold_valid_without_device():
    assert _fold() == NO_DEVICE
    assert _fold(n=0, dA=None, E=None) == NO_DEVICE  # no pieces before: A = 0


# ---------------------------------------------------------------- tc_decode_step_ragged
def _state(**kw):
    base = dict(B=2, H=2, dk=64, dv=64, W=16, t=0, kv_dtype=tc.TC_BF16, ring_k=0x10000,
                ring_v=0x10000, A=0x10000, lam=0x10000, eta=0x10000, g=0x10000, write_rule=0)
    base.update(kw)
    return tc.DecodeStateC(**base)


def _ragged(st, t_rows=FAKE):
    return _lib().tc_decode_step_ragged(ctypes.byref(st), t_rows, FAKE, FAKE, FAKE, FAKE, None)


def test_ragged_decode_rejects_invalid():
    assert _ragged(_state(), t_rows=None) == INVALID
    assert _ragged(_state(), t_rows=SKEW) == INVALID  # int64 clocks must be 8-byte aligned
    assert _ragged(_state(write_rule=2)) == INVALID
    assert _lib().tc_decode_step(ctypes.byref(_state(write_rule=-1)), FAKE, FAKE, FAKE, FAKE,
                                 None) == INVALID


@no_device_only
def test_ragged_decode_valid_without_device():
    st = _state(t=7, write_rule=tc.TC_WRITE_DELTA)
    assert _ragged(st) == NO_DEVICE
    assert st.t == 7  # the host clock is not used by the ragged step


# ---------------------------------------------------------------- tc_prefill_no_alloc
def _no_alloc(desc):
    return _lib().tc_prefill_no_alloc(ctypes.byref(desc), *[FAKE] * 8, None)


def test_no_alloc_rejects_invalid_and_oversized():
    assert _no_alloc(_desc(B=0)) == INVALID
    big = _desc(B=8, H=16, T=65536, W=64, C=64)  # float32 path: one state per chunk
    assert tc.prefill_workspace_size(big) > tc.NO_ALLOC_SCRATCH_BYTES
    assert _no_alloc(big) == WORKSPACE


def test_fused_workspace_fits_the_no_alloc_scratch():
    # the fused kernel's span summaries are bounded by about 4 matrices per SM
    # whatever the length; the general path keeps two states per chunk of 128 rows
    for B, H, T, W in [(8, 12, 4096, 512), (1, 16, 32768, 1024), (64, 64, 65536, 128)]:
        d = _desc(B=B, H=H, T=T, W=W, C=64, dtype=tc.TC_BF16)
        with tc.prefill_path("fused"):
            assert 0 <= tc.prefill_workspace_size(d) <= 4 * 148 * 64 * 64 * 4
        with tc.prefill_path("general"):
            chunks = B * H * ((T + 127) // 128)
            assert tc.prefill_workspace_size(d) >= 2 * chunks * 64 * 64 * 4


def test_prefill_path_setting():
    """tc_set_prefill_path / tc_get_prefill_path / tc_prefill_path_for: the
    choice between the two tensor-core paths for the calls both take, and
    which path a call takes (no device needed)."""
    assert tc.get_prefill_path() == "auto"
    lm = _desc(B=8, H=12, T=4096, W=512, C=64, dtype=tc.TC_BF16)
    odd = _desc(B=8, H=12, T=4096, W=500, C=64, dtype=tc.TC_BF16)  # W not a multiple of 128
    d128 = _desc(B=2, H=2, T=1000, dk=128, dv=128, W=256, C=64, dtype=tc.TC_BF16)
    f32 = _desc(dtype=tc.TC_F32)
    assert tc.prefill_path_for(lm) == "general"  # auto: fixed-length calls on the general path
    assert tc.prefill_path_for(odd) == "general" and tc.prefill_path_for(d128) == "general"
    assert tc.prefill_path_for(f32) is None      # float32: the SIMT path
    with tc.prefill_path("fused"):
        assert tc.get_prefill_path() == "fused"
        assert tc.prefill_path_for(lm) == "fused"
        assert tc.prefill_path_for(lm, 1024) == "fused"  # continuation at t0 >= W
        assert tc.prefill_path_for(lm, 100) == "general"  # partial halo: only the general path
        assert tc.prefill_path_for(odd) == "general"     # only the general path takes it
        l1 = _desc(B=8, H=12, T=4096, W=512, C=64, dtype=tc.TC_BF16, l1_only=True)
        assert tc.prefill_path_for(l1) == "fused"
        # the delta rule's window part runs on the fused kernel, its memory in chunks
        assert tc.prefill_path_for(_desc(B=8, H=12, T=4096, W=512, C=64, dtype=tc.TC_BF16,
                                         flags=tc.TC_PREFILL_DELTA_RULE)) == "fused"
    assert tc.get_prefill_path() == "auto"
    with tc.prefill_path(tc.TC_PATH_GENERAL):
        assert tc.prefill_path_for(lm) == "general"
    assert tc.prefill_path_for(_desc(B=0)) is None
    for bad in (3, -1, 100):
        with pytest.raises(tc.TCError):
            tc.set_prefill_path(bad)
    assert tc.get_prefill_path() == "auto"  # a refused value keeps the setting


@no_device_only
def test_no_alloc_valid_without_device():
    assert _no_alloc(_desc()) == NO_DEVICE


def test_prefill_path_binding_edge_cases():
    """The binding refuses unknown names, and the context manager restores
    the previous setting even when its body raises."""
    assert tc.get_prefill_path() == "auto"
    with pytest.raises(tc.TCError):
        tc.set_prefill_path("fastest")
    with pytest.raises(RuntimeError):
        with tc.prefill_path("general"):
            assert tc.get_prefill_path() == "general"
            raise RuntimeError("inside")
    assert tc.get_prefill_path() == "auto"
    with tc.prefill_path("fused"):
        with tc.prefill_path("general"):
            assert tc.get_prefill_path() == "general"
        assert tc.get_prefill_path() == "fused"
    assert tc.get_prefill_path() == "auto"
