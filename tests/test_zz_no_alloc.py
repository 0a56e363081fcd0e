"""tc_prefill_no_alloc against tc_prefill, on the GPU.

tc_prefill_no_alloc serves callers that cannot allocate device memory: it
runs the same prefill with the library's built-in scratch array in place of
a caller workspace.  These tests call it through the C-ABI twice in a row
with different inputs (the second call finds the first call's data in the
shared scratch) and require each result to equal tc_prefill's bit for bit:
both run the same deterministic kernels on the same inputs, so any
difference would be scratch data leaking from one call into the next.  This
file is named so that pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads as wl

pytestmark = pytest.mark.gpu


def _tc():
    import sliding_window_attention_tc_b200 as tc
    return tc


def _no_alloc(tc, x, dev):
    B, H, T, dk = x.q.shape
    dv = x.v.shape[-1]
    bf16 = x.q.dtype == torch.bfloat16
    desc = tc.make_prefill_desc(B, H, T, dk, dv, x.W, x.C, tc.TC_BF16 if bf16 else tc.TC_F32)
    args = [t.to(dev).contiguous() for t in (x.q, x.k, x.v, x.lam, x.eta, x.g)]
    y = torch.empty(B, H, T, dv, dtype=x.q.dtype, device=dev)
    A = torch.empty(B, H, dk, dv, dtype=torch.float32, device=dev)
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    st = tc.lib_handle().tc_prefill_no_alloc(ctypes.byref(desc), *[p(a) for a in args], p(y), p(A),
                                              ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, tc.status_string(st)
    return y, A, args


CASES = [
    # bf16, d = 64, W = 128: tensor-core path; several spans per head, so the
    # span summaries live in the scratch array
    (2, 2, 1000, 64, 64, 128, 64, "bf16"),
    # float32: portable path; the chunk states live in the scratch array
    (2, 3, 300, 64, 64, 37, 13, "f32"),
]


@pytest.mark.parametrize("case", CASES, ids=[c[-1] for c in CASES])
def test_no_alloc_matches_workspace_entry_point(cuda_device, case):
    tc = _tc()
    B, H, T, dk, dv, W, C, dtype = case
    desc = tc.make_prefill_desc(B, H, T, dk, dv, W, C, tc.TC_BF16 if dtype == "bf16" else tc.TC_F32)
    assert 0 < tc.prefill_workspace_size(desc) <= tc.NO_ALLOC_SCRATCH_BYTES
    for seed in (11, 12):  # two calls in a row, different inputs
        x = wl.random_prefill(B, H, T, dk, dv, W, C, dtype=dtype, seed=seed)
        y_na, A_na, args = _no_alloc(tc, x, cuda_device)
        y_ref, A_ref = tc.prefill(*args, W, C)
        torch.cuda.synchronize()
        assert tc.device_status() == 0
        assert torch.equal(y_na, y_ref)
        assert torch.equal(A_na, A_ref)
        assert np.isfinite(y_ref.float().cpu().numpy()).all()


def test_no_alloc_rejects_more_scratch_than_it_has(cuda_device):
    tc = _tc()
    # float32 with W = 1, C = 1: one 16x16 chunk state per eviction -> far
    # more than the built-in array holds
    desc = tc.make_prefill_desc(1, 8, 70000, 16, 16, 1, 1, tc.TC_F32)
    assert tc.prefill_workspace_size(desc) > tc.NO_ALLOC_SCRATCH_BYTES
    st = tc.lib_handle().tc_prefill_no_alloc(ctypes.byref(desc), *([None] * 8), None)
    assert st == 7  # TC_ERR_WORKSPACE, nothing enqueued


def test_no_alloc_runs_the_fused_kernel_when_only_its_scratch_fits(cuda_device):
    """The LM workload (8 x 12 x 4096, d = 64, W = 512): the general path
    would need 100 MiB of per-chunk states, the fused kernel fits the
    built-in array.  Under the automatic choice the call runs on the fused
    kernel and equals tc_prefill on that kernel bit for bit; with the general
    path chosen explicitly it is refused."""
    tc = _tc()
    x = wl.prefill_config("lm_prefill_bf16")
    B, H, T, d = x.q.shape
    desc = tc.make_prefill_desc(B, H, T, d, d, x.W, x.C, tc.TC_BF16)
    assert tc.get_prefill_path() == "auto"
    assert tc.prefill_workspace_size(desc) > tc.NO_ALLOC_SCRATCH_BYTES
    with tc.prefill_path("fused"):
        assert tc.prefill_workspace_size(desc) <= tc.NO_ALLOC_SCRATCH_BYTES
    y_na, A_na, args = _no_alloc(tc, x, cuda_device)
    with tc.prefill_path("fused"):
        y_ref, A_ref = tc.prefill(*args, x.W, x.C)
    torch.cuda.synchronize()
    assert tc.device_status() == 0
    assert torch.equal(y_na, y_ref) and torch.equal(A_na, A_ref)
    with tc.prefill_path("general"):
        p = lambda t: ctypes.c_void_p(t.data_ptr())
        st = tc.lib_handle().tc_prefill_no_alloc(ctypes.byref(desc), *[p(a) for a in args], p(y_na), p(A_na),
                                                  ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == 7  # TC_ERR_WORKSPACE, nothing enqueued
