"""The tensor-core prefill's bounded waits, made to run out on purpose.

Every wait inside the tensor-core kernels (for a copy, a tensor-core product
or another warp) gives up after a limit, records TC_ERR_DEVICE_TIMEOUT in the
device status word and lets every role drain its copies and products before
the kernel returns; a stalled pipeline therefore ends with an error instead
of a hung GPU.  The limit is 2 s by default; tc_set_wait_limit_ns lowers it.
With a 1 ns limit every wait that is not satisfied at its first try gives
up (a copy from memory, or a product the tensor core is still computing,
takes far longer), so the call must report the timeout, and the next call
with the default limit, on the same context, must again match the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl

pytestmark = pytest.mark.gpu

TC_ERR_DEVICE_TIMEOUT = 6


def _run(tc, x, dev):
    args = [t.to(dev).contiguous() for t in (x.q, x.k, x.v, x.lam, x.eta, x.g)]
    y, A = tc.prefill(*args, x.W, x.C)
    torch.cuda.synchronize()
    return y, A


def test_wait_limit_runs_out_and_the_context_stays_usable(cuda_device):
    import sliding_window_attention_tc_b200 as tc
    # bf16, d = 64, W = 128: the tensor-core path, several spans (pre-pass too)
    B, H, T = 2, 4, 2048
    x = wl.random_prefill(B, H, T, 64, 64, 128, 64, dtype="bf16", seed=31)
    desc = tc.make_prefill_desc(B, H, T, 64, 64, 128, 64, tc.TC_BF16)
    assert tc.prefill_launch_count(desc) == 3  # summaries, prefix, main kernel
    assert tc.device_status() == 0
    try:
        tc.set_wait_limit_ns(1)
        _run(tc, x, cuda_device)
        assert tc.device_status() == TC_ERR_DEVICE_TIMEOUT
    finally:
        tc.set_wait_limit_ns(0)
    assert tc.device_status() == 0  # read and cleared
    y, A = _run(tc, x, cuda_device)
    assert tc.device_status() == 0
    yo, Ao = oracle.prefill(x.q, x.k, x.v, x.lam, x.eta, x.g, x.W)
    y = y.float().cpu().numpy()
    A = A.cpu().numpy()
    assert np.linalg.norm(y - yo) <= 1e-2 * np.linalg.norm(yo)
    assert np.linalg.norm(A - Ao) <= 1e-3 * np.linalg.norm(Ao)
