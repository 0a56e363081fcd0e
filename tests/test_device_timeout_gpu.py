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
    # bf16, d = 64, W = 128 on the fused kernel: several spans (pre-pass too)
    B, H, T = 2, 4, 2048
    x = wl.random_prefill(B, H, T, 64, 64, 128, 64, dtype="bf16", seed=31)
    desc = tc.make_prefill_desc(B, H, T, 64, 64, 128, 64, tc.TC_BF16)
    with tc.prefill_path("fused"):
        assert tc.prefill_path_for(desc) == "fused"
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


def _rel(x, ref):
    return float(np.linalg.norm(np.asarray(x, np.float64) - ref) / np.linalg.norm(ref))


@pytest.mark.parametrize("d,W", [(64, 200), (128, 256)], ids=["d64_W200", "d128_W256"])
def test_general_path_wait_limit_runs_out(cuda_device, d, W):
    """The general tensor-core prefill (sums, window with the reads): the same bounded
    waits and drains, then a clean call on the same context."""
    import sliding_window_attention_tc_b200 as tc
    B, H, T = 2, 4, 1500
    x = wl.random_prefill(B, H, T, d, d, W, 64, dtype="bf16", seed=41)
    desc = tc.make_prefill_desc(B, H, T, d, d, W, 64, tc.TC_BF16)
    assert tc.prefill_launch_count(desc) == 3  # sums, scan, window (with the reads)
    assert tc.device_status() == 0
    try:
        tc.set_wait_limit_ns(1)
        _run(tc, x, cuda_device)
        assert tc.device_status() == TC_ERR_DEVICE_TIMEOUT
    finally:
        tc.set_wait_limit_ns(0)
    y, A = _run(tc, x, cuda_device)
    assert tc.device_status() == 0
    yo, Ao = oracle.prefill(x.q, x.k, x.v, x.lam, x.eta, x.g, x.W)
    assert _rel(y.float().cpu().numpy(), yo) <= 1e-2
    assert _rel(A.cpu().numpy(), Ao) <= 1e-3


def test_backward_wait_limit_runs_out(cuda_device):
    """The backward's tensor-core kernels (window, per-chunk sums and
    gradients): the waits give up and drain, then a clean call matches the
    oracle backward."""
    import sliding_window_attention_tc_b200 as tc
    B, H, T, d, W = 1, 2, 900, 64, 128
    x = wl.random_prefill(B, H, T, d, d, W, 64, dtype="bf16", seed=43)
    gen = torch.Generator().manual_seed(44)
    dy = (torch.randn(B, H, T, d, generator=gen) / 4).to(x.q.dtype)
    dev = cuda_device
    args = [t.to(dev).contiguous() for t in (x.q, x.k, x.v, x.lam, x.eta, x.g)]
    assert tc.backward_launch_count(x.q, W)[1]
    try:
        tc.set_wait_limit_ns(1)
        tc.backward(*args, W, dy.to(dev))
        torch.cuda.synchronize()
        assert tc.device_status() == TC_ERR_DEVICE_TIMEOUT
    finally:
        tc.set_wait_limit_ns(0)
    got = tc.backward(*args, W, dy.to(dev))
    torch.cuda.synchronize()
    assert tc.device_status() == 0
    ref = oracle.backward(x.q, x.k, x.v, x.lam, x.eta, x.g, W, dy)
    for a, b in zip(got[:3], ref[:3]):
        a = a.cpu().numpy()
        assert np.abs(a - b).max() <= 2e-4 * np.abs(b).max()
