"""GPU parity of tc_backward against the float64 oracle backward (itself
pinned by central differences of the forward oracle).  Both sides read the
same rounded inputs (bf16 values widened exactly).  The GPU accumulates in
float32; on the tensor-core path (bf16, d = 64) the products of the bf16
inputs are exact and P, dS and the float32 states enter as bf16 hi + lo
pairs (remainder below 2^-17 relative), so the bound is float32-level for
every input dtype: max|x - ref| / max|ref| <= 2e-4 per gradient tensor (sums
over up to T*d terms)."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl

pytestmark = pytest.mark.gpu


def max_rel(x, ref):
    x, ref = np.asarray(x, np.float64), np.asarray(ref, np.float64)
    den = np.abs(ref).max()
    return float(np.abs(x - ref).max() / den) if den > 0 else float(np.abs(x).max())


CASES = [
    # B, H, T, dk, dv, W, dtype
    (2, 2, 150, 16, 16, 8, "f32"),
    (1, 2, 300, 32, 32, 64, "f32"),
    (1, 1, 100, 16, 8, 5, "f32"),       # d_k != d_v
    (1, 2, 40, 16, 16, 64, "f32"),      # T < W: no eviction, L2 gradients of lambda, eta are 0
    (1, 2, 300, 64, 64, 128, "bf16"),   # bf16, d = 64: tensor-core window part
    (2, 3, 1000, 64, 64, 200, "bf16"),  # W not a multiple of the 64-row tiles, ragged T
    (1, 2, 77, 64, 64, 512, "bf16"),    # W > T, one partial 128-row block
    (1, 1, 700, 64, 64, 1, "bf16"),     # W = 1: every key its own query only
    (1, 2, 2100, 64, 64, 512, "bf16"),  # many tiles per block, 2 blocks per SM
    (1, 2, 200, 128, 128, 64, "bf16"),  # d = 128: tensor-core window, SIMT memory part
    (2, 2, 700, 128, 128, 200, "bf16"), # d = 128, W not a multiple of the tiles, several chunks
    (1, 1, 300, 128, 128, 512, "bf16"), # d = 128, W > T
    (1, 1, 150, 128, 40, 16, "f32"),    # d_k = 128, d_v not a multiple of 32
]


@pytest.mark.parametrize("case", CASES, ids=[f"{c[6]}_T{c[2]}_d{c[3]}x{c[4]}_W{c[5]}" for c in CASES])
def test_backward_matches_oracle(cuda_device, case):
    import sliding_window_attention_tc_b200 as tc
    B, H, T, dk, dv, W, dtype = case
    x = wl.random_prefill(B, H, T, dk, dv, W, 8, dtype=dtype, seed=70 + T)
    gen = torch.Generator().manual_seed(71)
    dy = (torch.randn(B, H, T, dv, generator=gen, dtype=torch.float64) / 4).to(x.q.dtype)
    dev = cuda_device
    d = lambda t: t.to(dev).contiguous()
    got = tc.backward(d(x.q), d(x.k), d(x.v), d(x.lam), d(x.eta), d(x.g), W, d(dy))
    torch.cuda.synchronize()
    assert tc.device_status() == 0
    # bf16 with d = 64 or 128 takes the tensor-core window kernels, every other case SIMT
    assert tc.backward_launch_count(x.q, W, x.v)[1] == (dtype == "bf16" and dk == dv and dk in (64, 128))
    ref = oracle.backward(x.q, x.k, x.v, x.lam, x.eta, x.g, W, dy)
    for name, a, b in zip(("dq", "dk", "dv", "dlam", "deta", "dg"), got, ref):
        if np.abs(b).max() == 0:
            assert float(a.abs().max()) <= 1e-6, name
        else:
            assert max_rel(a.cpu().numpy(), b) <= 2e-4, (name, max_rel(a.cpu().numpy(), b))


def test_backward_is_bit_for_bit_repeatable(cuda_device):
    """Every gradient is a fixed-order sum (no atomics): two calls on the
    same inputs give identical bits."""
    import sliding_window_attention_tc_b200 as tc
    B, H, T, d, W = 2, 4, 1100, 64, 128
    x = wl.random_prefill(B, H, T, d, d, W, 8, dtype="bf16", seed=5)
    gen = torch.Generator().manual_seed(6)
    dy = (torch.randn(B, H, T, d, generator=gen) / 4).to(x.q.dtype)
    dev = cuda_device
    args = [t.to(dev).contiguous() for t in (x.q, x.k, x.v, x.lam, x.eta, x.g)]
    a = tc.backward(*args, W, dy.to(dev))
    b = tc.backward(*args, W, dy.to(dev))
    torch.cuda.synchronize()
    assert tc.device_status() == 0
    for name, u, w in zip(("dq", "dk", "dv", "dlam", "deta", "dg"), a, b):
        assert torch.equal(u, w), name


def test_backward_full_lm_shape_one_head(cuda_device):
    """The LM workload at full size (8 x 12 x 4096, d = 64, W = 512), the
    launch configuration the benchmark times.  Heads are independent, and
    dlambda, deta, dg of head h sum over the batch only, so the oracle run on
    head h alone (all 8 batch rows) checks every output of that head."""
    import sliding_window_attention_tc_b200 as tc
    x = wl.prefill_config("lm_prefill_bf16")
    B, H, T, d = x.q.shape
    gen = torch.Generator().manual_seed(11)
    dy = (torch.randn(B, H, T, d, generator=gen) / 8).to(x.q.dtype)
    dev = cuda_device
    args = [t.to(dev).contiguous() for t in (x.q, x.k, x.v, x.lam, x.eta, x.g)]
    assert tc.backward_launch_count(x.q, x.W)[1]
    got = tc.backward(*args, x.W, dy.to(dev))
    torch.cuda.synchronize()
    assert tc.device_status() == 0
    h = 7
    sl = lambda t: t[:, h:h + 1]
    ref = oracle.backward(sl(x.q), sl(x.k), sl(x.v), x.lam[h:h + 1], x.eta[h:h + 1], x.g[h:h + 1],
                          x.W, sl(dy))
    for name, a, r in zip(("dq", "dk", "dv"), got[:3], ref[:3]):
        err = max_rel(sl(a).cpu().numpy(), r)
        assert err <= 2e-4, (name, err)
    for name, a, r in zip(("dlam", "deta", "dg"), got[3:], ref[3:]):
        err = abs(float(a[h]) - float(r[0])) / abs(float(r[0]))
        assert err <= 2e-4, (name, err)
