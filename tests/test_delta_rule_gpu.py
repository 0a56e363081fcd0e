"""GPU parity of the delta-rule write (Fig. 2 step (3), update =
k_old (v_old - k_old^T A)^T) against the float64 oracle running the same
rule: decode steps, the prefill, a continued prefill, and decode continuing a
prefill.

Tolerances as for the outer-product write: float32 max-relative 1e-5; bf16
relative L2 1e-2 on y and 1e-3 on A.
"""
import math

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


def rel_l2(x, ref):
    x, ref = np.asarray(x, np.float64), np.asarray(ref, np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(x - ref) / den) if den > 0 else float(np.linalg.norm(x))


def _tc():
    import sliding_window_attention_tc_b200 as tc
    return tc


def _close(dtype, y, y_ref, A, A_ref):
    if dtype == "f32":
        assert max_rel(y, y_ref) <= 1e-5
        assert max_rel(A, A_ref) <= 1e-5
    else:
        assert rel_l2(y, y_ref) <= 1e-2
        assert rel_l2(A, A_ref) <= 1e-3


@pytest.mark.parametrize("dtype,d", [("f32", 32), ("f32", 128), ("bf16", 64)])
def test_delta_decode_from_empty(cuda_device, dtype, d):
    tc = _tc()
    B, H, W, steps = 2, 2, 16, 50
    gen = torch.Generator().manual_seed(d)
    dt = wl.torch_dtype(dtype)
    s = 1.0 / math.sqrt(d)
    q, k, v = ((torch.randn(steps, B, H, d, generator=gen) * s).to(dt) for _ in range(3))
    lam = 0.9 + 0.09 * torch.rand(H, generator=gen)
    eta = 0.2 + torch.rand(H, generator=gen)
    g = torch.randn(H, generator=gen)
    dev = cuda_device
    st = tc.DecodeState.empty(B, H, W, d, d, lam.to(dev), eta.to(dev), g.to(dev), dtype=dt,
                              device=dev)
    st.write_rule = tc.TC_WRITE_DELTA
    ys = [tc.decode_step(st, q[i].to(dev), k[i].to(dev), v[i].to(dev)).float().cpu()
          for i in range(steps)]
    torch.cuda.synchronize()
    assert tc.device_status() == 0
    yo, rko, _, Ao = oracle.decode(np.zeros((B, H, W, d)), np.zeros((B, H, W, d)),
                                   np.zeros((B, H, d, d)), 0, q, k, v, lam, eta, g, rule="delta")
    _close(dtype, torch.stack(ys).numpy(), yo, st.A.cpu().numpy(), Ao)
    np.testing.assert_array_equal(st.ring_k.cpu().double().numpy(), rko)
    # the rule matters here: the outer-product oracle is far away
    yo_outer, *_ = oracle.decode(np.zeros((B, H, W, d)), np.zeros((B, H, W, d)),
                                 np.zeros((B, H, d, d)), 0, q, k, v, lam, eta, g)
    assert rel_l2(yo_outer, yo) > 1e-3


@pytest.mark.parametrize("B,H,T,d,W,dtype", [(1, 2, 200, 16, 8, "f32"), (2, 2, 500, 64, 128, "bf16")],
                         ids=["f32", "bf16"])
def test_delta_prefill_and_continuation(cuda_device, B, H, T, d, W, dtype):
    tc = _tc()
    x = wl.random_prefill(B, H, T, d, d, W, 16, dtype=dtype, seed=31 + d)
    dev = cuda_device
    dd = lambda t: t.to(dev).contiguous()
    y_ref, A_ref = oracle.prefill(x.q, x.k, x.v, x.lam, x.eta, x.g, W, rule="delta")
    y, A = tc.prefill(dd(x.q), dd(x.k), dd(x.v), dd(x.lam), dd(x.eta), dd(x.g), W, 16,
                      delta_rule=True)
    torch.cuda.synchronize()
    assert tc.device_status() == 0
    _close(dtype, y.float().cpu().numpy(), y_ref, A.cpu().numpy(), A_ref)
    # continued from t0 with the halo and the delta-rule state before t0
    t0 = T // 2
    _, A_pre = oracle.prefill(x.q[:, :, :t0], x.k[:, :, :t0], x.v[:, :, :t0], x.lam, x.eta,
                              x.g, W, rule="delta")
    n = min(t0, W)
    y2, A2 = tc.prefill_from_state(dd(x.q[:, :, t0:]), dd(x.k[:, :, t0:]), dd(x.v[:, :, t0:]),
                                   dd(x.lam), dd(x.eta), dd(x.g), W, 16, t0,
                                   dd(x.k[:, :, t0 - n:t0]), dd(x.v[:, :, t0 - n:t0]),
                                   torch.from_numpy(A_pre).float().to(dev), delta_rule=True)
    torch.cuda.synchronize()
    _close(dtype, y2.float().cpu().numpy(), y_ref[:, :, t0:], A2.cpu().numpy(), A_ref)


def test_delta_decode_continues_a_delta_prefill(cuda_device):
    tc = _tc()
    B, H, T, n, d, W = 2, 2, 120, 30, 32, 16
    x = wl.random_prefill(B, H, T + n, d, d, W, 8, dtype="f32", seed=41)
    dev = cuda_device
    dd = lambda t: t.to(dev).contiguous()
    lam, eta, g = dd(x.lam), dd(x.eta), dd(x.g)
    _, A = tc.prefill(dd(x.q[:, :, :T]), dd(x.k[:, :, :T]), dd(x.v[:, :, :T]), lam, eta, g, W, 8,
                      delta_rule=True)
    ring_k = torch.zeros(B, H, W, d, device=dev)
    ring_v = torch.zeros(B, H, W, d, device=dev)
    for j in range(T - W, T):
        ring_k[:, :, j % W] = x.k[:, :, j].to(dev)
        ring_v[:, :, j % W] = x.v[:, :, j].to(dev)
    st = tc.DecodeState(ring_k, ring_v, A, lam, eta, g, T, tc.TC_WRITE_DELTA)
    ys = [tc.decode_step(st, dd(x.q[:, :, j]), dd(x.k[:, :, j]), dd(x.v[:, :, j])).cpu()
          for j in range(T, T + n)]
    yo, Ao = oracle.prefill(x.q, x.k, x.v, x.lam, x.eta, x.g, W, rule="delta")
    assert max_rel(torch.stack(ys, 2).numpy(), yo[:, :, T:]) <= 1e-5
    assert max_rel(st.A.cpu().numpy(), Ao) <= 1e-5


# chunked memory (64 evictions per chunk): several chunks and a ragged last one
CHUNKED = [
    (1, 2, 1000, 32, 16, "f32"),    # 16 chunks, the last of 24 evictions
    (1, 1, 300, 128, 40, "f32"),    # d = 128
    (2, 2, 700, 64, 200, "bf16"),   # W not a multiple of 128: SIMT window part
    (1, 3, 1100, 64, 256, "bf16"),  # tensor-core window part, memory added into y
]


@pytest.mark.parametrize("B,H,T,d,W,dtype", CHUNKED, ids=[f"{c[5]}_T{c[2]}_d{c[3]}_W{c[4]}" for c in CHUNKED])
def test_delta_prefill_chunked(cuda_device, B, H, T, d, W, dtype):
    tc = _tc()
    x = wl.random_prefill(B, H, T, d, d, W, 16, dtype=dtype, seed=7 + T + d)
    dev = cuda_device
    dd = lambda t: t.to(dev).contiguous()
    y_ref, A_ref = oracle.prefill(x.q, x.k, x.v, x.lam, x.eta, x.g, W, rule="delta")
    y, A = tc.prefill(dd(x.q), dd(x.k), dd(x.v), dd(x.lam), dd(x.eta), dd(x.g), W, 16,
                      delta_rule=True)
    torch.cuda.synchronize()
    assert tc.device_status() == 0
    _close(dtype, y.float().cpu().numpy(), y_ref, A.cpu().numpy(), A_ref)

