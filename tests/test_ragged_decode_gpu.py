"""GPU parity of tc_decode_step_ragged: one decode batch whose rows sit at
different positions of their own sequences (some before the window is full,
some long past it), plus an empty row, against the float64 oracle prefill of
each row's whole sequence.

Tolerances are those of the decode parity tests: float32 max-relative 1e-5;
bf16 relative L2 1e-2 on y and 1e-3 on A.
"""
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


@pytest.mark.parametrize("dtype,d", [("f32", 32), ("bf16", 64)])
def test_ragged_rows_match_their_own_sequences(cuda_device, dtype, d):
    import sliding_window_attention_tc_b200 as tc
    H, W, steps, C = 2, 32, 9, 8
    clocks = [0, 7, W - 1, W, W + 37, -1]  # the last row is empty
    B = len(clocks)
    T_max = max(clocks) + steps
    x = wl.random_prefill(B, H, T_max, d, d, W, C, dtype=dtype, seed=900 + d)
    dev = cuda_device
    dt = x.k.dtype
    ring_k = torch.zeros(B, H, W, d, dtype=dt)
    ring_v = torch.zeros(B, H, W, d, dtype=dt)
    A = torch.zeros(B, H, d, d)
    for b, t in enumerate(clocks):
        if t <= 0:
            continue
        _, Ab = oracle.prefill(x.q[b:b + 1, :, :t], x.k[b:b + 1, :, :t], x.v[b:b + 1, :, :t],
                               x.lam, x.eta, x.g, W)
        A[b] = torch.from_numpy(Ab[0]).float()
        for j in range(max(0, t - W), t):
            ring_k[b, :, j % W] = x.k[b, :, j]
            ring_v[b, :, j % W] = x.v[b, :, j]
    # sentinel contents of the empty row
    ring_k[B - 1] = 3.0
    A[B - 1] = 5.0
    st = tc.DecodeState(ring_k.to(dev), ring_v.to(dev), A.to(dev), x.lam.to(dev), x.eta.to(dev),
                        x.g.to(dev), 0)
    t_rows = torch.tensor(clocks, dtype=torch.int64, device=dev)
    ys = []
    for i in range(steps):
        # row b reads token clocks[b] + i of its own sequence
        idx = [max(t, 0) + i for t in clocks]
        pick = lambda z: torch.stack([z[b, :, idx[b]] for b in range(B)]).to(dev).contiguous()
        y = torch.full((B, H, d), 7.0, dtype=dt, device=dev)
        tc.decode_step_ragged(st, t_rows, pick(x.q), pick(x.k), pick(x.v), y=y)
        ys.append(y.float().cpu())
    torch.cuda.synchronize()
    assert tc.device_status() == 0
    assert t_rows.cpu().tolist() == [t + steps if t >= 0 else -1 for t in clocks]
    y = torch.stack(ys, 2).numpy()  # [B,H,steps,d]
    tol_y, tol_A, err = (1e-5, 1e-5, max_rel) if dtype == "f32" else (1e-2, 1e-3, rel_l2)
    for b, t in enumerate(clocks[:-1]):
        yo, Ao = oracle.prefill(x.q[b:b + 1, :, :t + steps], x.k[b:b + 1, :, :t + steps],
                                x.v[b:b + 1, :, :t + steps], x.lam, x.eta, x.g, W)
        assert err(y[b], yo[0, :, t:t + steps]) <= tol_y, (b, t)
        assert err(st.A[b].cpu().numpy(), Ao[0]) <= tol_A, (b, t)
    # the empty row is untouched
    assert torch.all(st.ring_k[B - 1].float() == 3.0)
    assert torch.all(st.A[B - 1] == 5.0)
    assert np.all(y[B - 1] == 7.0)
