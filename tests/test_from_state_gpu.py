"""GPU parity of a continued sequence: tc_prefill_from_state, tc_state_fold
and the sequence-sharded prefill, against the float64 oracle run over the
whole unsplit sequence.

A sequence of T tokens is cut at t0.  The continuation gets the new tokens,
the keys and values of the min(t0, W) tokens before t0 (the window content),
and A after the evictions before t0.  With those it must produce exactly what
the layer produces for tokens t0 .. T-1 (Fig. 2 of the paper, token by
token), and the same final A.

Tolerances are those of the prefill parity tests:
- float32: max|x - ref| / max|ref| <= 1e-5;
- bf16: ||x - ref|| / ||ref|| <= 1e-2 on y and <= 1e-3 on A.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl

pytestmark = pytest.mark.gpu

F32_TOL = 1e-5
BF16_Y_TOL = 1e-2
BF16_A_TOL = 1e-3


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


def _check(x, y, A, y_ref, A_ref):
    if x.q.dtype == torch.float32:
        if y is not None:
            assert max_rel(y, y_ref) <= F32_TOL
        assert max_rel(A, A_ref) <= F32_TOL
    else:
        if y is not None:
            assert rel_l2(y, y_ref) <= BF16_Y_TOL
        assert rel_l2(A, A_ref) <= BF16_A_TOL


def _continue(x, t0, dev, state_only=False):
    """tc_prefill_from_state on tokens t0.. of x, with the halo and A_init the
    oracle gives for tokens ..t0-1."""
    tc = _tc()
    n = min(t0, x.W)
    A_init = None
    if t0 > 0:
        _, A_pre = oracle.prefill(x.q[:, :, :t0], x.k[:, :, :t0], x.v[:, :, :t0], x.lam, x.eta,
                                  x.g, x.W)
        A_init = torch.from_numpy(A_pre).float().to(dev)
    d = lambda t: t.to(dev).contiguous()
    halo_k = d(x.k[:, :, t0 - n:t0]) if n > 0 else None
    halo_v = d(x.v[:, :, t0 - n:t0]) if n > 0 else None
    y, A = tc.prefill_from_state(None if state_only else d(x.q[:, :, t0:]), d(x.k[:, :, t0:]),
                                 d(x.v[:, :, t0:]), d(x.lam), d(x.eta), d(x.g), x.W, x.C, t0,
                                 halo_k, halo_v, A_init, state_only=state_only)
    torch.cuda.synchronize()
    assert tc.device_status() == 0
    return (None if y is None else y.float().cpu().numpy()), A.cpu().numpy()


CASES = [
    # B, H, T, dk, dv, W, C, dtype, t0
    (2, 2, 700, 64, 64, 128, 64, "bf16", 0),      # tensor-core path, no halo
    (2, 2, 700, 64, 64, 128, 64, "bf16", 128),    # tensor-core path, full halo
    (2, 2, 700, 64, 64, 128, 64, "bf16", 300),    # t0 not a multiple of the tile
    (1, 3, 1000, 64, 64, 256, 64, "bf16", 600),   # W = 256, several spans
    (1, 2, 500, 64, 64, 128, 64, "bf16", 499),    # one new token
    (2, 2, 700, 64, 64, 128, 64, "bf16", 50),     # partial halo (t0 < W): portable path
    (1, 2, 300, 16, 16, 32, 8, "f32", 20),        # float32, partial halo
    (1, 2, 300, 16, 16, 32, 8, "f32", 150),       # float32, full halo
    (1, 2, 300, 32, 16, 48, 13, "f32", 299),      # d_k != d_v, ragged chunk, one token
]


@pytest.mark.parametrize("case", CASES, ids=[f"{c[7]}_W{c[5]}_t0{c[8]}" for c in CASES])
def test_prefill_from_state_matches_whole_sequence(cuda_device, case, both_paths):
    B, H, T, dk, dv, W, C, dtype, t0 = case
    x = wl.random_prefill(B, H, T, dk, dv, W, C, dtype=dtype, seed=600 + t0)
    y_ref, A_ref = oracle.prefill(x.q, x.k, x.v, x.lam, x.eta, x.g, W)
    y, A = _continue(x, t0, cuda_device)
    _check(x, y, A, y_ref[:, :, t0:], A_ref)


@pytest.mark.parametrize("case", [CASES[1], CASES[3], CASES[7]], ids=["bf16", "bf16_W256", "f32"])
def test_state_only_gives_the_final_state(cuda_device, case, both_paths):
    B, H, T, dk, dv, W, C, dtype, t0 = case
    x = wl.random_prefill(B, H, T, dk, dv, W, C, dtype=dtype, seed=700 + t0)
    _, A_ref = oracle.prefill(x.q, x.k, x.v, x.lam, x.eta, x.g, W)
    y, A = _continue(x, t0, cuda_device, state_only=True)
    assert y is None
    _check(x, None, A, None, A_ref)


def test_state_fold_is_the_decayed_sum(cuda_device):
    tc = _tc()
    gen = torch.Generator().manual_seed(5)
    n, B, H, dk, dv = 4, 2, 3, 8, 5
    dA = torch.randn(n, B, H, dk, dv, generator=gen, dtype=torch.float64)
    E = torch.tensor([7, 0, 130, 3], dtype=torch.int64)
    lam = torch.tensor([0.9, 0.99, 0.5], dtype=torch.float64)
    # closed form: sum_s lam^(E_{s+1} + ... + E_{n-1}) dA_s
    ref = torch.zeros(B, H, dk, dv, dtype=torch.float64)
    for s in range(n):
        ref += (lam ** float(E[s + 1:].sum())).view(1, H, 1, 1) * dA[s]
    out = tc.state_fold(dA.float().to(cuda_device), E.to(cuda_device), lam.float().to(cuda_device))
    torch.cuda.synchronize()
    assert max_rel(out.cpu().numpy(), ref.numpy()) <= 1e-6
    zero = tc.state_fold(dA[:0].float().to(cuda_device), E[:0].to(cuda_device),
                         lam.float().to(cuda_device))
    torch.cuda.synchronize()
    assert float(zero.abs().max()) == 0.0


SHARDED = [
    # lens per piece, B, H, d, W, C, dtype
    ([300, 150, 250], 2, 2, 64, 128, 64, "bf16"),   # every piece longer than W
    ([40, 30, 100, 60], 1, 2, 16, 64, 8, "f32"),    # short pieces: halos span pieces
]


@pytest.mark.parametrize("lens,B,H,d,W,C,dtype", SHARDED, ids=["bf16", "f32_short"])
def test_sharded_phases_on_one_gpu(cuda_device, lens, B, H, d, W, C, dtype):
    """The phases of the sequence-sharded prefill, run for each piece in turn
    on one GPU with the library (the all-gathers become stacks)."""
    from sliding_window_attention_tc_b200 import sharded
    x = wl.random_prefill(B, H, sum(lens), d, d, W, C, dtype=dtype, seed=800)
    y_ref, A_ref = oracle.prefill(x.q, x.k, x.v, x.lam, x.eta, x.g, W)
    dev = cuda_device
    lam, eta, g = (t.to(dev) for t in (x.lam, x.eta, x.g))
    bounds = np.cumsum([0] + lens)
    pieces = [[t[:, :, bounds[r]:bounds[r + 1]].to(dev).contiguous() for t in (x.q, x.k, x.v)]
              for r in range(len(lens))]
    tails = [sharded.tail(p[1], p[2], W) for p in pieces]
    tails_k = torch.stack([t[0] for t in tails])
    tails_v = torch.stack([t[1] for t in tails])
    info = [sharded.piece_of(r, lens, tails_k, tails_v, W) for r in range(len(lens))]
    dA_all = torch.stack([sharded.piece_state(info[r], pieces[r][1], pieces[r][2], lam, eta, g, W, C)
                          for r in range(len(lens))])
    E_all = torch.tensor([p.evictions for p in info], dtype=torch.int64, device=dev)
    for r in range(len(lens)):
        y, A = sharded.finish(r, info[r], dA_all, E_all, *pieces[r], lam, eta, g, W, C)
        torch.cuda.synchronize()
        assert _tc().device_status() == 0
        last = r == len(lens) - 1
        _check(x, y.float().cpu().numpy(), A.cpu().numpy() if last else A_ref,
               y_ref[:, :, bounds[r]:bounds[r + 1]], A_ref)
