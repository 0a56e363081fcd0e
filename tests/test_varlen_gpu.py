"""Variable-length prefill (tc_prefill_varlen) against the oracle run per
sequence.

Several sequences of different lengths share one call, packed token-major
([total, H, d]); each is the layer over its own tokens from an empty state
("Tensor Cache: Eviction-conditioned Associative Memory for Transformers",
§3.2 Fig. 2: every sequence runs its own streaming step).  The oracle runs
each sequence alone in the fixed-length layout.  Tolerances are the bf16 ones
of the fixed-length parity tests: ||x - ref|| / ||ref|| <= 1e-2 on y and
<= 1e-3 on A.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl

pytestmark = pytest.mark.gpu

BF16_Y_TOL = 1e-2
BF16_A_TOL = 1e-3
TC_ERR_DEVICE_BOUNDS = 5


def rel_l2(x, ref):
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(x - ref) / den) if den > 0 else float(np.linalg.norm(x))


def _run(tc, x, dev, cu=None, max_seqlen=None, l1_only=False):
    cu = x.cu_seqlens if cu is None else cu
    args = [t.to(dev).contiguous() for t in (x.q, x.k, x.v)]
    y, A = tc.prefill_varlen(*args, cu.to(dev), x.max_seqlen if max_seqlen is None else max_seqlen,
                             x.lam.to(dev), x.eta.to(dev), x.g.to(dev), x.W, x.C,
                             l1_only=l1_only)
    torch.cuda.synchronize()
    return y, A


def _check_sequence(x, b, y, A, yl1=None):
    """Sequence b of the packed outputs against the oracle run on it alone."""
    a, e = int(x.cu_seqlens[b]), int(x.cu_seqlens[b + 1])
    q, k, v = x.sequence(b)
    T = e - a
    if T == 0:
        assert np.all(A[b] == 0.0)
        return {}
    yo, Ao, ylo, _ = oracle.prefill(q, k, v, x.lam, x.eta, x.g, x.W, parts=True)
    ys = y[a:e].transpose(1, 0, 2)  # [H, T, d]
    out = {"T": T, "y": rel_l2(ys, yo[0])}
    assert out["y"] <= BF16_Y_TOL, out
    if T > x.W:
        out["A"] = rel_l2(A[b], Ao[0])
        assert out["A"] <= BF16_A_TOL, out
    else:
        assert np.all(A[b] == 0.0)
    if yl1 is not None:
        out["y_l1"] = rel_l2(yl1[a:e].transpose(1, 0, 2), ylo[0])
        assert out["y_l1"] <= BF16_Y_TOL, out
    return out


# lengths: T < W, T = 0, T not a multiple of 128, T = W, T >> W, one tile plus one
CASES = [
    ([100, 0, 1000, 128, 4133, 129, 2048], 4, 128, 64),
    ([700, 3, 2500, 512, 1537, 90, 640, 4096, 1], 2, 512, 128),
    ([5000, 17, 384], 3, 256, 64),
]


@pytest.mark.parametrize("case", CASES, ids=[str(c[0]) for c in CASES])
def test_varlen_matches_the_oracle_per_sequence(cuda_device, case):
    import sliding_window_attention_tc_b200 as tc
    lengths, H, W, C = case
    x = wl.random_varlen(lengths, H, 64, 64, W, C, dtype="bf16", seed=len(lengths) + W)
    assert tc.device_status() == 0
    y, A = _run(tc, x, cuda_device)
    yl1, _ = _run(tc, x, cuda_device, l1_only=True)
    assert tc.device_status() == 0
    y, yl1, A = y.float().cpu().numpy(), yl1.float().cpu().numpy(), A.cpu().numpy()
    assert np.isfinite(y).all() and np.isfinite(A).all()
    for b in range(len(lengths)):
        print(b, _check_sequence(x, b, y, A, yl1))


def test_varlen_of_equal_lengths_equals_the_batched_call(cuda_device, both_paths):
    """Equal lengths give the batched call's schedule (same rows, same spans
    or chunks), so on either tensor-core path the packed call must reproduce
    tc_prefill on that path bit for bit."""
    import sliding_window_attention_tc_b200 as tc
    B, H, T, W = 3, 4, 1500, 256
    assert tc.prefill_path_for(tc.make_prefill_desc(B, H, T, 64, 64, W, 64, tc.TC_BF16)) == both_paths
    x = wl.random_varlen([T] * B, H, 64, 64, W, 64, dtype="bf16", seed=7)
    y, A = _run(tc, x, cuda_device)
    dev = cuda_device
    to_bh = lambda t: t.view(B, T, H, 64).permute(0, 2, 1, 3).contiguous().to(dev)
    yb, Ab = tc.prefill(to_bh(x.q), to_bh(x.k), to_bh(x.v), x.lam.to(dev), x.eta.to(dev),
                        x.g.to(dev), W, 64)
    torch.cuda.synchronize()
    assert tc.device_status() == 0
    assert torch.equal(y.view(B, T, H, 64).permute(0, 2, 1, 3), yb)
    assert torch.equal(A, Ab)


def test_varlen_many_short_sequences(cuda_device):
    """More sequences than SMs, most shorter than one tile."""
    import sliding_window_attention_tc_b200 as tc
    gen = torch.Generator().manual_seed(3)
    lengths = torch.randint(1, 300, (200,), generator=gen).tolist()
    lengths[17] = 3000
    x = wl.random_varlen(lengths, 2, 64, 64, 128, 64, dtype="bf16", seed=11)
    y, A = _run(tc, x, cuda_device)
    assert tc.device_status() == 0
    y, A = y.float().cpu().numpy(), A.cpu().numpy()
    for b in (0, 17, 42, 199):
        _check_sequence(x, b, y, A)


def test_varlen_inconsistent_offsets_are_reported_and_skipped(cuda_device):
    """A sequence whose offsets decrease, or run past total, is skipped with
    TC_ERR_DEVICE_BOUNDS; the consistent sequences of the call are still
    right."""
    import sliding_window_attention_tc_b200 as tc
    x = wl.random_varlen([300, 200, 300], 2, 64, 64, 128, 64, dtype="bf16", seed=5)
    # sequence 1 runs 500 -> 100 (decreasing); sequences 0 and 2 are the
    # disjoint rows 200..499 and 100..149 (outputs of overlapping sequences
    # would race)
    bad = torch.tensor([200, 500, 100, 150], dtype=torch.int64)
    y, A = _run(tc, x, cuda_device, cu=bad, max_seqlen=300)
    assert tc.device_status() == TC_ERR_DEVICE_BOUNDS
    assert tc.device_status() == 0  # read and cleared
    y, A = y.float().cpu().numpy(), A.cpu().numpy()
    assert np.all(A[1] == 0.0)
    good = wl.VarlenInputs(x.q, x.k, x.v, bad, x.lam, x.eta, x.g, x.W, x.C)
    _check_sequence(good, 0, y, A)
    _check_sequence(good, 2, y, A)
    # past total, and longer than max_seqlen
    for cu, mx in (([0, 300, 200, 600], 400), ([0, 300, 500, 500], 250)):
        _run(tc, x, cuda_device, cu=torch.tensor(cu, dtype=torch.int64), max_seqlen=mx)
        assert tc.device_status() == TC_ERR_DEVICE_BOUNDS
    # the next consistent call is clean
    y, A = _run(tc, x, cuda_device)
    assert tc.device_status() == 0
    _check_sequence(x, 1, y.float().cpu().numpy(), A.cpu().numpy())


def test_varlen_with_no_tokens_zeroes_the_states(cuda_device):
    import sliding_window_attention_tc_b200 as tc
    x = wl.random_varlen([0, 0, 0], 2, 64, 64, 128, 64, dtype="bf16", seed=1)
    A = torch.full((3, 2, 64, 64), 7.0, device=cuda_device)
    y, A = tc.prefill_varlen(x.q.to(cuda_device), x.k.to(cuda_device), x.v.to(cuda_device),
                             x.cu_seqlens.to(cuda_device), 0, x.lam.to(cuda_device),
                             x.eta.to(cuda_device), x.g.to(cuda_device), x.W, x.C, A_final=A)
    torch.cuda.synchronize()
    assert y.numel() == 0
    assert torch.all(A == 0)
    assert tc.device_status() == 0


# general tensor-core path: W not a multiple of 128, d = 128, W = 1
GENERAL = [
    ([300, 0, 1000, 77, 2100], 3, 64, 200, 64),
    ([500, 1, 1300, 129], 2, 128, 256, 64),
    ([900, 64, 128, 5, 0], 2, 64, 1, 16),
]


@pytest.mark.parametrize("case", GENERAL, ids=[f"d{c[2]}_W{c[3]}" for c in GENERAL])
def test_varlen_general_path_matches_the_oracle(cuda_device, case):
    import sliding_window_attention_tc_b200 as tc
    lengths, H, d, W, C = case
    x = wl.random_varlen(lengths, H, d, d, W, C, dtype="bf16", seed=W + d)
    y, A = _run(tc, x, cuda_device)
    yl1, _ = _run(tc, x, cuda_device, l1_only=True)
    assert tc.device_status() == 0
    y, yl1, A = y.float().cpu().numpy(), yl1.float().cpu().numpy(), A.cpu().numpy()
    assert np.isfinite(y).all() and np.isfinite(A).all()
    for b in range(len(lengths)):
        print(b, _check_sequence(x, b, y, A, yl1))


def test_varlen_general_path_reports_inconsistent_offsets(cuda_device):
    import sliding_window_attention_tc_b200 as tc
    x = wl.random_varlen([300, 200, 300], 2, 64, 64, 200, 64, dtype="bf16", seed=9)
    bad = torch.tensor([200, 500, 100, 150], dtype=torch.int64)
    y, A = _run(tc, x, cuda_device, cu=bad, max_seqlen=300)
    assert tc.device_status() == TC_ERR_DEVICE_BOUNDS
    y, A = y.float().cpu().numpy(), A.cpu().numpy()
    assert np.all(A[1] == 0.0)
    good = wl.VarlenInputs(x.q, x.k, x.v, bad, x.lam, x.eta, x.g, x.W, x.C)
    _check_sequence(good, 0, y, A)
    _check_sequence(good, 2, y, A)
