"""GPU parity of the general tensor-core prefill (bf16, d_k = d_v in {64,
128}): the shapes the fused kernel does not take -- W not a multiple of 128,
W < 128, d = 128, continuations with a partial halo, state-only calls --
against the float64 oracle ("Tensor Cache: Eviction-conditioned Associative
Memory for Transformers", §3.1 eq. (1) and §3.2 Fig. 2).  Tolerances are the
bf16 ones of the other parity tests: ||y - ref|| / ||ref|| <= 1e-2 and
||A - ref|| / ||ref|| <= 1e-3.  Each case also checks the launch count of
the general path (combine copies, sums, scan, window with the reads), so a silent
switch to the SIMT kernels fails here."""
import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from test_parity_gpu import check_prefill, run_prefill

pytestmark = pytest.mark.gpu

BF16_Y_TOL = 1e-2
BF16_A_TOL = 1e-3


def rel_l2(x, ref):
    x, ref = np.asarray(x, np.float64), np.asarray(ref, np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(x - ref) / den) if den > 0 else float(np.linalg.norm(x))


def _tc():
    import sliding_window_attention_tc_b200 as tc
    return tc


def general_launches(T, W, n_halo=0, l1_only=False, state_only=False):
    """Launches of one call on the general path (see prefill_general_sm100.cu)."""
    Tc = n_halo + T
    E = max(0, Tc - min(W, Tc + 1))
    queries = not state_only and T > 0
    n = 2 if n_halo > 0 else 0
    if not l1_only:
        n += (1 if E > 0 else 0) + 1  # sums, scan
    return n + (1 if queries else 0)  # window (with the reads)


CASES = [
    # B, H, T, d, W
    (2, 3, 700, 64, 200),    # W not a multiple of 128, several chunks, ragged T
    (1, 2, 333, 64, 5),      # small W: most keys evicted
    (1, 2, 100, 64, 300),    # W > T: no eviction
    (2, 2, 1000, 128, 256),  # d = 128 (the decode workload's head size)
    (1, 3, 900, 128, 100),   # d = 128, W not a multiple of 128
    (1, 1, 129, 128, 1),     # W = 1
]


@pytest.mark.parametrize("case", CASES, ids=[str(c) for c in CASES])
def test_general_prefill(cuda_device, case):
    tc = _tc()
    B, H, T, d, W = case
    x = wl.random_prefill(B, H, T, d, d, W, 64, dtype="bf16", seed=17 + T + W)
    desc = tc.make_prefill_desc(B, H, T, d, d, W, 64, tc.TC_BF16)
    assert tc.prefill_launch_count(desc) == general_launches(T, W)
    y, A = run_prefill(x, cuda_device)
    yl1, _ = run_prefill(x, cuda_device, l1_only=True)
    check_prefill(x, y, A, l1_only_y=yl1)


@pytest.mark.parametrize("d,W,t0", [(64, 200, 70), (64, 200, 450), (128, 256, 100), (64, 512, 300)],
                         ids=["partial-halo", "full-halo", "d128-partial", "W512-partial"])
def test_general_continuation(cuda_device, d, W, t0):
    """tc_prefill_from_state at t0 with the halo of min(t0, W) tokens and the
    state of the evictions before the combined sequence, against the oracle
    over the whole sequence."""
    tc = _tc()
    B, H, T = 1, 2, 900
    x = wl.random_prefill(B, H, T, d, d, W, 64, dtype="bf16", seed=5 + t0)
    dev = cuda_device
    dd = lambda t: t.to(dev).contiguous()
    y_ref, A_ref = oracle.prefill(x.q, x.k, x.v, x.lam, x.eta, x.g, W)
    n = min(t0, W)
    # A after the steps before t0 (zero while t0 < W: nothing evicted yet)
    A_init = None
    if t0 >= W:
        _, A_pre = oracle.prefill(x.q[:, :, :t0], x.k[:, :, :t0], x.v[:, :, :t0], x.lam, x.eta, x.g, W)
        A_init = torch.from_numpy(A_pre).float().to(dev)
    y, A = tc.prefill_from_state(dd(x.q[:, :, t0:]), dd(x.k[:, :, t0:]), dd(x.v[:, :, t0:]),
                                 dd(x.lam), dd(x.eta), dd(x.g), W, 64, t0,
                                 dd(x.k[:, :, t0 - n:t0]), dd(x.v[:, :, t0 - n:t0]), A_init)
    torch.cuda.synchronize()
    assert tc.device_status() == 0
    assert rel_l2(y.float().cpu().numpy(), y_ref[:, :, t0:]) <= BF16_Y_TOL
    assert rel_l2(A.cpu().numpy(), A_ref) <= BF16_A_TOL


def test_general_state_only(cuda_device):
    """TC_PREFILL_STATE_ONLY: the chunk scan alone (sums and scan kernels)."""
    tc = _tc()
    B, H, T, d, W = 2, 2, 1500, 64, 200
    x = wl.random_prefill(B, H, T, d, d, W, 64, dtype="bf16", seed=23)
    dev = cuda_device
    dd = lambda t: t.to(dev).contiguous()
    desc = tc.make_prefill_desc(B, H, T, d, d, W, 64, tc.TC_BF16, state_only=True)
    assert tc.prefill_launch_count(desc) == general_launches(T, W, state_only=True)
    _, A = tc.prefill_from_state(None, dd(x.k), dd(x.v), dd(x.lam), dd(x.eta), dd(x.g), W, 64, 0,
                                 state_only=True)
    torch.cuda.synchronize()
    assert tc.device_status() == 0
    _, A_ref = oracle.prefill(x.q, x.k, x.v, x.lam, x.eta, x.g, W)
    assert rel_l2(A.cpu().numpy(), A_ref) <= BF16_A_TOL


def test_general_decode_shaped_prefill(cuda_device):
    """d = 128, W = 2048 (the decode workload's head size and window), two
    heads of 4000 tokens: the prefill that fills a decode ring."""
    tc = _tc()
    B, H, T, d, W = 1, 2, 4000, 128, 2048
    x = wl.random_prefill(B, H, T, d, d, W, 64, dtype="bf16", seed=29)
    desc = tc.make_prefill_desc(B, H, T, d, d, W, 64, tc.TC_BF16)
    assert tc.prefill_launch_count(desc) == general_launches(T, W)
    y, A = run_prefill(x, cuda_device)
    check_prefill(x, y, A)


def test_general_full_size_bench_workloads(cuda_device):
    """The two general-path workloads bench.py times, at full size, in the
    launch configuration it uses: the LM workload at W = 500, and d = 128,
    W = 2048 over 8 x 32 heads of 4096 tokens (inputs seeded as in bench.py).
    Sampled heads against the oracle run on each sampled head alone."""
    import math
    tc = _tc()
    dev = cuda_device
    x = wl.prefill_config("lm_prefill_bf16")
    y, A = tc.prefill(*(t.to(dev).contiguous() for t in (x.q, x.k, x.v, x.lam, x.eta, x.g)), 500, x.C)
    torch.cuda.synchronize()
    assert tc.device_status() == 0
    x500 = wl.PrefillInputs(x.q, x.k, x.v, x.lam, x.eta, x.g, 500, x.C)
    check_prefill(x500, y.float().cpu().numpy(), A.cpu().numpy(), heads=[(0, 0), (3, 7), (7, 11)])
    del y, A
    B, H, T, d, W = 8, 32, 4096, 128, 2048
    gen = torch.Generator(device=dev).manual_seed(1005)
    q, k, v = ((torch.randn(B, H, T, d, generator=gen, device=dev) / math.sqrt(d)).to(torch.bfloat16)
               for _ in range(3))
    lam = 0.99 + 0.0099 * torch.rand(H, generator=gen, device=dev)
    eta = 0.1 + 0.9 * torch.rand(H, generator=gen, device=dev)
    g = torch.randn(H, generator=gen, device=dev)
    y, A = tc.prefill(q, k, v, lam, eta, g, W, 128)
    torch.cuda.synchronize()
    assert tc.device_status() == 0
    for b, h in [(0, 0), (5, 31)]:
        sl = lambda t: t[b:b + 1, h:h + 1].cpu()
        yo, Ao = oracle.prefill(sl(q), sl(k), sl(v), lam[h:h + 1].cpu(), eta[h:h + 1].cpu(), g[h:h + 1].cpu(), W)
        assert rel_l2(y[b, h].float().cpu().numpy(), yo[0, 0]) <= BF16_Y_TOL
        assert rel_l2(A[b, h].cpu().numpy(), Ao[0, 0]) <= BF16_A_TOL


def test_general_prefill_fills_a_d128_decode_ring(cuda_device):
    """The decode workload's head size and window (d = 128, W = 256 here to
    keep the oracle short): a bf16 prefill on the general tensor-core path
    hands its state to the decode stream (ring slot j mod W holds token j,
    A = A_final, t = T), which continues; both match the oracle over all
    tokens."""
    tc = _tc()
    B, H, T, n, d, W = 1, 2, 700, 24, 128, 256
    x = wl.random_prefill(B, H, T + n, d, d, W, 64, dtype="bf16", seed=51)
    dev = cuda_device
    dd = lambda t: t.to(dev).contiguous()
    desc = tc.make_prefill_desc(B, H, T, d, d, W, 64, tc.TC_BF16)
    assert tc.prefill_launch_count(desc) == general_launches(T, W)
    lam, eta, g = dd(x.lam), dd(x.eta), dd(x.g)
    y, A = tc.prefill(dd(x.q[:, :, :T]), dd(x.k[:, :, :T]), dd(x.v[:, :, :T]), lam, eta, g, W, 64)
    ring_k = torch.zeros(B, H, W, d, dtype=torch.bfloat16, device=dev)
    ring_v = torch.zeros(B, H, W, d, dtype=torch.bfloat16, device=dev)
    for j in range(T - W, T):
        ring_k[:, :, j % W] = x.k[:, :, j].to(dev)
        ring_v[:, :, j % W] = x.v[:, :, j].to(dev)
    st = tc.DecodeState(ring_k, ring_v, A, lam, eta, g, T)
    ys = [tc.decode_step(st, dd(x.q[:, :, j]), dd(x.k[:, :, j]), dd(x.v[:, :, j])).float().cpu()
          for j in range(T, T + n)]
    torch.cuda.synchronize()
    assert tc.device_status() == 0
    yo, Ao = oracle.prefill(x.q, x.k, x.v, x.lam, x.eta, x.g, W)
    assert rel_l2(y.float().cpu().numpy(), yo[:, :, :T]) <= BF16_Y_TOL
    assert rel_l2(torch.stack(ys, 2).numpy(), yo[:, :, T:]) <= BF16_Y_TOL
    assert rel_l2(st.A.cpu().numpy(), Ao) <= BF16_A_TOL
