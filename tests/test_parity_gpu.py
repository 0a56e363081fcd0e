"""GPU parity: the CUDA path of libtc against the float64 CPU oracle.

Every comparison uses the same seeded inputs (workloads.py) on both sides; the
oracle reads the exact rounded values (float32 or bf16 widened to float64).

Tolerances (stated for the layer):
  float32 path:  max|x - ref| / max|ref| <= 1e-5 on y and on A;
  bf16 inputs, float32 accumulation and state:
                 ||x - ref||_2 / ||ref||_2 <= 1e-2 on y and <= 1e-3 on A.
Ring-buffer contents are byte copies and must match exactly.
Full-size workloads run on the GPU in the same launch configuration the
benchmark times; the oracle checks sampled heads of them.
"""
import math

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
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.abs(ref).max()
    return float(np.abs(x - ref).max() / den) if den > 0 else float(np.abs(x).max())


def rel_l2(x, ref):
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref)
    return float(np.linalg.norm(x - ref) / den) if den > 0 else float(np.linalg.norm(x))


def _tc():
    import sliding_window_attention_tc_b200 as tc
    return tc


def _dev(x, dev):
    return x.to(dev).contiguous()


def run_prefill(x: wl.PrefillInputs, dev, l1_only=False):
    tc = _tc()
    y, A = tc.prefill(_dev(x.q, dev), _dev(x.k, dev), _dev(x.v, dev), _dev(x.lam, dev),
                      _dev(x.eta, dev), _dev(x.g, dev), x.W, x.C, l1_only=l1_only)
    torch.cuda.synchronize()
    assert tc.device_status() == 0
    return y.float().cpu().numpy(), (None if A is None else A.cpu().numpy())


def check_prefill(x, y, A, heads=None, l1_only_y=None):
    """Compare GPU outputs with the oracle on the (b,h) pairs in heads (all
    when None).  Returns the error summary."""
    B, H = x.q.shape[:2]
    heads = heads if heads is not None else [(b, h) for b in range(B) for h in range(H)]
    f32 = x.q.dtype == torch.float32
    errs = {"y": [], "A": [], "y_l1": []}
    ys, yrs, As, Ars, yl1, yl1r = [], [], [], [], [], []
    by_h = {}
    for b, h in heads:
        by_h.setdefault(h, []).append(b)
    for h, bs in by_h.items():
        sl = (bs, slice(h, h + 1))
        yo, Ao, ylo, _ = oracle.prefill(x.q[sl], x.k[sl], x.v[sl], x.lam[h:h + 1],
                                        x.eta[h:h + 1], x.g[h:h + 1], x.W, parts=True)
        for i, b in enumerate(bs):
            ys.append(y[b, h]); yrs.append(yo[i, 0])
            As.append(A[b, h]); Ars.append(Ao[i, 0])
            if l1_only_y is not None:
                yl1.append(l1_only_y[b, h]); yl1r.append(ylo[i, 0])
    ys, yrs, As, Ars = map(np.stack, (ys, yrs, As, Ars))
    if f32:
        out = {"y": max_rel(ys, yrs), "A": max_rel(As, Ars) if np.abs(Ars).max() > 0 else
               float(np.abs(As).max())}
        assert out["y"] <= F32_TOL, out
        if np.abs(Ars).max() > 0:
            assert out["A"] <= F32_TOL, out
        else:
            assert np.all(As == 0.0)
        if yl1:
            out["y_l1"] = max_rel(np.stack(yl1), np.stack(yl1r))
            assert out["y_l1"] <= F32_TOL, out
    else:
        out = {"y": rel_l2(ys, yrs), "A": rel_l2(As, Ars) if np.linalg.norm(Ars) > 0 else
               float(np.abs(As).max())}
        assert out["y"] <= BF16_Y_TOL, out
        if np.linalg.norm(Ars) > 0:
            assert out["A"] <= BF16_A_TOL, out
        else:
            assert np.all(As == 0.0)
        if yl1:
            out["y_l1"] = rel_l2(np.stack(yl1), np.stack(yl1r))
            assert out["y_l1"] <= BF16_Y_TOL, out
    return out


# --- the named workloads --------------------------------------------------

def test_prefill_tiny_fp32(cuda_device):
    x = wl.prefill_config("tiny_fp32")
    y, A = run_prefill(x, cuda_device)
    out = check_prefill(x, y, A)
    print("tiny_fp32", out)


def test_prefill_recall_fp32(cuda_device):
    x = wl.prefill_config("recall_fp32")
    y, A = run_prefill(x, cuda_device)
    out = check_prefill(x, y, A)
    print("recall_fp32", out)


def _takes(x, path):
    """The call of workload x runs on the tensor-core path named path."""
    tc = _tc()
    B, H, T, d = x.q.shape
    desc = tc.make_prefill_desc(B, H, T, d, x.v.shape[-1], x.W, x.C, tc.TC_BF16)
    assert tc.prefill_path_for(desc) == path


def test_prefill_lm_bf16_full_size_sampled_heads(cuda_device, both_paths):
    x = wl.prefill_config("lm_prefill_bf16")
    _takes(x, both_paths)
    y, A = run_prefill(x, cuda_device)
    yl1, _ = run_prefill(x, cuda_device, l1_only=True)
    heads = [(0, 0), (1, 5), (3, 11), (5, 2), (7, 7), (7, 11)]
    out = check_prefill(x, y, A, heads, l1_only_y=yl1)
    assert np.isfinite(y).all()
    print("lm_prefill_bf16", out)


def test_prefill_long_bf16_full_size_sampled_heads(cuda_device, both_paths):
    x = wl.prefill_config("long_prefill_bf16")
    _takes(x, both_paths)
    y, A = run_prefill(x, cuda_device)
    yl1, _ = run_prefill(x, cuda_device, l1_only=True)
    out = check_prefill(x, y, A, [(0, 0), (0, 13)], l1_only_y=yl1)
    assert np.isfinite(y).all()
    print("long_prefill_bf16", out)


def test_prefill_lm_bf16_every_head(cuda_device, both_paths):
    """All 96 (b, h) rows of the LM workload (8 x 12 x 4096, W = 512), y and
    A_final, against one oracle call over every row, on each path."""
    x = wl.prefill_config("lm_prefill_bf16")
    _takes(x, both_paths)
    y, A = run_prefill(x, cuda_device)
    yo, Ao = oracle.prefill(x.q, x.k, x.v, x.lam, x.eta, x.g, x.W)
    B, H = x.q.shape[:2]
    worst = {"y": 0.0, "A": 0.0}
    for b in range(B):
        for h in range(H):
            ey, eA = rel_l2(y[b, h], yo[b, h]), rel_l2(A[b, h], Ao[b, h])
            assert ey <= BF16_Y_TOL and eA <= BF16_A_TOL, (b, h, ey, eA)
            worst = {"y": max(worst["y"], ey), "A": max(worst["A"], eA)}
    print("lm_prefill_bf16, every head", worst)


def test_prefill_long_bf16_every_head(cuda_device, both_paths):
    """All 16 heads of the long-context workload (1 x 16 x 32768, W = 1024),
    y and A_final, against one oracle call that runs the heads in parallel,
    on each path."""
    x = wl.prefill_config("long_prefill_bf16")
    _takes(x, both_paths)
    y, A = run_prefill(x, cuda_device)
    yo, Ao = oracle.prefill(x.q, x.k, x.v, x.lam, x.eta, x.g, x.W)
    H = x.q.shape[1]
    worst = {"y": 0.0, "A": 0.0}
    for h in range(H):
        ey, eA = rel_l2(y[0, h], yo[0, h]), rel_l2(A[0, h], Ao[0, h])
        assert ey <= BF16_Y_TOL and eA <= BF16_A_TOL, (h, ey, eA)
        worst = {"y": max(worst["y"], ey), "A": max(worst["A"], eA)}
    assert np.isfinite(y).all()
    print("long_prefill_bf16, every head", worst)


# --- edge shapes ----------------------------------------------------------

EDGE = [
    # B, H, T, dk, dv, W, C
    (1, 2, 50, 16, 16, 64, 16),     # T < W: nothing evicted, A_final = 0
    (1, 2, 64, 32, 32, 64, 8),      # T = W
    (1, 1, 65, 32, 32, 64, 8),      # one eviction
    (2, 3, 300, 64, 64, 37, 13),    # odd W, ragged last chunk
    (1, 2, 200, 24, 40, 20, 1),     # d_k != d_v, C = 1
    (1, 1, 150, 128, 128, 16, 1000),  # C larger than the number of evictions
    (1, 2, 77, 64, 64, 1, 5),       # W = 1
    (1, 1, 0, 64, 64, 16, 8),       # T = 0
    (2, 2, 1000, 64, 64, 128, 64),  # tile-aligned W, ragged T
    (1, 2, 777, 64, 64, 256, 128),  # C = 128, ragged T
    (1, 1, 100, 64, 64, 128, 64),   # T < W = one tile
    (1, 3, 1300, 64, 64, 512, 64),  # several tiles in the window
]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("shape", EDGE, ids=[str(s) for s in EDGE])
def test_prefill_edge_shapes(cuda_device, shape, dtype, both_paths):
    B, H, T, dk, dv, W, C = shape
    x = wl.random_prefill(B, H, T, dk, dv, W, C, dtype=dtype, seed=hash(shape) % 1000)
    y, A = run_prefill(x, cuda_device)
    if T == 0:
        assert y.size == 0 and np.all(A == 0.0)
        return
    yl1, _ = run_prefill(x, cuda_device, l1_only=True)
    check_prefill(x, y, A, l1_only_y=yl1)


def test_prefill_is_deterministic_and_keeps_inputs(cuda_device, both_paths):
    tc = _tc()
    x = wl.random_prefill(2, 3, 700, 64, 64, 128, 64, dtype="bf16", seed=3)
    q, k, v = (_dev(t, cuda_device) for t in (x.q, x.k, x.v))
    q0, k0, v0 = q.clone(), k.clone(), v.clone()
    args = (_dev(x.lam, cuda_device), _dev(x.eta, cuda_device), _dev(x.g, cuda_device))
    y1, A1 = tc.prefill(q, k, v, *args, x.W, x.C)
    y2, A2 = tc.prefill(q, k, v, *args, x.W, x.C)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2) and torch.equal(A1, A2)
    assert torch.equal(q, q0) and torch.equal(k, k0) and torch.equal(v, v0)


def test_prefill_host_variant_matches_device(cuda_device, both_paths):
    tc = _tc()
    x = wl.random_prefill(2, 2, 500, 64, 64, 128, 64, dtype="bf16", seed=4)
    yd, Ad = tc.prefill(*(_dev(t, cuda_device) for t in (x.q, x.k, x.v, x.lam, x.eta, x.g)),
                        x.W, x.C)
    desc = tc.make_prefill_desc(2, 2, 500, 64, 64, x.W, x.C, tc.TC_BF16)
    ws = torch.empty(tc.prefill_host_workspace_size(desc), dtype=torch.uint8, device=cuda_device)
    pin = lambda t: t.contiguous().pin_memory()
    yh = torch.empty(yd.shape, dtype=yd.dtype).pin_memory()
    Ah = torch.empty(Ad.shape, dtype=torch.float32).pin_memory()
    tc.prefill_host(pin(x.q), pin(x.k), pin(x.v), pin(x.lam), pin(x.eta), pin(x.g), x.W, x.C,
                    yh, Ah, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(yh, yd.cpu()) and torch.equal(Ah, Ad.cpu())


# --- decode ---------------------------------------------------------------

def _decode_run(B, H, W, d, steps, dtype, seed, t0=0, dev="cuda"):
    """Random stream from an empty state (t0 = 0) through `steps` steps."""
    tc = _tc()
    gen = torch.Generator().manual_seed(seed)
    dt = wl.torch_dtype(dtype)
    s = 1.0 / math.sqrt(d)
    q = (torch.randn(steps, B, H, d, generator=gen) * s).to(dt)
    k = (torch.randn(steps, B, H, d, generator=gen) * s).to(dt)
    v = (torch.randn(steps, B, H, d, generator=gen) * s).to(dt)
    lam = 0.9 + 0.09 * torch.rand(H, generator=gen)
    eta = 0.2 + torch.rand(H, generator=gen)
    g = torch.randn(H, generator=gen)
    st = tc.DecodeState.empty(B, H, W, d, d, lam.to(dev), eta.to(dev), g.to(dev), dtype=dt,
                              device=dev)
    ys = []
    for i in range(steps):
        ys.append(tc.decode_step(st, q[i].to(dev), k[i].to(dev), v[i].to(dev)).float().cpu())
    torch.cuda.synchronize()
    assert st.t == steps
    yo, rko, rvo, Ao = oracle.decode(np.zeros((B, H, W, d)), np.zeros((B, H, W, d)),
                                     np.zeros((B, H, d, d)), 0, q, k, v, lam, eta, g)
    return torch.stack(ys).numpy(), st, (yo, rko, rvo, Ao), (q, k, v)


@pytest.mark.parametrize("d", [16, 32, 64, 128])
def test_decode_fp32_from_empty(cuda_device, d):
    y, st, (yo, rko, rvo, Ao), _ = _decode_run(2, 3, 16, d, 40, "f32", seed=d)
    assert max_rel(y, yo) <= F32_TOL
    assert max_rel(st.A.cpu().numpy(), Ao) <= F32_TOL
    np.testing.assert_array_equal(st.ring_k.cpu().double().numpy(), rko)
    np.testing.assert_array_equal(st.ring_v.cpu().double().numpy(), rvo)


@pytest.mark.parametrize("d", [16, 32, 64, 128])
def test_decode_bf16_from_empty(cuda_device, d):
    y, st, (yo, rko, rvo, Ao), _ = _decode_run(2, 2, 24, d, 60, "bf16", seed=100 + d)
    assert rel_l2(y, yo) <= BF16_Y_TOL
    assert rel_l2(st.A.cpu().numpy(), Ao) <= BF16_A_TOL
    np.testing.assert_array_equal(st.ring_k.cpu().double().numpy(), rko)
    np.testing.assert_array_equal(st.ring_v.cpu().double().numpy(), rvo)


@pytest.mark.parametrize("W", [1, 5, 2048])
def test_decode_window_extremes(cuda_device, W):
    y, st, (yo, *_), _ = _decode_run(1, 2, W, 64, 12, "f32", seed=W)
    assert max_rel(y, yo) <= F32_TOL


def test_decode_continues_a_prefill(cuda_device):
    """Prefill T tokens on the GPU, hand the state to the stream (ring slot
    j mod W holds token j, A = A_final, t = T) and decode n more tokens; the
    result must match the oracle's prefill over all T + n tokens."""
    tc = _tc()
    B, H, T, n, d, W, C = 2, 2, 300, 40, 64, 64, 16
    x = wl.random_prefill(B, H, T + n, d, d, W, C, dtype="f32", seed=21)
    dev = cuda_device
    lam, eta, g = (_dev(t, dev) for t in (x.lam, x.eta, x.g))
    _, A = tc.prefill(_dev(x.q[:, :, :T], dev), _dev(x.k[:, :, :T], dev),
                      _dev(x.v[:, :, :T], dev), lam, eta, g, W, C)
    ring_k = torch.zeros(B, H, W, d, device=dev)
    ring_v = torch.zeros(B, H, W, d, device=dev)
    for j in range(T - W, T):
        ring_k[:, :, j % W] = x.k[:, :, j].to(dev)
        ring_v[:, :, j % W] = x.v[:, :, j].to(dev)
    st = tc.DecodeState(ring_k, ring_v, A, lam, eta, g, T)
    ys = [tc.decode_step(st, _dev(x.q[:, :, j], dev), _dev(x.k[:, :, j], dev),
                         _dev(x.v[:, :, j], dev)).cpu() for j in range(T, T + n)]
    yo, _ = oracle.prefill(x.q, x.k, x.v, x.lam, x.eta, x.g, W)
    y = torch.stack(ys, 2).numpy()
    assert max_rel(y, yo[:, :, T:]) <= F32_TOL


def test_decode_host_variant_matches_device(cuda_device):
    tc = _tc()
    B, H, W, d = 2, 2, 32, 128
    gen = torch.Generator().manual_seed(5)
    mk = lambda *s: (torch.randn(*s, generator=gen) / 11).to(torch.bfloat16)
    rk, rv = mk(B, H, W, d), mk(B, H, W, d)
    A = torch.randn(B, H, d, d, generator=gen) / 100
    prm = [torch.tensor([0.95, 0.99]), torch.tensor([0.3, 0.6]), torch.tensor([0.1, -0.5])]
    dev = cuda_device
    s1 = tc.DecodeState(rk.to(dev), rv.to(dev), A.to(dev), *(p.to(dev) for p in prm), 70)
    s2 = tc.DecodeState(rk.to(dev), rv.to(dev), A.to(dev), *(p.to(dev) for p in prm), 70)
    ws = torch.empty(tc.decode_step_host_workspace_size(s2), dtype=torch.uint8, device=dev)
    for i in range(3):
        q, k, v = mk(B, H, d), mk(B, H, d), mk(B, H, d)
        yd = tc.decode_step(s1, q.to(dev), k.to(dev), v.to(dev))
        yh = torch.empty(B, H, d, dtype=torch.bfloat16).pin_memory()
        tc.decode_step_host(s2, q.pin_memory(), k.pin_memory(), v.pin_memory(), yh, workspace=ws)
        torch.cuda.synchronize()
        assert torch.equal(yh, yd.cpu())
    assert torch.equal(s1.A, s2.A) and torch.equal(s1.ring_k, s2.ring_k)
    assert s1.t == s2.t == 73


def test_decode_full_size_sampled_heads(cuda_device):
    """The batched-decode workload (256 x 32 heads, d = 128, W = 2048, ring
    full, A the state left by 8192 evicted pairs, 512 steps) on the GPU; A is
    written through libtc.  The oracle writes the same pairs for 32 sampled
    heads with its own token loop, then replays them over all 512 steps."""
    import bench
    tc = _tc()
    x = wl.decode_workload(device=cuda_device)
    B, H = x.ring_k.shape[:2]
    rng = np.random.default_rng(0)
    flat = rng.choice(B * H, size=32, replace=False)
    sb, sh = torch.as_tensor(flat // H), torch.as_tensor(flat % H)
    x.A = bench.decode_state_from_prewarm(tc, x)
    prm = [t.cpu()[sh] for t in (x.lam, x.eta, x.g)]
    # the oracle's A for the sampled heads, from the same pairs (one oracle
    # "batch" entry, each sampled head with its own parameters)
    pk, pv = [], []
    for b, h in zip(sb.tolist(), sh.tolist()):
        k_ev, v_ev = wl.decode_prewarm_pairs(x, b, b + 1)
        pk.append(k_ev[0, h].cpu())
        pv.append(v_ev[0, h].cpu())
    pk, pv = torch.stack(pk).unsqueeze(0), torch.stack(pv).unsqueeze(0)
    pad = torch.zeros(1, len(flat), 1, pk.shape[-1], dtype=pk.dtype)
    kk, vv = torch.cat([pk, pad], dim=2), torch.cat([pv, pad], dim=2)
    _, A_o = oracle.prefill(torch.zeros_like(kk), kk, vv, prm[0], prm[1], prm[2], 1)
    A_err0 = rel_l2(x.A[sb, sh].cpu().numpy(), A_o[0])
    assert A_err0 <= 1e-4, A_err0  # a float32 scan of 8192 writes against float64
    init = [x.ring_k[sb, sh].cpu(), x.ring_v[sb, sh].cpu(), torch.from_numpy(A_o[0])]
    st = tc.DecodeState(x.ring_k, x.ring_v, x.A, x.lam, x.eta, x.g, x.t0)
    n = x.q.shape[0]
    ys = torch.empty(n, len(flat), x.v.shape[-1], dtype=torch.bfloat16)
    for i in range(n):
        y = tc.decode_step(st, x.q[i], x.k[i], x.v[i])
        ys[i] = y[sb, sh].cpu()
    torch.cuda.synchronize()
    assert tc.device_status() == 0
    q, k, v = (t[:, sb, sh].cpu().unsqueeze(1) for t in (x.q, x.k, x.v))
    yo, rko, rvo, Ao = oracle.decode(init[0].unsqueeze(0), init[1].unsqueeze(0),
                                     init[2].unsqueeze(0), x.t0, q, k, v, *prm)
    y_err = rel_l2(ys.float().numpy(), yo[:, 0])
    A_err = rel_l2(st.A[sb, sh].cpu().numpy(), Ao[0])
    print("decode full size: rel L2 y", y_err, "A", A_err)
    assert y_err <= BF16_Y_TOL and A_err <= BF16_A_TOL
    np.testing.assert_array_equal(st.ring_k[sb, sh].cpu().double().numpy(), rko[0])
