"""Pins of the CPU oracle against facts fixed by the pages and by mathematics.

Each test below checks the oracle against something other than itself: a
library routine (float64 scaled-dot-product attention), a closed form written
as one float64 matmul, brute force over tokens on tiny inputs, hand-worked
fixtures (tests/golden/), or an exact algebraic identity.  Together they are
chosen so that a plausible slip in the oracle (read before write, an
off-by-one window, a missing 1/sqrt(d_k), a transposed k (x) v, a dropped
decay, a wrong gate) fails at least one of them.

Source: "Tensor Cache: Eviction-conditioned Associative Memory for
Transformers" (arXiv 2605.22884), §3.1 eq. (1), §3.2 Fig. 2, abstract and §1
(read identity, chunk scan, chunk-mean shortcut).
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import workloads as wl

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _sdpa_band(q, k, v, W):
    """float64 torch SDPA with the window mask t-W < j <= t (library routine)."""
    T = q.shape[-2]
    t = torch.arange(T).view(T, 1)
    j = torch.arange(T).view(1, T)
    mask = (j <= t) & (j > t - W)
    return torch.nn.functional.scaled_dot_product_attention(
        torch.as_tensor(q, dtype=torch.float64), torch.as_tensor(k, dtype=torch.float64),
        torch.as_tensor(v, dtype=torch.float64), attn_mask=mask).numpy()


def _small(B=2, H=3, T=29, dk=8, dv=5, W=6, seed=7, lam=(0.6, 0.95), eta=(0.2, 1.5)):
    x = wl.random_prefill(B, H, T, dk, dv, W, 4, dtype="f32", seed=seed, lam_range=lam,
                          eta_range=eta)
    return x


# --- L1: the window path reduces to library softmax attention -------------

def test_window_covers_sequence_is_causal_softmax():
    """W >= T: nothing is evicted, A stays 0 and y is plain causal softmax
    attention (spec property 1; §3.2 token partition)."""
    x = _small(T=23, W=23)
    y, A = oracle.prefill(x.q, x.k, x.v, x.lam, x.eta, x.g, 23)
    ref = torch.nn.functional.scaled_dot_product_attention(
        x.q.double(), x.k.double(), x.v.double(), is_causal=True).numpy()
    np.testing.assert_allclose(y, ref, rtol=0, atol=1e-13)
    assert np.all(A == 0.0)
    y2, A2 = oracle.prefill(x.q, x.k, x.v, x.lam, x.eta, x.g, 100)
    np.testing.assert_allclose(y2, ref, rtol=0, atol=1e-13)
    assert np.all(A2 == 0.0)


@pytest.mark.parametrize("W", [1, 2, 5, 16])
def test_local_path_is_band_softmax(W):
    """y_local is exact softmax over keys t-W+1..t scaled by 1/sqrt(d_k)
    (§3.1 eq. (1)); the window includes the current token."""
    x = _small(T=31, W=W, dk=7, dv=3)
    _, _, yl, _ = oracle.prefill(x.q, x.k, x.v, x.lam, x.eta, x.g, W, parts=True)
    np.testing.assert_allclose(yl, _sdpa_band(x.q, x.k, x.v, W), rtol=0, atol=1e-13)
    if W == 1:
        np.testing.assert_array_equal(yl, x.v.double().numpy())


def test_gate_minus_infinity_is_pure_window_attention():
    """sigma(g) -> 0 leaves only the window path (spec L1-only run)."""
    x = _small(T=40, W=9)
    g = torch.full_like(x.g, -1e4)
    y, _ = oracle.prefill(x.q, x.k, x.v, x.lam, x.eta, g, 9)
    np.testing.assert_allclose(y, _sdpa_band(x.q, x.k, x.v, 9), rtol=0, atol=1e-13)


def test_gate_zero_is_half():
    """g = 0: y = y_local + m / 2 (Fig. 2 step (5), sigma = logistic)."""
    x = _small(T=40, W=9)
    g = torch.zeros_like(x.g)
    y, _, yl, m = oracle.prefill(x.q, x.k, x.v, x.lam, x.eta, g, 9, parts=True)
    np.testing.assert_allclose(y, yl + 0.5 * m, rtol=0, atol=1e-14)
    gg = torch.tensor([0.3, -1.2, 2.0])
    y, _, yl, m = oracle.prefill(x.q, x.k, x.v, x.lam, x.eta, gg, 9, parts=True)
    sig = 1.0 / (1.0 + np.exp(-gg.double().numpy()))
    np.testing.assert_allclose(y, yl + sig[None, :, None, None] * m, rtol=0, atol=1e-14)


# --- L2: state and read against closed forms and brute force --------------

def test_final_state_closed_form():
    """A_final = eta * sum_{i<=T-1-W} lam^(T-1-W-i) k_i v_i^T, as one float64
    matmul K^T diag(w) V (d_k != d_v so a transposed outer product fails)."""
    B, H, T, dk, dv, W = 2, 3, 57, 6, 4, 11
    x = _small(B=B, H=H, T=T, dk=dk, dv=dv, W=W)
    _, A = oracle.prefill(x.q, x.k, x.v, x.lam, x.eta, x.g, W)
    E = T - W
    for b in range(B):
        for h in range(H):
            lam, eta = float(x.lam[h]), float(x.eta[h])
            K = x.k[b, h, :E].double().numpy()
            V = x.v[b, h, :E].double().numpy()
            w = eta * lam ** (E - 1 - np.arange(E, dtype=np.float64))
            ref = K.T @ (w[:, None] * V)
            assert A[b, h].shape == (dk, dv)
            np.testing.assert_allclose(A[b, h], ref, rtol=1e-12, atol=1e-15)


def test_memory_read_brute_force():
    """m_t = sum_{i <= t-W} eta lam^(t-W-i) <q_t,k_i> v_i, by brute force over
    tokens.  The eviction of token t-W is included, so the write precedes the
    read within a step (Fig. 2 order; every earlier token reaches the query
    through exactly one path, §3.2)."""
    B, H, T, dk, dv, W = 1, 2, 24, 5, 3, 4
    x = _small(B=B, H=H, T=T, dk=dk, dv=dv, W=W)
    y, _, yl, m = oracle.prefill(x.q, x.k, x.v, x.lam, x.eta, x.g, W, parts=True)
    q, k, v = (t.double().numpy() for t in (x.q, x.k, x.v))
    for h in range(H):
        lam, eta = float(x.lam[h]), float(x.eta[h])
        for t in range(T):
            ref = np.zeros(dv)
            for i in range(0, t - W + 1):
                ref += eta * lam ** (t - W - i) * np.dot(q[0, h, t], k[0, h, i]) * v[0, h, i]
            np.testing.assert_allclose(m[0, h, t], ref, rtol=1e-12, atol=1e-15)
    # and the partition: the window part never sees an evicted token
    np.testing.assert_allclose(yl, _sdpa_band(x.q, x.k, x.v, W), rtol=0, atol=1e-13)


def test_read_identity():
    """q (k (x) v) = <q,k> v (abstract; §1): after the single eviction at
    t = W the state is eta k_0 v_0^T and the read is eta <q_W, k_0> v_0."""
    W, dk, dv = 3, 6, 4
    x = _small(B=1, H=1, T=W + 1, dk=dk, dv=dv, W=W)
    _, A, _, m = oracle.prefill(x.q, x.k, x.v, x.lam, x.eta, x.g, W, parts=True)
    q, k, v = (t.double().numpy()[0, 0] for t in (x.q, x.k, x.v))
    eta = float(x.eta[0])
    np.testing.assert_allclose(A[0, 0], eta * np.outer(k[0], v[0]), rtol=1e-15, atol=0)
    np.testing.assert_allclose(m[0, 0, W], eta * np.dot(q[W], k[0]) * v[0], rtol=1e-14, atol=1e-16)
    assert np.all(m[0, 0, :W] == 0.0)


def test_exact_recall_orthonormal_keys():
    """lam = eta = 1 and orthonormal evicted keys: querying with k_i returns
    v_i exactly (spec property 4)."""
    dk, dv, E, W = 16, 5, 12, 3
    rng = np.random.default_rng(3)
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    keys = Qm.T[:E]  # orthonormal rows
    vals = rng.standard_normal((E, dv))
    T = E + W  # the query at t = E-1+W sees tokens 0..E-1 through A only
    H = E
    q = np.zeros((1, H, T, dk))
    k = np.zeros((1, H, T, dk))
    v = np.zeros((1, H, T, dv))
    k[0, :, :E] = keys
    v[0, :, :E] = vals
    for h in range(H):
        q[0, h, T - 1] = keys[h]
    ones = np.ones(H)
    _, _, _, m = oracle.prefill(q, k, v, ones, ones, np.zeros(H), W, parts=True)
    for h in range(H):
        np.testing.assert_allclose(m[0, h, T - 1], vals[h], rtol=0, atol=1e-14)


# --- the optional delta-rule write (Fig. 2 step (3)) ------------------------

@pytest.mark.parametrize("lam,eta,n", [(1.0, 1.0, 3), (1.0, 0.5, 4), (0.9, 0.3, 6)])
def test_delta_rule_repeated_write_closed_form(lam, eta, n):
    """The same pair (unit key k, value v) written n times: with A = a k v^T
    the delta write gives a_n = (lam - eta) a_{n-1} + eta, so a_n =
    eta (1 - (lam - eta)^n) / (1 - (lam - eta)).  The outer product gives
    a_n = lam a_{n-1} + eta instead.  W = 1: token t evicts token t-1, so
    n + 1 identical tokens make n writes."""
    dk, dv = 4, 3
    rng = np.random.default_rng(11)
    kvec = rng.standard_normal(dk)
    kvec /= np.linalg.norm(kvec)
    vvec = rng.standard_normal(dv)
    T = n + 1
    q = np.zeros((1, 1, T, dk))
    k = np.tile(kvec, (1, 1, T, 1))
    v = np.tile(vvec, (1, 1, T, 1))
    prm = [np.array([lam]), np.array([eta]), np.zeros(1)]
    r = lam - eta
    a_delta = eta * n if abs(1 - r) < 1e-15 else eta * (1 - r ** n) / (1 - r)
    a_outer = sum(eta * lam ** j for j in range(n))
    _, A_d = oracle.prefill(q, k, v, *prm, 1, rule="delta")
    _, A_o = oracle.prefill(q, k, v, *prm, 1, rule="outer")
    np.testing.assert_allclose(A_d[0, 0], a_delta * np.outer(kvec, vvec), rtol=0, atol=1e-13)
    np.testing.assert_allclose(A_o[0, 0], a_outer * np.outer(kvec, vvec), rtol=0, atol=1e-13)


def test_delta_rule_equals_outer_product_on_orthonormal_keys():
    """Each evicted key orthogonal to every earlier one: k^T A = 0 before each
    write, so the delta write adds the same k v^T as the outer product."""
    dk, dv, E, W = 8, 3, 6, 2
    rng = np.random.default_rng(12)
    Qm, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    T = E + W
    q = rng.standard_normal((1, 2, T, dk))
    k = np.zeros((1, 2, T, dk))
    k[0, :, :E] = Qm.T[:E]
    v = rng.standard_normal((1, 2, T, dv))
    prm = [np.array([1.0, 1.0]), np.array([1.0, 1.0]), np.array([0.3, -0.2])]
    y_d, A_d = oracle.prefill(q, k, v, *prm, W, rule="delta")
    y_o, A_o = oracle.prefill(q, k, v, *prm, W, rule="outer")
    np.testing.assert_allclose(A_d, A_o, rtol=0, atol=1e-13)
    np.testing.assert_allclose(y_d, y_o, rtol=0, atol=1e-13)


def test_delta_rule_decode_continues_prefill():
    """The streaming form and the prefill form run the same token loop."""
    x = wl.random_prefill(1, 2, 50, 6, 5, 7, 4, dtype="f32", seed=13)
    T0 = 30
    y_full, A_full = oracle.prefill(x.q, x.k, x.v, x.lam, x.eta, x.g, 7, rule="delta")
    _, A0 = oracle.prefill(x.q[:, :, :T0], x.k[:, :, :T0], x.v[:, :, :T0], x.lam, x.eta, x.g,
                           7, rule="delta")
    ring_k = np.zeros((1, 2, 7, 6))
    ring_v = np.zeros((1, 2, 7, 5))
    for j in range(T0 - 7, T0):
        ring_k[:, :, j % 7] = x.k[:, :, j].double().numpy()
        ring_v[:, :, j % 7] = x.v[:, :, j].double().numpy()
    y, _, _, A = oracle.decode(ring_k, ring_v, A0, T0, x.q[:, :, T0:].permute(2, 0, 1, 3),
                               x.k[:, :, T0:].permute(2, 0, 1, 3),
                               x.v[:, :, T0:].permute(2, 0, 1, 3), x.lam, x.eta, x.g,
                               rule="delta")
    np.testing.assert_allclose(y.transpose(1, 2, 0, 3), y_full[:, :, T0:], rtol=0, atol=1e-12)
    np.testing.assert_allclose(A, A_full, rtol=0, atol=1e-12)


# --- backward: reverse-mode gradients against finite differences -----------

def test_backward_matches_central_differences():
    """Every gradient element of L = sum <dy, y> (q, k, v, lam, eta, g) agrees
    with a central difference of the forward oracle, on an input where the
    window fills and many pairs are evicted."""
    rng = np.random.default_rng(21)
    B, H, T, dk, dv, W = 1, 2, 11, 3, 2, 3
    q, k = (rng.standard_normal((B, H, T, dk)) * 0.6 for _ in range(2))
    v, dy = (rng.standard_normal((B, H, T, dv)) * 0.6 for _ in range(2))
    lam, eta, g = np.array([0.9, 0.75]), np.array([0.6, 1.2]), np.array([0.4, -0.7])
    grads = dict(zip(("q", "k", "v", "lam", "eta", "g"), oracle.backward(q, k, v, lam, eta, g, W, dy)))
    x = {"q": q, "k": k, "v": v, "lam": lam, "eta": eta, "g": g}

    def loss(**over):
        a = {**x, **over}
        y, _ = oracle.prefill(a["q"], a["k"], a["v"], a["lam"], a["eta"], a["g"], W)
        return float((y * dy).sum())

    h = 1e-6
    for name, base in x.items():
        fd = np.empty_like(base)
        for idx in np.ndindex(base.shape):
            xp, xm = base.copy(), base.copy()
            xp[idx] += h
            xm[idx] -= h
            fd[idx] = (loss(**{name: xp}) - loss(**{name: xm})) / (2 * h)
        np.testing.assert_allclose(grads[name], fd, rtol=0, atol=5e-8, err_msg=name)


# --- training form: chunk scan and the chunk-mean shortcut -----------------

@pytest.mark.parametrize("C", [1, 7, 16, 64, 300])
def test_chunk_scan_equals_token_writes_fp64(C):
    """The weighted-sum chunk scan is the per-token recurrence unrolled, so in
    float64 both agree to rounding, for any C including a ragged last chunk
    (abstract; §1 contributions)."""
    x = wl.prefill_config("tiny_fp32")
    E = 224
    k, v = x.k[0, 0, :E], x.v[0, 0, :E]
    At = oracle.scan_tokens(k, v, 0.95, 0.5)
    Ac = oracle.scan_chunks(k, v, 0.95, 0.5, C)
    assert np.linalg.norm(Ac - At) / np.linalg.norm(At) < 1e-14
    K, V = k.double().numpy(), v.double().numpy()
    w = 0.5 * 0.95 ** (E - 1 - np.arange(E, dtype=np.float64))
    np.testing.assert_allclose(At, K.T @ (w[:, None] * V), rtol=1e-12, atol=1e-16)


def test_chunk_scan_fp32_within_float32_rounding():
    """In float32 the chunk scan and the per-token writes both land within
    float32 rounding of the exact state (the pages: 'within float32 epsilon',
    'within 1e-7 relative').  Norm-wise relative error, bound 8 * 2^-23."""
    eps32 = 2.0 ** -23
    cases = []
    x = wl.prefill_config("tiny_fp32")
    cases.append((x.k[0, 0, :224], x.v[0, 0, :224], 0.95, 0.5, 16))
    x2 = wl.prefill_config("recall_fp32")
    for h in range(4):
        cases.append((x2.k[0, h, :1792], x2.v[0, h, :1792], float(x2.lam[h]),
                      float(x2.eta[h]), 64))
    for k, v, lam, eta, C in cases:
        exact = oracle.scan_tokens(k, v, lam, eta)
        nrm = np.linalg.norm(exact)
        tok32 = oracle.scan_tokens(k, v, lam, eta, fp32=True)
        chk32 = oracle.scan_chunks(k, v, lam, eta, C, fp32=True)
        assert np.linalg.norm(chk32 - exact) / nrm < 8 * eps32
        assert np.linalg.norm(tok32 - exact) / nrm < 8 * eps32
        assert np.linalg.norm(chk32 - tok32) / nrm < 8 * eps32


@pytest.mark.parametrize("C", [2, 5, 8])
def test_chunk_mean_adds_exactly_the_cross_terms(C):
    """With lam = eta = 1, C^2 * (kbar (x) vbar) summed over chunks minus the
    true writes equals the C^2 - C cross products k_i (x) v_j, i != j, of each
    chunk, computed by brute force (abstract; §1)."""
    rng = np.random.default_rng(C)
    n_chunks, dk, dv = 3, 4, 3
    E = C * n_chunks
    k = rng.standard_normal((E, dk))
    v = rng.standard_normal((E, dv))
    A_mean = oracle.scan_chunk_mean(k, v, 1.0, 1.0, C)
    A_true = oracle.scan_chunks(k, v, 1.0, 1.0, C)
    cross = np.zeros((dk, dv))
    count = 0
    for c in range(n_chunks):
        idx = range(c * C, (c + 1) * C)
        n_c = 0
        for i in idx:
            for j in idx:
                if i != j:
                    cross += np.outer(k[i], v[j])
                    n_c += 1
        assert n_c == C * C - C
        count += n_c
    assert count == n_chunks * (C * C - C)
    np.testing.assert_allclose(C * C * A_mean - A_true, cross, rtol=1e-12, atol=1e-12)
    # and the shortcut is a different state whenever C > 1
    assert np.linalg.norm(A_mean - A_true) > 1e-3 * np.linalg.norm(A_true)


def test_chunk_mean_with_decay_drops_per_token_weights():
    """With lam != 1 the shortcut also loses the per-token decay weights: for
    one chunk it equals eta * kbar (x) vbar, the exact write is
    eta * sum_i lam^(C-1-i) k_i (x) v_i."""
    rng = np.random.default_rng(11)
    C, dk, dv = 6, 3, 2
    k = rng.standard_normal((C, dk))
    v = rng.standard_normal((C, dv))
    lam, eta = 0.7, 0.4
    np.testing.assert_allclose(oracle.scan_chunk_mean(k, v, lam, eta, C),
                               eta * np.outer(k.mean(0), v.mean(0)), rtol=1e-14, atol=1e-15)
    w = eta * lam ** (C - 1 - np.arange(C))
    np.testing.assert_allclose(oracle.scan_chunks(k, v, lam, eta, C), k.T @ (w[:, None] * v),
                               rtol=1e-13, atol=1e-15)


# --- streaming form -------------------------------------------------------

def test_decode_from_empty_state_reproduces_prefill():
    """Decode steps from an empty ring, t0 = 0, reproduce prefill y and A."""
    B, H, T, dk, dv, W = 2, 2, 19, 4, 3, 5
    x = _small(B=B, H=H, T=T, dk=dk, dv=dv, W=W)
    y, A = oracle.prefill(x.q, x.k, x.v, x.lam, x.eta, x.g, W)
    z = lambda d: np.zeros((B, H, W, d))
    yd, rk, rv, Ad = oracle.decode(z(dk), z(dv), np.zeros((B, H, dk, dv)), 0,
                                   x.q.permute(2, 0, 1, 3), x.k.permute(2, 0, 1, 3),
                                   x.v.permute(2, 0, 1, 3), x.lam, x.eta, x.g)
    np.testing.assert_array_equal(yd.transpose(1, 2, 0, 3), y)
    np.testing.assert_array_equal(Ad, A)
    # the ring ends holding token j at slot j mod W
    for j in range(T - W, T):
        np.testing.assert_array_equal(rk[:, :, j % W], x.k[:, :, j].double().numpy())


def test_ring_slot_order_does_not_change_the_read():
    """Softmax over the window is permutation invariant: permuting the ring
    slots other than the one being overwritten leaves y unchanged (§3.2 ring
    buffer; eq. (1))."""
    rng = np.random.default_rng(5)
    B, H, W, dk, dv = 1, 2, 7, 4, 3
    rk = rng.standard_normal((B, H, W, dk))
    rv = rng.standard_normal((B, H, W, dv))
    A = rng.standard_normal((B, H, dk, dv))
    t0 = 3 * W + 2
    pos = t0 % W
    q = rng.standard_normal((1, B, H, dk))
    k = rng.standard_normal((1, B, H, dk))
    v = rng.standard_normal((1, B, H, dv))
    lam, eta, g = np.array([0.9, 0.8]), np.array([0.5, 1.1]), np.array([0.2, -0.4])
    y, *_ = oracle.decode(rk, rv, A, t0, q, k, v, lam, eta, g)
    perm = [i for i in range(W) if i != pos]
    shuffled = perm[::-1]
    rk2, rv2 = rk.copy(), rv.copy()
    rk2[:, :, perm] = rk[:, :, shuffled]
    rv2[:, :, perm] = rv[:, :, shuffled]
    y2, *_ = oracle.decode(rk2, rv2, A, t0, q, k, v, lam, eta, g)
    np.testing.assert_allclose(y2, y, rtol=1e-13, atol=1e-15)


def test_decode_before_ring_fills_masks_empty_slots():
    """t < W: no eviction and only slots 0..t take part; garbage in the
    unfilled slots must not change y (exact causal, §3.1)."""
    rng = np.random.default_rng(9)
    B, H, W, dk, dv = 1, 1, 8, 4, 4
    t0 = 3
    rk = np.zeros((B, H, W, dk))
    rv = np.zeros((B, H, W, dv))
    rk[:, :, :t0] = rng.standard_normal((B, H, t0, dk))
    rv[:, :, :t0] = rng.standard_normal((B, H, t0, dv))
    A = rng.standard_normal((B, H, dk, dv))
    q, k = rng.standard_normal((2, 1, B, H, dk))
    v = rng.standard_normal((1, B, H, dv))
    args = (q, k, v, [0.9], [0.5], [0.0])
    y, _, _, A1 = oracle.decode(rk, rv, A, t0, *args)
    rk[:, :, t0 + 1:] = 1e3
    rv[:, :, t0 + 1:] = -1e3
    y2, _, _, A2 = oracle.decode(rk, rv, A, t0, *args)
    np.testing.assert_array_equal(y, y2)
    np.testing.assert_array_equal(A1, A)  # no eviction: A untouched
    keys = np.concatenate([rk[0, 0, :t0], k[0, 0]], 0)
    vals = np.concatenate([rv[0, 0, :t0], v[0, 0]], 0)
    s = keys @ q[0, 0, 0] / 2.0
    p = np.exp(s - s.max())
    p /= p.sum()
    ref = p @ vals + 0.5 * (q[0, 0, 0] @ A[0, 0])
    np.testing.assert_allclose(y[0, 0, 0], ref, rtol=1e-13)


# --- hand-worked fixtures -------------------------------------------------

def _ev(e):
    return float(eval(str(e), {"__builtins__": {}}, {"sqrt": math.sqrt, "log": math.log,
                                                    "exp": math.exp}))


def test_golden_hand_d1_w1():
    with open(os.path.join(GOLDEN, "hand_d1_w1.json")) as f:
        gd = json.load(f)
    i = gd["inputs"]
    arr = lambda a: np.array(a, dtype=np.float64).reshape(1, 1, -1, 1)
    y, A, _, m = oracle.prefill(arr(i["q"]), arr(i["k"]), arr(i["v"]), [i["lam"]], [i["eta"]],
                                [i["g"]], i["W"], parts=True)
    np.testing.assert_array_equal(y.ravel(), gd["expected"]["y"])
    np.testing.assert_array_equal(m.ravel(), gd["expected"]["m"])
    assert A.item() == gd["expected"]["A_final"]


def test_golden_hand_d2_w2():
    with open(os.path.join(GOLDEN, "hand_d2_w2.json")) as f:
        gd = json.load(f)
    i = gd["inputs"]
    q = np.array([[_ev(e) for e in row] for row in i["q_expr"]])[None, None]
    k = np.array(i["k"], dtype=np.float64)[None, None]
    v = np.array(i["v"], dtype=np.float64)[None, None]
    y, A, _, m = oracle.prefill(q, k, v, [i["lam"]], [i["eta"]], [_ev(i["g_expr"])], i["W"],
                                parts=True)
    ex = gd["expected_expr"]
    np.testing.assert_allclose(y[0, 0], [[_ev(e) for e in r] for r in ex["y"]], rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(m[0, 0], [[_ev(e) for e in r] for r in ex["m"]], rtol=1e-14, atol=1e-15)
    np.testing.assert_allclose(A[0, 0], [[_ev(e) for e in r] for r in ex["A_final"]], rtol=0, atol=1e-15)


# --- workload generators (shape / distribution sanity, no layer math) ------

def test_recall_workload_layout():
    x = wl.prefill_config("recall_fp32")
    pos = x.meta["plant"]["positions"]
    assert pos[0] == 0 and pos[-1] == 504 and len(pos) == 64
    nk = torch.linalg.vector_norm(x.k[:, :, pos].double(), dim=-1)
    assert torch.allclose(nk, torch.ones_like(nk), atol=1e-6)
    # the query at 1800 + j re-issues planted key j mod 64 with small noise
    d = x.q[:, :, 1800 + 65].double() - x.k[:, :, pos[1]].double()
    assert float(d.norm(dim=-1).max()) < 0.05 * 64 ** 0.5 * 2


def test_lm_workload_is_rms_normalised():
    x = wl.prefill_config("lm_prefill_bf16")
    assert x.q.dtype == torch.bfloat16 and x.q.shape == (8, 12, 4096, 64)
    rms = x.k[0, 0, :100].double().pow(2).mean(-1).sqrt()
    assert torch.allclose(rms, torch.ones_like(rms), atol=1e-2)
    assert float(x.lam.min()) > 0.95 and float(x.lam.max()) < 0.9991
