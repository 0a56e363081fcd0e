"""The Python binding rejects tensors of the wrong dtype or shape before any
C-ABI call (CPU only).

The library sees only addresses, so a [H] parameter in float16, or a y buffer
one token short, would make a kernel read or write past the end of it.  The
binding checks every tensor against the shapes the call implies, and raises
TypeError or ValueError first.
"""
import pytest
import torch

import sliding_window_attention_tc_b200 as tc

B, H, T, D, W = 2, 3, 40, 16, 8


def _layer(dtype=torch.float32):
    q, k, v = (torch.randn(B, H, T, D).to(dtype) for _ in range(3))
    lam, eta, g = torch.full((H,), 0.9), torch.full((H,), 0.5), torch.zeros(H)
    return q, k, v, lam, eta, g


@pytest.mark.parametrize("bad, err", [
    (dict(lam=torch.full((H,), 0.9, dtype=torch.float16)), TypeError),
    (dict(eta=torch.full((H + 1,), 0.5)), ValueError),
    (dict(g=torch.zeros(1, H)), ValueError),
    (dict(k=torch.randn(B, H, T, D).to(torch.bfloat16)), TypeError),
    (dict(v=torch.randn(B, H, T - 1, D)), ValueError),
    (dict(y=torch.empty(B, H, T - 1, D)), ValueError),
    (dict(y=torch.empty(B, H, T, D, dtype=torch.bfloat16)), TypeError),
    (dict(A_final=torch.empty(B, H, D, D, dtype=torch.float64)), TypeError),
])
def test_prefill_rejects_mismatched_tensors(bad, err):
    q, k, v, lam, eta, g = _layer()
    args = dict(q=q, k=k, v=v, lam=lam, eta=eta, g=g)
    extra = {n: bad.pop(n) for n in ("y", "A_final") if n in bad}
    args.update(bad)
    with pytest.raises(err):
        tc.prefill(args["q"], args["k"], args["v"], args["lam"], args["eta"], args["g"], W, 8,
                   **extra)


def test_prefill_from_state_checks_halo_and_initial_state():
    q, k, v, lam, eta, g = _layer()
    t0 = 20  # halo of min(t0, W) = 8 tokens
    hk, hv = torch.randn(B, H, W, D), torch.randn(B, H, W, D)
    with pytest.raises(ValueError):
        tc.prefill_from_state(q, k, v, lam, eta, g, W, 8, t0, hk[:, :, 1:], hv)
    with pytest.raises(TypeError):
        tc.prefill_from_state(q, k, v, lam, eta, g, W, 8, t0, hk, hv.double())
    with pytest.raises(ValueError):
        tc.prefill_from_state(q, k, v, lam, eta, g, W, 8, t0, hk, hv, torch.zeros(B, H, D, D + 1))


def test_backward_checks_dy():
    q, k, v, lam, eta, g = _layer()
    with pytest.raises(ValueError):
        tc.backward(q, k, v, lam, eta, g, W, torch.randn(B, H, T, D + 1))
    with pytest.raises(TypeError):
        tc.backward(q, k, v, lam, eta, g, W, torch.randn(B, H, T, D).double())


def test_decode_checks_step_tensors_and_state():
    lam, eta, g = torch.full((H,), 0.9), torch.full((H,), 0.5), torch.zeros(H)
    st = tc.DecodeState.empty(B, H, W, D, D, lam, eta, g, dtype=torch.bfloat16, device="cpu")
    q = torch.randn(B, H, D).to(torch.bfloat16)
    with pytest.raises(TypeError):
        tc.decode_step(st, q.float(), q, q)
    with pytest.raises(ValueError):
        tc.decode_step(st, q, q, q[:, :, :-1])
    with pytest.raises(ValueError):
        tc.decode_step(st, q, q, q, y=torch.empty(B, H + 1, D, dtype=torch.bfloat16))
    with pytest.raises(ValueError):
        tc.decode_step_ragged(st, torch.zeros(B + 1, dtype=torch.int64), q, q, q)
    with pytest.raises(TypeError):
        tc.decode_step_ragged(st, torch.zeros(B, dtype=torch.int32), q, q, q)
    bad = tc.DecodeState(st.ring_k, st.ring_v, st.A.double(), lam, eta, g, 0)
    with pytest.raises(TypeError):
        tc.decode_step(bad, q, q, q)
    bad = tc.DecodeState(st.ring_k, st.ring_v, st.A, lam[:-1], eta, g, 0)
    with pytest.raises(ValueError):
        tc.decode_step(bad, q, q, q)


def test_state_fold_checks_shapes():
    dA = torch.zeros(2, B, H, D, D)
    with pytest.raises(ValueError):
        tc.state_fold(dA, torch.zeros(3, dtype=torch.int64), torch.full((H,), 0.9))
    with pytest.raises(ValueError):
        tc.state_fold(dA, torch.zeros(2, dtype=torch.int64), torch.full((H + 1,), 0.9))


def test_valid_tensors_pass_the_checks():
    # well-formed CPU tensors pass the checks; what stops the call is the
    # missing device (no CUDA stream here, or the library refusing host
    # memory), a RuntimeError, never the TypeError / ValueError of a check
    q, k, v, lam, eta, g = _layer()
    with pytest.raises(RuntimeError):
        tc.prefill(q, k, v, lam, eta, g, W, 8)


def test_prefill_varlen_checks_the_packed_layout():
    total = 50
    q, k, v = (torch.randn(total, H, 64).to(torch.bfloat16) for _ in range(3))
    lam, eta, g = torch.full((H,), 0.9), torch.full((H,), 0.5), torch.zeros(H)
    cu = torch.tensor([0, 20, 50], dtype=torch.int64)
    with pytest.raises(TypeError):  # offsets must be int64
        tc.prefill_varlen(q, k, v, cu.int(), 30, lam, eta, g, 128, 64)
    with pytest.raises(ValueError):  # q one token short
        tc.prefill_varlen(q[1:], k, v, cu, 30, lam, eta, g, 128, 64)
    with pytest.raises(TypeError):  # v in another dtype
        tc.prefill_varlen(q, k, v.float(), cu, 30, lam, eta, g, 128, 64)
    with pytest.raises(ValueError):  # A_final for the wrong number of sequences
        tc.prefill_varlen(q, k, v, cu, 30, lam, eta, g, 128, 64,
                          A_final=torch.empty(3, H, 64, 64))
    with pytest.raises(ValueError):  # no sequence at all
        tc.prefill_varlen(q, k, v, cu[:1], 30, lam, eta, g, 128, 64)
