"""Checkpoint and resume of a decode stream.

The streaming state of the layer is the ring of the last W keys and values,
the matrix A and the clock t ("Tensor Cache: Eviction-conditioned
Associative Memory for Transformers", §3.2 Fig. 2: each step reads and
writes only these).  Copying them out mid-stream to host memory, restoring
them into fresh device buffers and continuing must give the same outputs,
ring and A, bit for bit, as continuing without the copy.  Both continuations
also run the oracle's token loop from the saved state.
"""
import math

import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


def _stream(seed, steps, B, H, d, dtype):
    gen = torch.Generator().manual_seed(seed)
    s = 1.0 / math.sqrt(d)
    return [(torch.randn(steps, B, H, d, generator=gen) * s).to(dtype) for _ in range(3)]


@pytest.mark.parametrize("dtype, d, W", [(torch.bfloat16, 128, 64), (torch.float32, 64, 48),
                                         (torch.bfloat16, 64, 1)])
def test_decode_resumes_bit_for_bit_from_a_host_checkpoint(cuda_device, dtype, d, W):
    import sliding_window_attention_tc_b200 as tc
    dev = cuda_device
    B, H, n1, n2 = 3, 4, 2 * W + 17, W + 23  # the first leg wraps the ring twice
    q, k, v = _stream(7 + d + W, n1 + n2, B, H, d, dtype)
    gen = torch.Generator().manual_seed(99)
    lam = (0.9 + 0.09 * torch.rand(H, generator=gen)).to(dev)
    eta = (0.2 + torch.rand(H, generator=gen)).to(dev)
    g = torch.randn(H, generator=gen).to(dev)
    st = tc.DecodeState.empty(B, H, W, d, d, lam, eta, g, dtype=dtype, device=dev)
    for i in range(n1):
        tc.decode_step(st, q[i].to(dev), k[i].to(dev), v[i].to(dev))
    torch.cuda.synchronize()
    # checkpoint: the whole streaming state, in host memory
    ck = {"ring_k": st.ring_k.cpu(), "ring_v": st.ring_v.cpu(), "A": st.A.cpu(), "t": st.t}
    assert ck["t"] == n1

    def resume(state):
        ys = [tc.decode_step(state, q[n1 + i].to(dev), k[n1 + i].to(dev), v[n1 + i].to(dev))
              for i in range(n2)]
        torch.cuda.synchronize()
        return torch.stack(ys).cpu()

    y_direct = resume(st)
    restored = tc.DecodeState(ck["ring_k"].to(dev), ck["ring_v"].to(dev), ck["A"].to(dev),
                              lam, eta, g, ck["t"])
    y_restored = resume(restored)
    assert tc.device_status() == 0
    assert torch.equal(y_direct, y_restored)
    assert torch.equal(st.ring_k, restored.ring_k) and torch.equal(st.ring_v, restored.ring_v)
    assert torch.equal(st.A, restored.A)
    assert st.t == restored.t == n1 + n2
    # and the continuation is the layer's: the oracle from the saved state
    yo, rko, rvo, Ao = oracle.decode(ck["ring_k"].double().numpy(), ck["ring_v"].double().numpy(),
                                     ck["A"].double().numpy(), n1, q[n1:], k[n1:], v[n1:],
                                     lam.cpu(), eta.cpu(), g.cpu())
    y = y_restored.double().numpy()
    den = np.linalg.norm(yo)
    tol = 1e-2 if dtype == torch.bfloat16 else 1e-5
    assert np.linalg.norm(y - yo) <= tol * den
    np.testing.assert_array_equal(restored.ring_k.cpu().double().numpy(), rko)
    np.testing.assert_array_equal(restored.ring_v.cpu().double().numpy(), rvo)
