"""GPU checks of the chunk-mean ablation (TC_PREFILL_CHUNK_MEAN) against the
oracle's shortcut, and of the capacity diagnostic built on it."""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("C", [1, 7, 32])
def test_chunk_mean_ablation_matches_the_oracle_shortcut(cuda_device, C):
    import sliding_window_attention_tc_b200 as tc
    gen = torch.Generator().manual_seed(C)
    E, dk, dv, lam, eta = 300, 16, 12, 0.95, 0.7
    k = torch.randn(E + 1, dk, generator=gen) / 4
    v = torch.randn(E + 1, dv, generator=gen) / 4
    dev = cuda_device
    A_mean, A_scan = (tc.prefill_from_state(
        None, k.view(1, 1, E + 1, dk).to(dev), v.view(1, 1, E + 1, dv).to(dev),
        torch.tensor([lam], device=dev), torch.tensor([eta], device=dev),
        torch.zeros(1, device=dev), 1, C, 0, state_only=True, chunk_mean=cm)[1][0, 0].cpu().numpy()
        for cm in (True, False))
    ref_mean = oracle.scan_chunk_mean(k[:E], v[:E], lam, eta, C)
    ref_scan = oracle.scan_tokens(k[:E], v[:E], lam, eta)
    den = np.abs(ref_mean).max()
    assert np.abs(A_mean - ref_mean).max() <= 1e-5 * den
    assert np.abs(A_scan - ref_scan).max() <= 1e-5 * np.abs(ref_scan).max()
    if C == 1:  # one write per chunk: the shortcut is exact
        np.testing.assert_allclose(ref_mean, ref_scan, rtol=0, atol=1e-12)


def test_capacity_curve_scan_beats_chunk_mean(cuda_device):
    from sliding_window_attention_tc_b200.capacity import capacity_curve
    rows = capacity_curve(d=64, Ns=(16, 64, 256), C=16, device=cuda_device)
    assert rows[0]["scan_recall_top1"] == 1.0          # few pairs: every key retrieves its value
    for r in rows:
        assert r["scan_recall_cos"] > r["mean_recall_cos"]
    assert rows[0]["scan_recall_cos"] > rows[-1]["scan_recall_cos"]  # capacity falls off with N
