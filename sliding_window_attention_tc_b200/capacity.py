"""Capacity of the L2 memory, and the error of the chunk-mean shortcut,
measured on the GPU through libtc.

"Tensor Cache: Eviction-conditioned Associative Memory for Transformers"
(abstract; §1) trains A with a parallel weighted-sum chunk scan and warns
against the chunk-mean shortcut A <- lambda A + eta kbar vbar^T, which adds
C^2 - C spurious cross terms per chunk of C writes.  This diagnostic writes N
random pairs (unit keys, Gaussian values) into A with lambda = eta = 1 (a
plain associative memory), once by the exact scan and once by the shortcut
(TC_PREFILL_CHUNK_MEAN, an ablation of the portable scan).  Then every key
reads the memory, m_i = k_i A.  Reported per N:
  recall_cos   mean cosine between m_i and v_i
  recall_top1  fraction of keys whose read is closest (cosine) to its own value
Both the writes and the reads run in libtc.  The writes are
tc_prefill_from_state, state only: the N pairs are the evictions of an N + 1
token sequence with W = 1.  The reads are the layer's own L2 read: a
continuation (t0 = 1, W = 1) from A_init = A whose window holds only zero
values and whose writes add nothing (eta = 0), with the keys as queries and
sigmoid(g) = 1, so that y_i = k_i A.  Only the scores (cosines, argmax) are
computed here, with PyTorch, as analysis.
"""
from __future__ import annotations

from typing import Dict, List, Sequence

import torch


def _state(k: torch.Tensor, v: torch.Tensor, C: int, chunk_mean: bool) -> torch.Tensor:
    from . import prefill_from_state
    N, d = k.shape
    dev = k.device
    pad = torch.zeros(1, d, device=dev)
    ks = torch.cat([k, pad]).view(1, 1, N + 1, d).contiguous()
    vs = torch.cat([v, pad]).view(1, 1, N + 1, d).contiguous()
    one = torch.ones(1, device=dev)
    _, A = prefill_from_state(None, ks, vs, one, one, torch.zeros(1, device=dev), 1, C, 0,
                              state_only=True, chunk_mean=chunk_mean)
    return A[0, 0]


def _read(k: torch.Tensor, A: torch.Tensor) -> torch.Tensor:
    """m_i = k_i A through the layer: every window value is zero (y_local =
    0), eta = 0 keeps A fixed over the call, and g = 40 makes sigmoid(g) = 1
    in float32, so the output is the memory read alone."""
    from . import prefill_from_state
    N, d = k.shape
    dev = k.device
    zeros = torch.zeros(1, 1, N, d, device=dev)
    halo = torch.zeros(1, 1, 1, d, device=dev)
    y, _ = prefill_from_state(k.contiguous().view(1, 1, N, d), zeros, zeros,
                              torch.ones(1, device=dev), torch.zeros(1, device=dev),
                              torch.full((1,), 40.0, device=dev), 1, 1, 1, halo, halo,
                              A.contiguous().view(1, 1, d, d))
    return y[0, 0]


def _scores(k, v, A) -> Dict[str, float]:
    m = _read(k, A)
    mn = torch.nn.functional.normalize(m, dim=-1)
    vn = torch.nn.functional.normalize(v, dim=-1)
    cos = (mn * vn).sum(-1)
    top1 = ((mn @ vn.T).argmax(-1) == torch.arange(k.shape[0], device=k.device)).float()
    return {"recall_cos": float(cos.mean()), "recall_top1": float(top1.mean())}


def capacity_curve(d: int = 64, Ns: Sequence[int] = (16, 32, 64, 128, 256, 512), C: int = 16,
                   seed: int = 0, device: str = "cuda") -> List[Dict[str, float]]:
    """Recall against the number of stored pairs, for the exact scan and for
    the chunk-mean shortcut with chunks of C writes."""
    rows = []
    for N in Ns:
        gen = torch.Generator().manual_seed(seed + N)
        k = torch.nn.functional.normalize(torch.randn(N, d, generator=gen), dim=-1).to(device)
        v = torch.randn(N, d, generator=gen).to(device)
        exact = _scores(k, v, _state(k, v, C, False))
        mean = _scores(k, v, _state(k, v, C, True))
        rows.append({"N": N, "d": d, "C": C,
                     "scan_recall_cos": exact["recall_cos"], "scan_recall_top1": exact["recall_top1"],
                     "mean_recall_cos": mean["recall_cos"], "mean_recall_top1": mean["recall_top1"]})
    return rows


if __name__ == "__main__":
    import json
    for row in capacity_curve():
        print(json.dumps(row))
