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
The writes run in libtc (tc_prefill_from_state, state only: the N pairs are
the evictions of an N + 1 token sequence with W = 1); the read-out and the
scores are analysis and use PyTorch.
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


def _scores(k, v, A) -> Dict[str, float]:
    m = k @ A
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
