"""Sequence-sharded prefill on gloo ranks (CPU): the exchange logic of
sliding_window_attention_tc_b200.sharded with the float64 oracle as each
rank's compute, against the oracle on the unsplit sequence.

Each rank holds one contiguous piece of every (b,h) sequence.  The pieces
are coupled by the window (a halo of the W keys/values before the piece) and
by the L2 state (the decayed sum of every earlier eviction).  Exactly these
two couplings cross the process boundary, through all-gathers.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def oracle_prefill_fn(q, k, v, lam, eta, g, W, C, t0, halo_k, halo_v, A_init, state_only):
    """The layer over the new tokens from (halo, A_init) at position t0, by
    running the oracle's token loop from the corresponding ring state."""
    import oracle
    B, H, T, dk = k.shape
    dv = v.shape[-1]
    ring_k = np.zeros((B, H, W, dk))
    ring_v = np.zeros((B, H, W, dv))
    n = 0 if halo_k is None else halo_k.shape[2]
    for j in range(n):
        t = t0 - n + j
        ring_k[:, :, t % W] = halo_k[:, :, j].double().numpy()
        ring_v[:, :, t % W] = halo_v[:, :, j].double().numpy()
    A = np.zeros((B, H, dk, dv)) if A_init is None else A_init.double().numpy()
    qq = torch.zeros_like(k) if q is None else q
    y, _, _, A_out = oracle.decode(ring_k, ring_v, A, t0, qq.permute(2, 0, 1, 3).numpy(),
                                   k.permute(2, 0, 1, 3).numpy(), v.permute(2, 0, 1, 3).numpy(),
                                   lam.numpy(), eta.numpy(), g.numpy())
    y = torch.from_numpy(np.ascontiguousarray(y.transpose(1, 2, 0, 3)))
    return (None if state_only else y), torch.from_numpy(A_out)


def decayed_sum_fold(dA, E, lam):
    """The state before the next piece: A <- lam^E_s A + dA_s over the pieces."""
    A = torch.zeros(dA.shape[1:], dtype=torch.float64)
    for s in range(dA.shape[0]):
        dec = lam.double() ** float(E[s])
        A = dec.view(1, -1, 1, 1) * A + dA[s].double()
    return A


def _worker(rank, world, port, lens, W, out):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import datetime

    import torch.distributed as dist
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    from sliding_window_attention_tc_b200 import sharded
    x = _sequence(sum(lens), W)
    a, b = sum(lens[:rank]), sum(lens[:rank + 1])
    piece = [t[:, :, a:b].contiguous() for t in (x["q"], x["k"], x["v"])]
    y, A = sharded.sharded_prefill(*piece, x["lam"], x["eta"], x["g"], W, 16,
                                   prefill_fn=oracle_prefill_fn, fold_fn=decayed_sum_fold)
    out[rank] = (y.numpy(), A.numpy())
    dist.barrier()
    dist.destroy_process_group()


def _sequence(T, W, B=1, H=2, d=8, seed=77):
    gen = torch.Generator().manual_seed(seed)
    r = lambda *s: torch.randn(*s, generator=gen, dtype=torch.float64)
    return {"q": r(B, H, T, d) / 2, "k": r(B, H, T, d) / 2, "v": r(B, H, T, d) / 2,
            "lam": torch.tensor([0.97, 0.9], dtype=torch.float64),
            "eta": torch.tensor([0.5, 0.8], dtype=torch.float64),
            "g": torch.tensor([0.3, -0.4], dtype=torch.float64)}


CASES = [
    ([70, 50], 16),        # two ranks, pieces longer than W
    ([10, 30, 25], 16),    # the first piece is shorter than W: rank 2's halo spans pieces 0 and 1
    ([20, 5, 30], 16),     # a piece shorter than W in the middle
]


@pytest.mark.parametrize("lens,W", CASES, ids=["2ranks", "short_first", "short_middle"])
def test_sharded_prefill_matches_unsplit_sequence(lens, W):
    import oracle
    oracle.build()
    port = _free_port()
    manager = mp.get_context("spawn").Manager()
    out = manager.dict()
    world = len(lens)
    mp.start_processes(_worker, args=(world, port, lens, W, out), nprocs=world, join=True,
                       start_method="spawn")
    x = _sequence(sum(lens), W)
    y_ref, A_ref = oracle.prefill(x["q"].numpy(), x["k"].numpy(), x["v"].numpy(),
                                  x["lam"].numpy(), x["eta"].numpy(), x["g"].numpy(), W)
    for r in range(world):
        a, b = sum(lens[:r]), sum(lens[:r + 1])
        y, A = out[r]
        np.testing.assert_allclose(y, y_ref[:, :, a:b], rtol=0, atol=1e-12)
    np.testing.assert_allclose(out[world - 1][1], A_ref, rtol=0, atol=1e-12)


def test_piece_of_builds_halo_across_short_pieces():
    from sliding_window_attention_tc_b200 import sharded
    W = 4
    lens = [2, 1, 5]
    ks = [torch.arange(n, dtype=torch.float64).view(1, 1, n, 1) + 100 * s
          for s, n in enumerate(lens)]
    tails = [sharded.tail(k, k, W) for k in ks]
    p = sharded.piece_of(2, lens, [t[0] for t in tails], [t[1] for t in tails], W)
    assert p.t0 == 3
    # tokens 0, 1 (piece 0) and 2 (piece 1) are the 3 = min(t0, W) halo rows
    assert p.halo_k.flatten().tolist() == [0.0, 1.0, 100.0]
    assert p.evictions == 3 + 5 - 4
    p0 = sharded.piece_of(0, lens, [t[0] for t in tails], [t[1] for t in tails], W)
    assert p0.t0 == 0 and p0.halo_k is None and p0.evictions == 0
