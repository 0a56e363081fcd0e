"""Sequence-sharded prefill: one process per GPU, each holding a contiguous
piece of every (b,h) sequence.

"Tensor Cache: Eviction-conditioned Associative Memory for Transformers":
the layer couples consecutive tokens in two ways, so a piece cannot be
computed from its own tokens alone.

* Window (§3.1): the first W - 1 queries of a piece attend to keys of earlier
  pieces, and the evictions of its first W steps are earlier tokens.  So a
  rank needs a halo: the last min(t0, W) keys and values before its first
  token t0.
* State (§3.2, Fig. 2 step (3)): A at t0 sums every earlier eviction, each
  decayed by lambda once per later write.  Each rank computes what its own
  evictions add to a zero state (dA_r, after E_r evictions).  The ranks
  exchange (dA, E), and the state before piece r is their decayed sum.

Exchange: one all-gather of every rank's tail (its last W keys and values)
and piece length, and one all-gather of (dA_r, E_r).  That is
B*H*d_k*d_v float32 per rank, the same order as one head's state.
Compute per rank: one state-only chunk scan and one prefill from the state,
both in libtc (tc_prefill_from_state), plus tc_state_fold.  No remote memory
is read by a kernel; the collectives carry all data between GPUs.

The sharded prefill works in phases, so the single-process tests can run the same
code for several ranks in turn:
    tail      -> all-gather -> piece_state -> all-gather -> finish
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, List, Optional, Sequence

import torch


@dataclass
class Piece:
    """What a rank knows after the first exchange."""
    t0: int                           # global position of its first token
    halo_k: Optional[torch.Tensor]    # [B,H,n,dk], n = min(t0, W), oldest first
    halo_v: Optional[torch.Tensor]
    evictions: int                    # E_r: evictions that happen inside the piece


def tail(k: torch.Tensor, v: torch.Tensor, W: int):
    """The last min(T, W) keys and values of the local piece, right-aligned in
    [B,H,W,d] buffers (zeros in front), and the piece length."""
    B, H, T, dk = k.shape
    dv = v.shape[-1]
    n = min(T, W)
    tk = k.new_zeros((B, H, W, dk))
    tv = v.new_zeros((B, H, W, dv))
    if n > 0:
        tk[:, :, W - n:] = k[:, :, T - n:]
        tv[:, :, W - n:] = v[:, :, T - n:]
    return tk, tv, T


def piece_of(rank: int, lens: Sequence[int], tails_k: Sequence[torch.Tensor],
             tails_v: Sequence[torch.Tensor], W: int) -> Piece:
    """Halo and eviction count of piece `rank` from everyone's tails.  The halo
    may span several earlier pieces when they are shorter than W."""
    t0 = int(sum(lens[:rank]))
    n = min(t0, W)
    parts_k: List[torch.Tensor] = []
    parts_v: List[torch.Tensor] = []
    have = 0
    for s in range(rank - 1, -1, -1):
        take = min(int(lens[s]), W, n - have)
        if take <= 0:
            break
        parts_k.insert(0, tails_k[s][:, :, W - take:])
        parts_v.insert(0, tails_v[s][:, :, W - take:])
        have += take
    halo_k = torch.cat(parts_k, dim=2).contiguous() if n > 0 else None
    halo_v = torch.cat(parts_v, dim=2).contiguous() if n > 0 else None
    T = int(lens[rank])
    evictions = max(0, n + T - W)
    return Piece(t0, halo_k, halo_v, evictions)


def _library_prefill(q, k, v, lam, eta, g, W, C, t0, halo_k, halo_v, A_init, state_only):
    from . import prefill_from_state
    return prefill_from_state(q, k, v, lam, eta, g, W, C, t0, halo_k, halo_v, A_init,
                              state_only=state_only)


def _library_fold(dA, E, lam):
    from . import state_fold
    return state_fold(dA, E, lam)


def piece_state(piece: Piece, k, v, lam, eta, g, W: int, C: int,
                prefill_fn: Callable = _library_prefill) -> torch.Tensor:
    """dA_r: the state the piece's own evictions leave, started from zero."""
    _, A = prefill_fn(None, k, v, lam, eta, g, W, C, piece.t0, piece.halo_k, piece.halo_v, None,
                      True)
    return A


def finish(rank: int, piece: Piece, dA_all: torch.Tensor, E_all: torch.Tensor, q, k, v, lam,
           eta, g, W: int, C: int, prefill_fn: Callable = _library_prefill,
           fold_fn: Callable = _library_fold):
    """State before the piece from the earlier pieces' (dA, E), then the
    prefill of the piece from that state.  Returns (y, A after the piece)."""
    A_init = fold_fn(dA_all[:rank].contiguous(), E_all[:rank].contiguous(), lam)
    return prefill_fn(q, k, v, lam, eta, g, W, C, piece.t0, piece.halo_k, piece.halo_v, A_init,
                      False)


def sharded_prefill(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, lam: torch.Tensor,
                    eta: torch.Tensor, g: torch.Tensor, W: int, C: int, *, group=None,
                    prefill_fn: Callable = _library_prefill,
                    fold_fn: Callable = _library_fold):
    """Prefill of this rank's piece (q, k, v [B,H,T_r,d]) of a sequence split
    across the ranks of `group` in rank order.  Returns (y [B,H,T_r,dv],
    A_final); on the last rank A_final is A after the whole sequence.

    The tensors live where the process group's backend expects them (CUDA
    for NCCL).  prefill_fn / fold_fn default to libtc; tests on CPU ranks
    pass their own."""
    import torch.distributed as dist
    rank = dist.get_rank(group)
    world = dist.get_world_size(group)

    def gather(t: torch.Tensor) -> torch.Tensor:
        # [world, *t.shape]: concatenated along dim 0, which every backend takes
        out = torch.empty((world * t.shape[0],) + tuple(t.shape[1:]), dtype=t.dtype,
                          device=t.device)
        dist.all_gather_into_tensor(out, t.contiguous(), group=group)
        return out.view((world,) + tuple(t.shape))

    tk, tv, T = tail(k, v, W)
    lens = [int(x) for x in gather(torch.tensor([T], dtype=torch.int64, device=k.device)).flatten()]
    tails_k, tails_v = gather(tk), gather(tv)
    piece = piece_of(rank, lens, tails_k, tails_v, W)
    dA_all = gather(piece_state(piece, k, v, lam, eta, g, W, C, prefill_fn))
    E_all = gather(torch.tensor([piece.evictions], dtype=torch.int64, device=k.device)).flatten()
    return finish(rank, piece, dA_all, E_all, q, k, v, lam, eta, g, W, C, prefill_fn, fold_fn)
