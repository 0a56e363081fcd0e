"""CPU oracle for the Tensor Cache layer -- test infrastructure only.

The oracle is the plain float64 definition of the layer from "Tensor Cache:
Eviction-conditioned Associative Memory for Transformers" (arXiv 2605.22884),
computed token by token over a ring buffer and the memory matrix A (§3.1
eq. (1), §3.2 Fig. 2).  The arithmetic lives in ``tc_oracle.c``; this module
only builds it with gcc, converts arrays to contiguous float64 and calls it.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library never uses it, and it
imports nothing from the CUDA library.

Every function here is pinned by ``tests/test_oracle_pins.py`` against
closed forms, library routines (float64 scaled-dot-product attention), brute
force on tiny inputs and the hand-worked fixtures in ``tests/golden/``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "tc_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

_lib = None


def build(force: bool = False) -> str:
    """Compile ``tc_oracle.c`` into ``liboracle.so`` (gcc, OpenMP, no FMA
    contraction so the float32 scans round every operation)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
               "-shared", "-fPIC", "-o", _LIB + ".tmp", _SRC, "-lm"]
        subprocess.check_call(cmd)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        i64, dp, c_int, c_double = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int, ctypes.c_double
        lib.oracle_prefill_rule.argtypes = [i64] * 6 + [dp] * 10 + [c_int, c_int]
        lib.oracle_prefill_rule.restype = c_int
        lib.oracle_decode_rule.argtypes = [i64] * 7 + [dp] * 10 + [c_int, c_int]
        lib.oracle_decode_rule.restype = c_int
        lib.oracle_scan_tokens.argtypes = [i64, i64, i64, dp, dp, c_double, c_double, c_int, dp]
        lib.oracle_scan_chunks.argtypes = [i64, i64, i64, i64, dp, dp, c_double, c_double, c_int, dp]
        lib.oracle_scan_chunk_mean.argtypes = [i64, i64, i64, i64, dp, dp, c_double, c_double, dp]
        lib.oracle_backward.argtypes = [i64] * 6 + [dp] * 13 + [c_int]
        lib.oracle_backward.restype = c_int
        lib.oracle_max_threads.argtypes = [c_int]
        lib.oracle_max_threads.restype = c_int
        _lib = lib
    return _lib


def _f64(x) -> np.ndarray:
    """Exact widening of the caller's values (fp32 or bf16) to float64."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().to("cpu", torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _p(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def threads(nthreads: int = 0) -> int:
    """Number of OpenMP threads the oracle runs with (0 = runtime default)."""
    return int(_load().oracle_max_threads(int(nthreads)))


# Write rules of Fig. 2 step (3): the outer product (the layer as the paper
# trains it) or the optional delta rule (update = k (x) (v - k^T A)).
RULES = {"outer": 0, "delta": 1}


def prefill(q, k, v, lam, eta, g, W: int, *, parts: bool = False, nthreads: int = 0,
            rule: str = "outer"):
    """Token-by-token prefill from an empty state.

    q, k: [B,H,T,dk]; v: [B,H,T,dv]; lam, eta, g: [H].  Returns
    ``(y [B,H,T,dv], A_final [B,H,dk,dv])`` in float64, plus
    ``(y_local, m)`` when ``parts`` is set (y = y_local + sigmoid(g) m).
    ``rule`` selects the write of step (3): "outer" or "delta".
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    lam, eta, g = _f64(lam), _f64(eta), _f64(g)
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    assert k.shape == (B, H, T, dk) and v.shape == (B, H, T, dv)
    assert lam.shape == (H,) and eta.shape == (H,) and g.shape == (H,)
    y = np.empty((B, H, T, dv))
    A = np.empty((B, H, dk, dv))
    yl = np.empty_like(y) if parts else None
    m = np.empty_like(y) if parts else None
    rc = _load().oracle_prefill_rule(B, H, T, dk, dv, int(W), _p(q), _p(k), _p(v), _p(lam),
                                     _p(eta), _p(g), _p(y), _p(A), _p(yl) if parts else None,
                                     _p(m) if parts else None, RULES[rule], int(nthreads))
    if rc != 0:
        raise RuntimeError("oracle_prefill failed")
    return (y, A, yl, m) if parts else (y, A)


def decode(ring_k, ring_v, A, t0: int, q, k, v, lam, eta, g, *, nthreads: int = 0,
           rule: str = "outer"):
    """``nsteps`` streaming steps from the state (ring_k [B,H,W,dk],
    ring_v [B,H,W,dv], A [B,H,dk,dv], clock t0).  q, k: [nsteps,B,H,dk];
    v: [nsteps,B,H,dv].  Returns ``(y [nsteps,B,H,dv], ring_k, ring_v, A)``
    with the state after the last step (the inputs are not modified)."""
    ring_k, ring_v, A = _f64(ring_k).copy(), _f64(ring_v).copy(), _f64(A).copy()
    q, k, v = _f64(q), _f64(k), _f64(v)
    lam, eta, g = _f64(lam), _f64(eta), _f64(g)
    B, H, W, dk = ring_k.shape
    dv = ring_v.shape[-1]
    n = q.shape[0]
    assert q.shape == (n, B, H, dk) and k.shape == (n, B, H, dk) and v.shape == (n, B, H, dv)
    assert A.shape == (B, H, dk, dv)
    y = np.empty((n, B, H, dv))
    rc = _load().oracle_decode_rule(B, H, dk, dv, W, int(t0), n, _p(ring_k), _p(ring_v), _p(A),
                                    _p(q), _p(k), _p(v), _p(lam), _p(eta), _p(g), _p(y),
                                    RULES[rule], int(nthreads))
    if rc != 0:
        raise RuntimeError("oracle_decode failed")
    return y, ring_k, ring_v, A


def scan_tokens(k, v, lam: float, eta: float, *, fp32: bool = False) -> np.ndarray:
    """A after per-token writes of the pairs k [E,dk], v [E,dv] from A = 0."""
    k, v = _f64(k), _f64(v)
    E, dk = k.shape
    dv = v.shape[1]
    A = np.empty((dk, dv))
    _load().oracle_scan_tokens(E, dk, dv, _p(k), _p(v), float(lam), float(eta), int(fp32), _p(A))
    return A


def scan_chunks(k, v, lam: float, eta: float, C: int, *, fp32: bool = False) -> np.ndarray:
    """A after the weighted-sum chunk scan with chunk length C."""
    k, v = _f64(k), _f64(v)
    E, dk = k.shape
    dv = v.shape[1]
    A = np.empty((dk, dv))
    _load().oracle_scan_chunks(E, int(C), dk, dv, _p(k), _p(v), float(lam), float(eta),
                               int(fp32), _p(A))
    return A


def scan_chunk_mean(k, v, lam: float, eta: float, C: int) -> np.ndarray:
    """A after the chunk-mean shortcut A <- lam*A + eta*(kbar (x) vbar)."""
    k, v = _f64(k), _f64(v)
    E, dk = k.shape
    dv = v.shape[1]
    A = np.empty((dk, dv))
    _load().oracle_scan_chunk_mean(E, int(C), dk, dv, _p(k), _p(v), float(lam), float(eta), _p(A))
    return A


def backward(q, k, v, lam, eta, g, W: int, dy, *, nthreads: int = 0):
    """Gradients of L = sum_t <dy_t, y_t> for the layer from an empty state
    (outer-product write): returns (dq, dk, dv [B,H,T,d], dlam, deta, dg [H])
    in float64.  Reverse-mode through the token loop; small inputs only (it
    keeps every state A_t)."""
    q, k, v, dy = _f64(q), _f64(k), _f64(v), _f64(dy)
    lam, eta, g = _f64(lam), _f64(eta), _f64(g)
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    dq, dkk, dvv = np.empty_like(q), np.empty_like(k), np.empty_like(v)
    dl, de, dg_ = np.empty(H), np.empty(H), np.empty(H)
    rc = _load().oracle_backward(B, H, T, dk, dv, int(W), _p(q), _p(k), _p(v), _p(lam), _p(eta),
                                 _p(g), _p(dy), _p(dq), _p(dkk), _p(dvv), _p(dl), _p(de), _p(dg_),
                                 int(nthreads))
    if rc != 0:
        raise RuntimeError("oracle_backward failed")
    return dq, dkk, dvv, dl, de, dg_
