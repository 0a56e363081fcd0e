"""Python binding of libtc, the Tensor Cache layer for B200 (sm_100a).

This module only marshals arguments: it checks that tensors are contiguous
and of the right dtype, allocates outputs and workspace with PyTorch when the
caller does not pass them, and calls the C-ABI entry points declared in
``include/tc.h`` through ctypes.  Every step of the layer runs in the CUDA
kernels of ``libtc.so``; there is no CPU or PyTorch fallback.  Importing this
package fails if ``libtc.so`` has not been built
(``python sliding_window_attention_tc_b200/build.py``).

The layer ("Tensor Cache: Eviction-conditioned Associative Memory for
Transformers", §3.1-§3.2): per head, exact softmax attention over the last W
keys (L1) plus a d_k x d_v matrix A written only by pairs evicted from the
window, A <- lambda A + eta k v^T, read as m = q A (L2), fused as
y = y_local + sigmoid(g) m.  Within a step the eviction is written before the
read.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtc.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(f"libtc.so not found at {LIB_PATH}; build it with "
                      "`python sliding_window_attention_tc_b200/build.py`")

_lib = ctypes.CDLL(LIB_PATH)

TC_OK = 0
STATUS_NAMES = {0: "TC_OK", 1: "TC_ERR_INVALID_ARG", 2: "TC_ERR_UNSUPPORTED",
                3: "TC_ERR_NO_DEVICE", 4: "TC_ERR_CUDA", 5: "TC_ERR_DEVICE_BOUNDS",
                6: "TC_ERR_DEVICE_TIMEOUT", 7: "TC_ERR_WORKSPACE"}
TC_F32, TC_BF16 = 0, 1
TC_PREFILL_L1_ONLY = 1
TC_PREFILL_STATE_ONLY = 2
TC_PREFILL_DELTA_RULE = 4
TC_PREFILL_CHUNK_MEAN = 8
TC_WRITE_OUTER, TC_WRITE_DELTA = 0, 1
TC_PATH_AUTO, TC_PATH_FUSED, TC_PATH_GENERAL = 0, 1, 2

# Exported C symbols declared in include/tc.h.
EXPORTED = ("tc_prefill_workspace_size", "tc_prefill", "tc_prefill_launch_count", "tc_prefill_host_workspace_size",
            "tc_prefill_host", "tc_decode_step", "tc_decode_step_host_workspace_size",
            "tc_decode_step_host", "tc_get_device_status", "tc_status_string", "tc_version",
            "tc_prefill_no_alloc", "tc_prefill_from_state", "tc_prefill_from_state_workspace_size",
            "tc_state_fold", "tc_decode_step_ragged", "tc_backward", "tc_backward_workspace_size",
            "tc_set_wait_limit_ns", "tc_prefill_varlen", "tc_prefill_varlen_workspace_size",
            "tc_backward_launch_count", "tc_set_prefill_path", "tc_get_prefill_path",
            "tc_prefill_path_for")


class PrefillDesc(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int64), ("H", ctypes.c_int64), ("T", ctypes.c_int64),
                ("dk", ctypes.c_int64), ("dv", ctypes.c_int64), ("W", ctypes.c_int64),
                ("C", ctypes.c_int64), ("dtype", ctypes.c_int), ("flags", ctypes.c_uint32)]


class DecodeStateC(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int64), ("H", ctypes.c_int64), ("dk", ctypes.c_int64),
                ("dv", ctypes.c_int64), ("W", ctypes.c_int64), ("t", ctypes.c_int64),
                ("kv_dtype", ctypes.c_int), ("ring_k", ctypes.c_void_p),
                ("ring_v", ctypes.c_void_p), ("A", ctypes.c_void_p),
                ("lam", ctypes.c_void_p), ("eta", ctypes.c_void_p), ("g", ctypes.c_void_p),
                ("write_rule", ctypes.c_int)]


_vp, _sz, _int = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
_PD = ctypes.POINTER(PrefillDesc)
_DS = ctypes.POINTER(DecodeStateC)
_lib.tc_prefill_workspace_size.argtypes = [_PD]
_lib.tc_prefill_workspace_size.restype = _sz
_lib.tc_prefill.argtypes = [_PD] + [_vp] * 9 + [_sz, _vp]
_lib.tc_prefill.restype = _int
_lib.tc_backward_launch_count.argtypes = [_PD, ctypes.POINTER(_int)]
_lib.tc_backward_launch_count.restype = _int
_lib.tc_prefill_launch_count.argtypes = [_PD]
_lib.tc_prefill_launch_count.restype = _int
_lib.tc_prefill_host_workspace_size.argtypes = [_PD]
_lib.tc_prefill_host_workspace_size.restype = _sz
_lib.tc_prefill_host.argtypes = [_PD] + [_vp] * 9 + [_sz, _vp]
_lib.tc_prefill_host.restype = _int
_lib.tc_prefill_no_alloc.argtypes = [_PD] + [_vp] * 8 + [_vp]
_lib.tc_prefill_no_alloc.restype = _int
_lib.tc_prefill_from_state_workspace_size.argtypes = [_PD, ctypes.c_int64]
_lib.tc_prefill_from_state_workspace_size.restype = _sz
_lib.tc_prefill_from_state.argtypes = [_PD, ctypes.c_int64] + [_vp] * 12 + [_sz, _vp]
_lib.tc_prefill_from_state.restype = _int
_lib.tc_prefill_varlen_workspace_size.argtypes = [_PD]
_lib.tc_prefill_varlen_workspace_size.restype = _sz
_lib.tc_prefill_varlen.argtypes = [_PD, _vp, ctypes.c_int64] + [_vp] * 9 + [_sz, _vp]
_lib.tc_prefill_varlen.restype = _int
_lib.tc_backward_workspace_size.argtypes = [_PD]
_lib.tc_backward_workspace_size.restype = _sz
_lib.tc_backward.argtypes = [_PD] + [_vp] * 14 + [_sz, _vp]
_lib.tc_backward.restype = _int
_lib.tc_state_fold.argtypes = [ctypes.c_int64] * 5 + [_vp] * 4 + [_vp]
_lib.tc_state_fold.restype = _int
_lib.tc_decode_step.argtypes = [_DS] + [_vp] * 4 + [_vp]
_lib.tc_decode_step.restype = _int
_lib.tc_decode_step_ragged.argtypes = [_DS] + [_vp] * 5 + [_vp]
_lib.tc_decode_step_ragged.restype = _int
_lib.tc_decode_step_host_workspace_size.argtypes = [_DS]
_lib.tc_decode_step_host_workspace_size.restype = _sz
_lib.tc_decode_step_host.argtypes = [_DS] + [_vp] * 5 + [_sz, _vp]
_lib.tc_decode_step_host.restype = _int
_lib.tc_get_device_status.argtypes = [_vp]
_lib.tc_get_device_status.restype = _int
_lib.tc_status_string.argtypes = [_int]
_lib.tc_status_string.restype = ctypes.c_char_p
_lib.tc_version.argtypes = []
_lib.tc_version.restype = ctypes.c_char_p
_lib.tc_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
_lib.tc_set_wait_limit_ns.restype = None
_lib.tc_set_prefill_path.argtypes = [_int]
_lib.tc_set_prefill_path.restype = _int
_lib.tc_get_prefill_path.argtypes = []
_lib.tc_get_prefill_path.restype = _int
_lib.tc_prefill_path_for.argtypes = [_PD, ctypes.c_int64]
_lib.tc_prefill_path_for.restype = _int

SIZE_ERROR = ctypes.c_size_t(-1).value


class TCError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = int(status)
        super().__init__(f"{where}: {STATUS_NAMES.get(self.status, self.status)} "
                         f"({status_string(self.status)})")


def status_string(status: int) -> str:
    return _lib.tc_status_string(int(status)).decode()


def version() -> str:
    return _lib.tc_version().decode()


def lib_handle() -> ctypes.CDLL:
    """The loaded libtc (for tests that call the C-ABI directly)."""
    return _lib


def _check(st: int, where: str):
    if st != TC_OK:
        raise TCError(st, where)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return TC_F32
    if t.dtype == torch.bfloat16:
        return TC_BF16
    raise TypeError(f"unsupported dtype {t.dtype}; use float32 or bfloat16")


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _contig(*ts):
    for t in ts:
        if t is not None and not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


def _on_device(current: int, *ts):
    """Every CUDA tensor must live on the current device `current`: the
    kernels run there, and another GPU's buffer would be read over the peer
    link (or fault without peer access).  The library refuses such pointers
    too; checking here gives a clear Python error first."""
    for t in ts:
        if t is not None and t.device.type == "cuda" and t.device.index != current:
            raise ValueError(f"tensor on {t.device} but the current CUDA device is cuda:{current}; "
                             "call under torch.cuda.device(...) of the tensors' device")


def _dev_check(*ts):
    if any(t is not None and t.device.type == "cuda" for t in ts):
        _on_device(torch.cuda.current_device(), *ts)


# The C-ABI sees only addresses, so a tensor of the wrong size or element type
# would have a kernel read or write past its end: shapes and dtypes are
# checked here, before any call.
def _expect(t: Optional[torch.Tensor], name: str, shape, dtype):
    if t is None:
        return
    if t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}; expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}; expected {tuple(shape)}")


def _expect_layer(B, H, T, dk, dv, dt, q, k, v, lam, eta, g, y=None, A_final=None):
    """q, k [B,H,T,dk], v (and y) [B,H,T,dv] in dt; lam, eta, g [H] float32;
    A_final [B,H,dk,dv] float32 (None entries are not checked)."""
    _expect(q, "q", (B, H, T, dk), dt)
    _expect(k, "k", (B, H, T, dk), dt)
    _expect(v, "v", (B, H, T, dv), dt)
    for name, t in (("lam", lam), ("eta", eta), ("g", g)):
        if t is None:
            raise ValueError(f"{name} is required")
        _expect(t, name, (H,), torch.float32)
    _expect(y, "y", (B, H, T, dv), dt)
    _expect(A_final, "A_final", (B, H, dk, dv), torch.float32)


def make_prefill_desc(B, H, T, dk, dv, W, C, dtype: int, l1_only: bool = False,
                      state_only: bool = False, delta_rule: bool = False,
                      chunk_mean: bool = False) -> PrefillDesc:
    flags = ((TC_PREFILL_L1_ONLY if l1_only else 0) | (TC_PREFILL_STATE_ONLY if state_only else 0)
             | (TC_PREFILL_DELTA_RULE if delta_rule else 0)
             | (TC_PREFILL_CHUNK_MEAN if chunk_mean else 0))
    return PrefillDesc(int(B), int(H), int(T), int(dk), int(dv), int(W), int(C), int(dtype),
                       flags)


def prefill_workspace_size(desc: PrefillDesc) -> int:
    n = _lib.tc_prefill_workspace_size(ctypes.byref(desc))
    if n == SIZE_ERROR:
        raise TCError(1, "tc_prefill_workspace_size")
    return int(n)


def _desc_of(q, v, W, C, l1_only, delta_rule=False):
    B, H, T, dk = q.shape
    return make_prefill_desc(B, H, T, dk, v.shape[-1], W, C, _dtype_code(q), l1_only,
                             delta_rule=delta_rule)


def prefill(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, lam: torch.Tensor,
            eta: torch.Tensor, g: torch.Tensor, W: int, C: int, *, l1_only: bool = False,
            delta_rule: bool = False, y: Optional[torch.Tensor] = None,
            A_final: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
            stream=None):
    """tc_prefill on device tensors q, k [B,H,T,dk], v [B,H,T,dv] (float32 or
    bfloat16), lam, eta, g [H] float32.  Returns (y, A_final); A_final is
    None with l1_only.  delta_rule selects the delta-rule write."""
    desc = _desc_of(q, v, W, C, l1_only, delta_rule)
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    _expect_layer(B, H, T, dk, dv, q.dtype, q, k, v, lam, eta, g, y, A_final)
    if y is None:
        y = torch.empty((B, H, T, dv), dtype=q.dtype, device=q.device)
    if A_final is None and not l1_only:
        A_final = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    need = prefill_workspace_size(desc)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    _contig(q, k, v, lam, eta, g, y, A_final, workspace)
    _dev_check(q, k, v, lam, eta, g, y, A_final, workspace)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = _lib.tc_prefill(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(lam), _ptr(eta),
                         _ptr(g), _ptr(y), _ptr(A_final), _ptr(workspace), ws_bytes,
                         _stream(stream))
    _check(st, "tc_prefill")
    return y, A_final


def prefill_varlen(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cu_seqlens: torch.Tensor,
                   max_seqlen: int, lam: torch.Tensor, eta: torch.Tensor, g: torch.Tensor,
                   W: int, C: int, *, l1_only: bool = False, y: Optional[torch.Tensor] = None,
                   A_final: Optional[torch.Tensor] = None,
                   workspace: Optional[torch.Tensor] = None, stream=None):
    """tc_prefill_varlen: len(cu_seqlens) - 1 sequences packed token-major,
    q, k [total,H,dk], v [total,H,dv] bfloat16; sequence b is rows
    cu_seqlens[b] .. cu_seqlens[b+1]-1 (cu_seqlens int64 on the device),
    max_seqlen its longest length.  Each sequence starts from an empty
    state.  Returns (y [total,H,dv], A_final [B,H,dk,dv] float32 or None with
    l1_only)."""
    total, H, dk = k.shape
    dv = v.shape[-1]
    B = cu_seqlens.numel() - 1
    if B < 1:
        raise ValueError("cu_seqlens needs at least two entries")
    _expect(cu_seqlens, "cu_seqlens", (B + 1,), torch.int64)
    _expect(q, "q", (total, H, dk), k.dtype)
    _expect(v, "v", (total, H, dv), k.dtype)
    for name, t in (("lam", lam), ("eta", eta), ("g", g)):
        _expect(t, name, (H,), torch.float32)
    _expect(y, "y", (total, H, dv), k.dtype)
    _expect(A_final, "A_final", (B, H, dk, dv), torch.float32)
    desc = make_prefill_desc(B, H, int(max_seqlen), dk, dv, W, C, _dtype_code(k), l1_only)
    if y is None:
        y = torch.empty((total, H, dv), dtype=k.dtype, device=k.device)
    if A_final is None and not l1_only:
        A_final = torch.empty((B, H, dk, dv), dtype=torch.float32, device=k.device)
    need = _lib.tc_prefill_varlen_workspace_size(ctypes.byref(desc))
    if need == SIZE_ERROR:
        raise TCError(2, "tc_prefill_varlen_workspace_size")
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=k.device)
    _contig(q, k, v, cu_seqlens, lam, eta, g, y, A_final, workspace)
    _dev_check(q, k, v, cu_seqlens, lam, eta, g, y, A_final, workspace)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = _lib.tc_prefill_varlen(ctypes.byref(desc), _ptr(cu_seqlens), int(total), _ptr(q),
                                _ptr(k), _ptr(v), _ptr(lam), _ptr(eta), _ptr(g), _ptr(y),
                                _ptr(A_final), _ptr(workspace), ws_bytes, _stream(stream))
    _check(st, "tc_prefill_varlen")
    return y, A_final


def write_pairs(k: torch.Tensor, v: torch.Tensor, lam: torch.Tensor, eta: torch.Tensor,
                A: Optional[torch.Tensor] = None) -> torch.Tensor:
    """A after writing the pairs k [B,H,n,dk], v [B,H,n,dv] in order into an
    empty state with the layer's write, A <- lam A + eta k v^T per pair:
    tc_prefill_from_state, state only, over the n pairs plus one token with
    W = 1, so that exactly the n pairs are evicted (one chunk of n)."""
    B, H, n, dk = k.shape
    dv = v.shape[-1]
    pad_k = torch.zeros((B, H, 1, dk), dtype=k.dtype, device=k.device)
    pad_v = torch.zeros((B, H, 1, dv), dtype=v.dtype, device=v.device)
    ks = torch.cat([k, pad_k], dim=2).contiguous()
    vs = torch.cat([v, pad_v], dim=2).contiguous()
    g = torch.zeros(H, dtype=torch.float32, device=k.device)
    _, A = prefill_from_state(None, ks, vs, lam, eta, g, 1, max(n, 1), 0, state_only=True,
                              A_final=A)
    return A


def prefill_from_state(q: Optional[torch.Tensor], k: torch.Tensor, v: torch.Tensor,
                       lam: torch.Tensor, eta: torch.Tensor, g: torch.Tensor, W: int, C: int,
                       t0: int, halo_k: Optional[torch.Tensor] = None,
                       halo_v: Optional[torch.Tensor] = None, A_init: Optional[torch.Tensor] = None,
                       *, state_only: bool = False, l1_only: bool = False,
                       delta_rule: bool = False, chunk_mean: bool = False,
                       y: Optional[torch.Tensor] = None,
                       A_final: Optional[torch.Tensor] = None,
                       workspace: Optional[torch.Tensor] = None, stream=None):
    """tc_prefill_from_state: the layer over the new tokens k, v [B,H,T,d]
    (queries q, unless state_only) starting at global position t0, given the
    halo (keys / values of tokens t0 - min(t0, W) .. t0 - 1, oldest first) and
    A_init (A after the evictions before t0; None = zero).  Returns
    (y, A_final); y is None with state_only."""
    B, H, T, dk = k.shape
    dv = v.shape[-1]
    desc = make_prefill_desc(B, H, T, dk, dv, W, C, _dtype_code(k), l1_only, state_only,
                             delta_rule, chunk_mean)
    _expect_layer(B, H, T, dk, dv, k.dtype, q, k, v, lam, eta, g, y, A_final)
    n_halo = min(int(t0), int(W))
    _expect(halo_k, "halo_k", (B, H, n_halo, dk), k.dtype)
    _expect(halo_v, "halo_v", (B, H, n_halo, dv), k.dtype)
    _expect(A_init, "A_init", (B, H, dk, dv), torch.float32)
    if y is None and not state_only:
        y = torch.empty((B, H, T, dv), dtype=k.dtype, device=k.device)
    if A_final is None and not l1_only:
        A_final = torch.empty((B, H, dk, dv), dtype=torch.float32, device=k.device)
    need = _lib.tc_prefill_from_state_workspace_size(ctypes.byref(desc), int(t0))
    if need == SIZE_ERROR:
        raise TCError(1, "tc_prefill_from_state_workspace_size")
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=k.device)
    _contig(q, k, v, lam, eta, g, y, A_final, workspace, halo_k, halo_v, A_init)
    _dev_check(q, k, v, lam, eta, g, y, A_final, workspace, halo_k, halo_v, A_init)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = _lib.tc_prefill_from_state(ctypes.byref(desc), int(t0), _ptr(halo_k), _ptr(halo_v),
                                    _ptr(A_init), _ptr(q), _ptr(k), _ptr(v), _ptr(lam),
                                    _ptr(eta), _ptr(g), _ptr(y), _ptr(A_final), _ptr(workspace),
                                    ws_bytes, _stream(stream))
    _check(st, "tc_prefill_from_state")
    return y, A_final


def state_fold(dA: torch.Tensor, E: torch.Tensor, lam: torch.Tensor,
               A_out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """tc_state_fold: dA [n_parts,B,H,dk,dv] float32, E [n_parts] int64,
    lam [H] float32 (all on the device).  Returns the state before piece
    n_parts."""
    n, B, H, dk, dv = dA.shape
    if A_out is None:
        A_out = torch.empty((B, H, dk, dv), dtype=torch.float32, device=lam.device)
    _contig(dA, E, lam, A_out)
    _dev_check(dA, E, lam, A_out)
    if dA.dtype != torch.float32 or E.dtype != torch.int64:
        raise TypeError("dA must be float32 and E int64")
    _expect(E, "E", (n,), torch.int64)
    _expect(lam, "lam", (H,), torch.float32)
    _expect(A_out, "A_out", (B, H, dk, dv), torch.float32)
    st = _lib.tc_state_fold(B, H, dk, dv, n, _ptr(dA) if n else None, _ptr(E) if n else None,
                            _ptr(lam), _ptr(A_out), _stream(stream))
    _check(st, "tc_state_fold")
    return A_out


def backward(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, lam: torch.Tensor,
             eta: torch.Tensor, g: torch.Tensor, W: int, dy: torch.Tensor, *,
             workspace: Optional[torch.Tensor] = None, stream=None):
    """tc_backward: gradients of L = sum <dy, y> for the layer over q, k, v
    [B,H,T,d] (from an empty state, outer-product write).  Returns
    (dq, dk, dv [float32, input layout], dlam, deta, dg [H] float32)."""
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    desc = make_prefill_desc(B, H, T, dk, dv, W, 1, _dtype_code(q))
    _expect_layer(B, H, T, dk, dv, q.dtype, q, k, v, lam, eta, g)
    _expect(dy, "dy", (B, H, T, dv), q.dtype)
    f = dict(dtype=torch.float32, device=q.device)
    dq, dkk, dvv = torch.empty(B, H, T, dk, **f), torch.empty(B, H, T, dk, **f), torch.empty(B, H, T, dv, **f)
    dl, de, dg_ = torch.empty(H, **f), torch.empty(H, **f), torch.empty(H, **f)
    need = _lib.tc_backward_workspace_size(ctypes.byref(desc))
    if need == SIZE_ERROR:
        raise TCError(1, "tc_backward_workspace_size")
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    _contig(q, k, v, lam, eta, g, dy, workspace)
    _dev_check(q, k, v, lam, eta, g, dy, workspace)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = _lib.tc_backward(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(lam), _ptr(eta),
                          _ptr(g), _ptr(dy), _ptr(dq), _ptr(dkk), _ptr(dvv), _ptr(dl), _ptr(de),
                          _ptr(dg_), _ptr(workspace), ws_bytes, _stream(stream))
    _check(st, "tc_backward")
    return dq, dkk, dvv, dl, de, dg_


def backward_launch_count(q: torch.Tensor, W: int, v: Optional[torch.Tensor] = None):
    """(launches, tensor_cores) of one tc_backward call on tensors shaped like
    q [B,H,T,d_k] (and v [B,H,T,d_v], default q's shape) with window W."""
    B, H, T, dk = q.shape
    dv = dk if v is None else v.shape[-1]
    desc = make_prefill_desc(B, H, T, dk, dv, W, 1, _dtype_code(q))
    tcf = _int(0)
    n = _lib.tc_backward_launch_count(ctypes.byref(desc), ctypes.byref(tcf))
    if n < 0:
        raise TCError(1, "tc_backward_launch_count")
    return int(n), bool(tcf.value)


def prefill_launch_count(desc: PrefillDesc) -> int:
    """Kernel launches one tc_prefill call enqueues for desc."""
    n = _lib.tc_prefill_launch_count(ctypes.byref(desc))
    if n < 0:
        raise TCError(1, "tc_prefill_launch_count")
    return int(n)


_PATHS = {"auto": TC_PATH_AUTO, "fused": TC_PATH_FUSED, "general": TC_PATH_GENERAL}


def set_prefill_path(path) -> None:
    """tc_set_prefill_path: "auto" (default), "fused" or "general" (or the
    TC_PATH_* value), for calls both tensor-core paths can take.  Process-wide."""
    code = _PATHS.get(path, path) if isinstance(path, str) else int(path)
    if not isinstance(code, int):
        raise TCError(1, "tc_set_prefill_path")
    _check(_lib.tc_set_prefill_path(code), "tc_set_prefill_path")


def get_prefill_path() -> str:
    """The current tc_set_prefill_path setting, by name."""
    code = int(_lib.tc_get_prefill_path())
    return {v: k for k, v in _PATHS.items()}[code]


class prefill_path:
    """Context manager: tc_set_prefill_path(path) inside, the previous setting after."""

    def __init__(self, path):
        self.path = path

    def __enter__(self):
        self.prev = get_prefill_path()
        set_prefill_path(self.path)
        return self

    def __exit__(self, *exc):
        set_prefill_path(self.prev)
        return False


def prefill_path_for(desc: PrefillDesc, t0: int = 0):
    """tc_prefill_path_for: "fused" or "general", the tensor-core path a call
    described by desc (continuing at t0) would take now; None when neither takes it."""
    code = int(_lib.tc_prefill_path_for(ctypes.byref(desc), ctypes.c_int64(int(t0))))
    return None if code < 0 else {TC_PATH_FUSED: "fused", TC_PATH_GENERAL: "general"}[code]


NO_ALLOC_SCRATCH_BYTES = 16 << 20


def prefill_no_alloc(q, k, v, lam, eta, g, W, C, *, l1_only=False, y=None, A_final=None,
                     stream=None):
    """tc_prefill_no_alloc: tc_prefill using the library's built-in scratch
    array (no workspace argument) for callers that cannot allocate device
    memory.  y / A_final are allocated here by PyTorch only when not given."""
    desc = _desc_of(q, v, W, C, l1_only)
    B, H, T, dk = q.shape
    dv = v.shape[-1]
    _expect_layer(B, H, T, dk, dv, q.dtype, q, k, v, lam, eta, g, y, A_final)
    if y is None:
        y = torch.empty((B, H, T, dv), dtype=q.dtype, device=q.device)
    if A_final is None and not l1_only:
        A_final = torch.empty((B, H, dk, dv), dtype=torch.float32, device=q.device)
    _contig(q, k, v, lam, eta, g, y, A_final)
    _dev_check(q, k, v, lam, eta, g, y, A_final)
    st = _lib.tc_prefill_no_alloc(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(lam),
                                  _ptr(eta), _ptr(g), _ptr(y), _ptr(A_final), _stream(stream))
    _check(st, "tc_prefill_no_alloc")
    return y, A_final


def prefill_host_workspace_size(desc: PrefillDesc) -> int:
    n = _lib.tc_prefill_host_workspace_size(ctypes.byref(desc))
    if n == SIZE_ERROR:
        raise TCError(1, "tc_prefill_host_workspace_size")
    return int(n)


def prefill_host(q, k, v, lam, eta, g, W, C, y, A_final=None, *, workspace, l1_only=False,
                 stream=None):
    """tc_prefill_host: q, k, v, lam, eta, g, y (and A_final) are HOST tensors
    (pinned for asynchronous copies); workspace is a device byte tensor of
    prefill_host_workspace_size bytes.  Enqueued on stream; synchronize
    before reading y."""
    desc = _desc_of(q, v, W, C, l1_only)
    B, H, T, dk = q.shape
    _expect_layer(B, H, T, dk, v.shape[-1], q.dtype, q, k, v, lam, eta, g, y, A_final)
    if y is None:
        raise ValueError("y (a host tensor) is required")
    _contig(q, k, v, lam, eta, g, y, A_final, workspace)
    _dev_check(workspace)
    st = _lib.tc_prefill_host(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(lam),
                              _ptr(eta), _ptr(g), _ptr(y), _ptr(A_final), _ptr(workspace),
                              workspace.numel() * workspace.element_size(), _stream(stream))
    _check(st, "tc_prefill_host")
    return y, A_final


@dataclass
class DecodeState:
    """Streaming state (caller-owned device tensors, updated in place):
    ring_k [B,H,W,dk], ring_v [B,H,W,dv], A [B,H,dk,dv] float32, lam/eta/g
    [H] float32, the clock t (tokens consumed so far) and the write rule
    (TC_WRITE_OUTER, the paper's layer, or TC_WRITE_DELTA)."""
    ring_k: torch.Tensor
    ring_v: torch.Tensor
    A: torch.Tensor
    lam: torch.Tensor
    eta: torch.Tensor
    g: torch.Tensor
    t: int
    write_rule: int = 0

    def c_struct(self) -> DecodeStateC:
        B, H, W, dk = self.ring_k.shape
        dv = self.ring_v.shape[-1]
        _dtype_code(self.ring_k)
        _expect(self.ring_v, "ring_v", (B, H, W, dv), self.ring_k.dtype)
        _expect(self.A, "A", (B, H, dk, dv), torch.float32)
        for name, t in (("lam", self.lam), ("eta", self.eta), ("g", self.g)):
            _expect(t, name, (H,), torch.float32)
        _contig(self.ring_k, self.ring_v, self.A, self.lam, self.eta, self.g)
        _dev_check(self.ring_k, self.ring_v, self.A, self.lam, self.eta, self.g)
        return DecodeStateC(B, H, dk, dv, W, int(self.t), _dtype_code(self.ring_k),
                            self.ring_k.data_ptr(), self.ring_v.data_ptr(), self.A.data_ptr(),
                            self.lam.data_ptr(), self.eta.data_ptr(), self.g.data_ptr(),
                            int(self.write_rule))

    @staticmethod
    def empty(B, H, W, dk, dv, lam, eta, g, dtype=torch.bfloat16, device="cuda"):
        return DecodeState(torch.zeros((B, H, W, dk), dtype=dtype, device=device),
                           torch.zeros((B, H, W, dv), dtype=dtype, device=device),
                           torch.zeros((B, H, dk, dv), dtype=torch.float32, device=device),
                           lam, eta, g, 0)


def _expect_step(state: DecodeState, q, k, v, y):
    """q, k [B,H,dk], v and y [B,H,dv] in the ring's dtype."""
    B, H, _, dk = state.ring_k.shape
    dv = state.ring_v.shape[-1]
    dt = state.ring_k.dtype
    _expect(q, "q", (B, H, dk), dt)
    _expect(k, "k", (B, H, dk), dt)
    _expect(v, "v", (B, H, dv), dt)
    _expect(y, "y", (B, H, dv), dt)


def decode_step(state: DecodeState, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                y: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """tc_decode_step: q, k [B,H,dk], v [B,H,dv] device tensors in the ring's
    dtype.  Updates the ring and A in place, advances state.t, returns y."""
    cs = state.c_struct()
    _expect_step(state, q, k, v, y)
    if y is None:
        y = torch.empty(v.shape, dtype=v.dtype, device=v.device)
    _contig(q, k, v, y)
    _dev_check(q, k, v, y)
    st = _lib.tc_decode_step(ctypes.byref(cs), _ptr(q), _ptr(k), _ptr(v), _ptr(y),
                             _stream(stream))
    _check(st, "tc_decode_step")
    state.t = int(cs.t)
    return y


def decode_step_ragged(state: DecodeState, t_rows: torch.Tensor, q: torch.Tensor,
                       k: torch.Tensor, v: torch.Tensor, y: Optional[torch.Tensor] = None,
                       stream=None) -> torch.Tensor:
    """tc_decode_step_ragged: one step for every batch row b at its own clock
    t_rows[b] (device int64 [B]; negative = empty row, left untouched).  The
    library advances the non-negative clocks on the device; state.t is not
    used."""
    cs = state.c_struct()
    _expect_step(state, q, k, v, y)
    _expect(t_rows, "t_rows", (state.ring_k.shape[0],), torch.int64)
    if y is None:
        y = torch.empty(v.shape, dtype=v.dtype, device=v.device)
    _contig(q, k, v, y, t_rows)
    _dev_check(q, k, v, y, t_rows)
    st = _lib.tc_decode_step_ragged(ctypes.byref(cs), _ptr(t_rows), _ptr(q), _ptr(k), _ptr(v),
                                    _ptr(y), _stream(stream))
    _check(st, "tc_decode_step_ragged")
    return y


def decode_step_host_workspace_size(state: DecodeState) -> int:
    cs = state.c_struct()
    n = _lib.tc_decode_step_host_workspace_size(ctypes.byref(cs))
    if n == SIZE_ERROR:
        raise TCError(1, "tc_decode_step_host_workspace_size")
    return int(n)


def decode_step_host(state: DecodeState, q, k, v, y, *, workspace, stream=None):
    """tc_decode_step_host: q, k, v, y are HOST tensors (pinned); the state
    stays on the device.  Enqueued on stream; synchronize before reading y."""
    cs = state.c_struct()
    _expect_step(state, q, k, v, y)
    _contig(q, k, v, y, workspace)
    _dev_check(workspace)
    st = _lib.tc_decode_step_host(ctypes.byref(cs), _ptr(q), _ptr(k), _ptr(v), _ptr(y),
                                  _ptr(workspace), workspace.numel() * workspace.element_size(),
                                  _stream(stream))
    _check(st, "tc_decode_step_host")
    state.t = int(cs.t)
    return y


def set_wait_limit_ns(ns: int) -> None:
    """tc_set_wait_limit_ns: limit of the tensor-core kernels' bounded waits
    (0 restores the 2 s default).  Process-wide; meant for tests of the
    timeout path."""
    _lib.tc_set_wait_limit_ns(int(ns))


def device_status(stream=None) -> int:
    """tc_get_device_status: synchronizes stream, returns and clears the
    device status word."""
    return int(_lib.tc_get_device_status(_stream(stream)))
