"""Seeded synthetic inputs for the Tensor Cache layer.

This module only draws random numbers in the shapes and distributions of the
workloads described for "Tensor Cache: Eviction-conditioned Associative Memory
for Transformers" (arXiv 2605.22884): the associative-recall task (planted
key/value pairs re-issued as noisy queries), LM-shaped prefill, a long-context
run at 32x a 1024-token training length, and batched streaming decode.  It
holds none of the layer's arithmetic, so both the CUDA path and the CPU oracle
can take their inputs from it.  The pages use OpenWebText, Shakespeare and
trained weights; none of that is here, and these seeded tensors stand in for
them with the same shapes.

Prefill inputs (q, k, v, lam, eta, g) are drawn on the CPU with
``torch.Generator`` so every machine gets identical values.  The batched
decode workload is 9 GB and is drawn on the GPU with a seeded CUDA generator;
callers copy sampled heads to the host for checking.
"""
from __future__ import annotations

import math
from typing import Optional
from dataclasses import dataclass, field

import torch

# Name -> shape and parameter recipe.  seed = 1000 + position in this list.
PREFILL_CONFIGS = {
    # tiny case the oracle finishes in well under a second
    "tiny_fp32": dict(B=1, H=1, T=256, dk=16, dv=16, W=32, C=16, dtype="f32", seed=1001),
    # associative-recall shaped, fp32
    "recall_fp32": dict(B=8, H=4, T=2048, dk=64, dv=64, W=256, C=64, dtype="f32", seed=1002),
    # LM-shaped prefill, bf16 inputs, fp32 state
    "lm_prefill_bf16": dict(B=8, H=12, T=4096, dk=64, dv=64, W=512, C=64, dtype="bf16", seed=1003),
    # long-context prefill at 32 x 1024 tokens, bf16 inputs, fp32 state
    "long_prefill_bf16": dict(B=1, H=16, T=32768, dk=64, dv=64, W=1024, C=128, dtype="bf16",
                              seed=1004),
}
# variable-length prefill: the LM workload's 32768 tokens per head cut into
# 15 sequences of mixed lengths (shorter than W, ragged, and much longer)
VARLEN_CONFIG = dict(lengths=[8192, 6000, 4096, 3000, 2500, 2048, 1777, 1500, 1200, 1000, 700,
                              400, 200, 100, 55],
                     H=12, dk=64, dv=64, W=512, C=64, dtype="bf16", seed=1006)
DECODE_CONFIG = dict(B=256, H=32, dk=128, dv=128, W=2048, steps=512, history=10240,
                     prewarm_evictions=8192, dtype="bf16", seed=1005)

_TDTYPE = {"f32": torch.float32, "bf16": torch.bfloat16}


def torch_dtype(name: str) -> torch.dtype:
    return _TDTYPE[name]


@dataclass
class PrefillInputs:
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    lam: torch.Tensor  # [H] float32
    eta: torch.Tensor  # [H] float32
    g: torch.Tensor  # [H] float32
    W: int
    C: int
    meta: dict = field(default_factory=dict)


def _gen(seed: int) -> torch.Generator:
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    return gen


def _uniform(gen, n, lo, hi):
    return lo + (hi - lo) * torch.rand(n, generator=gen, dtype=torch.float64)


def prefill_config(name: str) -> PrefillInputs:
    """Inputs of one named prefill workload (CPU tensors)."""
    cfg = PREFILL_CONFIGS[name]
    B, H, T, dk, dv = cfg["B"], cfg["H"], cfg["T"], cfg["dk"], cfg["dv"]
    gen = _gen(cfg["seed"])
    dt = _TDTYPE[cfg["dtype"]]
    meta = {"name": name, **cfg}
    if name == "tiny_fp32":
        s = 1.0 / math.sqrt(dk)
        q = torch.randn(B, H, T, dk, generator=gen, dtype=torch.float64) * s
        k = torch.randn(B, H, T, dk, generator=gen, dtype=torch.float64) * s
        v = torch.randn(B, H, T, dv, generator=gen, dtype=torch.float64) * s
        lam = torch.full((H,), 0.95, dtype=torch.float64)
        eta = torch.full((H,), 0.5, dtype=torch.float64)
        g = torch.zeros(H, dtype=torch.float64)
    elif name == "recall_fp32":
        q, k, v, plant = _recall_qkv(gen, B, H, T, dk, dv)
        meta["plant"] = plant
        lam = _uniform(gen, H, 0.97, 0.999)
        eta = _uniform(gen, H, 0.1, 1.0)
        g = torch.randn(H, generator=gen, dtype=torch.float64)
    elif name == "lm_prefill_bf16":
        def rms_normed(d):
            x = torch.randn(B, H, T, d, generator=gen, dtype=torch.float64)
            return x / torch.sqrt(torch.mean(x * x, dim=-1, keepdim=True))
        q, k, v = rms_normed(dk), rms_normed(dk), rms_normed(dv)
        lam = torch.sigmoid(_uniform(gen, H, 3.0, 7.0))
        eta = torch.nn.functional.softplus(torch.randn(H, generator=gen, dtype=torch.float64))
        g = torch.randn(H, generator=gen, dtype=torch.float64)
    elif name == "long_prefill_bf16":
        q = torch.randn(B, H, T, dk, generator=gen, dtype=torch.float64) / 8
        k = torch.randn(B, H, T, dk, generator=gen, dtype=torch.float64) / 8
        v = torch.randn(B, H, T, dv, generator=gen, dtype=torch.float64) / 8
        lam = _uniform(gen, H, 0.99, 0.9999)
        eta = _uniform(gen, H, 0.05, 0.5)
        g = torch.randn(H, generator=gen, dtype=torch.float64)
    else:  # pragma: no cover
        raise KeyError(name)
    return PrefillInputs(q.to(dt).contiguous(), k.to(dt).contiguous(), v.to(dt).contiguous(),
                         lam.float(), eta.float(), g.float(), cfg["W"], cfg["C"], meta)


def _recall_qkv(gen, B, H, T, dk, dv, n_pairs=64, spacing=8, query_start=1800, noise=0.05):
    """Associative-recall layout: pair p sits at position spacing*p with a
    unit-norm Gaussian key and an N(0,1)/8 value; the queries at positions
    query_start + j re-issue key (j mod n_pairs) plus N(0, noise^2) noise.
    Everything else is N(0,1)/8 (norm close to 1 at d = 64)."""
    q = torch.randn(B, H, T, dk, generator=gen, dtype=torch.float64) / 8
    k = torch.randn(B, H, T, dk, generator=gen, dtype=torch.float64) / 8
    v = torch.randn(B, H, T, dv, generator=gen, dtype=torch.float64) / 8
    pk = torch.randn(B, H, n_pairs, dk, generator=gen, dtype=torch.float64)
    pk = pk / torch.linalg.vector_norm(pk, dim=-1, keepdim=True)
    pv = torch.randn(B, H, n_pairs, dv, generator=gen, dtype=torch.float64) / 8
    pos = torch.arange(n_pairs) * spacing
    k[:, :, pos] = pk
    v[:, :, pos] = pv
    qpos = torch.arange(query_start, T)
    which = (qpos - query_start) % n_pairs
    q[:, :, qpos] = pk[:, :, which] + noise * torch.randn(B, H, len(qpos), dk, generator=gen,
                                                         dtype=torch.float64)
    return q, k, v, {"positions": pos.tolist(), "query_start": query_start, "n_pairs": n_pairs}


def random_prefill(B, H, T, dk, dv, W, C, *, dtype="f32", seed=0, scale=None,
                   lam_range=(0.9, 0.999), eta_range=(0.1, 1.0)) -> PrefillInputs:
    """Generic seeded prefill inputs for parity cases at arbitrary shapes."""
    gen = _gen(seed)
    s = scale if scale is not None else 1.0 / math.sqrt(dk)
    q = torch.randn(B, H, T, dk, generator=gen, dtype=torch.float64) * s
    k = torch.randn(B, H, T, dk, generator=gen, dtype=torch.float64) * s
    v = torch.randn(B, H, T, dv, generator=gen, dtype=torch.float64) * s
    lam = _uniform(gen, H, *lam_range)
    eta = _uniform(gen, H, *eta_range)
    g = torch.randn(H, generator=gen, dtype=torch.float64)
    dt = _TDTYPE[dtype]
    return PrefillInputs(q.to(dt).contiguous(), k.to(dt).contiguous(), v.to(dt).contiguous(),
                         lam.float(), eta.float(), g.float(), W, C,
                         {"name": "random", "seed": seed, "dtype": dtype})


@dataclass
class VarlenInputs:
    q: torch.Tensor  # [total, H, dk], sequences packed token-major
    k: torch.Tensor
    v: torch.Tensor  # [total, H, dv]
    cu_seqlens: torch.Tensor  # int64 [n_seq + 1]
    lam: torch.Tensor  # [H] float32, shared by every sequence
    eta: torch.Tensor
    g: torch.Tensor
    W: int
    C: int

    @property
    def max_seqlen(self) -> int:
        return int((self.cu_seqlens[1:] - self.cu_seqlens[:-1]).max()) if len(self.cu_seqlens) > 1 else 0

    def sequence(self, b: int):
        """q, k, v of sequence b as [1, H, T_b, d] (the fixed-length layout)."""
        a, e = int(self.cu_seqlens[b]), int(self.cu_seqlens[b + 1])
        return tuple(t[a:e].permute(1, 0, 2).unsqueeze(0).contiguous()
                     for t in (self.q, self.k, self.v))


def random_varlen(lengths, H, dk, dv, W, C, *, dtype="bf16", seed=0, scale=None,
                  lam_range=(0.9, 0.999), eta_range=(0.1, 1.0)) -> VarlenInputs:
    """Seeded packed inputs: sequences of the given lengths, one after the
    other along the token axis, with the same per-head parameters."""
    gen = _gen(seed)
    s = scale if scale is not None else 1.0 / math.sqrt(dk)
    total = int(sum(lengths))
    q = torch.randn(total, H, dk, generator=gen, dtype=torch.float64) * s
    k = torch.randn(total, H, dk, generator=gen, dtype=torch.float64) * s
    v = torch.randn(total, H, dv, generator=gen, dtype=torch.float64) * s
    lam = _uniform(gen, H, *lam_range)
    eta = _uniform(gen, H, *eta_range)
    g = torch.randn(H, generator=gen, dtype=torch.float64)
    cu = torch.zeros(len(lengths) + 1, dtype=torch.int64)
    cu[1:] = torch.cumsum(torch.tensor(lengths, dtype=torch.int64), 0)
    dt = _TDTYPE[dtype]
    return VarlenInputs(q.to(dt).contiguous(), k.to(dt).contiguous(), v.to(dt).contiguous(), cu,
                        lam.float(), eta.float(), g.float(), W, C)


def varlen_config() -> "VarlenInputs":
    """Inputs of the variable-length prefill workload (CPU tensors)."""
    c = VARLEN_CONFIG
    return random_varlen(c["lengths"], c["H"], c["dk"], c["dv"], c["W"], c["C"],
                         dtype=c["dtype"], seed=c["seed"])


@dataclass
class DecodeInputs:
    ring_k: torch.Tensor  # [B,H,W,dk]
    ring_v: torch.Tensor  # [B,H,W,dv]
    A: Optional[torch.Tensor]  # [B,H,dk,dv] float32, or None: build it from prewarm_pairs
    q: torch.Tensor  # [steps,B,H,dk]
    k: torch.Tensor  # [steps,B,H,dk]
    v: torch.Tensor  # [steps,B,H,dv]
    lam: torch.Tensor
    eta: torch.Tensor
    g: torch.Tensor
    t0: int
    W: int
    n_prewarm: int = 0  # evicted pairs before the ring (decode_prewarm_pairs)
    seed: int = 0


def decode_prewarm_pairs(x: "DecodeInputs", b0: int, b1: int):
    """The n_prewarm (key, value) pairs evicted before the ring's tokens, for
    batch rows b0 .. b1-1: k [b1-b0, H, n, dk], v [b1-b0, H, n, dv] in the
    ring's dtype, pair e being token e (tokens n .. n+W-1 fill the ring).
    Drawn like the stream, N(0,1)/sqrt(d), from a generator seeded per batch
    row, so any subset of rows can be drawn again."""
    B, H, W, dk = x.ring_k.shape
    dv = x.ring_v.shape[-1]
    n = x.n_prewarm
    dev = x.ring_k.device
    gen = torch.Generator(device=dev)
    ks, vs = [], []
    for b in range(b0, b1):
        gen.manual_seed(x.seed * 1000003 + 17 + b)
        ks.append(torch.randn((H, n, dk), generator=gen, device=dev).mul_(1.0 / math.sqrt(dk)))
        vs.append(torch.randn((H, n, dv), generator=gen, device=dev).mul_(1.0 / math.sqrt(dv)))
    dt = x.ring_k.dtype
    return torch.stack(ks).to(dt), torch.stack(vs).to(dt)


def decode_workload(*, B=None, H=None, dk=None, dv=None, W=None, steps=None, history=None,
                    prewarm_evictions=None, dtype=None, seed=None, device="cuda") -> DecodeInputs:
    """Batched-decode workload: a full ring (tokens history-W..history-1 at
    slot t mod W) and ``steps`` fresh (q, k, v) per head.  A is left None:
    it is the state the ``prewarm_evictions`` pairs before the ring leave
    (decode_prewarm_pairs draws them; the caller writes them into A).
    Defaults are the full 256 x 32 head, d = 128, W = 2048, 512-step
    workload, with 8192 evicted pairs (history = 8192 + W)."""
    c = dict(DECODE_CONFIG)
    for key, val in dict(B=B, H=H, dk=dk, dv=dv, W=W, steps=steps, history=history,
                         prewarm_evictions=prewarm_evictions, dtype=dtype, seed=seed).items():
        if val is not None:
            c[key] = val
    B, H, dk, dv, W, n = c["B"], c["H"], c["dk"], c["dv"], c["W"], c["steps"]
    dt = _TDTYPE[c["dtype"]]
    dev = torch.device(device)
    cpu_gen = _gen(c["seed"])
    lam = _uniform(cpu_gen, H, 0.99, 0.9999)
    eta = _uniform(cpu_gen, H, 0.1, 1.0)
    g = torch.randn(H, generator=cpu_gen, dtype=torch.float64)
    gen = torch.Generator(device=dev)
    gen.manual_seed(c["seed"])
    sk, sv = 1.0 / math.sqrt(dk), 1.0 / math.sqrt(dv)

    def draw(shape, s):
        x = torch.randn(shape, generator=gen, device=dev, dtype=torch.float32)
        return x.mul_(s).to(dt)

    ring_k = draw((B, H, W, dk), sk)
    ring_v = draw((B, H, W, dv), sv)
    q = draw((n, B, H, dk), sk)
    k = draw((n, B, H, dk), sk)
    v = draw((n, B, H, dv), sv)
    return DecodeInputs(ring_k, ring_v, None, q, k, v, lam.float().to(dev), eta.float().to(dev),
                        g.float().to(dev), int(c["history"]), W, int(c["prewarm_evictions"]),
                        int(c["seed"]))
