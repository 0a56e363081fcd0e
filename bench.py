"""Benchmark of the Tensor Cache layer (libtc) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl tc|reference]

One step = one pass of the whole prefill hot path (L1 window softmax, L2
eviction chunk scan and memory read, gated fusion) over the LM-shaped prefill
workload: B=8, H=12, T=4096, d=64, W=512, C=64, bf16 inputs, float32 state.
The headline metric is prefill tokens/s (B*H*T per second) per GPU summed
over GPUs.  The same JSON line also carries the streaming-decode workload
(256 x 32 heads, d=128, W=2048, 512 consecutive decode steps), the
long-context prefill (1 x 16 x 32768, W=1024, C=128), the L1-only runs that
give the cost of the L2 path, the roofline of the dominant kernel, the
end-to-end number through the host-buffer entry point and the CPU oracle
timed on a bounded sample.

Multi-GPU: heads and batches are independent, so every rank runs its own
copy of the workload with no collective on the data path (weak scaling);
the timed region is bracketed by barriers and the max over ranks is taken.

--impl reference runs the CPU oracle (the float64 token-by-token definition)
on the host cores on a bounded sample of the same workload and prints the
same JSON line with "impl": "reference".
"""
from __future__ import annotations

import argparse
import ctypes
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as wl  # noqa: E402

HEADLINE = "lm_prefill_bf16"

# DRAM bytes (read + write) per launch from one ncu capture of the current
# kernels; they must be re-measured (or set to None) whenever a kernel changes.
#   prefill_main_kernel: one LM launch, 159.2 MB read + 31.9 MB written
#     (profiles/prefill_main_kernel_lm_prefill_bf16.md)
#   gen_window_kernel: one LM launch (W = 512), 195.1 MB read + 35.3 MB written
#     (profiles/gen_window_kernel_lm_prefill_bf16.md)
#   decode_kernel: the B = 32 capture scaled by heads to the 256 x 32 launch,
#     (1.1417 + 0.0172) GB x 8 (profiles/decode_kernel_b32_w2048_d128.md)
NCU_TRAFFIC_BYTES = {"prefill_main_kernel": 1.911e8, "gen_window_kernel": 2.304e8, "decode_kernel": 9.27e9}
# the kernel that dominates one prefill call on each tensor-core path
PATH_KERNEL = {"fused": "prefill_main_kernel", "general": "gen_window_kernel"}
METRIC = "prefill tokens/s & decode tok/s per B200; % of TC/HBM roofline"
UNIT = "tokens/s"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# ---------------------------------------------------------------------------
def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(PEAKS_FALLBACK), "fallback"


def prefill_flops(B, H, T, dk, dv, W):
    """Algorithmic FLOPs of one prefill: L1 = 2*(dk+dv) per (query, key in
    window); L2 = 2*dk*dv write + 2*dk*dv read per eviction / evicted read."""
    n_pairs = T * W - W * (W - 1) // 2 if T >= W else T * (T + 1) // 2
    E = max(0, T - W)
    l1 = 2 * (dk + dv) * n_pairs * B * H
    l2 = 4 * dk * dv * E * B * H
    return l1, l2


def prefill_executed_flops(B, H, T, W, tile=128, d=64):
    """Tensor-core FLOPs that prefill_main_kernel issues for one call (the
    bf16, d = 64 path): Q K^T and P V on every computed tile x tile block,
    masked parts included, plus the leading tile's P'V, Q S(n0) and hi/lo state
    MMAs for every query tile that has evictions.  (span_summary_kernel adds
    2*tile*d*tile*2 per eviction tile of the spans it summarises.)"""
    nT = (T + tile - 1) // tile
    wt = W // tile
    mma_tile = 2 * tile * tile * d                   # one 128 x 128 x 64 product
    l1 = l2 = 0
    for i in range(nT):
        lead = i >= wt
        nk = wt + 1 if lead else i + 1
        l1 += nk * 2 * mma_tile                      # Q K^T and P V
        if lead:
            l2 += mma_tile + tile * d * d * 2 + mma_tile  # P'V, Q S(n0), [hi; lo] K^T V
    return l1 * B * H, l2 * B * H


def general_executed_flops(B, H, T, W, d=64, l1_only=False):
    """Tensor-core FLOPs the general path issues for one call (bf16, no halo):
    per block of 128 query rows, Q K^T and P V on every 64-key tile from the
    first key it reads to the block's last row (masked parts included), P'V on
    the tiles that hold the block's chunk of evictions and Q A_b (hi + lo)
    after them; per-chunk sums: one 128 x 128 x 128 product pair (hi + lo)
    per CTA (two chunks of d = 64, or one of d = 128)."""
    G, X = 128, 64
    E = max(0, T - W)
    nC = (T + G - 1) // G
    win = mem = 0
    for b in range(nC):
        tau0 = G * b
        a = G * b - W
        e_lo = max(0, a)
        e_hi = max(e_lo, min(E, a + G))
        reads = not l1_only and e_hi > e_lo
        lo = e_lo if reads else max(0, tau0 - W + 1)
        hi = min(T - 1, tau0 + G - 1)
        xs = lo & ~(X - 1)
        n_tiles = (hi - xs) // X + 1
        win += n_tiles * 2 * (2 * G * X * d)
        if reads:
            n_read = sum(1 for n in range(n_tiles) if xs + X * n < e_hi and xs + X * n + X > e_lo)
            mem += n_read * 2 * G * X * d + 2 * (2 * G * d * d)
    if not l1_only and E > 0:
        ctas = (nC + 1) // 2 if d == 64 else nC
        mem += ctas * 2 * (2 * G * G * G)
    return win * B * H, mem * B * H


def decode_bytes(B, H, W, dk, dv, esz=2):
    ring = B * H * W * (dk + dv) * esz
    A = 2 * B * H * dk * dv * 4
    io = B * H * (2 * dk + 2 * dv) * esz + B * H * (dk + dv) * esz  # q,k,v,y + ring write
    return ring + A + io


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.samples = []
        self.windows = []
        self._stop = threading.Event()
        self._thread = None
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self._thread = threading.Thread(target=self._read, daemon=True)
        self._thread.start()

    def _read(self):
        for line in self.proc.stdout:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) >= 9:
                self.samples.append((time.time(), parts))

    def window(self, t0, t1):
        self.windows.append((t0, t1))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        inside = [p for (ts, p) in self.samples if any(a <= ts <= b for a, b in self.windows)]
        use = inside if inside else [p for _, p in self.samples]

        def num(x):
            try:
                return float(x)
            except ValueError:
                return None
        sm = [num(p[1]) for p in use if num(p[1]) is not None]
        mx = [num(p[2]) for p in use if num(p[2]) is not None]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for p in use for i in range(4) if p[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(use), "samples_in_timed_regions": len(inside)}


# ---------------------------------------------------------------------------
def _dist():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def _barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def _max_over_ranks(x: float, world: int, dev) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def timed_region(step, steps: int, world: int, dev) -> float:
    """Run step(i) for i < steps between barriers; return the elapsed time in
    ms, maximised over ranks.  On a CUDA device the time comes from CUDA
    events on the current stream with a synchronize on both sides; on the
    CPU (gloo ranks in tests) from a monotonic clock."""
    cuda = torch.device(dev).type == "cuda"
    if cuda:
        stream = torch.cuda.current_stream()
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        _barrier(world)
        torch.cuda.synchronize()
        start.record(stream)
        for i in range(steps):
            step(i)
        end.record(stream)
        torch.cuda.synchronize()
        _barrier(world)
        ms = start.elapsed_time(end)
    else:
        _barrier(world)
        t0 = time.perf_counter()
        for i in range(steps):
            step(i)
        ms = (time.perf_counter() - t0) * 1e3
        _barrier(world)
    return _max_over_ranks(ms, world, dev)


def _prefill_device_inputs(name, dev, copies):
    x = wl.prefill_config(name)
    sets = []
    for _ in range(copies):
        sets.append(tuple(t.to(dev) for t in (x.q, x.k, x.v)))
    prm = tuple(t.to(dev) for t in (x.lam, x.eta, x.g))
    return x, sets, prm


def time_prefill(tc, name, dev, steps, warmup, world, l1_only=False, clocks=None):
    """Device time of `steps` prefill calls on rotating input sets (so no
    step reads inputs left in L2 by the previous one).  Returns per-step
    event times (ms), the wall of the bracketed region, and launch count."""
    x, sets, prm = _prefill_device_inputs(name, dev, copies=3)
    B, H, T, dk = x.q.shape
    dv = x.v.shape[-1]
    y = [torch.empty(B, H, T, dv, dtype=x.q.dtype, device=dev) for _ in range(2)]
    A = torch.empty(B, H, dk, dv, dtype=torch.float32, device=dev)
    desc = tc.make_prefill_desc(B, H, T, dk, dv, x.W, x.C, tc.TC_BF16 if x.q.dtype ==
                                torch.bfloat16 else tc.TC_F32, l1_only)
    ws_n = tc.prefill_workspace_size(desc)
    ws = torch.empty(max(ws_n, 1), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()

    def step(i):
        q, k, v = sets[i % len(sets)]
        tc.prefill(q, k, v, *prm, x.W, x.C, l1_only=l1_only, y=y[i % 2],
                   A_final=None if l1_only else A, workspace=ws if ws_n else None, stream=stream)

    for i in range(warmup):
        step(i)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    _barrier(world)
    torch.cuda.synchronize()
    t0 = time.time()
    start.record(stream)
    for i in range(steps):
        ev[i][0].record(stream)
        step(i)
        ev[i][1].record(stream)
    end.record(stream)
    torch.cuda.synchronize()
    _barrier(world)
    t1 = time.time()
    if clocks:
        clocks.window(t0, t1)
    per = [a.elapsed_time(b) for a, b in ev]
    total_ms = start.elapsed_time(end)
    launches = tc_launches_per_prefill(tc, desc)
    return {"x": x, "per_step_ms": per, "total_ms": total_ms, "wall_s": t1 - t0,
            "launches_per_step": launches, "tokens_per_step": B * H * T}


def tc_launches_per_prefill(tc, desc):
    """Kernels one tc_prefill call enqueues (from the library's own report)."""
    fn = getattr(tc, "prefill_launch_count", None)
    return fn(desc) if fn else None


def decode_state_from_prewarm(tc, x, rows=16):
    """A of the decode workload: its n_prewarm evicted pairs written through
    libtc (state-only scan), rows batch rows at a time."""
    B, H, _, dk = x.ring_k.shape
    dv = x.ring_v.shape[-1]
    A = torch.empty((B, H, dk, dv), dtype=torch.float32, device=x.ring_k.device)
    for b0 in range(0, B, rows):
        b1 = min(B, b0 + rows)
        k, v = wl.decode_prewarm_pairs(x, b0, b1)
        tc.write_pairs(k, v, x.lam, x.eta, A=A[b0:b1])
        del k, v
    torch.cuda.synchronize()
    return A


def time_decode(tc, dev, world, clocks=None, steps=None, batch=None, e2e=True):
    x = wl.decode_workload(device=dev, B=batch, steps=None if steps is None else steps + 3)
    n = x.q.shape[0] - 3 if steps is not None else x.q.shape[0]
    x.A = decode_state_from_prewarm(tc, x)
    st = tc.DecodeState(x.ring_k, x.ring_v, x.A, x.lam, x.eta, x.g, x.t0)
    B, H, W, dk = x.ring_k.shape
    dv = x.ring_v.shape[-1]
    y = torch.empty(B, H, dv, dtype=x.v.dtype, device=dev)
    stream = torch.cuda.current_stream()
    # warm-up on scratch copies is not possible at 9 GB; warm up with 3 real
    # steps of a separate clock (the state they leave is still a valid state)
    for i in range(3):
        tc.decode_step(st, x.q[i], x.k[i], x.v[i], y=y, stream=stream)
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(n)]
    _barrier(world)
    torch.cuda.synchronize()
    t0 = time.time()
    off = 3 if steps is not None else 0
    for i in range(n):
        ev[i][0].record(stream)
        tc.decode_step(st, x.q[i + off], x.k[i + off], x.v[i + off], y=y, stream=stream)
        ev[i][1].record(stream)
    torch.cuda.synchronize()
    _barrier(world)
    t1 = time.time()
    if clocks:
        clocks.window(t0, t1)
    per = [a.elapsed_time(b) for a, b in ev]
    out = {"B": B, "H": H, "W": W, "d": dk, "steps": n, "per_step_ms": per,
           "bytes_per_step": decode_bytes(B, H, W, dk, dv)}
    if not e2e:
        return out
    # end to end: host q/k/v in, host y out, through tc_decode_step_host
    pin = [tuple(t[i].cpu().pin_memory() for t in (x.q, x.k, x.v)) for i in range(8)]
    yh = torch.empty(B, H, dv, dtype=x.v.dtype).pin_memory()
    ws = torch.empty(tc.decode_step_host_workspace_size(st), dtype=torch.uint8, device=dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ne = 32
    e0.record(stream)
    for i in range(ne):
        q, k, v = pin[i % len(pin)]
        tc.decode_step_host(st, q, k, v, yh, workspace=ws, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize()
    out["e2e_ms_per_step"] = e0.elapsed_time(e1) / ne
    out["e2e_h2d_bytes"] = sum(t.numel() * t.element_size() for t in pin[0])
    out["e2e_d2h_bytes"] = yh.numel() * yh.element_size()
    del x, st
    torch.cuda.empty_cache()
    return out


def time_prefill_e2e(tc, name, dev, steps):
    """Same workload through tc_prefill_host: pinned host q, k, v, lam, eta,
    g in, y and A_final back to pinned host memory, copies inside the timed
    region."""
    x = wl.prefill_config(name)
    B, H, T, dk = x.q.shape
    dv = x.v.shape[-1]
    pin = [t.contiguous().pin_memory() for t in (x.q, x.k, x.v, x.lam, x.eta, x.g)]
    yh = torch.empty(B, H, T, dv, dtype=x.q.dtype).pin_memory()
    Ah = torch.empty(B, H, dk, dv, dtype=torch.float32).pin_memory()
    desc = tc.make_prefill_desc(B, H, T, dk, dv, x.W, x.C, tc.TC_BF16)
    ws = torch.empty(tc.prefill_host_workspace_size(desc), dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream()
    for _ in range(2):
        tc.prefill_host(*pin, x.W, x.C, yh, Ah, workspace=ws, stream=stream)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        tc.prefill_host(*pin, x.W, x.C, yh, Ah, workspace=ws, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    h2d = sum(t.numel() * t.element_size() for t in pin)
    d2h = yh.numel() * yh.element_size() + Ah.numel() * 4
    return {"ms_per_step": ms, "tokens_per_s": B * H * T / (ms * 1e-3), "h2d": h2d, "d2h": d2h}


def state_size_ratio(T, W, d):
    """Per-head decode state of the layer (a W-slot bf16 ring of keys and
    values plus the d x d float32 A) against a full bf16 KV cache of T tokens:
    elements (W*2d + d^2) / (T*2d), and bytes.  Context only: the pages'
    2.4x figure is a whole-model peak-memory measurement."""
    elems = (W * 2 * d + d * d) / (T * 2 * d)
    nbytes = (W * 2 * d * 2 + d * d * 4) / (T * 2 * d * 2)
    return {"T": T, "W": W, "d": d, "elements_ratio": elems, "bytes_ratio": nbytes,
            "full_kv_over_state_bytes": 1.0 / nbytes}


def time_calls(fn, steps, warmup):
    """Per-call device times (ms) of fn() on the current stream, CUDA events."""
    stream = torch.cuda.current_stream()
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for a, b in ev:
        a.record(stream)
        fn()
        b.record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in ev]


def backward_flops(B, H, T, d, W):
    """Algorithmic FLOPs of one backward call: the window part takes five
    products per (query, key in window) pair (scores and dP recomputed, dV,
    dK, dQ) against the forward's two; the memory part twice the forward's
    write + read (the state's and its gradient's scans)."""
    l1, l2 = prefill_flops(B, H, T, d, d, W)
    return 2.5 * l1 + 2 * l2


def time_training_extras(tc, dev, peaks=None, peak_src="fallback", steps=5):
    """The backward pass (tensor-core window and memory parts for bf16, d = 64)
    and the delta-rule prefill (float32 SIMT, token-sequential memory) on the
    LM workload: ms per call and tokens/s."""
    peaks = peaks or dict(PEAKS_FALLBACK)
    x, sets, prm = _prefill_device_inputs(HEADLINE, dev, copies=1)
    q, k, v = sets[0]
    B, H, T, d = q.shape
    gen = torch.Generator(device=dev).manual_seed(7)
    dy = (torch.randn(B, H, T, d, generator=gen, device=dev) / 8).to(q.dtype)
    out = {}
    bwd_ms = statistics.median(time_calls(lambda: tc.backward(q, k, v, *prm, x.W, dy), steps, 3))
    fl = backward_flops(B, H, T, d, x.W)
    tf = fl / (bwd_ms * 1e-3) / 1e12
    peak_tf = float(peaks["bf16_tflops"])
    out["backward"] = {"workload": HEADLINE, "ms": bwd_ms, "tokens_per_s": B * H * T / (bwd_ms * 1e-3),
                       "launches_per_call": tc.backward_launch_count(q, x.W)[0],
                       "tensor_cores": tc.backward_launch_count(q, x.W)[1],
                       "roofline": {"bound": "tensor", "achieved": tf, "peak": peak_tf,
                                    "unit": "TFLOP/s", "frac": tf / peak_tf, "traffic": None,
                                    "peak_source": f"{peak_src} bf16 burst",
                                    "algorithmic_flops_per_call": fl,
                                    "note": "P, dS and the float32 states enter the tensor cores "
                                            "as bf16 hi + lo pairs, so the executed work is "
                                            "about twice the algorithmic"}}
    delta_ms = statistics.median(time_calls(
        lambda: tc.prefill(q, k, v, *prm, x.W, x.C, delta_rule=True), 3, 1))
    out["delta_rule_prefill"] = {"workload": HEADLINE, "ms": delta_ms,
                                 "tokens_per_s": B * H * T / (delta_ms * 1e-3)}
    del dy, sets
    torch.cuda.empty_cache()
    return out


def time_general(tc, dev, steps=10, warmup=3):
    """The general tensor-core prefill (the shapes the fused kernel does not
    take): the LM workload at W = 500 (not a multiple of 128), and d = 128 with
    W = 2048 (the decode workload's head size and window) over 8 x 32 heads
    of 4096 tokens.  Device-resident inputs, CUDA events, ms per call."""
    out = {}
    x, sets, prm = _prefill_device_inputs(HEADLINE, dev, copies=1)
    q, k, v = sets[0]
    B, H, T, d = q.shape
    W = 500
    ms = statistics.median(time_calls(lambda: tc.prefill(q, k, v, *prm, W, x.C), steps, warmup))
    l1f, l2f = prefill_flops(B, H, T, d, d, W)
    desc = tc.make_prefill_desc(B, H, T, d, d, W, x.C, tc.TC_BF16)
    out["lm_w500"] = {"B": B, "H": H, "T": T, "d": d, "W": W, "ms": ms,
                      "tokens_per_s": B * H * T / (ms * 1e-3),
                      "algorithmic_tflops": (l1f + l2f) / (ms * 1e-3) / 1e12,
                      "launches_per_call": tc.prefill_launch_count(desc)}
    del sets, q, k, v
    B, H, T, d, W = 8, 32, 4096, 128, 2048
    gen = torch.Generator(device=dev).manual_seed(1005)
    q, k, v = ((torch.randn(B, H, T, d, generator=gen, device=dev) / math.sqrt(d)).to(torch.bfloat16)
               for _ in range(3))
    lam = 0.99 + 0.0099 * torch.rand(H, generator=gen, device=dev)
    eta = 0.1 + 0.9 * torch.rand(H, generator=gen, device=dev)
    g = torch.randn(H, generator=gen, device=dev)
    ms = statistics.median(time_calls(lambda: tc.prefill(q, k, v, lam, eta, g, W, 128), steps, warmup))
    l1f, l2f = prefill_flops(B, H, T, d, d, W)
    desc = tc.make_prefill_desc(B, H, T, d, d, W, 128, tc.TC_BF16)
    out["d128_w2048"] = {"B": B, "H": H, "T": T, "d": d, "W": W, "ms": ms,
                         "tokens_per_s": B * H * T / (ms * 1e-3),
                         "algorithmic_tflops": (l1f + l2f) / (ms * 1e-3) / 1e12,
                         "launches_per_call": tc.prefill_launch_count(desc)}
    del q, k, v
    torch.cuda.empty_cache()
    return out


def time_varlen(tc, dev, steps=20, warmup=3):
    """The variable-length workload in one tc_prefill_varlen call, against the
    same sequences run as one tc_prefill call each (device-resident inputs,
    CUDA events, ms per whole batch)."""
    x = wl.varlen_config()
    q, k, v, cu = (t.to(dev) for t in (x.q, x.k, x.v, x.cu_seqlens))
    prm = tuple(t.to(dev) for t in (x.lam, x.eta, x.g))
    total, H, d = q.shape
    n = len(x.cu_seqlens) - 1
    y = torch.empty_like(v)
    A = torch.empty(n, H, d, d, dtype=torch.float32, device=dev)
    desc = tc.make_prefill_desc(n, H, x.max_seqlen, d, d, x.W, x.C, tc.TC_BF16)
    ws_n = tc.lib_handle().tc_prefill_varlen_workspace_size(ctypes.byref(desc))
    ws = torch.empty(max(ws_n, 1), dtype=torch.uint8, device=dev)
    one = statistics.median(time_calls(
        lambda: tc.prefill_varlen(q, k, v, cu, x.max_seqlen, *prm, x.W, x.C, y=y, A_final=A,
                                  workspace=ws if ws_n else None), steps, warmup))
    seqs = [tuple(t.to(dev) for t in x.sequence(b)) for b in range(n)]
    outs = [(torch.empty_like(s[2]), torch.empty(1, H, d, d, dtype=torch.float32, device=dev))
            for s in seqs]

    def per_sequence():
        for s, (ys, As) in zip(seqs, outs):
            tc.prefill(*s, *prm, x.W, x.C, y=ys, A_final=As)

    many = statistics.median(time_calls(per_sequence, max(5, steps // 4), warmup))
    tokens = total * H
    return {"workload": "varlen prefill, 15 sequences of 55..8192 tokens (32768 in all), "
                        "H=12, d=64, W=512, bf16",
            "lengths": list(wl.VARLEN_CONFIG["lengths"]), "ms": one, "tokens_per_s": tokens / (one * 1e-3),
            # the fixed-length launches plus the kernel that orders the rows by length
            "launches_per_call": tc.prefill_launch_count(desc) + 1,
            "per_sequence_calls_ms": many,
            "per_sequence_calls_tokens_per_s": tokens / (many * 1e-3)}


# ---------------------------------------------------------------------------
def _rows_per_call(B, H, threads):
    """Batch rows per oracle call: the fewest (at least one item per thread)
    whose B' * H items split evenly over the threads, else the most even."""
    best, best_eff = 1, -1.0
    for r in range(max(1, min(B, -(-threads // H))), B + 1):
        items = r * H
        eff = items / (-(-items // threads) * threads)
        if eff > best_eff + 1e-9:
            best, best_eff = r, eff
        if eff > 0.999:
            break
    return best


def _oracle_rows(x, b0, b1):
    """The oracle over batch rows b0..b1-1 and every head: one call, so that
    its OpenMP loop over (b, h) has (b1 - b0) * H items to share out."""
    import oracle
    oracle.prefill(x.q[b0:b1], x.k[b0:b1], x.v[b0:b1], x.lam, x.eta, x.g, x.W)


def oracle_sample(name, budget_s=12.0):
    """Time the CPU oracle as it stands on a bounded sample of a prefill
    workload: calls over whole batch rows (every head, from t = 0, as the
    layer requires), cycling through the rows until about budget_s seconds
    are spent.  Each call holds at least as many (b, h) items as the oracle
    has threads.  Returns tokens/s, the threads used and the sample."""
    import oracle
    x = wl.prefill_config(name)
    B, H, T = x.q.shape[:3]
    threads = oracle.threads(len(os.sched_getaffinity(0)))  # every core this process may use
    rows = _rows_per_call(B, H, threads)
    used = min(threads, rows * H)
    b0, spent, heads = 0, 0.0, 0
    while spent < budget_s:
        b1 = min(B, b0 + rows)
        t0 = time.perf_counter()
        _oracle_rows(x, b0, b1)
        spent += time.perf_counter() - t0
        heads += (b1 - b0) * H
        b0 = 0 if b1 == B else b1
    return {"value": heads * T / spent, "unit": UNIT, "cores": used, "kind": "oracle",
            "sample": f"{heads} heads x {T} tokens of {name} ({heads / (B * H):.2f} passes over "
                      f"its {B * H} heads; float64 token loop, OpenMP over heads on {used} "
                      f"threads), {spent:.1f} s"}


def run_reference(args):
    world, rank, _ = _dist()
    if world > 1 and rank != 0:
        return 0
    import oracle
    oracle.build()
    x = wl.prefill_config(HEADLINE)
    B, H, T = x.q.shape[:3]
    threads = oracle.threads(len(os.sched_getaffinity(0)))  # every core this process may use
    total_budget = 150.0
    per_step = total_budget / max(1, args.steps + args.warmup)
    # calibrate on one call that occupies every thread: seconds per batch row
    rows_cal = _rows_per_call(B, H, threads)
    t0 = time.perf_counter()
    _oracle_rows(x, 0, rows_cal)
    per_row = (time.perf_counter() - t0) / rows_cal
    rows = max(1, min(B, int(per_step / per_row)))  # batch rows (every head) per step
    cores = min(threads, rows * H)

    def step():
        _oracle_rows(x, 0, rows)
    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = time.perf_counter() - t0
    heads = rows * H
    tokens = heads * T * args.steps
    value = tokens / el
    sample = (f"{heads} of {B * H} heads x {T} tokens of {HEADLINE} per step "
              f"(float64 token loop, OpenMP over heads on {cores} threads)")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": HEADLINE, "B": B, "H": H, "T": T, "d": 64, "W": x.W,
                       "C": x.C},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_only(args, tc, dev, world, peaks):
    """One workload, numbers only: used for profiler runs (ncu), never for the
    benchmark line."""
    if args.only == "decode":
        d = time_decode(tc, dev, world, steps=args.decode_steps or 16, batch=args.decode_batch,
                        e2e=False)
        ms = statistics.mean(d["per_step_ms"])
        print(json.dumps({"only": "decode", "B": d["B"], "steps": d["steps"], "ms_per_step": ms,
                          "GB_per_s": d["bytes_per_step"] / (ms * 1e-3) / 1e9}))
        return 0
    if args.only == "varlen":
        print(json.dumps({"only": "varlen", **time_varlen(tc, dev, args.steps, args.warmup)}))
        return 0
    if args.only == "general":
        print(json.dumps({"only": "general", **time_general(tc, dev, args.steps, args.warmup)}))
        return 0
    if args.only == "delta":
        x, sets, prm = _prefill_device_inputs(HEADLINE, dev, copies=1)
        q, k, v = sets[0]
        ms = statistics.median(time_calls(lambda: tc.prefill(q, k, v, *prm, x.W, x.C, delta_rule=True),
                                          args.steps, args.warmup))
        print(json.dumps({"only": "delta", "workload": HEADLINE, "ms": ms}))
        return 0
    if args.only == "backward":
        print(json.dumps({"only": "backward",
                          **time_training_extras(tc, dev, peaks, steps=args.steps)["backward"]}))
        return 0
    name = HEADLINE if args.only == "prefill" else "long_prefill_bf16"
    r = time_prefill(tc, name, dev, args.steps, args.warmup, world)
    x = r["x"]
    B, H, T, dk = x.q.shape
    l1f, l2f = prefill_flops(B, H, T, dk, dk, x.W)
    ms = statistics.mean(r["per_step_ms"])
    print(json.dumps({"only": name, "ms_per_step": ms,
                      "tflops": (l1f + l2f) / (ms * 1e-3) / 1e12,
                      "launches_per_step": r["launches_per_step"]}))
    return 0


# ---------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="tc", choices=["tc", "reference"])
    ap.add_argument("--no-extras", action="store_true",
                    help="headline prefill only (skip decode, long prefill, oracle)")
    ap.add_argument("--only", choices=["prefill", "long", "decode", "varlen", "backward", "general", "delta"],
                    default=None,
                    help="time one workload only and print its numbers (profiling runs)")
    ap.add_argument("--decode-batch", type=int, default=None,
                    help="batch of the decode workload (default 256)")
    ap.add_argument("--decode-steps", type=int, default=None,
                    help="decode steps (default 512)")
    ap.add_argument("--path", choices=["auto", "fused", "general"], default="auto",
                    help="tensor-core prefill for the calls both paths take (tc_set_prefill_path; "
                         "profiling runs of one path)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        return run_reference(args)

    world, rank, local = _dist()
    if world != args.gpus:
        print(f"warning: --gpus {args.gpus} but WORLD_SIZE={world}", file=sys.stderr)
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    import sliding_window_attention_tc_b200 as tc
    tc.set_prefill_path(args.path)

    peaks, peak_src = load_peaks()
    if args.only:
        return run_only(args, tc, dev, world, peaks)
    clocks = ClockSampler(local)
    clocks.start()
    try:
        head = time_prefill(tc, HEADLINE, dev, args.steps, args.warmup, world, clocks=clocks)
        x = head["x"]
        B, H, T, dk = x.q.shape
        dv = x.v.shape[-1]
        total_ms = _max_over_ranks(head["total_ms"], world, dev)
        ms_step = total_ms / args.steps
        tokens = head["tokens_per_step"] * args.steps * world
        value = tokens / (total_ms * 1e-3)
        l1f, l2f = prefill_flops(B, H, T, dk, dv, x.W)
        mean_ms = statistics.mean(head["per_step_ms"])
        achieved_tflops = (l1f + l2f) / (mean_ms * 1e-3) / 1e12
        peak_tf = float(peaks["bf16_tflops"])
        path = tc.prefill_path_for(tc.make_prefill_desc(B, H, T, dk, dv, x.W, x.C, tc.TC_BF16))
        kern = PATH_KERNEL[path]
        roofline = {"bound": "tensor", "achieved": achieved_tflops, "peak": peak_tf,
                    "unit": "TFLOP/s", "frac": achieved_tflops / peak_tf,
                    "traffic": NCU_TRAFFIC_BYTES[kern],
                    "traffic_kernel": f"{kern} (ncu, one launch)",
                    "peak_source": f"{peak_src} bf16 burst",
                    "kernel": f"tc_prefill (all launches of one call, {path} path)",
                    "path": path,
                    "algorithmic_flops_per_launch": l1f + l2f}
        executed = prefill_executed_flops if path == "fused" else general_executed_flops
        e1, e2 = executed(B, H, T, x.W)
        roofline["executed_flops_per_launch"] = e1 + e2
        roofline["executed_tflops"] = (e1 + e2) / (mean_ms * 1e-3) / 1e12
        extras = {}
        if not args.no_extras:
            l1 = time_prefill(tc, HEADLINE, dev, max(20, args.steps // 4), 3, world,
                              l1_only=True, clocks=clocks)
            t_l1 = statistics.mean(l1["per_step_ms"])
            extras["l2_overhead_lm"] = {"tc_ms": mean_ms, "l1_only_ms": t_l1,
                                        "ratio": mean_ms / t_l1 - 1.0,
                                        "algorithmic_floor": l2f / l1f}
            lp = time_prefill(tc, "long_prefill_bf16", dev, 20, 3, world, clocks=clocks)
            lp1 = time_prefill(tc, "long_prefill_bf16", dev, 20, 3, world, l1_only=True,
                               clocks=clocks)
            xl = lp["x"]
            Bl, Hl, Tl, dl = xl.q.shape
            f1, f2 = prefill_flops(Bl, Hl, Tl, dl, dl, xl.W)
            t_lp = statistics.mean(lp["per_step_ms"])
            t_lp1 = statistics.mean(lp1["per_step_ms"])
            extras["long_prefill"] = {
                "workload": "long_prefill_bf16", "B": Bl, "H": Hl, "T": Tl, "d": dl, "W": xl.W,
                "C": xl.C, "ms": t_lp, "tokens_per_s": Bl * Hl * Tl / (t_lp * 1e-3),
                "achieved_tflops": (f1 + f2) / (t_lp * 1e-3) / 1e12,
                "frac_of_bf16_peak": (f1 + f2) / (t_lp * 1e-3) / 1e12 / peak_tf,
                "l1_only_ms": t_lp1, "l2_overhead_ratio": t_lp / t_lp1 - 1.0,
                "algorithmic_floor": f2 / f1,
                "path": tc.prefill_path_for(tc.make_prefill_desc(Bl, Hl, Tl, dl, dl, xl.W, xl.C, tc.TC_BF16)),
                "executed_tflops": sum((prefill_executed_flops if tc.prefill_path_for(
                    tc.make_prefill_desc(Bl, Hl, Tl, dl, dl, xl.W, xl.C, tc.TC_BF16)) == "fused"
                    else general_executed_flops)(Bl, Hl, Tl, xl.W)) / (t_lp * 1e-3) / 1e12,
                "state_size": state_size_ratio(Tl, xl.W, dl)}
            del lp, lp1
            dec = time_decode(tc, dev, world, clocks=clocks)
            dms = statistics.mean(dec["per_step_ms"])
            gbs = dec["bytes_per_step"] / (dms * 1e-3) / 1e9
            extras["decode"] = {
                "workload": "batched decode 256x32 heads, d=128, W=2048, bf16 ring, fp32 A",
                "steps": dec["steps"], "ms_per_step_mean": dms,
                "ms_per_step_p50": statistics.median(dec["per_step_ms"]),
                "tokens_per_s": dec["B"] / (dms * 1e-3),
                "roofline": {"bound": "hbm", "achieved": gbs, "peak": float(peaks["hbm_gbs"]),
                             "unit": "GB/s", "frac": gbs / float(peaks["hbm_gbs"]),
                             "traffic": NCU_TRAFFIC_BYTES["decode_kernel"], "peak_source": f"{peak_src} copy bandwidth",
                             "algorithmic_bytes_per_launch": dec["bytes_per_step"]},
                "e2e": {"ms_per_step": dec["e2e_ms_per_step"],
                        "tokens_per_s": dec["B"] / (dec["e2e_ms_per_step"] * 1e-3),
                        "h2d_bytes_per_step": dec["e2e_h2d_bytes"],
                        "d2h_bytes_per_step": dec["e2e_d2h_bytes"]}}
            extras["varlen_prefill"] = time_varlen(tc, dev)
            extras["general_prefill"] = time_general(tc, dev)
            extras.update(time_training_extras(tc, dev, peaks, peak_src))
        e2e = time_prefill_e2e(tc, HEADLINE, dev, max(5, min(20, args.steps // 10)))
    finally:
        clocks.stop()

    if rank != 0:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return 0
    launches = head["launches_per_step"]
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step,
        "ms_per_step_p50": statistics.median(head["per_step_ms"]), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": HEADLINE, "B": B, "H": H, "T": T, "d": dk, "W": x.W, "C": x.C,
                   "parallelism": f"replicas x{world} (heads independent, no collective)",
                   "l2_cache": "inputs rotate over 3 buffer sets (603 MB > 126 MB L2)"},
        "roofline": roofline,
        "e2e": {"value": e2e["tokens_per_s"] * world, "unit": UNIT,
                "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"]},
        "gpu_launches": None if launches is None else launches * args.steps,
        "clocks": clocks.summary(),
    }
    line.update(extras)
    if world == 1 and not args.no_extras:
        line["cpu_baseline"] = oracle_sample(HEADLINE)
    print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
