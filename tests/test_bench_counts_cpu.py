"""Host-side work counts that bench.py reports next to its timings.

The algorithmic FLOPs follow the definitions of the layer: L1 counts
2 (d_k + d_v) per (query, key in window) pair, and L2 counts 2 d_k d_v per
eviction plus 2 d_k d_v per token that reads the memory.  The executed counts
follow the tiling of the bf16 tensor-core kernel: 128 x 128 tiles, and each
query tile past the first W tokens has W/128 + 1 key tiles.  Each count is
checked against brute-force enumeration on small shapes and against the
closed form for the LM workload.
"""
import os
import sys

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

import bench  # noqa: E402


def _pairs_brute(T, W):
    return sum(min(t + 1, W) for t in range(T))


def test_algorithmic_flops_match_enumeration():
    for T, W, dk, dv in [(1, 4, 8, 8), (5, 8, 4, 2), (100, 7, 16, 32), (256, 32, 16, 16)]:
        l1, l2 = bench.prefill_flops(1, 1, T, dk, dv, W)
        assert l1 == 2 * (dk + dv) * _pairs_brute(T, W)
        assert l2 == 4 * dk * dv * max(0, T - W)


def test_executed_tiles_match_enumeration():
    # every (query tile, key tile) pair that overlaps the causal band is computed once
    for T, W in [(128, 128), (1000, 256), (4096, 512), (32768, 1024)]:
        nT = (T + 127) // 128
        blocks = 0
        lead_tiles = 0
        for i in range(nT):
            lo = max(0, i * 128 - W)  # first key any row of tile i sees (row 0 sees i*128-W+1..)
            first = lo // 128
            blocks += i - first + 1
            lead_tiles += i * 128 >= W
        e1, e2 = bench.prefill_executed_flops(1, 1, T, W)
        mma_tile = 2 * 128 * 128 * 64
        assert e1 == blocks * 2 * mma_tile, (T, W)
        assert e2 == lead_tiles * (2 * mma_tile + 128 * 64 * 64 * 2), (T, W)


def test_lm_workload_counts():
    l1, l2 = bench.prefill_flops(8, 12, 4096, 64, 64, 512)
    assert l1 + l2 == 53961818112
    e1, e2 = bench.prefill_executed_flops(8, 12, 4096, 512)
    # 150 computed tiles and 28 leading tiles per head
    assert e1 == 96 * 150 * 2 * (2 * 128 * 128 * 64)
    assert e2 == 96 * 28 * (2 * (2 * 128 * 128 * 64) + 128 * 64 * 64 * 2)


def test_oracle_calls_split_evenly_over_threads():
    # rows per call: at least one (b, h) item per thread, and whole waves where possible
    for B, H, threads in [(8, 12, 1), (8, 12, 8), (8, 12, 16), (8, 12, 32), (1, 16, 64), (8, 4, 6)]:
        r = bench._rows_per_call(B, H, threads)
        assert 1 <= r <= B
        items = r * H
        assert items >= min(threads, B * H)
        if any((k * H) % threads == 0 for k in range(-(-threads // H), B + 1)):
            assert items % threads == 0, (B, H, threads, r)


def test_cpu_baseline_reports_threads_used():
    out = bench.oracle_sample("lm_prefill_bf16", budget_s=0.05)
    cores = len(os.sched_getaffinity(0))
    assert 1 <= out["cores"] <= cores
    assert out["kind"] == "oracle" and out["value"] > 0
    assert "heads x 4096 tokens" in out["sample"]


def _general_brute(T, W, d):
    """Tensor-core FLOPs of the general path by enumerating keys: block b of
    128 query rows scores every 64-key tile that holds a key it reads (the
    window keys of its rows, and its chunk of evictions when it has one),
    P V on the same tiles, P'V on the tiles holding its chunk, Q A_b (hi +
    lo); one 128 x 128 x 128 sums product pair per CTA of chunks."""
    E = max(0, T - W)
    nC = -(-T // 128)
    tiles = reads = qa = 0
    for b in range(nC):
        rows = range(128 * b, min(T, 128 * b + 128))
        keys = {j for t in rows for j in range(max(0, t - W + 1), t + 1)}
        chunk = set(range(max(0, 128 * b - W), max(0, min(E, 128 * b + 128 - W))))
        keys |= chunk
        # the kernel's tiles run from the first key read to the block's last row
        lo, hi = min(keys), min(T - 1, 128 * b + 127)
        tiles += hi // 64 - lo // 64 + 1
        if chunk:
            reads += len({j // 64 for j in chunk})
            qa += 1
    mma = 2 * 128 * 64 * d
    sums = (((nC + 1) // 2) if d == 64 else nC) * 2 * (2 * 128 ** 3) if E > 0 else 0
    return tiles * 2 * mma, reads * mma + qa * 2 * (2 * 128 * d * d) + sums


def test_general_path_executed_flops_match_enumeration():
    for T, W, d in [(128, 128, 64), (700, 200, 64), (1000, 256, 128), (333, 5, 64), (100, 300, 64),
                    (4096, 500, 64), (2000, 512, 128)]:
        assert bench.general_executed_flops(1, 1, T, W, d) == _general_brute(T, W, d), (T, W, d)


def test_general_path_lm_counts():
    # per head: 300 key tiles (blocks 0-3: 2, 4, 6, 8; blocks 4-31: 10 each),
    # 56 tiles of P'V and 28 Q A_b products (blocks 4-31), 16 sums CTAs
    e1, e2 = bench.general_executed_flops(8, 12, 4096, 512)
    mma = 2 * 128 * 64 * 64
    assert e1 == 96 * 300 * 2 * mma
    assert e2 == 96 * (56 * mma + 28 * 2 * mma + 16 * 2 * (2 * 128 ** 3))
    l1, l2 = bench.prefill_flops(8, 12, 4096, 64, 64, 512)
    assert abs((e1 + e2) / (l1 + l2) - 1.567) < 1e-3
