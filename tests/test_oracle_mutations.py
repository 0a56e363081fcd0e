"""The oracle pins must catch plausible mistakes.

Each case copies the oracle's C source into a temporary directory, plants one
mistake by text substitution, builds it, points the oracle module at the
mutant and runs the pin tests; at least one pin must fail.  Only the CPU
oracle is mutated; nothing here touches a GPU.
"""
import ctypes
import os
import subprocess

import pytest

import oracle
import tests.test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "tc_oracle.c")

MUTATIONS = {
    "first eviction one step late (read before write)":
        ("if (t >= W) {\n        const double *k_old", "if (t > W) {\n        const double *k_old"),
    "missing 1/sqrt(d_k)":
        ("    const double scale = 1.0 / sqrt((double)dk);\n    double smax",
         "    const double scale = 1.0;\n    double smax"),
    "dropped decay":
        ("A[r * dv + c] = lam * A[r * dv + c] + eta * (k_old[r] * u[c]);",
         "A[r * dv + c] = A[r * dv + c] + eta * (k_old[r] * u[c]);"),
    "delta rule: correction with the wrong sign":
        ("u[c] = v_old[c] - pred;", "u[c] = v_old[c] + pred;"),
    "delta rule: prediction from the decayed state":
        ("for (int64_t r = 0; r < dk; ++r) pred += k_old[r] * A[r * dv + c];",
         "for (int64_t r = 0; r < dk; ++r) pred += k_old[r] * lam * A[r * dv + c];"),
    "delta rule: transposed prediction":
        ("for (int64_t r = 0; r < dk; ++r) pred += k_old[r] * A[r * dv + c];",
         "for (int64_t r = 0; r < dk && r < dv && c < dk; ++r) pred += k_old[r] * A[c * dv + r];"),
    "gate sign":
        ("const double gate = 1.0 / (1.0 + exp(-g));", "const double gate = 1.0 / (1.0 + exp(g));"),
    "window one key short":
        ("const int64_t n = (t + 1 < W) ? t + 1 : W;",
         "const int64_t n = (t + 1 < W) ? t + 1 : (W > 1 ? W - 1 : 1);"),
    "transposed read of A":
        ("for (int64_t r = 0; r < dk; ++r) mc += q[r] * A[r * dv + c];",
         "for (int64_t r = 0; r < dk; ++r) mc += q[r] * A[c * dv + r];"),
    "insert before evict":
        ("    memcpy(ring_k + pos * dk, k, (size_t)dk * sizeof(double));\n"
         "    memcpy(ring_v + pos * dv, v, (size_t)dv * sizeof(double));\n",
         ""),
    "backward: state gradient not decayed through a write":
        ("for (int64_t x = 0; x < nel; ++x) G[x] *= lam[h];", "for (int64_t x = 0; x < nel; ++x) G[x] *= 1.0;"),
    "backward: softmax gradient without the mean term":
        ("const double ds = p[i] * (dp - Dt);", "const double ds = p[i] * dp;"),
    "backward: lambda gradient against A_t instead of A_{t-1}":
        ("const double *Ap = As + t * nel; /* A_{t-1} */", "const double *Ap = As + (t + 1) * nel;"),
    "chunk decay exponent off by one":
        ("const double wd = eta * pow(lam, (double)(Cc - 1 - i));",
         "const double wd = eta * pow(lam, (double)(Cc - i));"),
}

# Pins with d_k >= d_v only, so a transposed index stays inside the buffers.
PIN_CALLS = [
    pins.test_window_covers_sequence_is_causal_softmax,
    lambda: pins.test_local_path_is_band_softmax(5),
    pins.test_gate_minus_infinity_is_pure_window_attention,
    pins.test_gate_zero_is_half,
    pins.test_final_state_closed_form,
    pins.test_memory_read_brute_force,
    pins.test_read_identity,
    pins.test_exact_recall_orthonormal_keys,
    lambda: pins.test_chunk_scan_equals_token_writes_fp64(16),
    lambda: pins.test_chunk_mean_adds_exactly_the_cross_terms(5),
    pins.test_chunk_mean_with_decay_drops_per_token_weights,
    pins.test_golden_hand_d1_w1,
    pins.test_golden_hand_d2_w2,
    lambda: pins.test_delta_rule_repeated_write_closed_form(1.0, 1.0, 3),
    lambda: pins.test_delta_rule_repeated_write_closed_form(1.0, 0.5, 4),
    lambda: pins.test_delta_rule_repeated_write_closed_form(0.9, 0.3, 6),
    pins.test_delta_rule_equals_outer_product_on_orthonormal_keys,
    pins.test_backward_matches_central_differences,
]


def _build_mutant(tmp_path, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor not unique: {old!r}"
    if new == "":  # move the insert ahead of the eviction block
        src = src.replace(old, "")
        anchor = "    if (t >= W) {\n        const double *k_old"
        assert src.count(anchor) == 1
        src = src.replace(anchor, old + anchor)
    else:
        src = src.replace(old, new)
    c = tmp_path / "mut.c"
    c.write_text(src)
    so = tmp_path / "libmut.so"
    subprocess.check_call(["gcc", "-O1", "-fopenmp", "-ffp-contract=off", "-shared", "-fPIC",
                           "-o", str(so), str(c), "-lm"])
    return str(so)


@pytest.mark.parametrize("name", list(MUTATIONS))
def test_pins_catch_planted_mistake(name, tmp_path):
    old, new = MUTATIONS[name]
    so = _build_mutant(tmp_path, old, new)
    good = oracle._load()
    mut = ctypes.CDLL(so)
    for fn in ("oracle_prefill_rule", "oracle_decode_rule", "oracle_scan_tokens",
               "oracle_scan_chunks", "oracle_scan_chunk_mean", "oracle_backward",
               "oracle_max_threads"):
        getattr(mut, fn).argtypes = getattr(good, fn).argtypes
        getattr(mut, fn).restype = getattr(good, fn).restype
    failed = []
    oracle._lib = mut
    try:
        for call in PIN_CALLS:
            try:
                call()
            except AssertionError:
                failed.append(call)
    finally:
        oracle._lib = good
    assert failed, f"no pin caught the planted mistake: {name}"
