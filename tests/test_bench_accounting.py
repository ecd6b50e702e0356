"""The work the benchmark divides by, checked against the oracle's explicit
sets (CPU): the visible (query, key) pairs behind the prefill FLOP count and
the cache rows behind the decode byte count."""

from __future__ import annotations

import pytest

import bench
import oracle


@pytest.mark.parametrize("L,L_m,n", [
    (6, 3, 2), (9, 0, 2), (40, 13, 5), (33, 33, 4), (50, 10, 100), (64, 1, 1), (17, 0, 40),
])
def test_visible_pairs_counts_the_packed_mask(L, L_m, n):
    assert bench.visible_pairs(L, L_m, n) == int(oracle.packed_mask(L, L_m, n).sum())


def test_visible_pairs_at_the_32k_config():
    # the closed form at the full config agrees with a row-by-row count of
    # the visible sets (without building the 32K x 32K mask)
    L, L_m, n = 32768, 12832, 128
    rows = sum(min(p, L_m) if p <= L_m else L_m + min(n, p - L_m) for p in range(1, L + 1))
    assert bench.visible_pairs(L, L_m, n) == rows == 340_698_960


def test_decode_bytes_per_launch_match_the_occupancy_law():
    # K and V rows of Eq.(6) at T >= n, plus q, o, k_new, v_new
    w = dict(bench.WORKLOADS["single_doc"])
    lens = bench.ref_lens_for(w)
    rows = sum(oracle.occupancy_rswa(w["n"] + 1, L, w["n"]) for L in lens)
    s = 2  # bf16
    want = w["H"] * (2 * rows * w["d"] * s) + w["B"] * w["H"] * 4 * w["d"] * s
    assert bench.bytes_per_launch(w, lens) == want == 13_936_640


@pytest.mark.parametrize("L,L_m,n", [(6, 3, 2), (40, 13, 5), (50, 10, 100), (17, 0, 4)])
def test_visible_keys_per_row_match_the_oracle(L, L_m, n):
    # the per-row count behind the prefill oracle baseline's FLOPs
    for r in range(L):
        assert bench.visible_keys(r, L_m, n) == len(oracle.packed_visible_positions(r + 1, L_m, n)), r


def test_prefill_oracle_baseline_runs_on_a_small_pack():
    w = dict(L=300, L_m=100, n=16, H=2, d=16)
    v, threads, sample = bench.oracle_prefill_sample(w, budget_s=0.05, n_random=8)
    assert v > 0 and threads >= 1 and "query rows" in sample


def test_curve_cache_rows_and_ratio_follow_eq5_to_eq7():
    w = dict(bench.WORKLOADS["single_doc"])
    lens = bench.ref_lens_for(w)
    n = w["n"]
    for T in bench.CURVE_T:
        assert bench.cache_rows(lens, n, T, False) == sum(oracle.occupancy_rswa(T, L, n) for L in lens)
        assert bench.cache_rows(lens, n, T, True) == sum(oracle.occupancy_full(T, L) for L in lens)
    ratios = bench.curve_cache_ratio(lens, n, bench.CURVE_T)
    assert len(lens) == 1 and len(ratios) == len(bench.CURVE_T)
    for T, r in zip(bench.CURVE_T, ratios):
        assert r == pytest.approx(oracle.cache_ratio(T, lens[0], n), abs=1e-6)
    # ragged batch: the ratio of summed rows
    assert bench.curve_cache_ratio([5, 7], 2, [1, 4]) == [1.0, round((7 + 9) / (9 + 11), 6)]


@pytest.mark.parametrize("cu,refs,n", [([0, 5, 9, 12], [2, 1, 0], 2), ([0, 30, 31, 80], [10, 1, 49], 4),
                                       ([0, 17], [17], 3)])
def test_pack_visible_pairs_count_the_varlen_mask(cu, refs, n):
    assert bench.pack_visible_pairs(cu, refs, n) == int(oracle.varlen_mask(cu, refs, n).sum())


def test_pack_oracle_baseline_runs_on_a_small_pack():
    w = dict(L=300, L_m=100, n=16, H=2, d=16)
    v, threads, sample = bench.oracle_prefill_sample(w, budget_s=0.05, n_random=4,
                                                     docs=([0, 120, 121, 300], [40, 1, 0]))
    assert v > 0 and "3 documents" in sample


def test_step_plan_times_exactly_the_steps_asked_and_ends_at_the_target():
    for T_target, n, steps, warmup in [(6144, 128, 20, 5), (100000, 128, 64, 8), (6144, 128, 6144, 8),
                                       (300, 128, 7, 3)]:
        T0, first, last = bench.step_plan(T_target, n, steps, warmup)
        assert T0 >= n  # the ring is full before the first timed step
        assert last - first + 1 == steps
        assert first == T0 + warmup + bench.GRAPH_STEPS + 1
        if T_target - warmup - bench.GRAPH_STEPS - steps >= n:
            assert last == T_target


def test_oracle_sample_weighs_a_ragged_batch_by_quantiles():
    w = dict(bench.WORKLOADS["ragged"])
    w.update(H=1, d=16)
    lens = [100, 200, 300, 400, 500, 600, 700, 800]
    v, threads, sample = bench.oracle_sample(w, lens, budget_s=0.05, max_seqs=4)
    assert v > 0 and threads >= 1
    assert "4 of 8 sequences (L_m [200, 400, 600, 800])" in sample
