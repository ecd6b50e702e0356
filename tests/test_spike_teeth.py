"""CPU proof that the spike inputs give the bf16 parity tests teeth.

With N(0,1) inputs an attention output averages thousands of values, so a
kernel that drops or adds one key (or the whole window) can stay inside the
2e-2 bf16 tolerance.  The spiked inputs of ``tests/spikes.py`` fix that: for
every probe, the oracle's output with the probed key's visibility flipped
(the mistake a one-key mask error makes) is far from the true output.  The
GPU tests run these same constructions; these tests show on the CPU that a
one-key error anywhere on the probed edges cannot pass them, and that the
probes make the running row maximum jump, so the tensor-core kernel's
rescale of its accumulator runs.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from reference_sliding_window_b200 import synth
from tests import spikes
from tests.gpu_util import BF16_ABS

TEETH = 0.1  # a flipped key must move the output by at least this (5x the bf16 tolerance)


def flipped_gap_packed(Q, K, V, L_m, n, row, key, bidir=False):
    """max |o(true set) - o(true set with `key` flipped)| over heads and dims."""
    vis_fn = oracle.bidir_prefix_visible_positions if bidir else oracle.packed_visible_positions
    vis = vis_fn(row + 1, L_m, n) - 1
    flip = np.setdiff1d(vis, [key]) if key in vis else np.union1d(vis, [key])
    if flip.size == 0:  # the probed key is the only visible one: dropping it leaves 0/0
        return float("inf")
    d = Q.shape[-1]
    sc = 1.0 / np.sqrt(d)
    gap = 0.0
    for h in range(Q.shape[1]):
        a = oracle.attend(Q[row, h], K[vis, h], V[vis, h], sc)
        b = oracle.attend(Q[row, h], K[flip, h], V[flip, h], sc)
        gap = max(gap, float(np.abs(a - b).max()))
    return gap


def rescale_growth_log2(Q, K, L_m, n, row, bidir=False, tile=128):
    """How far (log2 units) the row maximum over the visible keys rises
    beyond the maximum of the first visible key tile, for head 0."""
    vis_fn = oracle.bidir_prefix_visible_positions if bidir else oracle.packed_visible_positions
    vis = vis_fn(row + 1, L_m, n) - 1
    s = (K[vis, 0] @ Q[row, 0]) / np.sqrt(Q.shape[-1]) * np.log2(np.e)
    first = vis // tile == vis[0] // tile
    return float(s.max() - s[first].max())


PACKED_CASES = [
    # L, L_m, n, H, bidir
    (1000, 300, 128, 2, False),
    (700, 256, 64, 2, False),
    (700, 0, 128, 2, False),
    (640, 384, 5, 2, True),
    (1000, 513, 200, 2, False),
]


@pytest.mark.parametrize("L,L_m,n,H,bidir", PACKED_CASES)
def test_packed_probes_flip_far_beyond_tolerance(L, L_m, n, H, bidir):
    Q, K, V = synth.prefill_case(L, H, 128, "bf16", seed=L + n + 3)
    probes = spikes.packed_edge_probes(L, L_m, n)
    assert len(probes) >= 20
    Qs = synth.spike_packed_queries(Q, K, probes)
    Qd, Kd, Vd = (t.double().numpy() for t in (Qs, K, V))
    gaps = [flipped_gap_packed(Qd, Kd, Vd, L_m, n, i, j, bidir) for i, j in probes]
    worst = int(np.argmin(gaps))
    assert gaps[worst] > TEETH, f"probe {probes[worst]} moves the output by only {gaps[worst]:.3g}"
    assert TEETH > 4 * BF16_ABS


@pytest.mark.parametrize("L,L_m,n,H,bidir", [c for c in PACKED_CASES if c[1] >= 256])
def test_packed_probes_exercise_the_rescale(L, L_m, n, H, bidir):
    """Where the reference spans several key tiles, many probed keys lie
    beyond a row's first key tile and lift its maximum by more than 2^8, the
    threshold of the tensor-core kernel's lazy rescale."""
    Q, K, V = synth.prefill_case(L, H, 128, "bf16", seed=L + n + 3)
    probes = spikes.packed_edge_probes(L, L_m, n)
    Qd = synth.spike_packed_queries(Q, K, probes).double().numpy()
    Kd = K.double().numpy()
    grow = [rescale_growth_log2(Qd, Kd, L_m, n, i, bidir) for i, _ in probes]
    assert sum(g > 8.0 for g in grow) >= len(probes) // 4


def test_packed_probes_at_the_32k_config():
    """The 32K teacher-forced shape (L_m = 12832, n = 128), one head: every
    probed key still dominates its row."""
    L, L_m, n = 32768, 12832, 128
    Q, K, V = synth.prefill_case(L, 1, 128, "bf16", seed=77)
    probes = spikes.packed_edge_probes(L, L_m, n, limit=96)
    Qs = synth.spike_packed_queries(Q, K, probes)
    Qd, Kd, Vd = (t.double().numpy() for t in (Qs, K, V))
    gaps = [flipped_gap_packed(Qd, Kd, Vd, L_m, n, i, j) for i, j in probes]
    assert min(gaps) > TEETH


def test_whole_window_dropped_is_seen_with_spikes():
    """The failure N(0,1) inputs hide at L_m = 12832: a kernel that ignores
    the window entirely.  With the query spiked on a window key the output
    moves by O(1)."""
    L, L_m, n = 13200, 12832, 128
    Q, K, V = synth.prefill_case(L, 1, 128, "bf16", seed=78)
    i = L_m + 200
    Qs = synth.spike_packed_queries(Q, K, [(i, i - 5)])
    Qd, Kd, Vd = (t.double().numpy() for t in (Qs, K, V))
    vis = oracle.packed_visible_positions(i + 1, L_m, n) - 1
    sc = 1 / np.sqrt(128)
    a = oracle.attend(Qd[i, 0], Kd[vis, 0], Vd[vis, 0], sc)
    b = oracle.attend(Qd[i, 0], Kd[:L_m, 0], Vd[:L_m, 0], sc)
    assert np.abs(a - b).max() > 1.0


def flipped_gap_decode(case, t, b, pos):
    """The same for decode step t of sequence b with the key at logical
    position pos flipped in or out of the visible set."""
    L = case.ref_lens[b]
    Kh, Vh = synth.history(case, b, t)
    q = case.q[t - 1, b].double().cpu().numpy()
    vis = oracle.decode_visible_positions(t, L, case.n) - 1
    p = pos - 1
    flip = np.setdiff1d(vis, [p]) if p in vis else np.union1d(vis, [p])
    if flip.size == 0:
        return float("inf")
    sc = 1.0 / np.sqrt(case.d)
    gap = 0.0
    for h in range(case.H):
        a = oracle.attend(q[h], Kh[vis, h], Vh[vis, h], sc)
        c = oracle.attend(q[h], Kh[flip, h], Vh[flip, h], sc)
        gap = max(gap, float(np.abs(a - c).max()))
    return gap


@pytest.mark.parametrize("ref_lens,H,n,T", [
    ([2592], 2, 128, 300),            # single-document shape
    ([12832, 544, 3000], 2, 128, 260),  # ragged shapes, 50 and 2 pages
    ([40, 13], 2, 8, 30),
])
def test_decode_probes_flip_far_beyond_tolerance(ref_lens, H, n, T):
    case = synth.decode_case(B=len(ref_lens), H=H, d=128, ref_lens=ref_lens, n=n, T=T, dtype="bf16", seed=5)
    steps = sorted({1, 2, n - 1, n, n + 1, 2 * n, 2 * n + 1, T - 1, T})
    probes = spikes.decode_edge_probes(steps, ref_lens, n)
    kinds_seen = set()
    synth.spike_decode_queries(case, probes)
    for t, b, pos in probes:
        gap = flipped_gap_decode(case, t, b, pos)
        assert gap > TEETH, f"step {t} seq {b} pos {pos}: {gap:.3g}"
        kinds_seen.add(pos - ref_lens[b] if pos > ref_lens[b] else "ref")
    assert len(kinds_seen) >= 3
