"""Where to put spiked keys: (query, key) pairs on the edges of R-SWA's
visible sets.

A spiked query is a multiple of one key (``synth.spike_*``), so its output is
almost exactly that key's value row when the key is visible and something
else when it is not.  Each pair below puts the key on or next to an edge of
the visible set of "Unlimited OCR Works" 方法展开 §3, Eq.(1)-(2): the oldest
key of the output window and the one just before it, the last reference key
and the first output key, the diagonal and the key just after it, and the
same edges where they fall on a 128-key tile seam or a 256-query tile-pair
seam of the tensor-core kernel (or a 32-row stage seam of the decode
kernel).  Whether a probed key is visible is not decided here: the tests
compare with the oracle, and ``test_spike_teeth.py`` checks on the CPU that
flipping the visibility of any probed key moves the oracle's output far
beyond the bf16 tolerance.
"""

from __future__ import annotations

from typing import Dict, List, Sequence, Tuple

TILE = 128


def packed_edge_probes(L: int, L_m: int, n: int, tile: int = TILE, limit: int = 0) -> List[Tuple[int, int]]:
    """(row, key) pairs, 0-based, one per query row, for a packed sequence of
    L rows with L_m reference rows and window n.  ``limit`` > 0 keeps at
    most that many pairs (spread over the kinds)."""
    by_row: Dict[int, int] = {}

    def add(i: int, j: int) -> None:
        if 0 <= i < L and 0 <= j < L and i not in by_row:
            by_row[i] = j

    first_out = L_m  # 0-based row of the first output
    # window edges: the key just outside the window and the oldest one inside
    for i in (first_out + n, first_out + n + 1, first_out + 2 * n + 3, L - 1, L - 2):
        add(i, i - n)           # just outside the window (a reference key if i - n < L_m)
    for i in (first_out + n + 5, first_out + 3 * n // 2, L - 3):
        add(i, i - n + 1)       # the oldest key of the window
    # reference seam: the last reference key and the first output key
    if L_m >= 1:
        for i in (first_out, first_out + 1, first_out + n - 1, first_out + n, first_out + 2 * n):
            add(i, L_m - 1)
        for i in (first_out + n - 2, first_out + n + 2, L - 5):
            add(i, L_m)
        for i in (0, 1, L_m // 2, L_m - 2, L_m - 1):  # prefix rows: the last reference key
            add(i, L_m - 1)
    # diagonal and the key just after it
    for i in (first_out + 7, first_out + n // 2, L - 7, L_m // 3):
        add(i, i)
    for i in (first_out + 9, L_m // 4, L - 9, L_m - 3):
        add(i, i + 1)
    # the same edges on tile seams (key tiles of `tile` keys, query pairs of 2*tile rows)
    for s in range(tile, L, tile):
        add(s - 1, s)           # the next tile's first key, just past the diagonal
        add(s, s)               # diagonal on the seam
        add(s + n - 1, s - 1)   # window starts at the seam: the key before it is outside
        add(s + n - 2, s - 1)   # window starts one key before the seam
        add(s + n, s)           # window starts one key after the seam
        if (s // tile) % 2 == 0:
            add(s + 1, s - 1)   # pair seam: the previous pair's last key
    pairs = sorted(by_row.items())
    if limit and len(pairs) > limit:
        step = len(pairs) / limit
        pairs = [pairs[int(k * step)] for k in range(limit)]
    return pairs


def decode_edge_probes(steps: Sequence[int], ref_lens: Sequence[int], n: int,
                       seqs: Sequence[int] = None, stage: int = 32) -> List[Tuple[int, int, int]]:
    """(t, b, pos) triples: at decode step t (after t appends) the query of
    sequence b spikes on the key at 1-based logical position pos.  The kinds
    cycle over steps and sequences: the just-evicted output t - n, the oldest
    output still in the window, the newest output (the query's own key), the
    last and the first reference row, and a reference row on a 32-row stage
    seam."""
    out = []
    kinds = ("evicted", "oldest", "newest", "last_ref", "first_ref", "stage_seam")
    bs = list(range(len(ref_lens))) if seqs is None else list(seqs)
    c = 0
    for t in steps:
        for b in bs:
            L = int(ref_lens[b])
            for _ in range(len(kinds)):
                kind = kinds[c % len(kinds)]
                c += 1
                if kind == "evicted" and t - n >= 1:
                    pos = L + t - n
                elif kind == "oldest" and t >= 1:
                    pos = L + max(1, t - n + 1)
                elif kind == "newest" and t >= 1:
                    pos = L + t
                elif kind == "last_ref":
                    pos = L
                elif kind == "first_ref":
                    pos = 1
                elif kind == "stage_seam" and L > stage:
                    pos = stage * ((L // stage) // 2) + 1 - (c % 2)  # 32k + 1 or 32k (1-based)
                else:
                    continue
                out.append((int(t), int(b), int(pos)))
                break
    return out
