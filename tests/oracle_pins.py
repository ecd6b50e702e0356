"""Checks that pin the CPU oracle to things other than itself.

Each ``pin_*`` function takes the oracle module (or a mutated copy of it) and
raises AssertionError if the oracle disagrees with what the pages and the
mathematics fix:

* hand-evaluated values of Eq.(2), Eq.(5)-(7) and of the packed mask
  (``tests/golden``),
* special cases that reduce to a library routine (T <= n is plain causal
  attention: torch's fp64 scaled_dot_product_attention),
* closed forms (identical keys -> mean of the visible values; identical
  values -> that value; q = 0 -> uniform mean),
* brute force with scalar loops on tiny inputs,
* the queue of fixed capacity L_m + n that evicts position m+1
  ("多模态文档解析开源新进展:Unlimited OCR技术方案", KV cache 恒定).

``test_oracle.py`` runs every pin on the real oracle and, to show the pins
have teeth, on copies with planted mistakes.
"""

from __future__ import annotations

import math
import os
from fractions import Fraction

import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    out = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                out.append([int(x) for x in line.split()])
    return out


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


# --------------------------------------------------------------- index sets

def pin_eq2_small(o):
    for row in _rows("eq2_visible_sets_Lm3_n2.txt"):
        t, pos = row[0], row[1:]
        got = o.visible_positions(t, 3, 2).tolist()
        assert got == pos, (t, got, pos)


def pin_eq2_default_window(o):
    for t, lo, hi, size in _rows("eq2_window_Lm272_n128.txt"):
        w = o.window_positions(t, 272, 128)
        assert len(w) == size, (t, len(w), size)
        if size:
            assert (int(w[0]), int(w[-1])) == (lo, hi), (t, w[0], w[-1])


def pin_packed_mask_small(o):
    want = np.array(_rows("packed_mask_L6_Lm3_n2.txt"), dtype=bool)
    got = o.packed_mask(6, 3, 2)
    assert got.shape == want.shape and (got == want).all(), got.astype(int)


def pin_swa_mask_small(o):
    # L_m = 0: no reference segment, the plain sliding window (reading R6).
    want = np.array(_rows("swa_mask_L6_n2.txt"), dtype=bool)
    got = o.packed_mask(6, 0, 2)
    assert got.shape == want.shape and (got == want).all(), got.astype(int)


def pin_bidir_prefix_mask_small(o):
    want = np.array(_rows("packed_mask_bidir_L6_Lm3_n2.txt"), dtype=bool)
    got = o.packed_mask(6, 3, 2, bidir_prefix=True)
    assert got.shape == want.shape and (got == want).all(), got.astype(int)


def pin_swa_and_bidir_predicates(o):
    # Brute-force predicates, written independently of the set construction.
    for n, L in ((1, 5), (2, 9), (3, 14), (7, 11), (20, 12)):
        M = o.packed_mask(L, 0, n)
        for p in range(1, L + 1):
            for j in range(1, L + 1):
                assert bool(M[p - 1, j - 1]) == (p - n < j <= p), (n, p, j)
    for L_m, n, L in ((3, 2, 9), (1, 1, 6), (5, 3, 14), (6, 8, 10)):
        M = o.packed_mask(L, L_m, n, bidir_prefix=True)
        for p in range(1, L + 1):
            for j in range(1, L + 1):
                want = (j <= L_m) if p <= L_m else (j <= p and (j <= L_m or j > p - n))
                assert bool(M[p - 1, j - 1]) == want, (L_m, n, p, j)


def pin_cache_sizes(o):
    for L_m, n, T, c_mha, c_rswa, num, den in _rows("eq5_eq7_cache_sizes.txt"):
        assert o.occupancy_full(T, L_m) == c_mha
        assert o.occupancy_rswa(T, L_m, n) == c_rswa
        assert o.cache_ratio(T, L_m, n) == num / den


def pin_ratio_limits(o):
    # Eq.(8): for T >= n the ratio is exactly (L_m + n) / (L_m + T);
    # Eq.(9): for T >> L_m + n it approaches (L_m + n) / T and goes to 0.
    L_m, n = 2592, 128
    for T in (128, 129, 6144, 100000):
        assert Fraction(o.occupancy_rswa(T, L_m, n), o.occupancy_full(T, L_m)) == \
            Fraction(L_m + n, L_m + T)
    T = 10**9
    r = o.cache_ratio(T, L_m, n)
    assert abs(r - (L_m + n) / T) / r < 1e-5 and r < 1e-5


def pin_decode_occupancy(o):
    # |N(T+1)| = L_m + min(n, T) = Eq.(6), for every T (reading: the newest
    # output is the query).
    for L_m in (1, 5, 17):
        for n in (1, 3, 8):
            for T in range(0, 3 * n + 6):
                vis = o.decode_visible_positions(T, L_m, n)
                assert len(vis) == L_m + min(n, T), (L_m, n, T)
                assert len(set(vis.tolist())) == len(vis)
                # reference rows always visible ("encoded once, never updated")
                assert set(range(1, L_m + 1)) <= set(vis.tolist())
                # the newest output is visible to its own query
                if T > 0:
                    assert L_m + T in set(vis.tolist())


def pin_packed_mask_predicate(o):
    # Brute-force predicate, written independently of the set construction:
    # key j is visible from query p iff j <= p and (p is a prefix query, or j
    # is a reference key, or j lies within the last n positions up to p).
    for L_m, n, L in ((3, 2, 9), (1, 1, 6), (5, 3, 14), (4, 8, 11)):
        M = o.packed_mask(L, L_m, n)
        for p in range(1, L + 1):
            for j in range(1, L + 1):
                want = j <= p and (p <= L_m or j <= L_m or j >= p - n + 1)
                assert bool(M[p - 1, j - 1]) == want, (L_m, n, p, j)


def pin_window_of_one_is_reference_plus_self(o):
    # n = 1: an output query sees P and itself, nothing else (closed form).
    for L_m in (1, 4, 9):
        P = list(range(1, L_m + 1))
        for p in range(L_m + 1, L_m + 7):
            assert o.packed_visible_positions(p, L_m, 1).tolist() == P + [p], (L_m, p)
        for T in range(1, 6):
            assert o.decode_visible_positions(T, L_m, 1).tolist() == P + [L_m + T], (L_m, T)


# ----------------------------------------------------------------- numerics

def pin_short_output_is_causal(o):
    # T <= n: the window covers every output, so R-SWA is plain causal
    # attention over prefix + outputs (torch's fp64 SDPA as the library
    # routine).  Also n >= L for any L_m.
    for L, L_m, n, H, d in ((20, 7, 13, 2, 5), (33, 1, 40, 3, 4), (16, 16, 1, 1, 8)):
        Q, K, V = _rand((L, H, d), 1), _rand((L, H, d), 2), _rand((L, H, d), 3)
        got = o.masked_forward(Q, K, V, L_m, n)
        tq = torch.from_numpy(Q).permute(1, 0, 2)
        tk = torch.from_numpy(K).permute(1, 0, 2)
        tv = torch.from_numpy(V).permute(1, 0, 2)
        ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True)
        ref = ref.permute(1, 0, 2).numpy()
        assert np.allclose(got, ref, rtol=1e-12, atol=1e-12), np.abs(got - ref).max()


def pin_swa_wide_window_is_causal(o):
    # L_m = 0 and n >= L: the window covers every earlier token, so the form
    # is plain causal attention (torch's fp64 SDPA as the library routine).
    for L, n, H, d in ((17, 17, 2, 5), (9, 40, 1, 3)):
        Q, K, V = _rand((L, H, d), 31), _rand((L, H, d), 32), _rand((L, H, d), 33)
        got = o.masked_forward(Q, K, V, 0, n)
        tq, tk, tv = (torch.from_numpy(x).permute(1, 0, 2) for x in (Q, K, V))
        ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=True)
        ref = ref.permute(1, 0, 2).numpy()
        assert np.allclose(got, ref, rtol=1e-12, atol=1e-12), np.abs(got - ref).max()


def pin_bidir_prefix_rows_are_full_attention(o):
    # Bidirectional prefix: prefix rows are plain (non-causal) attention over
    # the prefix block (torch's fp64 SDPA); output rows are those of the
    # default form.
    L, L_m, n, H, d = 15, 6, 3, 2, 4
    Q, K, V = _rand((L, H, d), 34), _rand((L, H, d), 35), _rand((L, H, d), 36)
    got = o.masked_forward(Q, K, V, L_m, n, bidir_prefix=True)
    tq, tk, tv = (torch.from_numpy(x[:L_m]).permute(1, 0, 2) for x in (Q, K, V))
    ref = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, is_causal=False).permute(1, 0, 2).numpy()
    assert np.allclose(got[:L_m], ref, rtol=1e-12, atol=1e-12), np.abs(got[:L_m] - ref).max()
    base = o.masked_forward(Q, K, V, L_m, n)
    assert np.allclose(got[L_m:], base[L_m:], rtol=0, atol=0)
    rows = [0, L_m - 1, L_m, L - 1]
    sub = o.masked_forward_rows(Q, K, V, L_m, n, rows, bidir_prefix=True)
    assert np.allclose(sub, got[rows], rtol=1e-13, atol=1e-13)


def pin_swa_brute_force(o):
    # Scalar loops, math.exp, explicit window predicate; L_m = 0, tiny sizes.
    L, n, H, d = 8, 3, 2, 3
    Q, K, V = _rand((L, H, d), 37), _rand((L, H, d), 38), _rand((L, H, d), 39)
    got = o.masked_forward(Q, K, V, 0, n)
    scale = 1.0 / math.sqrt(d)
    for h in range(H):
        for p in range(1, L + 1):
            vis = [j for j in range(1, L + 1) if p - n < j <= p]
            s = {j: sum(Q[p - 1, h, c] * K[j - 1, h, c] for c in range(d)) * scale for j in vis}
            mx = max(s.values())
            w = {j: math.exp(s[j] - mx) for j in vis}
            z = sum(w.values())
            for c in range(d):
                want = sum(w[j] * V[j - 1, h, c] for j in vis) / z
                assert abs(got[p - 1, h, c] - want) < 1e-12, (h, p, c)


def pin_identical_keys_mean(o):
    # All keys equal -> all scores equal -> o = mean of the visible values.
    L, L_m, n, H, d = 6, 3, 2, 2, 4
    Q = _rand((L, H, d), 4)
    K = np.broadcast_to(_rand((1, H, d), 5), (L, H, d)).copy()
    V = _rand((L, H, d), 6)
    got = o.masked_forward(Q, K, V, L_m, n)
    mask = np.array(_rows("packed_mask_L6_Lm3_n2.txt"), dtype=bool)
    for p in range(L):
        want = V[mask[p]].mean(axis=0)
        assert np.allclose(got[p], want, rtol=1e-13, atol=1e-13), (p, got[p], want)


def pin_identical_values(o):
    L, L_m, n, H, d = 11, 4, 3, 2, 5
    Q, K = _rand((L, H, d), 7), _rand((L, H, d), 8)
    v0 = _rand((1, H, d), 9)
    V = np.broadcast_to(v0, (L, H, d)).copy()
    got = o.masked_forward(Q, K, V, L_m, n)
    assert np.allclose(got, V, rtol=1e-13, atol=1e-13)


def pin_zero_query_uniform(o):
    # q = 0 -> uniform weights over N(t): the output is the mean of the
    # visible values; the divisor is |N(t)|, checked against Eq.(6).
    L_m, n, T, H, d = 5, 3, 7, 2, 4
    Kh, Vh = _rand((L_m + T, H, d), 10), _rand((L_m + T, H, d), 11)
    for t in range(0, T + 1):
        got = o.decode_step(np.zeros((H, d)), Kh, Vh, L_m, t, n)
        rows = list(range(L_m)) + list(range(L_m + max(0, t - n), L_m + t))
        assert len(rows) == L_m + min(n, t)
        assert np.allclose(got, Vh[rows].mean(axis=0), rtol=1e-13, atol=1e-13), t


def pin_brute_force(o):
    # Scalar loops, math.exp, explicit predicate; tiny sizes.
    L, L_m, n, H, d = 9, 3, 2, 2, 3
    Q, K, V = _rand((L, H, d), 12), _rand((L, H, d), 13), _rand((L, H, d), 14)
    got = o.masked_forward(Q, K, V, L_m, n)
    scale = 1.0 / math.sqrt(d)
    for h in range(H):
        for p in range(1, L + 1):
            vis = [j for j in range(1, L + 1)
                   if j <= p and (p <= L_m or j <= L_m or j > p - n)]
            s = {j: sum(Q[p - 1, h, c] * K[j - 1, h, c] for c in range(d)) * scale for j in vis}
            mx = max(s.values())
            w = {j: math.exp(s[j] - mx) for j in vis}
            z = sum(w.values())
            for c in range(d):
                want = sum(w[j] * V[j - 1, h, c] for j in vis) / z
                assert abs(got[p - 1, h, c] - want) < 1e-12, (h, p, c)


def pin_scale_is_inverse_sqrt_d(o):
    L, L_m, n, H, d = 8, 2, 3, 1, 16
    Q, K, V = _rand((L, H, d), 15), _rand((L, H, d), 16), _rand((L, H, d), 17)
    a = o.masked_forward(Q, K, V, L_m, n)
    b = o.masked_forward(Q, K, V, L_m, n, scale=0.25)
    assert np.allclose(a, b, rtol=1e-14, atol=1e-14)
    c = o.masked_forward(Q, K, V, L_m, n, scale=0.5)
    assert not np.allclose(a, c)


def pin_decode_equals_packed_row(o):
    # Decode after T appends with q = Q[L_m + T - 1] equals row L_m + T - 1 of
    # the packed form (both describe the query producing output T+1).
    L_m, n, T, H, d = 4, 3, 9, 2, 5
    L = L_m + T
    Q, K, V = _rand((L, H, d), 18), _rand((L, H, d), 19), _rand((L, H, d), 20)
    full = o.masked_forward(Q, K, V, L_m, n)
    for t in range(1, T + 1):
        got = o.decode_step(Q[L_m + t - 1], K, V, L_m, t, n)
        assert np.allclose(got, full[L_m + t - 1], rtol=1e-13, atol=1e-13), t


def pin_queue_replay(o):
    # The literal queue (capacity L_m + n, evict position m+1) holds exactly
    # N(T+1) after T pushes, and attention over its contents equals the
    # from-scratch masked recomputation.  The n-slot ring holds the same set,
    # and output j overwrites what the queue evicts when j arrives.
    for L_m in (1, 5, 17):
        for n in (1, 3, 8):
            H, d = 2, 3
            T_max = 3 * n + 5
            Kh = _rand((L_m + T_max, H, d), 100 + L_m * 10 + n)
            Vh = _rand((L_m + T_max, H, d), 200 + L_m * 10 + n)
            qs = _rand((T_max + 1, H, d), 300 + L_m * 10 + n)
            for h in range(H):
                qc = o.QueueCache(L_m, n, Kh[:L_m, h], Vh[:L_m, h])
                ring = {}
                for T in range(0, T_max + 1):
                    if T > 0:
                        before = qc.positions().tolist()
                        qc.push(Kh[L_m + T - 1, h], Vh[L_m + T - 1, h])
                        slot = o.ring_slot(T, n)
                        old = ring.get(slot)
                        ring[slot] = L_m + T
                        if len(before) == L_m + n:
                            evicted = set(before) - set(qc.positions().tolist())
                            assert evicted == {old}, (T, evicted, old)
                    vis = o.decode_visible_positions(T, L_m, n).tolist()
                    assert qc.positions().tolist() == vis, (L_m, n, T)
                    stored = o.ring_storage_positions(T, L_m, n).tolist()
                    assert stored[:L_m] == list(range(1, L_m + 1))
                    assert stored[L_m:] == [ring[s] for s in range(min(n, T))]
                    assert sorted(stored) == vis
                    a = o.attend(qs[T, h], qc.keys(), qc.values(), 1.0 / math.sqrt(d))
                    b = o.decode_step(qs[T], Kh, Vh, L_m, T, n)[h]
                    assert np.allclose(a, b, rtol=1e-13, atol=1e-13)


def pin_order_independence(o):
    # Storage order of the rows does not change the result (softmax over a
    # set), which is what lets the ring store outputs out of logical order.
    rng = np.random.default_rng(21)
    q, K, V = rng.standard_normal(6), rng.standard_normal((40, 6)), rng.standard_normal((40, 6))
    perm = rng.permutation(40)
    assert np.allclose(o.attend(q, K, V, 0.3), o.attend(q, K[perm], V[perm], 0.3),
                       rtol=1e-13, atol=1e-13)


def pin_full_mode(o):
    # Full attention (Eq.(5) cache) equals R-SWA with n >= T.
    L_m, T, H, d = 6, 10, 2, 4
    Kh, Vh, q = _rand((L_m + T, H, d), 22), _rand((L_m + T, H, d), 23), _rand((H, d), 24)
    for t in range(T + 1):
        a = o.decode_step_full(q, Kh, Vh, L_m, t)
        b = o.decode_step(q, Kh, Vh, L_m, t, T + 1)
        assert np.allclose(a, b, rtol=1e-13, atol=1e-13)
    # and with n < T it differs (the window really cuts).
    a = o.decode_step_full(q, Kh, Vh, L_m, T)
    b = o.decode_step(q, Kh, Vh, L_m, T, 2)
    assert not np.allclose(a, b)


# ------------------------------------------------- several documents per pack

def pin_varlen_mask_small(o):
    want = np.array(_rows("varlen_mask_docs_5_4_3_n2.txt"), dtype=bool)
    got = o.varlen_mask([0, 5, 9, 12], [2, 1, 0], 2)
    assert got.shape == want.shape and (got == want).all(), got.astype(int)


def pin_varlen_predicate(o):
    # Brute-force predicate, written independently of the set construction:
    # same document, and j <= p and (j <= L_m or j > p - n) at local positions.
    rng = np.random.default_rng(61)
    for _ in range(12):
        lens = rng.integers(1, 9, rng.integers(1, 5)).tolist()
        refs = [int(rng.integers(0, x + 1)) for x in lens]
        n = int(rng.integers(1, 6))
        cu = np.concatenate([[0], np.cumsum(lens)]).tolist()
        doc = np.repeat(np.arange(len(lens)), lens)
        M = o.varlen_mask(cu, refs, n)
        for g in range(cu[-1]):
            for k in range(cu[-1]):
                i = doc[g]
                p, j, L_m = g - cu[i] + 1, k - cu[i] + 1, refs[i]
                want = doc[k] == i and j <= p and (j <= L_m or j > p - n)
                assert bool(M[g, k]) == want, (cu, refs, n, g, k)


def pin_varlen_single_document(o):
    # One document is the single-sequence packed form.
    for L, L_m, n in ((6, 3, 2), (9, 0, 3), (7, 7, 1), (11, 4, 20)):
        for bidir in (False, True):
            assert (o.varlen_mask([0, L], [L_m], n, bidir) == o.packed_mask(L, L_m, n, bidir)).all()


def pin_varlen_documents_independent(o):
    # The pack's output is each document's own output, and a document's
    # output does not move when another document's K/V change.
    lens, refs, n, H, d = [7, 3, 9], [3, 0, 9], 2, 2, 4
    cu = np.concatenate([[0], np.cumsum(lens)]).tolist()
    Q, K, V = _rand((cu[-1], H, d), 62), _rand((cu[-1], H, d), 63), _rand((cu[-1], H, d), 64)
    got = o.masked_forward_varlen(Q, K, V, cu, refs, n)
    for i in range(len(lens)):
        a, b = cu[i], cu[i + 1]
        want = o.masked_forward(Q[a:b], K[a:b], V[a:b], refs[i], n)
        assert np.allclose(got[a:b], want, rtol=1e-13, atol=1e-13), i
    K2, V2 = K.copy(), V.copy()
    K2[cu[1]:cu[2]] += 5.0
    V2[cu[1]:cu[2]] -= 3.0
    got2 = o.masked_forward_varlen(Q, K2, V2, cu, refs, n)
    keep = np.r_[0:cu[1], cu[2]:cu[3]]
    assert np.array_equal(got2[keep], got[keep])
    rows = [0, cu[1] - 1, cu[1], cu[2], cu[3] - 1]
    sub = o.masked_forward_varlen_rows(Q, K, V, cu, refs, n, rows)
    assert np.allclose(sub, got[rows], rtol=1e-13, atol=1e-13)


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
