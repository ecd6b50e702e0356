"""CPU tests: the oracle against its pins, and planted mistakes that the pins
must catch (each mistake is planted in a private copy of the oracle)."""

from __future__ import annotations

import importlib.util
import math
import os

import numpy as np
import pytest

import oracle
from tests import oracle_pins as pins

ORACLE_FILE = os.path.join(os.path.dirname(os.path.dirname(__file__)), "oracle", "rswa_oracle.py")


@pytest.mark.parametrize("pin", pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(oracle)


def _fresh_oracle():
    spec = importlib.util.spec_from_file_location("rswa_oracle_mutant", ORACLE_FILE)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _mut_window_short(m):
    def window_positions(t, L_m, n):
        lo, hi = max(L_m + 1, L_m + t - n + 1), L_m + t - 1
        return np.arange(lo, hi + 1) if hi >= lo else np.zeros(0, np.int64)
    m.window_positions = window_positions


def _mut_window_long(m):
    def window_positions(t, L_m, n):
        lo, hi = max(L_m + 1, L_m + t - n), L_m + t
        return np.arange(lo, hi + 1) if hi >= lo else np.zeros(0, np.int64)
    m.window_positions = window_positions


def _mut_query_index(m):
    # query at packed position p taken as output t = p - L_m (drops itself)
    orig = m.visible_positions

    def packed_visible_positions(p, L_m, n):
        if p <= L_m:
            return np.arange(1, p + 1)
        return orig(p - L_m, L_m, n)
    m.packed_visible_positions = packed_visible_positions


def _mut_prefix_bidirectional(m):
    orig = m.packed_visible_positions

    def packed_visible_positions(p, L_m, n):
        if p <= L_m:
            return np.arange(1, L_m + 1)
        return orig(p, L_m, n)
    m.packed_visible_positions = packed_visible_positions


def _mut_no_scale(m):
    orig = m.attend
    m.attend = lambda q, K, V, scale: orig(q, K, V, 1.0)
    m._default_scale = lambda d, scale: 1.0


def _mut_swap_kv(m):
    orig = m.attend
    m.attend = lambda q, K, V, scale: orig(q, V, K, scale)
    orig_mf = m.masked_forward
    m.masked_forward = lambda Q, K, V, L_m, n, scale=None: orig_mf(Q, V, K, L_m, n, scale)


def _mut_sign(m):
    orig = m.attend
    m.attend = lambda q, K, V, scale: orig(-np.asarray(q), K, V, scale)
    orig_mf = m.masked_forward
    m.masked_forward = lambda Q, K, V, L_m, n, scale=None: orig_mf(-np.asarray(Q), K, V, L_m, n, scale)


def _mut_softmax_axis(m):
    def masked_forward(Q, K, V, L_m, n, scale=None):
        Q, K, V = (np.asarray(x, np.float64) for x in (Q, K, V))
        L, H, d = Q.shape
        sc = 1.0 / math.sqrt(d) if not scale else scale
        M = m.packed_mask(L, L_m, n)
        O = np.empty_like(Q)
        for h in range(H):
            S = np.where(M, (Q[:, h] @ K[:, h].T) * sc, -np.inf)
            W = np.exp(S - S.max(axis=1, keepdims=True))
            W = W / W.sum(axis=0, keepdims=True)          # wrong axis
            O[:, h] = W @ V[:, h]
        return O
    m.masked_forward = masked_forward


def _mut_ring_slot(m):
    m.ring_slot = lambda j, n: j % n


def _mut_queue_evicts_reference(m):
    class Q(m.QueueCache):
        def push(self, k, v):
            if len(self.entries) == self.L_m + self.n:
                del self.entries[self.L_m - 1]
            self.T += 1
            self.entries.append((self.L_m + self.T, np.array(k, float), np.array(v, float)))
    m.QueueCache = Q


def _mut_occupancy(m):
    m.occupancy_rswa = lambda T, L_m, n: L_m + min(n, T + 1)


def _mut_decode_window(m):
    orig = m.visible_positions
    m.decode_visible_positions = lambda T, L_m, n: orig(max(T, 1), L_m, n)


def _mut_swa_keeps_first_token(m):
    # the window forgets that there is no reference segment: key 1 stays visible
    orig = m.packed_visible_positions

    def packed_visible_positions(p, L_m, n):
        vis = orig(p, L_m, n)
        return np.union1d(vis, [1]) if L_m == 0 else vis
    m.packed_visible_positions = packed_visible_positions


def _mut_bidir_stays_causal(m):
    m.bidir_prefix_visible_positions = lambda p, L_m, n: m.packed_visible_positions(p, L_m, n)


def _mut_bidir_sees_outputs(m):
    # prefix queries also see the first output
    orig = m.bidir_prefix_visible_positions
    m.bidir_prefix_visible_positions = lambda p, L_m, n: (
        np.arange(1, L_m + 2) if p <= L_m else orig(p, L_m, n))


def _mut_varlen_global_positions(m):
    # forgets to shift a document's local positions back to pack positions
    def varlen_visible_positions(g, cu_seqlens, ref_lens, n, bidir_prefix=False):
        cu = [int(x) for x in cu_seqlens]
        i = next(k for k in range(len(cu) - 1) if cu[k] < g <= cu[k + 1])
        return m.packed_visible_positions(g, int(ref_lens[i]), n)
    m.varlen_visible_positions = varlen_visible_positions


def _mut_varlen_crosses_documents(m):
    # the whole pack treated as one sequence with the first document's L_m
    m.varlen_mask = lambda cu, refs, n, bidir_prefix=False: m.packed_mask(int(cu[-1]), int(refs[0]), n,
                                                                        bidir_prefix)


def _mut_varlen_wrong_document(m):
    # a query on a document's first row is taken as the last row of the previous one
    orig = m.varlen_visible_positions

    def varlen_visible_positions(g, cu_seqlens, ref_lens, n, bidir_prefix=False):
        cu = [int(x) for x in cu_seqlens]
        if g - 1 in cu[1:-1]:
            return orig(g - 1, cu_seqlens, ref_lens, n, bidir_prefix)
        return orig(g, cu_seqlens, ref_lens, n, bidir_prefix)
    m.varlen_visible_positions = varlen_visible_positions


MUTANTS = [
    _mut_window_short, _mut_window_long, _mut_query_index, _mut_prefix_bidirectional,
    _mut_no_scale, _mut_swap_kv, _mut_sign, _mut_softmax_axis, _mut_ring_slot,
    _mut_queue_evicts_reference, _mut_occupancy, _mut_decode_window,
    _mut_swa_keeps_first_token, _mut_bidir_stays_causal, _mut_bidir_sees_outputs,
    _mut_varlen_global_positions, _mut_varlen_crosses_documents, _mut_varlen_wrong_document,
]


# a planted mistake can leave a query with no visible key (a row of -inf)
@pytest.mark.filterwarnings("ignore:invalid value encountered:RuntimeWarning")
@pytest.mark.parametrize("mutate", MUTANTS, ids=lambda f: f.__name__[5:])
def test_pins_catch_planted_mistake(mutate):
    m = _fresh_oracle()
    mutate(m)
    failed = []
    for pin in pins.ALL_PINS:
        try:
            pin(m)
        except Exception:  # any failure means the pin noticed
            failed.append(pin.__name__)
    assert failed, f"no pin caught {mutate.__name__}"


def test_oracle_rejects_bad_arguments():
    for cu, refs in (([1, 4], [1]), ([0, 4, 4], [1, 0]), ([0, 4], [5]), ([0, 4], [1, 1]), ([0, 3], [-1])):
        with pytest.raises(ValueError):
            oracle.varlen_mask(cu, refs, 2)
    with pytest.raises(ValueError):
        oracle.window_positions(0, 3, 2)
    with pytest.raises(ValueError):
        oracle.window_positions(1, 3, 0)
    with pytest.raises(ValueError):
        oracle.decode_visible_positions(-1, 3, 2)
    with pytest.raises(ValueError):
        oracle.ring_slot(0, 4)
