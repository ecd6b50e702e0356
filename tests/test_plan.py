"""CPU tests of the decode launch planner (the production code, through the
host-only rswa_plan_decode call): every planned row of every slab is
streamed exactly once, the split-K bookkeeping is consistent, and the work
is balanced.  Both plans: spans over all slabs, and one 8-CTA cluster per
slab."""

from __future__ import annotations

import ctypes as C

import numpy as np
import pytest

from reference_sliding_window_b200 import _native

NSM = 148


def plan(lens, H, window, S_cap, num_sms=NSM, max_clusters=0):
    lib = _native.lib()
    B = len(lens)
    cap_items, cap_ctas = B * H + 1024, 1025
    items = (C.c_int32 * (8 * cap_items))()
    begin = (C.c_int32 * cap_ctas)()
    ni, nc, cl = C.c_int(), C.c_int(), C.c_int()
    st = lib.rswa_plan_decode(B, H, (C.c_int32 * B)(*lens), window, S_cap, num_sms, max_clusters,
                              items, cap_items, begin, cap_ctas, C.byref(ni), C.byref(nc), C.byref(cl))
    _native.check(st)
    it = np.frombuffer(items, dtype=np.int32, count=8 * ni.value).reshape(-1, 8)
    return it, np.frombuffer(begin, dtype=np.int32, count=nc.value + 1).copy(), bool(cl.value)


def check_common(it, begin, lens, H, window, S_cap):
    rows_bh = [min(L + window, S_cap) for L in lens for _ in range(H)]
    nbh = len(rows_bh)
    # every row of every slab exactly once, in contiguous pieces
    cover = [np.zeros(r, dtype=np.int32) for r in rows_bh]
    for bh, row0, rows, part, pfirst, nparts, last, pad in it:
        assert 0 <= bh < nbh and rows >= 0 and pad == 0
        assert row0 % 32 == 0 and row0 + rows <= rows_bh[bh]
        cover[bh][row0:row0 + rows] += 1
    for c in cover:
        assert (c == 1).all()
    # CTAs take consecutive items
    assert begin[0] == 0 and begin[-1] == len(it) and (np.diff(begin) >= 0).all()
    # split-K bookkeeping: a slab's partials are consecutive and agree
    for bh in range(nbh):
        idx = np.nonzero(it[:, 0] == bh)[0]
        assert len(idx) >= 1 and (np.diff(idx) == 1).all()
        assert (it[idx, 4] == idx[0]).all() and (it[idx, 5] == len(idx)).all()
        assert it[idx[-1], 6] == 1 and (it[idx[:-1], 6] == 0).all()
        assert sorted(it[idx, 1].tolist()) == it[idx, 1].tolist()


@pytest.mark.parametrize("seed", range(6))
def test_span_plan(seed):
    rng = np.random.default_rng(seed)
    B, H, n = int(rng.integers(1, 70)), int(rng.integers(1, 12)), int(rng.integers(1, 200))
    lens = [int(x) for x in rng.integers(1, 13000, B)]
    S_cap = max(lens) + n
    it, begin, cluster = plan(lens, H, n, S_cap)
    assert not cluster
    check_common(it, begin, lens, H, n, S_cap)
    G = len(begin) - 1
    assert 1 <= G <= NSM
    assert (it[:, 3] == np.arange(len(it))).all()  # item i is partial i
    # 32-row stages per CTA differ by at most one (the last stage of a slab may be partial)
    stages = [sum((r + 31) // 32 for r in it[begin[c]:begin[c + 1], 2]) for c in range(G)]
    assert max(stages) - min(stages) <= 1
    # at most two items of a CTA share their slab with another CTA
    for c in range(G):
        assert sum(1 for x in it[begin[c]:begin[c + 1]] if x[5] > 1) <= 2


def test_single_document_plans():
    lens, H, n = [2592], 10, 128
    it, begin, cluster = plan(lens, H, n, 2720, max_clusters=16)
    assert cluster and len(begin) - 1 == 80
    check_common(it, begin, lens, H, n, 2720)
    assert (np.diff(begin) == 1).all()                      # one item per CTA
    assert (it[:, 5] == 8).all() and (it[:, 4] == (it[:, 0] * 8)).all()
    assert (it[:, 0] == np.arange(80) // 8).all()           # cluster c holds slab c
    it2, begin2, cluster2 = plan(lens, H, n, 2720, max_clusters=0)
    assert not cluster2 and len(begin2) - 1 == NSM
    check_common(it2, begin2, lens, H, n, 2720)


def test_cluster_plan_needs_a_resident_cluster_per_slab():
    # 17 slabs, 16 resident clusters: the span plan
    _, _, cluster = plan([700] * 17, 1, 128, 828, max_clusters=16)
    assert not cluster
    it, begin, cluster = plan([700] * 16, 1, 128, 828, max_clusters=16)
    assert cluster and len(begin) - 1 == 128
    check_common(it, begin, [700] * 16, 1, 128, 828)


def test_tiny_slabs_leave_some_cluster_ctas_empty():
    it, begin, cluster = plan([3, 40], 2, 8, 48, max_clusters=16)
    assert cluster
    check_common(it, begin, [3, 40], 2, 8, 48)
    assert (it[:, 2] == 0).any()  # fewer 32-row stages than CTAs in a cluster


def test_plan_capacity_and_argument_errors():
    lib = _native.lib()
    items = (C.c_int32 * 8)()
    begin = (C.c_int32 * 2)()
    ni, nc, cl = C.c_int(), C.c_int(), C.c_int()
    st = lib.rswa_plan_decode(1, 10, (C.c_int32 * 1)(2592), 128, 2720, NSM, 0, items, 1, begin, 2,
                              C.byref(ni), C.byref(nc), C.byref(cl))
    assert st == _native.ERR_CAPACITY and ni.value > 1
    st = lib.rswa_plan_decode(1, 10, (C.c_int32 * 1)(0), 128, 2720, NSM, 0, items, 1, begin, 2,
                              C.byref(ni), C.byref(nc), C.byref(cl))
    assert st == _native.ERR_ARG
