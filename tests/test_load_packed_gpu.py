"""GPU tests of rswa_load_packed, the seam from the packed (teacher-forced)
layout to the decode cache: the cache it writes equals, bit for bit, the one
that a reference load plus T0 appends leaves, and decoding continues from it
in agreement with the oracle."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from reference_sliding_window_b200 import MODE_FULL, MODE_RSWA, RSWA, RSWAError, masked_forward, synth
from tests.gpu_util import assert_close, compare_steps, make_attn, run_steps

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


@pytest.fixture(params=["auto", "span"])
def plan(request, monkeypatch):
    if request.param == "span":
        monkeypatch.setenv("RSWA_DECODE_PLAN", "span")
    else:
        monkeypatch.delenv("RSWA_DECODE_PLAN", raising=False)
    return request.param


def packed_kv(case: synth.DecodeCase, T0: int, pad: int = 3):
    """[B, L, H, d] packed K, V of the case's first T0 outputs: reference rows
    [0, L_m[b]), output t at row L_m[b] + t - 1, the rest filled with a
    constant that must never reach the cache."""
    L = case.L_m_cap + T0 + pad
    shape = (case.B, L, case.H, case.d)
    K = torch.full(shape, 7.0, dtype=case.K_ref.dtype)
    V = torch.full(shape, -7.0, dtype=case.K_ref.dtype)
    for b, Lb in enumerate(case.ref_lens):
        K[b, :Lb] = case.K_ref[b, :, :Lb].transpose(0, 1)
        V[b, :Lb] = case.V_ref[b, :, :Lb].transpose(0, 1)
        K[b, Lb:Lb + T0] = case.k[:T0, b]
        V[b, Lb:Lb + T0] = case.v[:T0, b]
    return K.cuda(), V.cuda()


def check_cache(a: RSWA, case, Kp, Vp, T0: int, full: bool):
    kc, vc = a.k_cache.cpu(), a.v_cache.cpu()
    Kp, Vp = Kp.cpu(), Vp.cpu()
    assert a.step_count() == [T0] * case.B
    for b, L in enumerate(case.ref_lens):
        want = (np.arange(1, L + T0 + 1, dtype=np.int64) if full
                else oracle.ring_storage_positions(T0, L, case.n))
        assert np.array_equal(a.cache_positions(b), want)
        for r, pos in enumerate(want):
            assert torch.equal(kc[b, :, r], Kp[b, int(pos) - 1]), (b, r, int(pos))
            assert torch.equal(vc[b, :, r], Vp[b, int(pos) - 1]), (b, r, int(pos))
        # rows past the occupied ones are untouched (zero since allocation)
        assert not kc[b, :, len(want):].any() and not vc[b, :, len(want):].any()


@pytest.mark.parametrize("dtype,d", [("f32", 64), ("bf16", 128)])
@pytest.mark.parametrize("T0", [0, 5, 8, 9, 29])
def test_load_packed_equals_reference_load_plus_appends(dtype, d, T0, plan):
    n = 8
    case = synth.decode_case(B=3, H=2, d=d, ref_lens=[5, 37, 1], n=n, T=T0 + 2 * n + 1, dtype=dtype,
                             seed=40 + T0)
    Kp, Vp = packed_kv(case, T0)
    a = RSWA(case.L_m_cap, n, case.H, d, case.B, synth.torch_dtype(dtype))
    a.load_packed(Kp, Vp, case.ref_lens, T0)
    torch.cuda.synchronize()
    assert a.cache_len() == [oracle.occupancy_rswa(T0, L, n) for L in case.ref_lens]
    check_cache(a, case, Kp, Vp, T0, full=False)
    # the incremental path reaches the same occupied rows
    b_ = make_attn(case)
    run_steps(b_, case, T0, sample=set())
    for b, L in enumerate(case.ref_lens):
        occ = oracle.occupancy_rswa(T0, L, n)
        assert torch.equal(a.k_cache[b, :, :occ], b_.k_cache[b, :, :occ])
        assert torch.equal(a.v_cache[b, :, :occ], b_.v_cache[b, :, :occ])
    # decoding continues: outputs T0+1 .. T0+2n+1 against the oracle
    outs = run_steps(a, case, case.T, start=T0 + 1)
    compare_steps(case, outs)


def test_load_packed_full_mode():
    T0, T_cap = 13, 40
    case = synth.decode_case(B=2, H=2, d=128, ref_lens=[70, 9], n=4, T=T_cap, dtype="bf16", seed=50)
    Kp, Vp = packed_kv(case, T0)
    a = RSWA(case.L_m_cap, case.n, case.H, case.d, case.B, torch.bfloat16, mode=MODE_FULL, T_cap=T_cap)
    a.load_packed(Kp, Vp, case.ref_lens, T0)
    torch.cuda.synchronize()
    assert a.cache_len() == [L + T0 for L in case.ref_lens]
    check_cache(a, case, Kp, Vp, T0, full=True)
    outs = run_steps(a, case, T_cap, start=T0 + 1)
    compare_steps(case, outs, full=True)
    with pytest.raises(RSWAError, match="CAPACITY"):
        a.load_packed(Kp, Vp, case.ref_lens, T_cap + 1)


def test_prefill_then_decode(plan):
    """Teacher-forced prefill of L_m reference tokens + T0 outputs, its K/V
    loaded into the cache, then decode steps: each step's output is the
    packed form's row for that output (same visible set), and both agree
    with the oracle."""
    L_m, n, T0, extra, H, d = 300, 16, 50, 6, 2, 128
    L = L_m + T0 + extra
    Q, K, V = synth.prefill_case(L, H, d, "bf16", seed=51)
    O = masked_forward(Q.cuda(), K.cuda(), V.cuda(), L_m=L_m, n=n)
    a = RSWA(L_m, n, H, d, 1, torch.bfloat16)
    a.load_packed(K[:L_m + T0].cuda(), V[:L_m + T0].cuda(), [L_m], T0)
    rows = list(range(L_m + T0, L))
    want = oracle.masked_forward_rows(Q.double().numpy(), K.double().numpy(), V.double().numpy(), L_m, n, rows)
    for i, p in enumerate(rows):
        o = a.append_decode(K[p].unsqueeze(0).cuda(), V[p].unsqueeze(0).cuda(), Q[p].unsqueeze(0).cuda())
        torch.cuda.synchronize()
        assert_close(o[0], want[i], "bf16", f"decode row {p}")
        assert_close(O[p], want[i], "bf16", f"packed row {p}")
    a.check()


def test_load_packed_rejects_bad_sizes():
    case = synth.decode_case(B=2, H=2, d=64, ref_lens=[6, 3], n=4, T=4, dtype="f32", seed=52)
    Kp, Vp = packed_kv(case, 2, pad=0)  # L = 6 + 2
    a = RSWA(case.L_m_cap, case.n, case.H, case.d, case.B, torch.float32)
    with pytest.raises(RSWAError, match="CAPACITY"):
        a.load_packed(Kp, Vp, case.ref_lens, 3)  # 6 + 3 rows > L = 8
    with pytest.raises(RSWAError, match="ARG"):
        a.load_packed(Kp, Vp, case.ref_lens, -1)
    with pytest.raises(RSWAError, match="CAPACITY"):
        a.load_packed(Kp, Vp, [7, 3], 0)  # above L_m_cap = 6
    with pytest.raises(ValueError):
        a.load_packed(Kp[:1], Vp[:1], case.ref_lens, 0)
    with pytest.raises(RSWAError, match="STATE"):
        a.decode(torch.zeros(2, 2, 64, device="cuda"))  # nothing loaded yet


@pytest.mark.parametrize("dtype,d,L,L_m,n,mode,bidir", [
    ("bf16", 128, 1000, 300, 128, MODE_RSWA, False),   # the ring's rows span two key tiles
    ("bf16", 128, 700, 256, 64, MODE_RSWA, False),     # L_m on a tile boundary
    ("bf16", 128, 2000, 513, 200, MODE_RSWA, True),    # ring wider than a tile; bidirectional prefix
    ("bf16", 128, 300, 300, 16, MODE_RSWA, False),     # no outputs yet: reference only
    ("bf16", 128, 400, 399, 16, MODE_RSWA, False),     # one output
    ("bf16", 128, 700, 300, 16, MODE_FULL, False),     # full cache: every output kept
    ("f32", 64, 500, 200, 32, MODE_RSWA, False),       # CUDA-core path: attention, then a copy
])
def test_prefill_fill_leaves_the_cache_of_a_load_plus_appends(dtype, d, L, L_m, n, mode, bidir, plan):
    """rswa_masked_forward_fill: O bit for bit the plain masked forward's,
    the cache bit for bit rswa_load_packed's (which tests above pin to a
    reference load plus appends), and decoding continues in agreement with
    the oracle, on spiked queries."""
    H, T0, extra = 2, L - L_m, 9
    Q, K, V = synth.prefill_case(L + extra, H, d, dtype, seed=L + n + 61)
    full = mode == MODE_FULL
    T_cap = T0 + extra if full else 0
    n_att = L if full else n
    Qc, Kc, Vc = Q[:L].cuda(), K[:L].cuda(), V[:L].cuda()
    a = RSWA(L_m, n, H, d, 1, synth.torch_dtype(dtype), mode=mode, T_cap=T_cap)
    O = a.prefill(Qc, Kc, Vc, L_m=L_m, bidir_prefix=bidir)
    O_ref = masked_forward(Qc, Kc, Vc, L_m=L_m, n=n_att, bidir_prefix=bidir)
    ref = RSWA(L_m, n, H, d, 1, synth.torch_dtype(dtype), mode=mode, T_cap=T_cap)
    ref.load_packed(Kc, Vc, [L_m], T0)
    torch.cuda.synchronize()
    assert torch.equal(O, O_ref)
    assert a.step_count() == [T0]
    assert np.array_equal(a.cache_positions(0), ref.cache_positions(0))
    occ = a.cache_len()[0]
    assert torch.equal(a.k_cache[0, :, :occ], ref.k_cache[0, :, :occ])
    assert torch.equal(a.v_cache[0, :, :occ], ref.v_cache[0, :, :occ])
    # decode outputs T0+1 .. T0+extra: packed rows L .. L+extra-1 are their tokens
    rows = list(range(L, L + extra))
    Qs = synth.spike_packed_queries(Q, K, [(r, r - (n if not full else 1) + 1) for r in rows])
    Kd, Vd, Qd = K.double().numpy(), V.double().numpy(), Qs.double().numpy()
    want = oracle.masked_forward_rows(Qd, Kd, Vd, L_m, n_att, rows, bidir_prefix=bidir)
    for i, r in enumerate(rows):
        o = a.append_decode(K[r].unsqueeze(0).cuda(), V[r].unsqueeze(0).cuda(), Qs[r].unsqueeze(0).cuda())
        torch.cuda.synchronize()
        assert_close(o[0], want[i], dtype, f"decode after fill, row {r}")
    a.check()


def test_prefill_fill_rejects_bad_arguments():
    a = RSWA(100, 8, 2, 128, 2, torch.bfloat16)
    Q = torch.zeros(120, 2, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(RSWAError, match="UNSUPPORTED"):  # batch 2
        a.prefill(Q, Q, Q, L_m=100)
    b = RSWA(100, 8, 2, 128, 1, torch.bfloat16)
    with pytest.raises(RSWAError, match="CAPACITY"):
        b.prefill(Q, Q, Q, L_m=101)
    with pytest.raises(RSWAError, match="ARG"):
        b.prefill(Q, Q, Q, L_m=0)
    c = RSWA(100, 8, 2, 128, 1, torch.bfloat16, mode=MODE_FULL, T_cap=10)
    with pytest.raises(RSWAError, match="CAPACITY"):
        c.prefill(Q, Q, Q, L_m=100)  # 20 outputs > T_cap
