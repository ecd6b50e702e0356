"""GPU parity tests of the decode path (append, decode, fused append+decode)
against the fp64 oracle, through the C ABI."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from reference_sliding_window_b200 import MODE_FULL, MODE_RSWA, RSWA, RSWAError, synth
from tests.gpu_util import assert_close, compare_steps, make_attn, oracle_decode, run_steps

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


@pytest.fixture(params=["auto", "span"])
def plan(request, monkeypatch):
    """Both decode plans: the library's choice (the cluster merge for these
    few-slab cases) and the span plan with its merge across CTAs."""
    if request.param == "span":
        monkeypatch.setenv("RSWA_DECODE_PLAN", "span")
    else:
        monkeypatch.delenv("RSWA_DECODE_PLAN", raising=False)
    return request.param


# ------------------------------------------------------------ index parity

@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_ring_slots_and_reference_rows_bit_exact(dtype):
    """Which output sits in which cache row, bit for bit, after every step;
    the reference rows never change; occupancy follows Eq.(6)."""
    case = synth.decode_case(B=3, H=2, d=64, ref_lens=[5, 37, 1], n=8, T=30, dtype=dtype, seed=1)
    a = make_attn(case)
    dev = a.device
    k, v, q = (t.to(dev) for t in (case.k, case.v, case.q))
    for t in range(0, case.T + 1):
        if t > 0:
            a.append_decode(k[t - 1], v[t - 1], q[t - 1])
        torch.cuda.synchronize()
        assert a.cache_len() == [oracle.occupancy_rswa(t, L, case.n) for L in case.ref_lens]
        assert a.step_count() == [t] * case.B
        kc, vc = a.k_cache.cpu(), a.v_cache.cpu()
        for b, L in enumerate(case.ref_lens):
            want_pos = oracle.ring_storage_positions(t, L, case.n)
            assert np.array_equal(a.cache_positions(b), want_pos)
            assert torch.equal(kc[b, :, :L], case.K_ref[b, :, :L])
            assert torch.equal(vc[b, :, :L], case.V_ref[b, :, :L])
            for s, pos in enumerate(want_pos[L:]):
                j = int(pos) - L  # output index stored in ring slot s
                assert torch.equal(kc[b, :, L + s], case.k[j - 1, b]), (t, b, s, j)
                assert torch.equal(vc[b, :, L + s], case.v[j - 1, b]), (t, b, s, j)
    a.check()


def test_standalone_append_writes_the_same_rows():
    case = synth.decode_case(B=2, H=3, d=128, ref_lens=[10, 3], n=4, T=11, dtype="bf16", seed=2)
    a = make_attn(case)
    dev = a.device
    for t in range(1, case.T + 1):
        a.append(case.k[t - 1].to(dev), case.v[t - 1].to(dev))
    kc = a.k_cache.cpu()
    for b, L in enumerate(case.ref_lens):
        for s, pos in enumerate(oracle.ring_storage_positions(case.T, L, case.n)[L:]):
            assert torch.equal(kc[b, :, L + s], case.k[int(pos) - L - 1, b])
    a.check()


# ---------------------------------------------------------- numeric parity

def test_config_tiny_f32_every_step():
    """Batch 1, 2 heads, d=64, L_m=272 (256 vision + 16 prompt), n=128,
    T=512, float32: every step against the oracle."""
    case = synth.decode_case(B=1, H=2, d=64, ref_lens=[272], n=128, T=512, dtype="f32", seed=3)
    a = make_attn(case)
    outs = run_steps(a, case, case.T)
    compare_steps(case, outs)


def test_decode_before_any_output_sees_reference_only():
    case = synth.decode_case(B=2, H=2, d=128, ref_lens=[40, 7], n=16, T=1, dtype="f32", seed=4)
    a = make_attn(case)
    q = case.q[0].cuda()
    o = a.decode(q)
    torch.cuda.synchronize()
    for b, L in enumerate(case.ref_lens):
        Kh, Vh = synth.history(case, b, 0)
        want = oracle.decode_step(case.q[0, b].double().numpy(), Kh, Vh, L, 0, case.n)
        assert_close(o[b], want, "f32")
    a.check()


@pytest.mark.parametrize("dtype,d,n,ref_lens,fused", [
    ("f32", 64, 1, [3], True),
    ("f32", 128, 8, [100, 1], False),
    ("bf16", 128, 4, [1, 50], True),
    ("bf16", 64, 16, [33, 2, 17], False),
    ("bf16", 128, 33, [257, 31, 96, 128], True),
    ("f32", 64, 5, [500], True),
])
def test_small_shapes_every_step(dtype, d, n, ref_lens, fused, plan):
    T = 3 * n + 5
    case = synth.decode_case(B=len(ref_lens), H=2, d=d, ref_lens=ref_lens, n=n, T=T, dtype=dtype, seed=5 + n)
    a = make_attn(case)
    outs = run_steps(a, case, T, fused=fused)
    compare_steps(case, outs)


def test_window_wider_than_output_is_full_attention():
    case = synth.decode_case(B=1, H=2, d=64, ref_lens=[60], n=1000, T=50, dtype="f32", seed=6)
    a = make_attn(case)
    outs = run_steps(a, case, case.T)
    compare_steps(case, outs, full=True)


def test_full_mode_and_its_capacity():
    case = synth.decode_case(B=2, H=2, d=128, ref_lens=[70, 9], n=8, T=40, dtype="bf16", seed=7)
    a = make_attn(case, mode=MODE_FULL, T_cap=40)
    outs = run_steps(a, case, case.T)
    compare_steps(case, outs, full=True)
    assert a.cache_len() == [L + 40 for L in case.ref_lens]
    with pytest.raises(RSWAError, match="CAPACITY"):
        a.append(case.k[0].cuda(), case.v[0].cuda())
    a.check()


def test_full_mode_replans_past_first_window(plan):
    # FULL mode plans 64 output rows at a time; cross several boundaries.
    case = synth.decode_case(B=1, H=2, d=64, ref_lens=[30], n=8, T=530, dtype="f32", seed=8)
    a = make_attn(case, mode=MODE_FULL, T_cap=600)
    outs = run_steps(a, case, case.T, sample={1, 511, 512, 513, 530})
    compare_steps(case, outs, full=True)


def test_reset_restarts_outputs_keeps_reference():
    case = synth.decode_case(B=1, H=2, d=64, ref_lens=[20], n=4, T=9, dtype="f32", seed=9)
    a = make_attn(case)
    run_steps(a, case, case.T, sample=set())
    a.reset()
    assert a.step_count() == [0]
    outs = run_steps(a, case, 6)
    compare_steps(case, outs)


def test_state_errors():
    case = synth.decode_case(B=1, H=2, d=64, ref_lens=[20], n=4, T=2, dtype="f32", seed=10)
    a = RSWA(case.L_m_cap, case.n, case.H, case.d, case.B, torch.float32)
    with pytest.raises(RSWAError, match="STATE"):
        a.append(case.k[0].cuda(), case.v[0].cuda())
    with pytest.raises(RSWAError, match="STATE"):
        a.decode(case.q[0].cuda())
    with pytest.raises(RSWAError, match="CAPACITY"):
        a.load_reference(case.K_ref.cuda(), case.V_ref.cuda(), [21])
    with pytest.raises(ValueError):
        a.decode(case.q[0].cuda().to(torch.bfloat16))
    a.check()


# ------------------------------------------------------------- CUDA graphs

def test_graph_replay_advances_the_ring(plan):
    """One captured append+decode replayed step after step: the device step
    counter and slot index make the graph reusable."""
    case = synth.decode_case(B=2, H=2, d=128, ref_lens=[300, 45], n=16, T=60, dtype="bf16", seed=11)
    a = make_attn(case)
    dev = a.device
    k, v, q = (t.to(dev) for t in (case.k, case.v, case.q))
    kin, vin, qin = k[0].clone(), v[0].clone(), q[0].clone()
    out = torch.empty_like(qin)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for t in range(1, 21):          # eager warm-up, also past n
            a.append_decode(k[t - 1], v[t - 1], q[t - 1], out=out)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            a.append_decode(kin, vin, qin, out=out)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    assert a.step_count() == [20, 20]
    for t in range(21, case.T + 1):
        kin.copy_(k[t - 1]); vin.copy_(v[t - 1]); qin.copy_(q[t - 1])
        g.replay()
        if t in (21, 37, 60):
            torch.cuda.synchronize()
            compare_steps(case, {t: out.clone()})
    assert a.step_count() == [case.T, case.T]
    a.check()


# ------------------------------------------------- full-size, sampled outputs

def _device_case(B, H, d, ref_lens, n, T, seed):
    return synth.decode_case(B=B, H=H, d=d, ref_lens=ref_lens, n=n, T=T, dtype="bf16",
                             seed=seed, device="cuda")


def test_single_document_full_size_sampled(plan):
    """Batch 1, 10 heads, d=128, L_m=2592 (10 pages x 256 + 32 prompt),
    n=128, T=6144 steps, bf16: outputs sampled across the run."""
    case = _device_case(1, 10, 128, [2592], 128, 6144, 12)
    a = make_attn(case)
    sample = {1, 2, 127, 128, 129, 130, 256, 3000, 6143, 6144}
    outs = run_steps(a, case, case.T, sample=sample)
    compare_steps(case, outs)


def test_ragged_batch_full_size_sampled():
    """64 sequences, 10 heads, d=128, 2-50 pages each (L_m = 256*pages + 32),
    n=128, T=6144 steps: sampled steps and sequences."""
    pages = synth.ragged_page_counts(64, seed=13)
    lens = [synth.reference_length(p, 32) for p in pages]
    case = _device_case(64, 10, 128, lens, 128, 6144, 13)
    a = make_attn(case)
    outs = run_steps(a, case, case.T, sample={1, 128, 129, 6144})
    bs = sorted({int(np.argmax(lens)), int(np.argmin(lens)), 0, 63})
    compare_steps(case, outs, bs=bs)
