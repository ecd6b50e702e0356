"""GPU parity tests on spiked inputs: one-key mask errors become O(1) errors.

Each probed query is a multiple of one key placed on an edge of its visible
set (``tests/spikes.py``): the window's oldest key and the one before it, the
reference seam, the diagonal, and the same edges on key-tile, query-pair and
decode-stage seams.  A kernel that gets one of those keys' visibility wrong
misses the oracle by about 3, against a bf16 tolerance of 2e-2; every test
here also checks, on these very inputs, that the oracle's output with the
probed key flipped is more than 0.1 away.  The spikes also lift the running
row maximum far above its first tile's, which drives the tensor-core
kernel's lazy rescale of its accumulator and the decode kernel's correction
factor.  Spec: "Unlimited OCR Works", 方法展开 §3 Eq.(1)-(4); the decode cache
of §4 Eq.(6) and its queue.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from reference_sliding_window_b200 import MODE_FULL, RSWA, masked_forward, synth
from tests import spikes
from tests.gpu_util import assert_close, compare_steps, make_attn, oracle_decode, run_steps
from tests.test_spike_teeth import PACKED_CASES, TEETH, flipped_gap_decode, flipped_gap_packed

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


# ------------------------------------------------------------ packed form

@pytest.mark.parametrize("L,L_m,n,H,bidir", PACKED_CASES)
@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 128), ("f32", 64)])
def test_packed_spikes_every_row(L, L_m, n, H, bidir, dtype, d):
    """Every row against the oracle; the probed rows have teeth.  bf16 with
    d = 128 runs the tcgen05 kernel, the others the CUDA-core kernel."""
    Q, K, V = synth.prefill_case(L, H, d, dtype, seed=L + n + 3)
    probes = spikes.packed_edge_probes(L, L_m, n)
    Qs = synth.spike_packed_queries(Q, K, probes)
    O = masked_forward(Qs.cuda(), K.cuda(), V.cuda(), L_m=L_m, n=n, bidir_prefix=bidir)
    torch.cuda.synchronize()
    Qd, Kd, Vd = (t.double().numpy() for t in (Qs, K, V))
    want = oracle.masked_forward(Qd, Kd, Vd, L_m, n, bidir_prefix=bidir)
    assert_close(O, want, dtype, "spiked masked forward")
    for i, j in probes[::5]:
        assert flipped_gap_packed(Qd, Kd, Vd, L_m, n, i, j, bidir) > TEETH


def test_packed_spikes_32k_config():
    """The 32K teacher-forced config (L_m = 12832 + 19936 outputs, n = 128,
    10 heads, bf16) with 96 probes on its edges, plus random rows."""
    L, L_m, n, H = 32768, 12832, 128, 10
    Q, K, V = synth.prefill_case(L, H, 128, "bf16", seed=79)
    probes = spikes.packed_edge_probes(L, L_m, n, limit=96)
    Qs = synth.spike_packed_queries(Q, K, probes)
    O = masked_forward(Qs.cuda(), K.cuda(), V.cuda(), L_m=L_m, n=n)
    torch.cuda.synchronize()
    rng = np.random.default_rng(79)
    rows = sorted({i for i, _ in probes} | set(rng.integers(0, L, 24).tolist()))
    Qd, Kd, Vd = (t.double().numpy() for t in (Qs, K, V))
    want = oracle.masked_forward_rows(Qd, Kd, Vd, L_m, n, rows)
    assert_close(O[rows], want, "bf16", "spiked 32K")
    for i, j in probes[::8]:
        assert flipped_gap_packed(Qd[:, :2], Kd[:, :2], Vd[:, :2], L_m, n, i, j) > TEETH


# ------------------------------------------------------------------ decode

def _spiked_decode(case, steps, seqs=None):
    probes = spikes.decode_edge_probes(sorted(steps), case.ref_lens, case.n, seqs=seqs)
    synth.spike_decode_queries(case, probes)
    return probes


def _teeth(case, probes, every=3):
    for t, b, pos in probes[::every]:
        assert flipped_gap_decode(case, t, b, pos) > TEETH, (t, b, pos)


@pytest.mark.parametrize("dtype,d,n,ref_lens,fused", [
    ("bf16", 128, 8, [40, 13, 97], True),
    ("bf16", 128, 16, [300, 33], False),
    ("f32", 128, 8, [70, 9], True),
    ("f32", 64, 5, [500], True),
    ("bf16", 64, 16, [33, 2, 17], True),
])
def test_decode_spikes_every_step(dtype, d, n, ref_lens, fused, plan):
    T = 3 * n + 5
    case = synth.decode_case(B=len(ref_lens), H=2, d=d, ref_lens=ref_lens, n=n, T=T, dtype=dtype, seed=90 + n)
    probes = _spiked_decode(case, range(1, T + 1))
    a = make_attn(case)
    outs = run_steps(a, case, T, fused=fused)
    compare_steps(case, outs)
    if dtype == "bf16":
        _teeth(case, probes)


def test_decode_spikes_single_document_full_size(plan):
    """Batch 1, 10 heads, d = 128, L_m = 2592, n = 128, T = 6144, bf16: the
    ring's wrap steps and the run's end, each with a spiked query."""
    case = synth.decode_case(B=1, H=10, d=128, ref_lens=[2592], n=128, T=6144, dtype="bf16", seed=91)
    steps = {1, 2, 127, 128, 129, 130, 255, 256, 257, 3000, 6143, 6144}
    probes = _spiked_decode(case, steps)
    a = make_attn(case)
    outs = run_steps(a, case, case.T, sample=steps)
    compare_steps(case, outs)
    _teeth(case, probes, every=1)


def test_decode_spikes_ragged_full_size():
    """64 sequences of 2-50 pages, 10 heads, n = 128, T = 6144: spiked
    queries at the wrap steps for the longest, shortest, first and last
    sequences."""
    pages = synth.ragged_page_counts(64, seed=13)
    lens = [synth.reference_length(p, 32) for p in pages]
    case = synth.decode_case(B=64, H=10, d=128, ref_lens=lens, n=128, T=6144, dtype="bf16", seed=92,
                             device="cuda")
    bs = sorted({int(np.argmax(lens)), int(np.argmin(lens)), 0, 63})
    steps = {1, 128, 129, 256, 6144}
    probes = _spiked_decode(case, steps, seqs=bs)
    a = make_attn(case)
    outs = run_steps(a, case, case.T, sample=steps)
    compare_steps(case, outs, bs=bs)
    _teeth(case, [p for p in probes if p[0] <= 256], every=2)


def test_decode_spikes_full_mode(plan):
    """The same kernel over the full cache (every output kept, Eq.(5))."""
    case = synth.decode_case(B=2, H=2, d=128, ref_lens=[300, 41], n=8, T=200, dtype="bf16", seed=93)
    steps = {1, 8, 9, 64, 65, 128, 129, 200}
    probes = spikes.decode_edge_probes(sorted(steps), case.ref_lens, case.T)
    synth.spike_decode_queries(case, probes)
    a = make_attn(case, mode=MODE_FULL, T_cap=200)
    outs = run_steps(a, case, case.T, sample=steps)
    compare_steps(case, outs, full=True)


def test_decode_long_horizon_100k_steps():
    """Config of the long-horizon run: batch 8, L_m = 12832 (50 pages),
    n = 128, T = 100000 outputs with ring eviction (heads cut to 2 for
    time).  Spiked queries at sampled steps; occupancy and the position held
    by every cache row bit-exact there; the ring's contents bit-exact at the
    end."""
    B, H, d, n, T, L = 8, 2, 128, 128, 100000, 12832
    case = synth.decode_case(B=B, H=H, d=d, ref_lens=[L] * B, n=n, T=T, dtype="bf16", seed=94, device="cuda")
    steps = {1, n, n + 1, 50000, T - 1, T}
    bs = [0, 5]
    probes = _spiked_decode(case, steps, seqs=bs)
    a = make_attn(case)
    k, v, q = case.k, case.v, case.q
    outs = {}
    for t in range(1, T + 1):
        o = a.append_decode(k[t - 1], v[t - 1], q[t - 1])
        if t in steps:
            outs[t] = o.clone()
            torch.cuda.synchronize()
            assert a.cache_len() == [oracle.occupancy_rswa(t, L, n)] * B
            for b in bs:
                assert np.array_equal(a.cache_positions(b), oracle.ring_storage_positions(t, L, n))
        if t % 4096 == 0:
            torch.cuda.synchronize()
            a.check()
    torch.cuda.synchronize()
    a.check()
    assert a.step_count() == [T] * B
    compare_steps(case, outs, bs=bs)
    _teeth(case, [p for p in probes if p[0] <= n + 1], every=1)
    kc = a.k_cache[:, :, L:L + n].cpu()
    for b in bs:
        for s_, pos in enumerate(oracle.ring_storage_positions(T, L, n)[L:]):
            assert torch.equal(kc[b, :, s_], k[int(pos) - L - 1, b].cpu())
