"""GPU tests of two library features around the decode step:

* rswa_load_reference_chunk: a reference written chunk by chunk (say page
  by page) gives, bit for bit, the cache of one rswa_load_reference of the
  concatenated rows, and decoding from it matches the oracle;
* rswa_append_decode_layers: one decode step over R layer handles (an
  R-layer decoder's attention), eager and replayed from a CUDA graph, every
  layer checked against the oracle at sampled steps.

Spec: "Unlimited OCR Works", 方法展开 §3-§4 (the reference is encoded once
and never updated; the Eq.(6) cache of each layer).
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

from reference_sliding_window_b200 import RSWA, LayerStep, RSWAError, append_decode_layers, synth
from tests import spikes
from tests.gpu_util import compare_steps, make_attn, run_steps

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _chunks(ref_lens, sizes):
    """Per-chunk row counts per sequence: consecutive pieces of `sizes` rows
    until each sequence's reference is used up (0 once it is)."""
    out, done = [], [0] * len(ref_lens)
    for sz in sizes:
        rows = [max(0, min(sz, L - d)) for L, d in zip(ref_lens, done)]
        out.append(rows)
        done = [d + r for d, r in zip(done, rows)]
    assert done == list(ref_lens)
    return out


@pytest.mark.parametrize("dtype,d", [("bf16", 128), ("f32", 64)])
def test_reference_in_chunks_equals_one_load(dtype, d):
    ref_lens = [2592, 300, 517]
    case = synth.decode_case(B=3, H=2, d=d, ref_lens=ref_lens, n=16, T=40, dtype=dtype, seed=60)
    one = make_attn(case)
    dev = one.device
    a = RSWA(case.L_m_cap, case.n, case.H, case.d, case.B, synth.torch_dtype(dtype), device=dev)
    with pytest.raises(RSWAError, match="STATE"):
        a.decode(case.q[0].to(dev))  # nothing loaded yet
    Kr, Vr = case.K_ref.to(dev), case.V_ref.to(dev)
    done = [0] * case.B
    for rows in _chunks(ref_lens, [256, 256, 1000, 256, 2000]):  # page-sized, then larger pieces
        width = max(rows) or 1
        Kc = torch.zeros((case.B, case.H, width, d), dtype=Kr.dtype, device=dev)
        Vc = torch.zeros_like(Kc)
        for b, r in enumerate(rows):
            Kc[b, :, :r] = Kr[b, :, done[b]:done[b] + r]
            Vc[b, :, :r] = Vr[b, :, done[b]:done[b] + r]
        a.load_reference_chunk(Kc, Vc, rows)
        done = [x + r for x, r in zip(done, rows)]
    torch.cuda.synchronize()
    assert a.cache_len() == ref_lens
    for b, L in enumerate(ref_lens):
        assert torch.equal(a.k_cache[b, :, :L], one.k_cache[b, :, :L])
        assert torch.equal(a.v_cache[b, :, :L], one.v_cache[b, :, :L])
    outs = run_steps(a, case, case.T, sample={1, 16, 17, 40})
    compare_steps(case, outs)
    with pytest.raises(RSWAError, match="STATE"):  # the ring now follows the reference rows
        a.load_reference_chunk(Kc, Vc, [1] * case.B)
    a.reset()
    with pytest.raises(RSWAError, match="CAPACITY"):  # past L_m_cap
        a.load_reference_chunk(Kc, Vc, [1] * case.B)
    a.check()


@pytest.mark.parametrize("graph,R", [(False, 4), (True, 4), ("step", 4), ("graphstep", 4), ("graphstep", 2)])
def test_layers_call_every_layer_matches_the_oracle(graph, R):
    """R layers of different reference lengths and the same batch; the
    queries spike on window edges at the sampled steps.  With R = 2 each
    decode's previous kernel is the other layer's, the tightest case for
    copying ring rows before the dependency wait."""
    T, n = 150, 16
    cases = [synth.decode_case(B=2, H=2, d=128, ref_lens=[300 + 37 * r, 41 + r], n=n, T=T, dtype="bf16",
                               seed=70 + r) for r in range(R)]
    edge_steps = {1, n, n + 1, 2 * n + 1, T}
    prev_steps = {n + 5, T - 1}  # queries on the output the previous step appended
    steps = edge_steps | prev_steps
    for c in cases:
        synth.spike_decode_queries(c, spikes.decode_edge_probes(sorted(edge_steps), c.ref_lens, n))
        synth.spike_decode_queries(c, [(t, b, c.ref_lens[b] + t - 1) for t in sorted(prev_steps) for b in range(c.B)])
    layers = [make_attn(c) for c in cases]
    dev = layers[0].device
    ins = [tuple(t.to(dev) for t in (c.k, c.v, c.q)) for c in cases]
    outs = [torch.empty_like(ins[r][2][0]) for r in range(R)]
    got = {r: {} for r in range(R)}
    if graph in ("step", "graphstep"):  # fixed buffers refilled in place, one prebuilt call per step
        kin = [x[0][0].clone() for x in ins]
        vin = [x[1][0].clone() for x in ins]
        qin = [x[2][0].clone() for x in ins]
        step = LayerStep(layers, kin, vin, qin, outs, graph=graph == "graphstep")
        for t in range(1, T + 1):
            for r in range(R):
                kin[r].copy_(ins[r][0][t - 1])
                vin[r].copy_(ins[r][1][t - 1])
                qin[r].copy_(ins[r][2][t - 1])
            step()
            if t in steps:
                for r in range(R):
                    got[r][t] = outs[r].clone()
    elif not graph:
        for t in range(1, T + 1):
            append_decode_layers(layers, [x[0][t - 1] for x in ins], [x[1][t - 1] for x in ins],
                                 [x[2][t - 1] for x in ins], out=outs)
            if t in steps:
                for r in range(R):
                    got[r][t] = outs[r].clone()
    else:
        kin = [x[0][0].clone() for x in ins]
        vin = [x[1][0].clone() for x in ins]
        qin = [x[2][0].clone() for x in ins]
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            append_decode_layers(layers, kin, vin, qin, out=outs)  # step 1, eager
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                append_decode_layers(layers, kin, vin, qin, out=outs)
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        for r in range(R):
            got[r][1] = outs[r].clone()
        for t in range(2, T + 1):
            for r in range(R):
                kin[r].copy_(ins[r][0][t - 1])
                vin[r].copy_(ins[r][1][t - 1])
                qin[r].copy_(ins[r][2][t - 1])
            g.replay()
            if t in steps:
                torch.cuda.synchronize()
                for r in range(R):
                    got[r][t] = outs[r].clone()
    torch.cuda.synchronize()
    for r in range(R):
        assert layers[r].step_count() == [T, T]
        layers[r].check()
        compare_steps(cases[r], got[r])


def test_layers_call_checks_everything_before_launching():
    case = synth.decode_case(B=1, H=2, d=64, ref_lens=[20], n=4, T=2, dtype="f32", seed=80)
    a, b = make_attn(case), make_attn(case)
    k = case.k[0].cuda()
    bad = torch.zeros(1, 2, 32, device="cuda")
    with pytest.raises(ValueError):
        append_decode_layers([a, b], [k, bad], [k, k], [k, k])
    with pytest.raises(RSWAError, match="ARG"):
        append_decode_layers([a, a], [k, k], [k, k], [k, k])  # the same handle twice
    torch.cuda.synchronize()
    assert a.step_count() == [0] and b.step_count() == [0]  # nothing ran
