"""GPU tests of consecutive decode launches on one handle with nothing in
between, captured in one CUDA graph, so each launch may start (and copy
reference rows) while the previous step is still running.  The library
then copies ring rows only after the dependency wait: the previous kernel
on the stream is a decode of the same handle, which may still be writing
its slot row.  Every step is checked against the oracle, with queries
spiked on the output the previous step appended, so a stale copy of that
row fails by O(1).  Also after a packed load and after a reset, and in
FULL mode.

Spec: "Unlimited OCR Works", 方法展开 §3-§4 (Eq.(3)-(4) over the Eq.(6)
cache; output T overwrites the slot of output T - n).
"""

from __future__ import annotations

import pytest
import torch

from reference_sliding_window_b200 import MODE_FULL, synth
from tests.gpu_util import assert_close, compare_steps, make_attn, oracle_decode

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


def _spike_newest(case, steps):
    """At each step t in `steps`, point q at output t - 1 (the row the
    previous launch wrote) so that a stale copy of it moves the output."""
    probes = [(t, b, case.ref_lens[b] + t - 1) for t in steps if t >= 2 for b in range(case.B)]
    synth.spike_decode_queries(case, probes)


def _graph_steps(a, case, t0, t1, with_plain=False):
    """Captures steps t0..t1 of `a` back to back in one graph (and, with
    with_plain, a plain decode of the same query after each), replays it once
    and returns {t: output} (and {t: plain output})."""
    dev = a.device
    k, v, q = (x.to(dev) for x in (case.k, case.v, case.q))
    outs = torch.empty((t1 - t0 + 1,) + tuple(q.shape[1:]), dtype=q.dtype, device=dev)
    plain = torch.empty_like(outs)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            for t in range(t0, t1 + 1):
                a.append_decode(k[t - 1], v[t - 1], q[t - 1], out=outs[t - t0])
                if with_plain:
                    a.decode(q[t - 1], out=plain[t - t0])
    torch.cuda.current_stream().wait_stream(s)
    g.replay()
    torch.cuda.synchronize()
    a.check()
    got = {t: outs[t - t0].clone() for t in range(t0, t1 + 1)}
    got_plain = {t: plain[t - t0].clone() for t in range(t0, t1 + 1)} if with_plain else {}
    del g
    return got, got_plain


@pytest.mark.parametrize("dtype,d,n", [("bf16", 128, 16), ("bf16", 128, 1), ("f32", 64, 5), ("bf16", 64, 3)])
def test_back_to_back_steps_every_output(dtype, d, n, plan):
    T = 3 * max(n, 8) + 7
    case = synth.decode_case(B=2, H=2, d=d, ref_lens=[300, 41], n=n, T=T, dtype=dtype, seed=90 + n)
    _spike_newest(case, range(2, T + 1))
    a = make_attn(case)
    # steps 1..5 eagerly (the graph then starts from a handle with T = 5)
    dev = a.device
    k, v, q = (x.to(dev) for x in (case.k, case.v, case.q))
    for t in range(1, 6):
        a.append_decode(k[t - 1], v[t - 1], q[t - 1])
    got, plain = _graph_steps(a, case, 6, T, with_plain=True)
    compare_steps(case, got)
    for t in got:  # a plain decode after the append sees the same cache and query
        assert torch.equal(got[t], plain[t]), f"step {t}: plain decode differs from the fused step"
    assert a.step_count() == [T, T]


def test_back_to_back_full_mode(plan):
    T = 70
    case = synth.decode_case(B=1, H=2, d=128, ref_lens=[200], n=8, T=T, dtype="bf16", seed=95)
    _spike_newest(case, range(2, T + 1))
    a = make_attn(case, mode=MODE_FULL, T_cap=T)
    got, _ = _graph_steps(a, case, 1, T)
    compare_steps(case, got, full=True)


def test_packed_load_then_back_to_back_steps(plan):
    """After rswa_load_packed the step counter is not a decode's own, so no
    row is replaced; the first graph step must see the packed rows."""
    n, T0, T = 16, 40, 60
    case = synth.decode_case(B=2, H=2, d=128, ref_lens=[300, 41], n=n, T=T, dtype="bf16", seed=97)
    _spike_newest(case, range(T0 + 1, T + 1))
    a = make_attn(case)
    dev = a.device
    # run some steps first so the side copy holds a token that the packed load replaces
    k, v, q = (x.to(dev) for x in (case.k, case.v, case.q))
    for t in range(1, 12):
        a.append_decode(k[t - 1] * 3, v[t - 1] * 3, q[t - 1])
    L = max(case.ref_lens) + T0
    K = torch.zeros((case.B, L, case.H, case.d), dtype=k.dtype, device=dev)
    V = torch.zeros_like(K)
    for b in range(case.B):
        Kh, Vh = synth.history(case, b, T0)
        Lb = case.ref_lens[b] + T0
        K[b, :Lb] = torch.as_tensor(Kh, device=dev).to(k.dtype)
        V[b, :Lb] = torch.as_tensor(Vh, device=dev).to(k.dtype)
    a.load_packed(K, V, case.ref_lens, T0)
    got, _ = _graph_steps(a, case, T0 + 1, T)
    compare_steps(case, got)


def test_reset_then_back_to_back_steps(plan):
    case = synth.decode_case(B=1, H=2, d=128, ref_lens=[150], n=4, T=20, dtype="bf16", seed=99)
    _spike_newest(case, range(2, 21))
    a = make_attn(case)
    dev = a.device
    k, v, q = (x.to(dev) for x in (case.k, case.v, case.q))
    for t in range(1, 9):  # other tokens into the ring and the side copy
        a.append_decode(-k[t - 1], -v[t - 1], q[t - 1])
    a.reset()
    got, _ = _graph_steps(a, case, 1, 20)
    compare_steps(case, got)
    want = oracle_decode(case, 20, 0)
    assert_close(got[20][0], want, "bf16", "step 20 after reset")
