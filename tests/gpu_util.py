"""Helpers shared by the GPU parity tests: drive the library through its
binding and compare with the CPU oracle at the tolerances the tests use.

Tolerances:
* float32 storage: per output row, max |o - o*| <= 1e-5 * max(max|o*|, 1e-3)
  (a relative bound that does not blow up when o* is near zero);
* bfloat16 storage (float32 accumulation, bf16 output): max |o - o*| <= 2e-2.
"""

from __future__ import annotations

import numpy as np
import torch

import oracle
from reference_sliding_window_b200 import MODE_FULL, MODE_RSWA, RSWA, synth

F32_REL = 1e-5
BF16_ABS = 2e-2


def assert_close(got: torch.Tensor, want: np.ndarray, dtype: str, what: str = "") -> float:
    """got: [..., d] tensor; want: same shape float64.  Returns the max error."""
    g = got.detach().to(torch.float64).cpu().numpy()
    assert g.shape == want.shape, (g.shape, want.shape)
    assert np.isfinite(g).all(), f"{what}: non-finite output"
    err = np.abs(g - want)
    if dtype == "f32":
        scale = np.maximum(np.abs(want).max(axis=-1, keepdims=True), 1e-3)
        rel = (err / scale).max()
        assert rel <= F32_REL, f"{what}: relative error {rel:.3e} > {F32_REL}"
        return float(rel)
    m = float(err.max())
    assert m <= BF16_ABS, f"{what}: max abs error {m:.3e} > {BF16_ABS}"
    return m


def make_attn(case: synth.DecodeCase, mode: int = MODE_RSWA, T_cap: int = 0) -> RSWA:
    dev = torch.device("cuda")
    a = RSWA(case.L_m_cap, case.n, case.H, case.d, case.B, synth.torch_dtype(case.dtype),
             mode=mode, T_cap=T_cap, device=dev)
    a.load_reference(case.K_ref.to(dev).contiguous(), case.V_ref.to(dev).contiguous(), case.ref_lens)
    return a


def run_steps(a: RSWA, case: synth.DecodeCase, steps, sample=None, fused: bool = True,
              start: int = 1) -> dict:
    """Appends outputs start..steps and decodes after each; returns the
    outputs of the sampled steps (all if sample is None)."""
    dev = a.device
    k, v, q = (t.to(dev) for t in (case.k, case.v, case.q))
    outs = {}
    for t in range(start, steps + 1):
        if fused:
            o = a.append_decode(k[t - 1], v[t - 1], q[t - 1])
        else:
            a.append(k[t - 1], v[t - 1])
            o = a.decode(q[t - 1])
        if sample is None or t in sample:
            outs[t] = o.clone()
        if t % 512 == 0:  # localise any device-side error to a window of steps
            torch.cuda.synchronize()
            a.check()
    torch.cuda.synchronize()
    a.check()
    return outs


def oracle_decode(case: synth.DecodeCase, t: int, b: int, full: bool = False) -> np.ndarray:
    """fp64 oracle output of sequence b after t appends, from the full history."""
    Kh, Vh = synth.history(case, b, t)
    q = case.q[t - 1, b].to(torch.float64).cpu().numpy()
    if full:
        return oracle.decode_step_full(q, Kh, Vh, case.ref_lens[b], t)
    return oracle.decode_step(q, Kh, Vh, case.ref_lens[b], t, case.n)


def compare_steps(case, outs, bs=None, full: bool = False) -> float:
    worst = 0.0
    for t, o in outs.items():
        for b in (range(case.B) if bs is None else bs):
            want = oracle_decode(case, t, b, full)
            worst = max(worst, assert_close(o[b], want, case.dtype, f"step {t} seq {b}"))
    return worst
