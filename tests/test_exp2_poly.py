"""CPU check of the FMA-pipe 2^x used by the tensor-core prefill kernel.

The kernel's constants must be the ones the committed fit script produces,
and the float32 evaluation (Cody-Waite rounding with the 1.5*2^23 shifter,
cubic for 2^f on [-1/2, 1/2], exponent add) must stay within its stated
relative error bound of exp2 over the range the kernel uses."""

from __future__ import annotations

import importlib.util
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "reference_sliding_window_b200", "csrc")


def _fit_module():
    spec = importlib.util.spec_from_file_location("fit_exp2", os.path.join(CSRC, "fit_exp2.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def _kernel_constants():
    src = open(os.path.join(CSRC, "masked_tc.cu")).read()
    m = re.search(r"kC0 = ([0-9.e-]+)f, kC1 = ([0-9.e-]+)f, kC2 = ([0-9.e-]+)f, kC3 = ([0-9.e-]+)f", src)
    assert m, "constants not found in masked_tc.cu"
    return [np.float32(float(x)) for x in m.groups()]


def _exp2_fma_f32(x: np.ndarray, c) -> np.ndarray:
    f32 = np.float32
    x = np.maximum(x.astype(f32), f32(-126.0))
    shift = f32(12582912.0)
    y = (x + shift).astype(f32)
    f = (x - (y - shift)).astype(f32)
    p = f32(c[3])
    for ck in (c[2], c[1], c[0]):
        p = (p * f + f32(ck)).astype(f32)  # the kernel uses fused multiply-add
    n = y.view(np.int32) - np.array(shift, dtype=f32).view(np.int32)
    return (p.view(np.int32) + (n << 23)).view(f32)


def test_kernel_constants_come_from_the_fit():
    fit = _fit_module().fit()
    k = _kernel_constants()
    assert np.allclose(np.array(k, dtype=np.float64), fit.astype(np.float32).astype(np.float64), rtol=0, atol=0)


def test_exp2_fma_relative_error_bound():
    c = _kernel_constants()
    x = np.concatenate([np.linspace(-126.0, 8.0, 400001), np.linspace(-2, 2, 100001)]).astype(np.float32)
    got = _exp2_fma_f32(x, c).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got / want - 1.0)
    assert rel.max() < 1.5e-4, rel.max()          # far below bf16 rounding of P (2^-9)
    assert _fit_module().max_rel_error(np.array(c, dtype=np.float64)) < 1e-4
