"""GPU test of rswa_decode_noalloc, the decode entry point that allocates
nothing (its scratch is a static device array inside the library).

It exists for callers that cannot allocate device memory: a plugin inside a
framework whose own allocator owns every device allocation, or code that must
avoid the implicit synchronisation of cudaMalloc / cudaFree.  Two calls in a
row, through the C ABI, must match the handle-based rswa_decode on the same
caches and the fp64 oracle, within the tolerances the other GPU tests use,
and leave the device error word clear.  This file is collected last so that
a failure here leaves every other test already run.
"""

from __future__ import annotations

import ctypes as C

import pytest
import torch

import oracle
from reference_sliding_window_b200 import RSWAError, _native, synth
from tests.gpu_util import assert_close, make_attn

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _decode_noalloc(a, q: torch.Tensor, o: torch.Tensor) -> None:
    lens = (C.c_int32 * a.batch)(*a.cache_len())
    dt = _native.BF16 if a.dtype == torch.bfloat16 else _native.F32
    _native.check(_native.lib().rswa_decode_noalloc(
        a.k_cache.data_ptr(), a.v_cache.data_ptr(), a.S_cap, lens, q.data_ptr(), o.data_ptr(),
        a.batch, a.H, a.d, dt, 0.0, _stream()))


@pytest.mark.parametrize("dtype,d,ref_lens,H,n,T", [
    ("bf16", 128, [2592], 10, 128, 140),          # single document: slabs split over many CTAs
    ("bf16", 128, [300, 45, 1000], 4, 16, 40),    # ragged batch
    ("f32", 64, [272], 2, 128, 30),               # tiny float32 case
    ("bf16", 128, [20000], 1, 128, 130),          # one slab spread over every CTA
])
def test_noalloc_matches_handle_decode_two_calls(dtype, d, ref_lens, H, n, T):
    case = synth.decode_case(B=len(ref_lens), H=H, d=d, ref_lens=ref_lens, n=n, T=T + 2,
                             dtype=dtype, seed=41 + d)
    a = make_attn(case)
    dev = a.device
    for t in range(1, T + 1):
        a.append(case.k[t - 1].to(dev), case.v[t - 1].to(dev))
    for call in range(2):  # the second call reuses the scratch the first left behind
        q = case.q[T + call].to(dev)
        ref = a.decode(q)
        got = torch.full_like(q, float("nan"))
        _decode_noalloc(a, q, got)
        torch.cuda.synchronize()
        assert_close(got, ref.to(torch.float64).cpu().numpy(), dtype, f"no-alloc call {call + 1}")
        for b in range(case.B):
            # the state after T appends, queried with the query of step T + call + 1
            Kh, Vh = synth.history(case, b, T)
            want = oracle.decode_step(case.q[T + call, b].double().numpy(), Kh, Vh, case.ref_lens[b], T, n)
            assert_close(got[b], want, dtype, f"no-alloc call {call + 1} vs oracle, seq {b}")
        _native.check(_native.lib().rswa_decode_noalloc_check(_stream()))
    a.check()


def test_noalloc_rejects_sizes_beyond_its_scratch():
    buf = torch.zeros(64, dtype=torch.bfloat16, device="cuda")
    lens = (C.c_int32 * 1025)(*([1] * 1025))
    st = _native.lib().rswa_decode_noalloc(buf.data_ptr(), buf.data_ptr(), 1, lens, buf.data_ptr(),
                                           buf.data_ptr(), 1025, 1, 64, _native.BF16, 0.0, None)
    with pytest.raises(RSWAError, match="CAPACITY.*1024"):
        _native.check(st)
