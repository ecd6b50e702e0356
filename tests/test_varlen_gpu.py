"""GPU parity tests of the teacher-forced form over a pack of several
documents (rswa_masked_forward_varlen) against the fp64 oracle, through the
C ABI.  Documents see only their own keys; each document's rows must also
equal, bit for bit, a standalone call on that document.  This file is
collected after the other GPU tests so that a failure here leaves them run.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from reference_sliding_window_b200 import RSWAError, masked_forward, masked_forward_varlen, synth
from tests.gpu_util import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


@pytest.mark.parametrize("cu,refs,n,H,d,dtype,bidir", [
    # tensor-core kernel (bf16, d=128): a window document, a one-tile
    # document, a plain-window document (L_m = 0), an all-prefix document
    ([0, 300, 428, 956, 1127], [100, 128, 0, 171], 16, 2, 128, "bf16", False),
    ([0, 384, 700], [200, 300], 8, 2, 128, "bf16", True),
    ([0, 256, 640, 1024], [3, 129, 384], 5, 1, 128, "bf16", False),  # documents on tile-pair edges
    # CUDA-core kernel: a one-row document; bf16 with d=64
    ([0, 1, 258, 400], [1, 5, 100], 7, 2, 64, "f32", False),
    ([0, 130, 390], [64, 0], 300, 2, 64, "bf16", False),
])
def test_varlen_every_row(cu, refs, n, H, d, dtype, bidir):
    L = cu[-1]
    Q, K, V = synth.prefill_case(L, H, d, dtype, seed=L + n + 3)
    O = masked_forward_varlen(Q.cuda(), K.cuda(), V.cuda(), cu, refs, n, bidir_prefix=bidir)
    torch.cuda.synchronize()
    want = oracle.masked_forward_varlen(Q.double().numpy(), K.double().numpy(), V.double().numpy(), cu, refs,
                                        n, bidir_prefix=bidir)
    assert_close(O, want, dtype, "varlen forward")
    for i in range(len(refs)):
        a, b = cu[i], cu[i + 1]
        Oi = masked_forward(Q[a:b].cuda(), K[a:b].cuda(), V[a:b].cuda(), L_m=refs[i], n=n, bidir_prefix=bidir)
        torch.cuda.synchronize()
        assert torch.equal(O[a:b], Oi), f"document {i}"


def test_varlen_32k_pack_sampled_rows():
    """A 32768-row pack of documents (single-page and 2-50 page documents in
    a 9:1 mix, each its reference segment then its outputs), 10 heads,
    d=128, n=128, bf16: every document's edge rows plus random rows."""
    L, H, d, n = 32768, 10, 128, 128
    cu, refs = synth.pack_documents(L, seed=32)
    assert len(refs) > 1
    Q, K, V = synth.prefill_case(L, H, d, "bf16", seed=24, device="cuda")
    O = masked_forward_varlen(Q, K, V, cu, refs, n)
    torch.cuda.synchronize()
    rows = set(np.random.default_rng(24).integers(0, L, 32).tolist())
    for i, Lm in enumerate(refs):
        a, b = cu[i], cu[i + 1]
        rows |= {r for r in (a, a + 1, a + Lm - 1, a + Lm, a + Lm + 1, a + Lm + n - 1, a + Lm + n, b - 1)
                 if a <= r < b}
    rows = sorted(rows)
    Qc, Kc, Vc = (t.double().cpu().numpy() for t in (Q, K, V))
    want = oracle.masked_forward_varlen_rows(Qc, Kc, Vc, cu, refs, n, rows)
    assert_close(O[rows], want, "bf16", "varlen 32K pack")


def test_varlen_rejects_bad_documents():
    Q = torch.zeros(16, 2, 64, device="cuda")
    with pytest.raises(ValueError):
        masked_forward_varlen(Q, Q, Q, [0, 8, 15], [1, 1], 2)   # does not end at L
    with pytest.raises(ValueError):
        masked_forward_varlen(Q, Q, Q, [0, 16], [1, 1], 2)      # one entry short
    with pytest.raises(RSWAError, match="ARG"):
        masked_forward_varlen(Q, Q, Q, [0, 8, 16], [9, 1], 2)   # more reference rows than rows
    with pytest.raises(RSWAError, match="ARG"):
        masked_forward_varlen(Q, Q, Q, [0, 8, 8, 16], [1, 0, 1], 2)


@pytest.mark.parametrize("L,L_m,n", [(1, 1, 1), (77, 30, 8), (127, 0, 16), (100, 100, 4)])
def test_tensor_core_kernel_shorter_than_one_tile(L, L_m, n):
    """bf16, d=128 takes the tensor-core kernel; with L < 128 its only query
    tile is part padding (the tensor maps zero-fill rows past L)."""
    Q, K, V = synth.prefill_case(L, 2, 128, "bf16", seed=L + 90)
    O = masked_forward(Q.cuda(), K.cuda(), V.cuda(), L_m=L_m, n=n)
    torch.cuda.synchronize()
    want = oracle.masked_forward(Q.double().numpy(), K.double().numpy(), V.double().numpy(), L_m, n)
    assert_close(O, want, "bf16", "short sequence, tensor-core kernel")


def test_varlen_pack_with_short_documents_on_tensor_cores():
    cu, refs, n = [0, 5, 133, 200, 201, 500], [5, 60, 0, 1, 288], 16
    L = cu[-1]
    Q, K, V = synth.prefill_case(L, 2, 128, "bf16", seed=95)
    O = masked_forward_varlen(Q.cuda(), K.cuda(), V.cuda(), cu, refs, n)
    torch.cuda.synchronize()
    want = oracle.masked_forward_varlen(Q.double().numpy(), K.double().numpy(), V.double().numpy(), cu, refs, n)
    assert_close(O, want, "bf16", "pack with short documents")
