"""GPU parity tests of the teacher-forced (packed prefill) form against the
fp64 oracle, through the C ABI."""

from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from reference_sliding_window_b200 import RSWAError, masked_forward, synth
from tests.gpu_util import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _run(L, L_m, n, H, d, dtype, seed):
    Q, K, V = synth.prefill_case(L, H, d, dtype, seed)
    O = masked_forward(Q.cuda(), K.cuda(), V.cuda(), L_m=L_m, n=n)
    torch.cuda.synchronize()
    return Q, K, V, O


@pytest.mark.parametrize("L,L_m,n,H,d,dtype", [
    (300, 100, 16, 2, 64, "f32"),
    (257, 1, 7, 1, 128, "f32"),
    (64, 64, 4, 2, 64, "f32"),        # all prefix: plain causal
    (1, 1, 1, 1, 64, "f32"),
    (700, 300, 128, 2, 128, "bf16"),
    (520, 129, 1, 3, 128, "bf16"),
    (400, 255, 300, 2, 64, "bf16"),   # window wider than the outputs
    # tensor-core kernel (bf16, d=128), which takes query tiles in pairs:
    (128, 128, 16, 1, 128, "bf16"),   # one tile; its partner lies wholly past L
    (1000, 513, 200, 2, 128, "bf16"), # ragged last pair
    (768, 256, 64, 2, 128, "bf16"),   # L_m on a pair boundary
    (640, 384, 5, 3, 128, "bf16"),    # L_m on a tile boundary inside a pair
    (600, 600, 8, 2, 128, "bf16"),    # L_m = L: causal everywhere
    (900, 100, 10000, 1, 128, "bf16"),  # window wider than the sequence: full causal
])
def test_masked_forward_every_row(L, L_m, n, H, d, dtype):
    Q, K, V, O = _run(L, L_m, n, H, d, dtype, seed=L + n)
    want = oracle.masked_forward(Q.double().numpy(), K.double().numpy(), V.double().numpy(), L_m, n)
    assert_close(O, want, dtype, "masked forward")


@pytest.mark.parametrize("L,L_m,n,H,d,dtype,bidir", [
    # L_m = 0: no reference segment, the plain sliding window
    (300, 0, 16, 2, 64, "f32", False),
    (700, 0, 128, 2, 128, "bf16", False),
    (520, 0, 1, 2, 128, "bf16", False),
    (257, 0, 300, 1, 128, "f32", False),
    # bidirectional prefix
    (300, 100, 16, 2, 64, "f32", True),
    (700, 300, 128, 2, 128, "bf16", True),
    (640, 384, 5, 2, 128, "bf16", True),   # L_m on a tile boundary inside a pair
    (200, 200, 8, 1, 128, "bf16", True),   # all prefix: full attention
])
def test_masked_forward_window_and_prefix_options(L, L_m, n, H, d, dtype, bidir):
    Q, K, V = synth.prefill_case(L, H, d, dtype, seed=L + n + 7)
    O = masked_forward(Q.cuda(), K.cuda(), V.cuda(), L_m=L_m, n=n, bidir_prefix=bidir)
    torch.cuda.synchronize()
    want = oracle.masked_forward(Q.double().numpy(), K.double().numpy(), V.double().numpy(), L_m, n,
                                 bidir_prefix=bidir)
    assert_close(O, want, dtype, "masked forward options")


def test_teacher_forced_full_size_sampled_rows():
    """Packed 32768-token sequence, 10 heads, d=128, L_m=12832 reference
    tokens + 19936 outputs with n=128, bf16: boundary rows plus random rows."""
    L, L_m, n, H, d = 32768, 12832, 128, 10, 128
    Q, K, V = synth.prefill_case(L, H, d, "bf16", seed=21, device="cuda")
    O = masked_forward(Q, K, V, L_m=L_m, n=n)
    torch.cuda.synchronize()
    rng = np.random.default_rng(21)
    rows = sorted({0, 1, 127, 128, L_m - 1, L_m, L_m + 1, L_m + n - 1, L_m + n, L_m + n + 1, L - 1}
                  | set(rng.integers(0, L, 48).tolist()))
    Qc, Kc, Vc = (t.double().cpu().numpy() for t in (Q, K, V))
    want = oracle.masked_forward_rows(Qc, Kc, Vc, L_m, n, rows)
    assert_close(O[rows], want, "bf16", "teacher-forced 32K")


def test_decode_and_packed_forms_agree():
    """The packed row of output t and the decode step that produces it see the
    same keys; both GPU paths must agree with the oracle and each other."""
    from reference_sliding_window_b200 import RSWA
    L_m, n, T, H, d = 90, 8, 30, 2, 64
    L = L_m + T
    Q, K, V = synth.prefill_case(L, H, d, "f32", seed=22)
    O = masked_forward(Q.cuda(), K.cuda(), V.cuda(), L_m=L_m, n=n)
    a = RSWA(L_m, n, H, d, 1, torch.float32)
    Kr = K[:L_m].transpose(0, 1).unsqueeze(0).contiguous().cuda()
    Vr = V[:L_m].transpose(0, 1).unsqueeze(0).contiguous().cuda()
    a.load_reference(Kr, Vr, [L_m])
    for t in range(1, T + 1):
        p = L_m + t - 1  # 0-based row of output t's token
        o = a.append_decode(K[p].unsqueeze(0).contiguous().cuda(), V[p].unsqueeze(0).contiguous().cuda(),
                            Q[p].unsqueeze(0).contiguous().cuda())
        torch.cuda.synchronize()
        assert_close(o[0], O[p].double().cpu().numpy(), "f32", f"t={t}")
    a.check()


def test_masked_forward_rejects_mismatched_tensors():
    Q = torch.zeros(16, 2, 64, device="cuda")
    with pytest.raises(ValueError):
        masked_forward(Q, torch.zeros(16, 2, 32, device="cuda"), Q, L_m=4, n=2)
    with pytest.raises(RSWAError, match="ARG"):
        masked_forward(Q, Q, Q, L_m=17, n=2)
