"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module only draws random numbers and lays them out; it holds none of the
attention arithmetic and no visibility logic.  Values are drawn i.i.d.
N(0, 1) in float32 and then rounded once to the storage dtype, so every
consumer (CUDA path and CPU oracle) reads the same rounded numbers.

Workload shapes follow the pages: a 1024x1024 page is 256 vision tokens
("Unlimited OCR Works：一篇读懂 R-SWA 如何把长文档 OCR 从 for-loop 推向
one-shot", 方法展开 §2), documents have 2 to 50 pages and training sequences
are packed to 32K tokens (实验与证据 §1), and the default output window is
n = 128 (核心导读).
"""

from __future__ import annotations

from dataclasses import dataclass
from typing import List, Optional, Sequence

import numpy as np
import torch

VISION_TOKENS_PER_PAGE = 256

DTYPES = {"f32": torch.float32, "bf16": torch.bfloat16}


def torch_dtype(name: str) -> torch.dtype:
    return DTYPES[name]


def normal(shape: Sequence[int], seed: int, dtype: str = "f32",
           device: str = "cpu") -> torch.Tensor:
    """i.i.d. N(0,1) tensor of ``shape`` rounded to ``dtype``.

    On the CPU the numbers come from numpy's PCG64 (stable across torch
    versions); on a CUDA device from a seeded torch generator on that device
    (used only for inputs too large to draw on the host)."""
    shape = tuple(int(s) for s in shape)
    if device == "cpu":
        x = np.random.default_rng(seed).standard_normal(shape, dtype=np.float32)
        return torch.from_numpy(x).to(DTYPES[dtype])
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32).to(DTYPES[dtype])


def ragged_page_counts(batch: int, seed: int, lo: int = 2, hi: int = 50) -> List[int]:
    """Pages per document, uniform in [lo, hi] (the pages' 2-50 page documents)."""
    rng = np.random.default_rng(seed)
    return [int(x) for x in rng.integers(lo, hi + 1, size=batch)]


def reference_length(pages: int, prompt_tokens: int) -> int:
    """L_m = 256 vision tokens per page + prompt tokens."""
    return VISION_TOKENS_PER_PAGE * pages + prompt_tokens


# Output (text) tokens per page: the pages do not give one.  400 is the ratio
# of the 32K teacher-forced workload (19936 outputs after a 50-page
# reference); each document draws its own from 400 x U[0.5, 1.5].
OUTPUT_TOKENS_PER_PAGE = 400


def pack_documents(total: int, seed: int, prompt_tokens: int = 32,
                   multi_page_share: float = 0.1) -> tuple:
    """Documents packed back to back into one sequence of ``total`` rows, as
    the training data is packed to 32K tokens: single-page documents and
    multi-page ones (2-50 pages) in a 9:1 mix (实验与证据 §1).  Each document is
    its reference segment (256 per page + prompt) followed by its outputs; the
    last one is cut where the pack ends.  -> (cu_seqlens, ref_lens)."""
    rng = np.random.default_rng(seed)
    cu, refs = [0], []
    while cu[-1] < total:
        pages = int(rng.integers(2, 51)) if rng.random() < multi_page_share else 1
        outs = int(round(OUTPUT_TOKENS_PER_PAGE * pages * rng.uniform(0.5, 1.5)))
        room = total - cu[-1]
        L_m = min(reference_length(pages, prompt_tokens), room)
        cu.append(cu[-1] + min(L_m + outs, room))
        refs.append(L_m)
    return cu, refs


@dataclass
class DecodeCase:
    """Inputs of a decode run.

    K_ref, V_ref: [B, H, L_m_cap, d] (rows >= ref_lens[b] are padding, zero).
    k, v, q:      [T, B, H, d] per-step new key/value and query.
    """
    B: int
    H: int
    d: int
    n: int
    T: int
    ref_lens: List[int]
    dtype: str
    K_ref: torch.Tensor
    V_ref: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    q: torch.Tensor

    @property
    def L_m_cap(self) -> int:
        return self.K_ref.shape[2]


def decode_case(B: int, H: int, d: int, ref_lens: Sequence[int], n: int, T: int,
                dtype: str, seed: int, device: str = "cpu",
                L_m_cap: Optional[int] = None) -> DecodeCase:
    ref_lens = [int(x) for x in ref_lens]
    assert len(ref_lens) == B
    cap = max(ref_lens) if L_m_cap is None else int(L_m_cap)
    K_ref = normal((B, H, cap, d), seed * 7 + 1, dtype, device)
    V_ref = normal((B, H, cap, d), seed * 7 + 2, dtype, device)
    for b, L in enumerate(ref_lens):
        K_ref[b, :, L:] = 0
        V_ref[b, :, L:] = 0
    k = normal((T, B, H, d), seed * 7 + 3, dtype, device)
    v = normal((T, B, H, d), seed * 7 + 4, dtype, device)
    q = normal((T, B, H, d), seed * 7 + 5, dtype, device)
    return DecodeCase(B, H, d, n, T, ref_lens, dtype, K_ref, V_ref, k, v, q)


def history(case: DecodeCase, b: int, T: int) -> tuple:
    """Full (never evicted) history of sequence b after T appends, as float64
    numpy arrays [L_m + T, H, d]: reference rows, then outputs 1..T.  Pure
    re-layout of the generated tensors (for the oracle)."""
    L = case.ref_lens[b]
    Kh = torch.cat([case.K_ref[b, :, :L].transpose(0, 1), case.k[:T, b]], dim=0)
    Vh = torch.cat([case.V_ref[b, :, :L].transpose(0, 1), case.v[:T, b]], dim=0)
    return (Kh.to(torch.float64).cpu().numpy(), Vh.to(torch.float64).cpu().numpy())


def prefill_case(L: int, H: int, d: int, dtype: str, seed: int, device: str = "cpu"):
    """Packed Q, K, V of shape [L, H, d]."""
    Q = normal((L, H, d), seed * 11 + 1, dtype, device)
    K = normal((L, H, d), seed * 11 + 2, dtype, device)
    V = normal((L, H, d), seed * 11 + 3, dtype, device)
    return Q, K, V


# ---------------------------------------------------------------- spike inputs
#
# A query set to a multiple of one key makes that key's score stand far above
# every other score, so the attention output is (almost exactly) that key's
# value row when the key is visible, and something else entirely when it is
# not.  Placing the key on an edge of the visible set turns a one-key error in
# the mask into an O(1) error in the output.  Which (query, key) pairs sit on
# an edge is decided by the caller; these functions only copy rows.

SPIKE_GAIN = 4.0


def spike_packed_queries(Q: torch.Tensor, K: torch.Tensor, probes, gain: float = SPIKE_GAIN) -> torch.Tensor:
    """Copy of Q ([L, H, d]) where, for each (row, key) in ``probes``
    (0-based packed rows, distinct rows), Q[row, h] = gain * K[key, h] for
    every head h, rounded to Q's dtype."""
    Q = Q.clone()
    rows = [int(r) for r, _ in probes]
    if len(set(rows)) != len(rows):
        raise ValueError("one probe per query row")
    if probes:
        r = torch.tensor(rows, device=Q.device)
        k = torch.tensor([int(j) for _, j in probes], device=Q.device)
        Q[r] = (K[k].to(torch.float32) * gain).to(Q.dtype)
    return Q


def history_key(case: DecodeCase, b: int, pos: int) -> torch.Tensor:
    """Key [H, d] at 1-based logical position ``pos`` of sequence b: the
    reference rows 1..L_m[b], then output j at position L_m[b] + j."""
    L = case.ref_lens[b]
    if 1 <= pos <= L:
        return case.K_ref[b, :, pos - 1]
    j = pos - L
    if not 1 <= j <= case.T:
        raise ValueError("position outside the generated history")
    return case.k[j - 1, b]


def spike_decode_queries(case: DecodeCase, probes, gain: float = SPIKE_GAIN) -> None:
    """In place: for each (t, b, pos) in ``probes``, the query of decode step
    t (``case.q[t-1, b]``) becomes gain * (key at logical position pos of
    sequence b), for every head, rounded to the case's dtype."""
    for t, b, pos in probes:
        key = history_key(case, int(b), int(pos)).to(torch.float32)
        case.q[int(t) - 1, int(b)] = (key * gain).to(case.q.dtype)
