"""Plain, slow, fp64 CPU oracle for Reference Sliding Window Attention (R-SWA).

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports, calls or
executes this module: only the tests, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` use it.  It
shares no code, tables or helpers with the CUDA library; it works on numpy
arrays in float64 and builds the R-SWA visibility set explicitly.

Sources (page title, then the section / equation followed):

[UOW-1] "Unlimited OCR Works：一篇读懂 R-SWA 如何把长文档 OCR 从 for-loop 推向
        one-shot" (WeThinkIn article)
        - 方法展开 §3 "R-SWA 的 attention 计算": Eq.(1) N(t) = P ∪ D_n(t),
          P = {1..L_m}; Eq.(2) D_n(t) = {j | max(L_m+1, L_m+t-n) <= j <= L_m+t-1};
          Eq.(3) softmax of q_t.k_j / sqrt(d_k) normalised over N(t);
          Eq.(4) o_t = sum_{j in N(t)} alpha_tj v_j.
        - 方法展开 §4 "KV cache 管理": Eq.(5) C_MHA(T) = L_m + T;
          Eq.(6) C_R-SWA(T) = L_m + min(n, T) <= L_m + n; Eq.(7)-(9) the ratio.
[UOW-3] "多模态文档解析开源新进展:Unlimited OCR技术方案", section
        "为什么它能“无限”读下去？关键在 KV cache 恒定": the cache is a queue of
        fixed capacity m + n; each new token evicts the oldest output entry,
        the one at position m+1 (m = L_m there).

Readings where the pages leave a step open (each one is also listed in the
design notes):

R1  Query indexing.  Eq.(2) is written for "output token t" and its window
    ends at position L_m+t-1.  We read t as the output being *produced*: the
    query that produces output t is the hidden state at position L_m+t-1.
    So D_n(1) is empty (the last prompt token sees only P) and, in the
    packed form, a query at position p > L_m produces output t = p-L_m+1 and
    sees P plus positions max(L_m+1, p-n+1) .. p (itself included).
R2  Prefix queries (p <= L_m) are causal inside the prefix.  Eq.(1) only
    speaks of output tokens; the decoder is a causal LM with MHA replaced
    one for one, so the prefix keeps the causal mask.
R3  Scale 1/sqrt(d) (Eq.(3)); ``scale`` may be overridden by the caller.
R4  Multi-head attention with H query heads = H key/value heads; heads are
    independent.
R5  Decode after T appends: the query of the newest output T produces
    output T+1 and sees N(T+1) = P ∪ outputs max(1, T+1-n) .. T, which is
    L_m + min(n, T) rows, Eq.(6).
R6  L_m = 0 in the packed form leaves no reference segment: every query p
    sees max(1, p-n+1) .. p, the plain sliding window the pages contrast
    R-SWA with ([UOW-1] 核心导读 Fig. 1 and 方法展开 §1, "vanilla SWA").
R7  Bidirectional prefix (an option; the pages are silent and R2 is the
    default): every prefix query p <= L_m sees all of P = 1..L_m; outputs
    are unchanged.
R8  Several documents in one pack ([UOW-1] 实验与证据 §1 训练设置: samples
    are packed to 32K tokens).  The pages do not say how packed documents
    see each other; we take the plain reading: document i occupies packed
    rows cu_seqlens[i] .. cu_seqlens[i+1]-1 with its own reference length
    ref_lens[i], its queries see only its own keys, and inside it the
    single-sequence mask applies at local positions.
"""

from __future__ import annotations

import math
from typing import List, Sequence

import numpy as np

__all__ = [
    "reference_positions",
    "window_positions",
    "visible_positions",
    "packed_visible_positions",
    "bidir_prefix_visible_positions",
    "packed_mask",
    "attend",
    "masked_forward",
    "masked_forward_rows",
    "varlen_visible_positions",
    "varlen_mask",
    "masked_forward_varlen",
    "masked_forward_varlen_rows",
    "decode_visible_positions",
    "decode_step",
    "occupancy_rswa",
    "occupancy_full",
    "cache_ratio",
    "ring_slot",
    "ring_storage_positions",
    "QueueCache",
]


# --------------------------------------------------------------------------
# Index sets: [UOW-1] Eq.(1)-(2), readings R1, R2, R5.  Positions are 1-based.
# --------------------------------------------------------------------------

def reference_positions(L_m: int) -> np.ndarray:
    """P = {1, ..., L_m} of [UOW-1] Eq.(1)."""
    return np.arange(1, L_m + 1, dtype=np.int64)


def window_positions(t: int, L_m: int, n: int) -> np.ndarray:
    """D_n(t) of [UOW-1] Eq.(2): {j | max(L_m+1, L_m+t-n) <= j <= L_m+t-1}."""
    if t < 1 or n < 1:
        raise ValueError("t and n must be >= 1")
    lo = max(L_m + 1, L_m + t - n)
    hi = L_m + t - 1
    if hi < lo:
        return np.zeros(0, dtype=np.int64)
    return np.arange(lo, hi + 1, dtype=np.int64)


def visible_positions(t: int, L_m: int, n: int) -> np.ndarray:
    """N(t) = P ∪ D_n(t) of [UOW-1] Eq.(1), sorted ascending."""
    return np.concatenate([reference_positions(L_m), window_positions(t, L_m, n)])


def packed_visible_positions(p: int, L_m: int, n: int) -> np.ndarray:
    """Keys visible to the query at packed position p (1-based).

    p <= L_m: causal inside the prefix (reading R2).
    p >  L_m: this query produces output t = p - L_m + 1 (reading R1), so it
    sees N(t) of Eq.(1)-(2).
    """
    if p < 1:
        raise ValueError("p must be >= 1")
    if p <= L_m:
        return np.arange(1, p + 1, dtype=np.int64)
    return visible_positions(p - L_m + 1, L_m, n)


def bidir_prefix_visible_positions(p: int, L_m: int, n: int) -> np.ndarray:
    """As ``packed_visible_positions`` with a bidirectional prefix (reading
    R7): a prefix query p <= L_m sees all of P."""
    if 1 <= p <= L_m:
        return reference_positions(L_m)
    return packed_visible_positions(p, L_m, n)


def packed_mask(L: int, L_m: int, n: int, bidir_prefix: bool = False) -> np.ndarray:
    """Explicit boolean mask M[p-1, j-1] = (j visible from query p), shape [L, L]."""
    vis = bidir_prefix_visible_positions if bidir_prefix else packed_visible_positions
    M = np.zeros((L, L), dtype=bool)
    for p in range(1, L + 1):
        M[p - 1, vis(p, L_m, n) - 1] = True
    return M


def decode_visible_positions(T: int, L_m: int, n: int) -> np.ndarray:
    """Rows the decode query sees after T outputs were appended (reading R5).

    The newest output T is the query; it produces output T+1, so the set is
    N(T+1) = P ∪ D_n(T+1).  T = 0 gives P alone.
    """
    if T < 0:
        raise ValueError("T must be >= 0")
    return visible_positions(T + 1, L_m, n)


# --------------------------------------------------------------------------
# Cache-size laws: [UOW-1] Eq.(5)-(7).
# --------------------------------------------------------------------------

def occupancy_rswa(T: int, L_m: int, n: int) -> int:
    """C_R-SWA(T) = L_m + min(n, T), [UOW-1] Eq.(6)."""
    return L_m + min(n, T)


def occupancy_full(T: int, L_m: int) -> int:
    """C_MHA(T) = L_m + T, [UOW-1] Eq.(5)."""
    return L_m + T


def cache_ratio(T: int, L_m: int, n: int) -> float:
    """rho(T) = C_R-SWA(T) / C_MHA(T), [UOW-1] Eq.(7)."""
    return occupancy_rswa(T, L_m, n) / occupancy_full(T, L_m)


# --------------------------------------------------------------------------
# The queue of [UOW-3] and the ring-slot storage order used by the library.
# --------------------------------------------------------------------------

class QueueCache:
    """The fixed-capacity queue of [UOW-3] written out literally.

    Capacity L_m + n.  The first L_m entries are the reference rows and are
    never touched again.  Pushing an output when the queue is full first
    removes the entry at 1-based queue index L_m + 1 (the oldest output,
    "position m+1"), then appends the new one at the tail.  Each entry is
    (logical position, k, v).
    """

    def __init__(self, L_m: int, n: int, K_ref: np.ndarray, V_ref: np.ndarray):
        if n < 1:
            raise ValueError("n must be >= 1")
        self.L_m, self.n = L_m, n
        self.entries: List[tuple] = [
            (j + 1, np.array(K_ref[j], dtype=np.float64), np.array(V_ref[j], dtype=np.float64))
            for j in range(L_m)
        ]
        self.T = 0

    def push(self, k: np.ndarray, v: np.ndarray) -> None:
        if len(self.entries) == self.L_m + self.n:
            del self.entries[self.L_m]          # queue index m+1 (1-based)
        self.T += 1
        self.entries.append((self.L_m + self.T, np.array(k, dtype=np.float64),
                             np.array(v, dtype=np.float64)))

    def positions(self) -> np.ndarray:
        return np.array([e[0] for e in self.entries], dtype=np.int64)

    def keys(self) -> np.ndarray:
        return np.stack([e[1] for e in self.entries])

    def values(self) -> np.ndarray:
        return np.stack([e[2] for e in self.entries])


def ring_slot(j: int, n: int) -> int:
    """Storage slot of output j (1-based) in an n-slot ring: (j - 1) mod n.

    Output j lands in the slot that held output j - n, which is exactly the
    entry the queue of [UOW-3] evicts when output j arrives.
    """
    if j < 1:
        raise ValueError("j must be >= 1")
    return (j - 1) % n


def ring_storage_positions(T: int, L_m: int, n: int) -> np.ndarray:
    """Logical position held by each valid cache row, in storage order.

    Rows 0..L_m-1 hold the reference positions 1..L_m.  Row L_m + s holds
    the newest output j <= T with ring_slot(j, n) == s, for s < min(n, T).
    """
    pos = list(range(1, L_m + 1))
    for s in range(min(n, T)):
        # newest j <= T with (j - 1) % n == s
        j = T - ((T - 1 - s) % n)
        pos.append(L_m + j)
    return np.array(pos, dtype=np.int64)


# --------------------------------------------------------------------------
# Attention: [UOW-1] Eq.(3)-(4) in float64, over an explicit visible set.
# --------------------------------------------------------------------------

def attend(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float) -> np.ndarray:
    """o = sum_j alpha_j v_j with alpha = softmax_j(q.k_j * scale) over the
    rows given, [UOW-1] Eq.(3)-(4).  q [d], K [m, d], V [m, d] -> [d].
    The row maximum is subtracted before exp (same value, no overflow)."""
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    s = (K @ q) * scale
    s = s - s.max()
    w = np.exp(s)
    w = w / w.sum()
    return w @ V


def _default_scale(d: int, scale) -> float:
    return 1.0 / math.sqrt(d) if (scale is None or scale <= 0) else float(scale)


def masked_forward(Q: np.ndarray, K: np.ndarray, V: np.ndarray, L_m: int, n: int,
                   scale=None, bidir_prefix: bool = False) -> np.ndarray:
    """Teacher-forced form: O = softmax(Q K^T * scale + M) V per head with the
    explicit mask M of ``packed_mask`` (-inf where not visible).
    Q, K, V: [L, H, d]  ->  O: [L, H, d] float64."""
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    L, H, d = Q.shape
    sc = _default_scale(d, scale)
    M = packed_mask(L, L_m, n, bidir_prefix)
    O = np.empty((L, H, d), dtype=np.float64)
    for h in range(H):
        S = (Q[:, h, :] @ K[:, h, :].T) * sc
        S = np.where(M, S, -np.inf)
        S = S - S.max(axis=1, keepdims=True)
        W = np.exp(S)
        W = W / W.sum(axis=1, keepdims=True)
        O[:, h, :] = W @ V[:, h, :]
    return O


def masked_forward_rows(Q: np.ndarray, K: np.ndarray, V: np.ndarray, L_m: int, n: int,
                        rows: Sequence[int], scale=None, bidir_prefix: bool = False) -> np.ndarray:
    """Same as ``masked_forward`` for the selected 0-based query rows only
    (for sequences too long for the full [L, L] mask).  -> [len(rows), H, d]."""
    L, H, d = Q.shape
    sc = _default_scale(d, scale)
    out = np.empty((len(rows), H, d), dtype=np.float64)
    for i, r in enumerate(rows):
        vis = (bidir_prefix_visible_positions if bidir_prefix else packed_visible_positions)(int(r) + 1, L_m, n) - 1
        for h in range(H):
            out[i, h] = attend(Q[r, h], K[vis, h], V[vis, h], sc)
    return out


# --------------------------------------------------------------------------
# Several documents per pack (reading R8).
# --------------------------------------------------------------------------

def _check_docs(cu_seqlens: Sequence[int], ref_lens: Sequence[int], n: int) -> List[int]:
    cu = [int(x) for x in cu_seqlens]
    if len(cu) < 2 or cu[0] != 0 or len(ref_lens) != len(cu) - 1:
        raise ValueError("cu_seqlens must start at 0 and have one more entry than ref_lens")
    for i in range(len(cu) - 1):
        if cu[i + 1] <= cu[i]:
            raise ValueError("every document needs at least one row")
        if not 0 <= int(ref_lens[i]) <= cu[i + 1] - cu[i]:
            raise ValueError("ref_lens[i] must lie in [0, document length]")
    if n < 1:
        raise ValueError("n must be >= 1")
    return cu


def varlen_visible_positions(g: int, cu_seqlens: Sequence[int], ref_lens: Sequence[int], n: int,
                             bidir_prefix: bool = False) -> np.ndarray:
    """Keys (1-based pack positions) visible to the query at pack position g:
    find g's document, apply the single-sequence visible set at the local
    position, shift back to pack positions (reading R8)."""
    cu = _check_docs(cu_seqlens, ref_lens, n)
    if not 1 <= g <= cu[-1]:
        raise ValueError("g outside the pack")
    i = next(k for k in range(len(cu) - 1) if cu[k] < g <= cu[k + 1])
    vis = bidir_prefix_visible_positions if bidir_prefix else packed_visible_positions
    return vis(g - cu[i], int(ref_lens[i]), n) + cu[i]


def varlen_mask(cu_seqlens: Sequence[int], ref_lens: Sequence[int], n: int,
                bidir_prefix: bool = False) -> np.ndarray:
    """Explicit [L, L] mask of a pack, L = cu_seqlens[-1]."""
    L = int(cu_seqlens[-1])
    M = np.zeros((L, L), dtype=bool)
    for g in range(1, L + 1):
        M[g - 1, varlen_visible_positions(g, cu_seqlens, ref_lens, n, bidir_prefix) - 1] = True
    return M


def masked_forward_varlen(Q: np.ndarray, K: np.ndarray, V: np.ndarray, cu_seqlens: Sequence[int],
                          ref_lens: Sequence[int], n: int, scale=None,
                          bidir_prefix: bool = False) -> np.ndarray:
    """Teacher-forced form over a pack of documents: softmax(Q K^T * scale + M) V
    per head with M = ``varlen_mask`` over the whole pack.
    Q, K, V: [L, H, d], L = cu_seqlens[-1]  ->  O: [L, H, d] float64."""
    Q = np.asarray(Q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    L, H, d = Q.shape
    if L != int(cu_seqlens[-1]):
        raise ValueError("Q rows must equal cu_seqlens[-1]")
    sc = _default_scale(d, scale)
    M = varlen_mask(cu_seqlens, ref_lens, n, bidir_prefix)
    O = np.empty((L, H, d), dtype=np.float64)
    for h in range(H):
        S = (Q[:, h, :] @ K[:, h, :].T) * sc
        S = np.where(M, S, -np.inf)
        S = S - S.max(axis=1, keepdims=True)
        W = np.exp(S)
        W = W / W.sum(axis=1, keepdims=True)
        O[:, h, :] = W @ V[:, h, :]
    return O


def masked_forward_varlen_rows(Q: np.ndarray, K: np.ndarray, V: np.ndarray, cu_seqlens: Sequence[int],
                               ref_lens: Sequence[int], n: int, rows: Sequence[int], scale=None,
                               bidir_prefix: bool = False) -> np.ndarray:
    """``masked_forward_varlen`` for the selected 0-based pack rows only.
    -> [len(rows), H, d]."""
    L, H, d = Q.shape
    sc = _default_scale(d, scale)
    out = np.empty((len(rows), H, d), dtype=np.float64)
    for i, r in enumerate(rows):
        vis = varlen_visible_positions(int(r) + 1, cu_seqlens, ref_lens, n, bidir_prefix) - 1
        for h in range(H):
            out[i, h] = attend(Q[r, h], K[vis, h], V[vis, h], sc)
    return out


def decode_step(q: np.ndarray, K_hist: np.ndarray, V_hist: np.ndarray, L_m: int, T: int,
                n: int, scale=None) -> np.ndarray:
    """Decode output after T appends, recomputed from the FULL history.

    K_hist, V_hist: [>= L_m + T, H, d]; row i holds logical position i+1
    (reference rows first, then outputs 1..T).  q: [H, d].  The visible set
    is N(T+1) (reading R5); no ring buffer is involved, so this checks the
    library's ring logic independently.  -> [H, d] float64.
    """
    q = np.asarray(q, dtype=np.float64)
    H, d = q.shape
    sc = _default_scale(d, scale)
    vis = decode_visible_positions(T, L_m, n) - 1
    out = np.empty((H, d), dtype=np.float64)
    for h in range(H):
        out[h] = attend(q[h], K_hist[vis, h], V_hist[vis, h], sc)
    return out


def decode_step_full(q: np.ndarray, K_hist: np.ndarray, V_hist: np.ndarray, L_m: int, T: int,
                     scale=None) -> np.ndarray:
    """Full-attention (MHA) decode, the Eq.(5) cache: all L_m + T rows."""
    q = np.asarray(q, dtype=np.float64)
    H, d = q.shape
    sc = _default_scale(d, scale)
    out = np.empty((H, d), dtype=np.float64)
    for h in range(H):
        out[h] = attend(q[h], K_hist[: L_m + T, h], V_hist[: L_m + T, h], sc)
    return out
