"""B200 (sm_100a) Reference Sliding Window Attention.

Thin Python binding over the C ABI of librswa.so (include/rswa.h).  It only
checks and marshals arguments: torch tensors supply device memory and the
current CUDA stream; every step of the attention runs in the library's CUDA
kernels.  If the library is missing or the device is not a B200 the calls
raise; nothing is computed any other way.

    attn = RSWA(L_m_cap=2592, n=128, H=10, d=128, batch=1, dtype=torch.bfloat16)
    attn.load_reference(K_ref, V_ref, ref_lens)        # [B, H, L_m_cap, d]
    o = attn.append_decode(k, v, q)                    # [B, H, d] each
    O = masked_forward(Q, K, V, L_m=..., n=128)        # [L, H, d]
"""

from __future__ import annotations

import ctypes as C
from typing import Optional, Sequence

import numpy as np
import torch

from . import _native
from ._native import MODE_FULL, MODE_RSWA, RSWAError, check

__all__ = ["RSWA", "LayerStep", "append_decode_layers", "masked_forward", "masked_forward_varlen", "RSWAError", "MODE_RSWA", "MODE_FULL", "library_version"]

_DT = {torch.float32: _native.F32, torch.bfloat16: _native.BF16}


def library_version() -> str:
    return _native.lib().rswa_version().decode()


# The raw current-stream query avoids building a Stream object on every call.
_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream_ptr(device: torch.device) -> int:
    if _raw_stream is not None:
        return _raw_stream(device.index)
    return torch.cuda.current_stream(device).cuda_stream


def _check_tensor(name: str, t: torch.Tensor, shape, dtype, device) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


class RSWA:
    """Decode-side R-SWA state over caller-owned device memory.

    The K/V caches ([B, H, L_m_cap + window, d] each) and the workspace are
    torch tensors owned by this object; the library itself allocates
    nothing.  mode MODE_RSWA keeps an n-slot output ring (cache L_m + n);
    MODE_FULL keeps every output (cache L_m + T_cap), the full-attention
    baseline.
    """

    def __init__(self, L_m_cap: int, n: int, H: int, d: int, batch: int,
                 dtype: torch.dtype = torch.bfloat16, mode: int = MODE_RSWA, T_cap: int = 0,
                 device: Optional[torch.device] = None):
        if dtype not in _DT:
            raise ValueError(f"dtype {dtype} not supported (float32, bfloat16)")
        dev = torch.device(device) if device is not None else torch.device("cuda")
        if dev.type != "cuda":
            raise ValueError(f"RSWA needs a CUDA device, got {dev}")
        if dev.index is None:
            dev = torch.device("cuda", torch.cuda.current_device())
        self.device = dev
        self._dev_index = dev.index
        self._vec_shape = torch.Size((batch, H, d))
        self.L_m_cap, self.n, self.H, self.d, self.batch = L_m_cap, n, H, d, batch
        self.dtype, self.mode, self.T_cap = dtype, mode, T_cap
        self.window = n if mode == MODE_RSWA else T_cap
        L = _native.lib()
        cache_bytes = L.rswa_cache_bytes(L_m_cap, self.window, H, d, batch, _DT[dtype])
        ws_bytes = L.rswa_workspace_bytes(L_m_cap, self.window, H, d, batch)
        if cache_bytes == 0 or ws_bytes == 0:
            raise ValueError("invalid sizes for RSWA")
        self.S_cap = L_m_cap + self.window
        self.k_cache = torch.zeros((batch, H, self.S_cap, d), dtype=dtype, device=self.device)
        self.v_cache = torch.zeros((batch, H, self.S_cap, d), dtype=dtype, device=self.device)
        self.workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=self.device)
        self._stream = _stream_ptr(self.device)
        h = C.c_void_p()
        with torch.cuda.device(self.device):
            check(L.rswa_init(C.byref(h), mode, L_m_cap, n, T_cap, H, d, batch, _DT[dtype],
                              self.k_cache.data_ptr(), self.v_cache.data_ptr(),
                              self.workspace.data_ptr(), ws_bytes, self._stream))
        self._h = h
        self._lib = L

    # -- plumbing
    def _sync_stream(self) -> None:
        s = _stream_ptr(self.device)
        if s != self._stream:
            check(_native.lib().rswa_set_stream(self._h, s))
            self._stream = s

    def _vec(self, name, t):
        # fast path of _check_tensor on cached values; the slow one names the problem
        if not (isinstance(t, torch.Tensor) and t.dtype == self.dtype and t.shape == self._vec_shape
                and t.get_device() == self._dev_index and t.is_contiguous()):
            _check_tensor(name, t, (self.batch, self.H, self.d), self.dtype, self.device)

    def close(self) -> None:
        if getattr(self, "_h", None):
            _native.lib().rswa_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    # -- API
    def load_reference(self, K_ref: torch.Tensor, V_ref: torch.Tensor, ref_lens: Sequence[int]) -> None:
        """K_ref, V_ref: [B, H, stride, d] on the device; rows [0, ref_lens[b]) are used."""
        if K_ref.dim() != 4:
            raise ValueError("K_ref must be [B, H, stride, d]")
        stride = K_ref.shape[2]
        _check_tensor("K_ref", K_ref, (self.batch, self.H, stride, self.d), self.dtype, self.device)
        _check_tensor("V_ref", V_ref, (self.batch, self.H, stride, self.d), self.dtype, self.device)
        if len(ref_lens) != self.batch:
            raise ValueError("ref_lens must have one entry per sequence")
        lens = (C.c_int32 * self.batch)(*[int(x) for x in ref_lens])
        self._sync_stream()
        check(_native.lib().rswa_load_reference(self._h, K_ref.data_ptr(), V_ref.data_ptr(), stride, lens))

    def load_packed(self, K: torch.Tensor, V: torch.Tensor, ref_lens: Sequence[int], T0: int) -> None:
        """Cache as after load_reference + T0 appends, from the packed layout
        K, V: [B, L, H, d] (or [L, H, d] for one sequence) on the device, where
        row p of sequence b holds position p+1: the reference rows
        [0, ref_lens[b]), then output t at row ref_lens[b] + t - 1."""
        if K.dim() == 3 and self.batch == 1:
            K, V = K.unsqueeze(0), V.unsqueeze(0)
        if K.dim() != 4:
            raise ValueError("K must be [B, L, H, d]")
        L = K.shape[1]
        _check_tensor("K", K, (self.batch, L, self.H, self.d), self.dtype, self.device)
        _check_tensor("V", V, (self.batch, L, self.H, self.d), self.dtype, self.device)
        if len(ref_lens) != self.batch:
            raise ValueError("ref_lens must have one entry per sequence")
        lens = (C.c_int32 * self.batch)(*[int(x) for x in ref_lens])
        self._sync_stream()
        check(_native.lib().rswa_load_packed(self._h, K.data_ptr(), V.data_ptr(), L, lens, int(T0)))

    def load_reference_chunk(self, K: torch.Tensor, V: torch.Tensor, rows: Sequence[int]) -> None:
        """Appends rows [0, rows[b]) of K, V ([B, H, stride, d] on the device)
        to sequence b's reference, after the rows already loaded; only
        before the first output is appended."""
        if K.dim() != 4:
            raise ValueError("K must be [B, H, stride, d]")
        stride = K.shape[2]
        _check_tensor("K", K, (self.batch, self.H, stride, self.d), self.dtype, self.device)
        _check_tensor("V", V, (self.batch, self.H, stride, self.d), self.dtype, self.device)
        if len(rows) != self.batch:
            raise ValueError("rows must have one entry per sequence")
        r = (C.c_int32 * self.batch)(*[int(x) for x in rows])
        self._sync_stream()
        check(_native.lib().rswa_load_reference_chunk(self._h, K.data_ptr(), V.data_ptr(), stride, r))

    def prefill(self, Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, L_m: int, scale: float = 0.0,
                out: Optional[torch.Tensor] = None, bidir_prefix: bool = False) -> torch.Tensor:
        """Teacher-forced attention of one sequence (Q, K, V: [L, H, d]) with
        this handle's window, that also fills the cache as a reference load of
        rows [0, L_m) plus L - L_m appends would; decoding continues at output
        L - L_m + 1.  Batch-1 handles only."""
        if Q.dim() != 3:
            raise ValueError("Q must be [L, H, d]")
        L = Q.shape[0]
        for name, t in (("Q", Q), ("K", K), ("V", V)):
            _check_tensor(name, t, (L, self.H, self.d), self.dtype, self.device)
        O = torch.empty_like(Q) if out is None else out
        _check_tensor("out", O, (L, self.H, self.d), self.dtype, self.device)
        self._sync_stream()
        check(_native.lib().rswa_masked_forward_fill(self._h, Q.data_ptr(), K.data_ptr(), V.data_ptr(), O.data_ptr(),
                                                      L, int(L_m), float(scale),
                                                      _native.FLAG_BIDIR_PREFIX if bidir_prefix else 0))
        return O

    def append(self, k: torch.Tensor, v: torch.Tensor) -> None:
        self._vec("k", k)
        self._vec("v", v)
        self._sync_stream()
        check(_native.lib().rswa_append(self._h, k.data_ptr(), v.data_ptr()))

    def decode(self, q: torch.Tensor, out: Optional[torch.Tensor] = None, scale: float = 0.0) -> torch.Tensor:
        self._vec("q", q)
        o = torch.empty_like(q) if out is None else out
        self._vec("out", o)
        self._sync_stream()
        check(self._lib.rswa_decode(self._h, q.data_ptr(), o.data_ptr(), float(scale)))
        return o

    def append_decode(self, k: torch.Tensor, v: torch.Tensor, q: torch.Tensor,
                      out: Optional[torch.Tensor] = None, scale: float = 0.0) -> torch.Tensor:
        self._vec("k", k)
        self._vec("v", v)
        self._vec("q", q)
        o = torch.empty_like(q) if out is None else out
        self._vec("out", o)
        self._sync_stream()
        check(self._lib.rswa_append_decode(self._h, k.data_ptr(), v.data_ptr(), q.data_ptr(),
                                           o.data_ptr(), float(scale)))
        return o

    def cache_len(self) -> list:
        out = (C.c_int32 * self.batch)()
        self._sync_stream()
        check(_native.lib().rswa_cache_len(self._h, out))
        return list(out)

    def step_count(self) -> list:
        out = (C.c_int32 * self.batch)()
        self._sync_stream()
        check(_native.lib().rswa_step_count(self._h, out))
        return list(out)

    def cache_positions(self, b: int) -> np.ndarray:
        cap = self.S_cap
        out = (C.c_int64 * cap)()
        cnt = C.c_int()
        self._sync_stream()
        check(_native.lib().rswa_cache_positions(self._h, int(b), out, cap, C.byref(cnt)))
        return np.frombuffer(out, dtype=np.int64, count=cnt.value).copy()

    def reset(self) -> None:
        self._sync_stream()
        check(_native.lib().rswa_reset(self._h))

    def check(self) -> None:
        """Raises RSWAError if a kernel flagged a device-side error."""
        self._sync_stream()
        check(_native.lib().rswa_check(self._h))


def append_decode_layers(layers: Sequence[RSWA], k: Sequence[torch.Tensor], v: Sequence[torch.Tensor],
                         q: Sequence[torch.Tensor], out: Optional[Sequence[torch.Tensor]] = None,
                         scale: float = 0.0) -> list:
    """One decode step of an R-layer decoder: append_decode on every layer
    handle in order (one C call, one kernel per layer).  k[r], v[r], q[r],
    out[r]: [B, H, d] tensors of layer r's handle.  Returns the outputs."""
    R = len(layers)
    if not (len(k) == len(v) == len(q) == R) or (out is not None and len(out) != R):
        raise ValueError("one k, v, q (and out) per layer")
    outs = [torch.empty_like(q[r]) for r in range(R)] if out is None else list(out)
    for r, a in enumerate(layers):
        a._vec("k", k[r])
        a._vec("v", v[r])
        a._vec("q", q[r])
        a._vec("out", outs[r])
        a._sync_stream()
    P = C.c_void_p * R
    hs = P(*[a._h.value for a in layers])
    check(_native.lib().rswa_append_decode_layers(
        hs, R, P(*[t.data_ptr() for t in k]), P(*[t.data_ptr() for t in v]), P(*[t.data_ptr() for t in q]),
        P(*[t.data_ptr() for t in outs]), float(scale)))
    return outs


class LayerStep:
    """One decode step over fixed layer handles and fixed device buffers (a
    model's per-layer k, v, q and output tensors, refilled in place every
    step): the checks and the pointer arrays are done once, so each call is
    a single C call of rswa_append_decode_layers.

    graph=True (RSWA-mode handles only) captures that call once into a CUDA
    graph and replays it on each call: the step counter lives on the device,
    so every replay is the next step.  Capture and replays do not keep the
    handles' host-side step count (read only by FULL-mode planning and the
    reference-chunk loader); step_count() reads the device counter and
    refreshes it."""

    def __init__(self, layers: Sequence[RSWA], k: Sequence[torch.Tensor], v: Sequence[torch.Tensor],
                 q: Sequence[torch.Tensor], out: Sequence[torch.Tensor], scale: float = 0.0,
                 graph: bool = False):
        R = len(layers)
        if not (len(k) == len(v) == len(q) == len(out) == R) or R < 1:
            raise ValueError("one k, v, q and out per layer")
        for r, a in enumerate(layers):
            a._vec("k", k[r])
            a._vec("v", v[r])
            a._vec("q", q[r])
            a._vec("out", out[r])
        P = C.c_void_p * R
        self._layers = list(layers)
        self._keep = (list(k), list(v), list(q), list(out))  # the tensors must outlive the step
        self._args = (P(*[a._h.value for a in layers]), R, P(*[t.data_ptr() for t in k]),
                      P(*[t.data_ptr() for t in v]), P(*[t.data_ptr() for t in q]),
                      P(*[t.data_ptr() for t in out]), float(scale))
        self._fn = _native.lib().rswa_append_decode_layers
        self._graph = None
        if graph:
            if any(a.mode != MODE_RSWA for a in layers):
                raise ValueError("graph=True needs RSWA-mode handles (FULL mode re-plans on the host)")
            dev = layers[0].device
            side = torch.cuda.Stream(dev)
            side.wait_stream(torch.cuda.current_stream(dev))
            g = torch.cuda.CUDAGraph()
            with torch.cuda.stream(side):
                with torch.cuda.graph(g, stream=side):
                    self._launch()
            torch.cuda.current_stream(dev).wait_stream(side)
            self._graph = g

    def _launch(self) -> None:
        for a in self._layers:
            a._sync_stream()
        check(self._fn(*self._args))

    def __call__(self) -> None:
        if self._graph is not None:
            self._graph.replay()
        else:
            self._launch()


def masked_forward(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, L_m: int, n: int,
                   scale: float = 0.0, out: Optional[torch.Tensor] = None,
                   bidir_prefix: bool = False) -> torch.Tensor:
    """Teacher-forced R-SWA attention.  Q, K, V, out: [L, H, d] on a B200.
    L_m = 0: no reference segment (the plain sliding window of n).
    bidir_prefix: prefix queries see every reference key (default: causal)."""
    if Q.dim() != 3:
        raise ValueError("Q must be [L, H, d]")
    L, H, d = Q.shape
    if Q.dtype not in _DT:
        raise ValueError(f"dtype {Q.dtype} not supported")
    for name, t in (("K", K), ("V", V)):
        _check_tensor(name, t, (L, H, d), Q.dtype, Q.device)
    _check_tensor("Q", Q, (L, H, d), Q.dtype, Q.device)
    O = torch.empty_like(Q) if out is None else out
    _check_tensor("out", O, (L, H, d), Q.dtype, Q.device)
    with torch.cuda.device(Q.device):
        check(_native.lib().rswa_masked_forward_ex(Q.data_ptr(), K.data_ptr(), V.data_ptr(), O.data_ptr(),
                                                   L, int(L_m), int(n), H, d, _DT[Q.dtype], float(scale),
                                                   _native.FLAG_BIDIR_PREFIX if bidir_prefix else 0,
                                                   _stream_ptr(Q.device)))
    return O


def masked_forward_varlen(Q: torch.Tensor, K: torch.Tensor, V: torch.Tensor, cu_seqlens: Sequence[int],
                          ref_lens: Sequence[int], n: int, scale: float = 0.0,
                          out: Optional[torch.Tensor] = None, bidir_prefix: bool = False) -> torch.Tensor:
    """Teacher-forced R-SWA attention over a pack of documents.  Q, K, V, out:
    [L, H, d] on a B200, L = cu_seqlens[-1]; document i holds rows
    cu_seqlens[i] .. cu_seqlens[i+1]-1 with ref_lens[i] reference rows and
    sees only its own keys."""
    if Q.dim() != 3:
        raise ValueError("Q must be [L, H, d]")
    L, H, d = Q.shape
    if Q.dtype not in _DT:
        raise ValueError(f"dtype {Q.dtype} not supported")
    n_docs = len(ref_lens)
    if len(cu_seqlens) != n_docs + 1 or int(cu_seqlens[-1]) != L:
        raise ValueError("cu_seqlens must have len(ref_lens) + 1 entries ending at L")
    for name, t in (("Q", Q), ("K", K), ("V", V)):
        _check_tensor(name, t, (L, H, d), Q.dtype, Q.device)
    O = torch.empty_like(Q) if out is None else out
    _check_tensor("out", O, (L, H, d), Q.dtype, Q.device)
    cu = (C.c_int32 * (n_docs + 1))(*[int(x) for x in cu_seqlens])
    refs = (C.c_int32 * n_docs)(*[int(x) for x in ref_lens])
    with torch.cuda.device(Q.device):
        check(_native.lib().rswa_masked_forward_varlen(
            Q.data_ptr(), K.data_ptr(), V.data_ptr(), O.data_ptr(), cu, refs, n_docs, int(n), H, d,
            _DT[Q.dtype], float(scale), _native.FLAG_BIDIR_PREFIX if bidir_prefix else 0,
            _stream_ptr(Q.device)))
    return O
