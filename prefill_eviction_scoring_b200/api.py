"""Python binding of libwaits.so: argument marshalling for torch tensors.

Every step of the path runs in the library's CUDA kernels; this module only
checks tensor shapes/dtypes, allocates outputs with torch, and passes raw
pointers and the current CUDA stream.  Names follow the WAITS README
Quickstart (``sigmoid_a``, ``recent_budget``, ``select_budget``/``budget``)
and Evaluation (``window`` = b).
"""

from __future__ import annotations

import ctypes
from typing import Optional, Tuple

import torch

from . import _lib


def _ptr(t: Optional[torch.Tensor]):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _need_cuda(name, t, dtype):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def make_shape(cu_seqlens: torch.Tensor, total_tokens: int, max_seqlen: int,
               num_q_heads: int, num_kv_heads: int, head_dim: int) -> _lib.Shape:
    return _lib.Shape(int(cu_seqlens.numel() - 1), int(total_tokens),
                      int(max_seqlen), int(num_q_heads), int(num_kv_heads),
                      int(head_dim), cu_seqlens.data_ptr())


def workspace_bytes(shape: _lib.Shape) -> int:
    lib = _lib.load()
    n = ctypes.c_size_t(0)
    _lib.check("waits_workspace_size", lib.waits_workspace_size(ctypes.byref(shape), ctypes.byref(n)))
    return int(n.value)


def _max_seqlen(cu_seqlens, max_seqlen):
    if max_seqlen is not None:
        return int(max_seqlen)
    cu = cu_seqlens.to("cpu")
    return int((cu[1:] - cu[:-1]).max()) if cu.numel() > 1 else 0


class Compressor:
    """Reusable workspace + outputs for one packed-batch shape.

    ``Compressor(cu_seqlens, T, max_seqlen, Hq, Hkv, d, budget)`` allocates
    the workspace and the output tensors once; each call enqueues
    score -> select -> compact on the current stream.
    """

    def __init__(self, cu_seqlens: torch.Tensor, total_tokens: int,
                 max_seqlen: int, num_q_heads: int, num_kv_heads: int,
                 head_dim: int, budget: int):
        _need_cuda("cu_seqlens", cu_seqlens, torch.int32)
        self.lib = _lib.load()
        self.cu = cu_seqlens
        self.dev = cu_seqlens.device
        self.shape = make_shape(cu_seqlens, total_tokens, max_seqlen,
                                num_q_heads, num_kv_heads, head_dim)
        self.nseq = cu_seqlens.numel() - 1
        self.T, self.Hq, self.Hkv, self.d = total_tokens, num_q_heads, num_kv_heads, head_dim
        self.B = int(budget)
        self.ws_bytes = workspace_bytes(self.shape)
        self.workspace = torch.empty(self.ws_bytes, dtype=torch.uint8, device=self.dev)
        self.scores = torch.empty((num_kv_heads, total_tokens), dtype=torch.float32, device=self.dev)
        self.idx = torch.empty((self.nseq, num_kv_heads, self.B), dtype=torch.int32, device=self.dev)
        self.kept_len = torch.empty((self.nseq,), dtype=torch.int32, device=self.dev)
        self.K_out = torch.empty((self.nseq, num_kv_heads, self.B, head_dim), dtype=torch.bfloat16, device=self.dev)
        self.V_out = torch.empty_like(self.K_out)

    def check_inputs(self, Q, K, V=None):
        _need_cuda("Q", Q, torch.bfloat16)
        _need_cuda("K", K, torch.bfloat16)
        if tuple(Q.shape) != (self.T, self.Hq, self.d) or tuple(K.shape) != (self.T, self.Hkv, self.d):
            raise ValueError("Q/K shapes do not match the compressor's shape")
        if V is not None:
            _need_cuda("V", V, torch.bfloat16)
            if V.shape != K.shape:
                raise ValueError("V must have K's shape")

    def __call__(self, Q, K, V, sigmoid_a: float, window: int, recent_budget: int):
        self.check_inputs(Q, K, V)
        st = self.lib.waits_compress(
            ctypes.byref(self.shape), _ptr(Q), _ptr(K), _ptr(V), float(sigmoid_a),
            int(window), int(recent_budget), self.B, _ptr(self.scores), _ptr(self.idx),
            _ptr(self.kept_len), _ptr(self.K_out), _ptr(self.V_out), _ptr(self.workspace),
            self.ws_bytes, _stream(self.dev))
        _lib.check("waits_compress", st)
        return self.K_out, self.V_out, self.idx, self.kept_len, self.scores

    def score(self, Q, K, sigmoid_a: float, window: int):
        self.check_inputs(Q, K)
        st = self.lib.waits_score(ctypes.byref(self.shape), _ptr(Q), _ptr(K), float(sigmoid_a),
                                  int(window), _ptr(self.scores), _ptr(self.workspace),
                                  self.ws_bytes, _stream(self.dev))
        _lib.check("waits_score", st)
        return self.scores

    def compress_routed(self, Q, K, V, sigmoid_a: torch.Tensor, window: torch.Tensor,
                        recent_budget: int):
        """``waits_compress_routed``: per-sequence curves, ``sigmoid_a`` fp32
        ``[nseq]`` and ``window`` int32 ``[nseq]`` on the device."""
        self.check_inputs(Q, K, V)
        _need_cuda("sigmoid_a", sigmoid_a, torch.float32)
        _need_cuda("window", window, torch.int32)
        if sigmoid_a.numel() != self.nseq or window.numel() != self.nseq:
            raise ValueError("one sigmoid_a and one window per sequence")
        st = self.lib.waits_compress_routed(
            ctypes.byref(self.shape), _ptr(Q), _ptr(K), _ptr(V), _ptr(sigmoid_a), _ptr(window),
            int(recent_budget), self.B, _ptr(self.scores), _ptr(self.idx), _ptr(self.kept_len),
            _ptr(self.K_out), _ptr(self.V_out), _ptr(self.workspace), self.ws_bytes,
            _stream(self.dev))
        _lib.check("waits_compress_routed", st)
        return self.K_out, self.V_out, self.idx, self.kept_len, self.scores

    def score_routed(self, Q, K, sigmoid_a: torch.Tensor, window: torch.Tensor):
        """``waits_score_routed``: per-sequence ``sigmoid_a`` (fp32) and
        ``window`` (int32) device tensors of ``nseq`` values."""
        self.check_inputs(Q, K)
        _need_cuda("sigmoid_a", sigmoid_a, torch.float32)
        _need_cuda("window", window, torch.int32)
        if sigmoid_a.numel() != self.nseq or window.numel() != self.nseq:
            raise ValueError("one sigmoid_a and one window per sequence")
        st = self.lib.waits_score_routed(
            ctypes.byref(self.shape), _ptr(Q), _ptr(K), _ptr(sigmoid_a), _ptr(window),
            _ptr(self.scores), _ptr(self.workspace), self.ws_bytes, _stream(self.dev))
        _lib.check("waits_score_routed", st)
        return self.scores

    def score_with_lse(self, Q, K, lse, sigmoid_a: float, window: int):
        """``waits_score_with_lse``: the scores from the caller's row LSE
        (fp32 ``[Hq, T]``, natural log), without the row-statistics pass."""
        self.check_inputs(Q, K)
        _need_cuda("lse", lse, torch.float32)
        if tuple(lse.shape) != (self.Hq, self.T) or not lse.is_contiguous():
            raise ValueError("lse must be a contiguous fp32 [Hq, T] tensor")
        st = self.lib.waits_score_with_lse(
            ctypes.byref(self.shape), _ptr(Q), _ptr(K), _ptr(lse), float(sigmoid_a), int(window),
            _ptr(self.scores), _ptr(self.workspace), self.ws_bytes, _stream(self.dev))
        _lib.check("waits_score_with_lse", st)
        return self.scores

    def device_status(self) -> int:
        v = ctypes.c_uint32(0)
        _lib.check("waits_read_device_status", self.lib.waits_read_device_status(
            _ptr(self.workspace), self.ws_bytes, _stream(self.dev), ctypes.byref(v)))
        return int(v.value)


def score(Q: torch.Tensor, K: torch.Tensor, cu_seqlens: torch.Tensor, *,
          sigmoid_a: float, window: int, max_seqlen: Optional[int] = None) -> torch.Tensor:
    """fp32 scores ``[Hkv, T]`` (``waits_score``)."""
    T, Hq, d = Q.shape
    c = Compressor(cu_seqlens, T, _max_seqlen(cu_seqlens, max_seqlen), Hq, K.shape[1], d, 1)
    return c.score(Q, K, sigmoid_a, window)


def compress_heads(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cu_seqlens: torch.Tensor,
                   kv_heads: Tuple[int, int], *, sigmoid_a: float, window: int,
                   recent_budget: int, budget: int, max_seqlen: Optional[int] = None):
    """``waits_compress_heads``: score, select and compact the KV heads
    ``[kv_heads[0], kv_heads[1])`` of the layer, reading ``q, k, v`` in place
    (a tensor-parallel rank's share).  Returns ``(K_out, V_out, idx,
    kept_len, scores)`` for those heads only."""
    _need_cuda("q", q, torch.bfloat16)
    _need_cuda("k", k, torch.bfloat16)
    _need_cuda("v", v, torch.bfloat16)
    _need_cuda("cu_seqlens", cu_seqlens, torch.int32)
    T, Hq, d = q.shape
    Hkv = k.shape[1]
    g0, g1 = int(kv_heads[0]), int(kv_heads[1])
    Hs = g1 - g0
    nseq = cu_seqlens.numel() - 1
    dev = q.device
    lib = _lib.load()
    shape = make_shape(cu_seqlens, T, _max_seqlen(cu_seqlens, max_seqlen), Hq, Hkv, d)
    ws_bytes = workspace_bytes(shape)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    scores = torch.empty((max(Hs, 0), T), dtype=torch.float32, device=dev)
    idx = torch.empty((nseq, max(Hs, 0), budget), dtype=torch.int32, device=dev)
    kept = torch.empty((nseq,), dtype=torch.int32, device=dev)
    Ko = torch.empty((nseq, max(Hs, 0), budget, d), dtype=torch.bfloat16, device=dev)
    Vo = torch.empty_like(Ko)
    st = lib.waits_compress_heads(ctypes.byref(shape), g0, g1, _ptr(q), _ptr(k), _ptr(v),
                                  float(sigmoid_a), int(window), int(recent_budget), int(budget),
                                  _ptr(scores), _ptr(idx), _ptr(kept), _ptr(Ko), _ptr(Vo),
                                  _ptr(ws), ws_bytes, _stream(dev))
    _lib.check("waits_compress_heads", st)
    return Ko, Vo, idx, kept, scores


def decode_attention(q: torch.Tensor, K_cache: torch.Tensor, V_cache: torch.Tensor,
                     cache_len: torch.Tensor, with_lse: bool = False):
    """One decode step over the compacted cache (``waits_decode_attention``).

    ``q`` bf16 ``[nseq, Hq, d]``; ``K_cache``, ``V_cache`` bf16 ``[nseq, Hkv,
    C, d]`` (e.g. waits_compress's outputs); ``cache_len`` int32 ``[nseq]``.
    Returns fp32 ``[nseq, Hq, d]`` (and the fp32 ``[nseq, Hq]`` row LSE).
    """
    _need_cuda("q", q, torch.bfloat16)
    _need_cuda("K_cache", K_cache, torch.bfloat16)
    _need_cuda("V_cache", V_cache, torch.bfloat16)
    _need_cuda("cache_len", cache_len, torch.int32)
    nseq, Hq, d = q.shape
    Hkv, C = K_cache.shape[1], K_cache.shape[2]
    if tuple(K_cache.shape) != (nseq, Hkv, C, d) or V_cache.shape != K_cache.shape:
        raise ValueError("caches must be [nseq, Hkv, C, d] like q's [nseq, Hq, d]")
    lib = _lib.load()
    n = ctypes.c_size_t(0)
    _lib.check("waits_decode_workspace_size",
               lib.waits_decode_workspace_size(nseq, Hq, d, C, ctypes.byref(n)))
    ws = torch.empty(max(n.value, 16), dtype=torch.uint8, device=q.device)
    out = torch.empty((nseq, Hq, d), dtype=torch.float32, device=q.device)
    lse = torch.empty((nseq, Hq), dtype=torch.float32, device=q.device) if with_lse else None
    st = lib.waits_decode_attention(nseq, Hq, Hkv, d, C, _ptr(q), _ptr(K_cache), _ptr(V_cache),
                                    _ptr(cache_len), _ptr(out), _ptr(lse), _ptr(ws), ws.numel(),
                                    _stream(q.device))
    _lib.check("waits_decode_attention", st)
    return (out, lse) if with_lse else out


def score_with_lse(Q: torch.Tensor, K: torch.Tensor, cu_seqlens: torch.Tensor,
                   lse: torch.Tensor, *, sigmoid_a: float, window: int,
                   max_seqlen: Optional[int] = None) -> torch.Tensor:
    """fp32 ``[Hkv, T]`` scores (``waits_score_with_lse``) from the caller's
    natural-log row LSE ``[Hq, T]`` (a FlashAttention forward's
    ``softmax_lse``): only the weighted column-sum pass runs."""
    _need_cuda("cu_seqlens", cu_seqlens, torch.int32)
    T, Hq, d = Q.shape
    c = Compressor(cu_seqlens, T, _max_seqlen(cu_seqlens, max_seqlen), Hq, K.shape[1], d, 1)
    return c.score_with_lse(Q, K, lse, sigmoid_a, window)


def score_static(Q: torch.Tensor, K: torch.Tensor, cu_seqlens: torch.Tensor, *,
                 sigmoid_a: float, window: int, max_seqlen: Optional[int] = None,
                 out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """``waits_score_static``: the scores of :func:`score` with the library's
    own static scratch instead of a workspace, for callers that must not
    allocate device memory (pass ``out``, fp32 ``[Hkv, T]``, to allocate
    nothing here either).  Shapes whose workspace would exceed
    ``_lib.STATIC_WORKSPACE_BYTES`` are rejected; calls that overlap on the
    GPU share the scratch and must be serialised."""
    _need_cuda("Q", Q, torch.bfloat16)
    _need_cuda("K", K, torch.bfloat16)
    _need_cuda("cu_seqlens", cu_seqlens, torch.int32)
    T, Hq, d = Q.shape
    Hkv = K.shape[1]
    if out is None:
        out = torch.empty((Hkv, T), dtype=torch.float32, device=Q.device)
    _need_cuda("out", out, torch.float32)
    lib = _lib.load()
    shape = make_shape(cu_seqlens, T, _max_seqlen(cu_seqlens, max_seqlen), Hq, Hkv, d)
    st = lib.waits_score_static(ctypes.byref(shape), _ptr(Q), _ptr(K), float(sigmoid_a),
                                int(window), _ptr(out), _stream(Q.device))
    _lib.check("waits_score_static", st)
    return out


def select(scores: torch.Tensor, cu_seqlens: torch.Tensor, *, recent_budget: int,
           budget: int, max_seqlen: Optional[int] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """``(idx [nseq, Hkv, B] int32, kept_len [nseq] int32)`` (``waits_select``)."""
    _need_cuda("scores", scores, torch.float32)
    _need_cuda("cu_seqlens", cu_seqlens, torch.int32)
    lib = _lib.load()
    Hkv, T = scores.shape
    nseq = cu_seqlens.numel() - 1
    shape = make_shape(cu_seqlens, T, _max_seqlen(cu_seqlens, max_seqlen), Hkv, Hkv, 64)
    idx = torch.empty((nseq, Hkv, int(budget)), dtype=torch.int32, device=scores.device)
    kept = torch.empty((nseq,), dtype=torch.int32, device=scores.device)
    st = lib.waits_select(ctypes.byref(shape), _ptr(scores), int(recent_budget), int(budget),
                          _ptr(idx), _ptr(kept), None, 0, _stream(scores.device))
    _lib.check("waits_select", st)
    return idx, kept


def compact(K: torch.Tensor, V: torch.Tensor, cu_seqlens: torch.Tensor, idx: torch.Tensor,
            kept_len: torch.Tensor, *, max_seqlen: Optional[int] = None,
            workspace: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """``(K_out, V_out)`` bf16 ``[nseq, Hkv, B, d]`` (``waits_compact``)."""
    _need_cuda("K", K, torch.bfloat16)
    _need_cuda("V", V, torch.bfloat16)
    _need_cuda("idx", idx, torch.int32)
    _need_cuda("kept_len", kept_len, torch.int32)
    lib = _lib.load()
    T, Hkv, d = K.shape
    nseq, _, B = idx.shape
    shape = make_shape(cu_seqlens, T, _max_seqlen(cu_seqlens, max_seqlen), Hkv, Hkv, d)
    Ko = torch.empty((nseq, Hkv, B, d), dtype=torch.bfloat16, device=K.device)
    Vo = torch.empty_like(Ko)
    ws_b = 0 if workspace is None else workspace.numel()
    st = lib.waits_compact(ctypes.byref(shape), _ptr(K), _ptr(V), _ptr(idx), _ptr(kept_len),
                           int(B), _ptr(Ko), _ptr(Vo), _ptr(workspace), ws_b,
                           _stream(K.device))
    _lib.check("waits_compact", st)
    return Ko, Vo


def select_compact(scores: torch.Tensor, K: torch.Tensor, V: torch.Tensor,
                   cu_seqlens: torch.Tensor, *, recent_budget: int, budget: int,
                   max_seqlen: Optional[int] = None
                   ) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor, torch.Tensor]:
    """``(idx, kept_len, K_out, V_out)``: ``select`` then ``compact`` in one
    kernel (``waits_select_compact``)."""
    _need_cuda("scores", scores, torch.float32)
    _need_cuda("K", K, torch.bfloat16)
    _need_cuda("V", V, torch.bfloat16)
    _need_cuda("cu_seqlens", cu_seqlens, torch.int32)
    lib = _lib.load()
    T, Hkv, d = K.shape
    nseq = cu_seqlens.numel() - 1
    B = int(budget)
    shape = make_shape(cu_seqlens, T, _max_seqlen(cu_seqlens, max_seqlen), Hkv, Hkv, d)
    idx = torch.empty((nseq, Hkv, B), dtype=torch.int32, device=K.device)
    kept = torch.empty((nseq,), dtype=torch.int32, device=K.device)
    Ko = torch.empty((nseq, Hkv, B, d), dtype=torch.bfloat16, device=K.device)
    Vo = torch.empty_like(Ko)
    st = lib.waits_select_compact(ctypes.byref(shape), _ptr(scores), _ptr(K), _ptr(V),
                                  int(recent_budget), B, _ptr(idx), _ptr(kept), _ptr(Ko),
                                  _ptr(Vo), None, 0, _stream(K.device))
    _lib.check("waits_select_compact", st)
    return idx, kept, Ko, Vo


def compress(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cu_seqlens: torch.Tensor, *,
             sigmoid_a: float, window: int, recent_budget: int, budget: int,
             max_seqlen: Optional[int] = None):
    """WAITS prefill compression of one layer (``waits_compress``).

    Returns ``(K_out, V_out, idx, kept_len, scores)``.
    """
    T, Hq, d = q.shape
    c = Compressor(cu_seqlens, T, _max_seqlen(cu_seqlens, max_seqlen), Hq, k.shape[1], d,
                   budget)
    return c(q, k, v, sigmoid_a, window, recent_budget)


class HostCompressor:
    """``waits_compress_host``: inputs and outputs in (pinned) host memory,
    device staging buffers owned here."""

    def __init__(self, cu_seqlens_host: torch.Tensor, num_q_heads: int, num_kv_heads: int,
                 head_dim: int, budget: int, device="cuda"):
        self.lib = _lib.load()
        cu = cu_seqlens_host.to(torch.int32).contiguous()
        self.cu_host = cu.pin_memory() if not cu.is_pinned() else cu
        self.nseq = cu.numel() - 1
        self.T = int(cu[-1])
        self.max_seqlen = int((cu[1:] - cu[:-1]).max())
        self.B = int(budget)
        self.Hq, self.Hkv, self.d = num_q_heads, num_kv_heads, head_dim
        dev = torch.device(device)
        self.dev = dev
        bf = torch.bfloat16
        self.dQ = torch.zeros((self.T, num_q_heads, head_dim), dtype=bf, device=dev)
        self.dK = torch.empty((self.T, num_kv_heads, head_dim), dtype=bf, device=dev)
        self.dV = torch.empty_like(self.dK)
        self.dcu = torch.empty((self.nseq + 1,), dtype=torch.int32, device=dev)
        self.dscores = torch.empty((num_kv_heads, self.T), dtype=torch.float32, device=dev)
        self.didx = torch.empty((self.nseq, num_kv_heads, self.B), dtype=torch.int32, device=dev)
        self.dkept = torch.empty((self.nseq,), dtype=torch.int32, device=dev)
        self.dKo = torch.empty((self.nseq, num_kv_heads, self.B, head_dim), dtype=bf, device=dev)
        self.dVo = torch.empty_like(self.dKo)
        self.shape = make_shape(self.dcu, self.T, self.max_seqlen, num_q_heads, num_kv_heads,
                                head_dim)
        self.ws_bytes = workspace_bytes(self.shape)
        self.workspace = torch.empty(self.ws_bytes, dtype=torch.uint8, device=dev)
        self.bufs = _lib.DeviceBuffers(
            self.dQ.data_ptr(), self.dK.data_ptr(), self.dV.data_ptr(), self.dscores.data_ptr(),
            self.didx.data_ptr(), self.dkept.data_ptr(), self.dKo.data_ptr(),
            self.dVo.data_ptr(), self.dcu.data_ptr())
        pin = dict(pin_memory=True)
        self.idx = torch.empty((self.nseq, num_kv_heads, self.B), dtype=torch.int32, **pin)
        self.kept_len = torch.empty((self.nseq,), dtype=torch.int32, **pin)
        self.K_out = torch.empty((self.nseq, num_kv_heads, self.B, head_dim), dtype=bf, **pin)
        self.V_out = torch.empty_like(self.K_out).pin_memory()
        self.h2d_bytes = 0
        self.d2h_bytes = 0

    def __call__(self, Q_host, K_host, V_host, sigmoid_a: float, window: int,
                 recent_budget: int):
        for n, t in (("Q", Q_host), ("K", K_host), ("V", V_host)):
            if t.is_cuda or t.dtype != torch.bfloat16 or not t.is_contiguous():
                raise ValueError(f"{n} must be a contiguous bf16 host tensor")
        up, down = ctypes.c_size_t(0), ctypes.c_size_t(0)
        st = self.lib.waits_compress_host(
            ctypes.byref(self.shape), _ptr(self.cu_host), _ptr(Q_host), _ptr(K_host),
            _ptr(V_host), float(sigmoid_a), int(window), int(recent_budget), self.B,
            _ptr(self.idx), _ptr(self.kept_len), _ptr(self.K_out), _ptr(self.V_out),
            ctypes.byref(self.bufs), _ptr(self.workspace), self.ws_bytes, _stream(self.dev),
            ctypes.byref(up), ctypes.byref(down))
        _lib.check("waits_compress_host", st)
        self.h2d_bytes, self.d2h_bytes = int(up.value), int(down.value)
        return self.K_out, self.V_out, self.idx, self.kept_len
