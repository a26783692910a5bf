"""Tensor-level binding of libcsa.so: argument marshalling only.

Every function takes CUDA torch tensors, checks dtype / shape / contiguity, and calls the C ABI
on the current torch stream. All arithmetic of the layer runs in the library's kernels; there
is no Python or CPU implementation here.

Citations for what each call computes are in include/csa.h (pages: "DeepSeek-V4-Pro 架构：一个 token
的旅程" and "图解DeepSeek V4：详细计算流程解析").
"""

from __future__ import annotations

import ctypes
import math
from typing import Optional

import torch

from . import _lib
from ._lib import CompressorCfg, DecodeArgs, HcaDecodeArgs, check


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream() -> int:
    return torch.cuda.current_stream().cuda_stream


def _need(t: torch.Tensor, name: str, dtype: torch.dtype, shape=None) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (the layer runs only in libcsa.so's kernels)")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _bstride(t: torch.Tensor, name: str) -> int:
    """Batch stride in elements of a [B, rows, d] tensor whose rows are contiguous."""
    if t.dim() != 3 or t.stride(2) != 1 or t.stride(1) != t.shape[2]:
        raise ValueError(f"{name} must be [B, rows, d] with contiguous rows")
    return t.stride(0)


def compressor_cfg(ratio: int, d: int, rope_dim: int = 64, rope_base: float = 10000.0,
                   eps: float = 1e-6) -> CompressorCfg:
    return CompressorCfg(ratio, 1 if ratio == 4 else 0, d, rope_dim, rope_base, eps)


def workspace_size(kind: int, B: int, S: int, max_entries: int, topk: int = 1) -> int:
    n = ctypes.c_size_t(0)
    check(_lib.load().csa_workspace_size(kind, B, S, max_entries, topk, ctypes.byref(n)), "csa_workspace_size")
    return n.value


def workspace(kind: int, B: int, S: int, max_entries: int, topk: int = 1, device=None) -> torch.Tensor:
    """A zeroed workspace (its first 256 bytes are the device status word)."""
    return torch.zeros(workspace_size(kind, B, S, max_entries, topk), dtype=torch.uint8, device=device or "cuda")


def state_reset(cfg: CompressorCfg, state_kv: torch.Tensor, state_score: torch.Tensor) -> None:
    _need(state_kv, "state_kv", torch.bfloat16)
    _need(state_score, "state_score", torch.bfloat16, state_kv.shape)
    check(_lib.load().csa_state_reset(ctypes.byref(cfg), state_kv.shape[0], state_kv.data_ptr(),
                                      state_score.data_ptr(), _stream()), "csa_state_reset")


def compress(cfg: CompressorCfg, start_pos: torch.Tensor, kv: torch.Tensor, score: torch.Tensor,
             gamma: torch.Tensor, state_kv: torch.Tensor, state_score: torch.Tensor, cache: torch.Tensor,
             cache_f32: Optional[torch.Tensor] = None) -> None:
    """C4A / C128A over a segment: kv, score [B, S, width]; writes completed entries of cache
    [B, max_entries, d] (and cache_f32) and advances the state."""
    B, S, width = kv.shape
    _need(start_pos, "start_pos", torch.int32, (B,))
    _need(kv, "kv", torch.bfloat16)
    _need(score, "score", torch.bfloat16, kv.shape)
    _need(gamma, "gamma", torch.bfloat16, (cfg.d,))
    _need(state_kv, "state_kv", torch.bfloat16)
    _need(state_score, "state_score", torch.bfloat16, state_kv.shape)
    _need(cache, "cache", torch.bfloat16)
    if cache_f32 is not None:
        _need(cache_f32, "cache_f32", torch.float32, cache.shape)
    check(_lib.load().csa_compress(ctypes.byref(cfg), B, S, start_pos.data_ptr(), kv.data_ptr(), score.data_ptr(),
                                   gamma.data_ptr(), state_kv.data_ptr(), state_score.data_ptr(), cache.data_ptr(),
                                   _bstride(cache, "cache"), cache.shape[1], _ptr(cache_f32), _stream()),
          "csa_compress")


def indexer_topk(q_pos: torch.Tensor, q_idx: torch.Tensor, w: torch.Tensor, idx_cache: torch.Tensor, topk: int,
                 ratio: int = 4, topk_idx: Optional[torch.Tensor] = None, scores: Optional[torch.Tensor] = None,
                 ws: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Lightning indexer + top-k. q_pos [B,S] int32, q_idx [B,S,H_I,d_I] bf16, w [B,S,H_I] fp32,
    idx_cache [B, max_entries, d_I] bf16. Returns topk_idx [B,S,topk] int32 (ascending, -1 padded)."""
    B, S, H_I, d_I = q_idx.shape
    E = idx_cache.shape[1]
    _need(q_pos, "q_pos", torch.int32, (B, S))
    _need(q_idx, "q_idx", torch.bfloat16)
    _need(w, "w", torch.float32, (B, S, H_I))
    if topk_idx is None:
        topk_idx = torch.empty(B, S, topk, dtype=torch.int32, device=q_idx.device)
    _need(topk_idx, "topk_idx", torch.int32, (B, S, topk))
    if scores is not None:
        _need(scores, "scores", torch.float32, (B, S, E))
    if ws is None:
        ws = workspace(_lib.CSA_WS_INDEXER_TOPK, B, S, E, topk, q_idx.device)
    check(_lib.load().csa_indexer_topk(B, S, H_I, d_I, ratio, topk, q_pos.data_ptr(), q_idx.data_ptr(), w.data_ptr(),
                                       idx_cache.data_ptr(), _bstride(idx_cache, "idx_cache"), E,
                                       topk_idx.data_ptr(), _ptr(scores), ws.data_ptr(), ws.numel(), _stream()),
          "csa_indexer_topk")
    return topk_idx


def indexer_scores(q_pos: torch.Tensor, q_idx: torch.Tensor, w: torch.Tensor, idx_cache: torch.Tensor,
                   ratio: int = 4, scores: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None
                   ) -> torch.Tensor:
    """Indexer scores over this call's heads only (no selection): scores [B,S,max_entries] fp32, the
    visible s < (t+1)//ratio written. With the heads split over ranks, these are partial scores."""
    B, S, H_I, d_I = q_idx.shape
    E = idx_cache.shape[1]
    _need(q_pos, "q_pos", torch.int32, (B, S))
    _need(q_idx, "q_idx", torch.bfloat16)
    _need(w, "w", torch.float32, (B, S, H_I))
    if scores is None:
        scores = torch.empty(B, S, E, dtype=torch.float32, device=q_idx.device)
    _need(scores, "scores", torch.float32, (B, S, E))
    if ws is None:
        ws = workspace(_lib.CSA_WS_SPARSE_ATTN, B, S, E, 1, q_idx.device)
    check(_lib.load().csa_indexer_scores(B, S, H_I, d_I, ratio, q_pos.data_ptr(), q_idx.data_ptr(), w.data_ptr(),
                                         idx_cache.data_ptr(), _bstride(idx_cache, "idx_cache"), E, scores.data_ptr(),
                                         ws.data_ptr(), ws.numel(), _stream()), "csa_indexer_scores")
    return scores


def topk(q_pos: torch.Tensor, scores: torch.Tensor, k: int, ratio: int = 4, topk_idx: Optional[torch.Tensor] = None,
         ws: Optional[torch.Tensor] = None) -> torch.Tensor:
    """The selection of csa_indexer_topk over given scores [B,S,max_entries] fp32: the min(k, E)
    largest of the visible s < E, ties to the lower index, ascending, -1 padded."""
    B, S, E = scores.shape
    _need(q_pos, "q_pos", torch.int32, (B, S))
    _need(scores, "scores", torch.float32)
    if topk_idx is None:
        topk_idx = torch.empty(B, S, k, dtype=torch.int32, device=scores.device)
    _need(topk_idx, "topk_idx", torch.int32, (B, S, k))
    if ws is None:
        ws = workspace(_lib.CSA_WS_INDEXER_TOPK, B, S, E, k, scores.device)
    check(_lib.load().csa_topk(B, S, ratio, k, q_pos.data_ptr(), scores.data_ptr(), E, topk_idx.data_ptr(),
                               ws.data_ptr(), ws.numel(), _stream()), "csa_topk")
    return topk_idx


def _attn_common(q_pos, q, ring, cache, sink, out):
    B, S, H, d = q.shape
    _need(q_pos, "q_pos", torch.int32, (B, S))
    _need(q, "q", torch.bfloat16)
    _need(sink, "sink", torch.float32, (H,))
    if ring.dtype != torch.bfloat16 or not ring.is_cuda:
        raise TypeError("ring must be a bf16 CUDA tensor")
    if cache.dtype != torch.bfloat16 or not cache.is_cuda:
        raise TypeError("cache must be a bf16 CUDA tensor")
    if out is None:
        out = torch.empty(B, S, H, d, dtype=torch.bfloat16, device=q.device)
    if out.dtype not in (torch.bfloat16, torch.float32):
        raise TypeError("out must be bf16 or fp32")
    _need(out, "out", out.dtype, (B, S, H, d))
    return B, S, H, d, out


def sparse_attn(q_pos: torch.Tensor, q: torch.Tensor, ring: torch.Tensor, cache: torch.Tensor,
                topk_idx: torch.Tensor, sink: torch.Tensor, window: int, out: Optional[torch.Tensor] = None,
                scale: Optional[float] = None, rope_dim: int = 64, rope_base: float = 10000.0,
                ws: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Sparse MQA with sink + inverse RoPE over window rows (ring [B, ring_cap, d]) and the
    selected entries (cache [B, max_entries, d], topk_idx [B, S, k])."""
    B, S, H, d, out = _attn_common(q_pos, q, ring, cache, sink, out)
    _need(topk_idx, "topk_idx", torch.int32)
    if topk_idx.shape[:2] != (B, S):
        raise ValueError("topk_idx must be [B, S, k]")
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    if ws is None:
        ws = workspace(_lib.CSA_WS_SPARSE_ATTN, B, S, 1, 1, q.device)
    check(_lib.load().csa_sparse_attn(B, S, H, d, rope_dim, rope_base, scale, q_pos.data_ptr(), q.data_ptr(),
                                      ring.data_ptr(), _bstride(ring, "ring"), ring.shape[1], window,
                                      cache.data_ptr(), _bstride(cache, "cache"), cache.shape[1],
                                      topk_idx.data_ptr(), topk_idx.shape[2], sink.data_ptr(), out.data_ptr(),
                                      int(out.dtype == torch.float32), ws.data_ptr(), ws.numel(), _stream()),
          "csa_sparse_attn")
    return out


def hca_attn(q_pos: torch.Tensor, q: torch.Tensor, ring: torch.Tensor, cache: torch.Tensor, sink: torch.Tensor,
             window: int, ratio: int = 128, out: Optional[torch.Tensor] = None, scale: Optional[float] = None,
             rope_dim: int = 64, rope_base: float = 10000.0, ws: Optional[torch.Tensor] = None) -> torch.Tensor:
    """HCA attention: window rows plus every visible entry s < (t+1)//ratio."""
    B, S, H, d, out = _attn_common(q_pos, q, ring, cache, sink, out)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    if ws is None:
        ws = workspace(_lib.CSA_WS_HCA_ATTN, B, S, 1, 1, q.device)
    check(_lib.load().hca_attn(B, S, H, d, rope_dim, rope_base, scale, ratio, q_pos.data_ptr(), q.data_ptr(),
                               ring.data_ptr(), _bstride(ring, "ring"), ring.shape[1], window, cache.data_ptr(),
                               _bstride(cache, "cache"), cache.shape[1], sink.data_ptr(), out.data_ptr(),
                               int(out.dtype == torch.float32), ws.data_ptr(), ws.numel(), _stream()),
          "hca_attn")
    return out


class CsaDecodeState:
    """Device-resident per-request state of one CSA layer for decode: the two compressor
    states, the two compressed caches, the window ring, and a reusable workspace."""

    def __init__(self, B: int, max_entries: int, H: int = 128, d: int = 512, H_I: int = 64, d_I: int = 128,
                 window: int = 128, topk: int = 1024, ratio: int = 4, rope_dim: int = 64,
                 rope_base: float = 10000.0, eps: float = 1e-6, device="cuda"):
        self.B, self.max_entries, self.H, self.d, self.H_I, self.d_I = B, max_entries, H, d, H_I, d_I
        self.window, self.topk, self.ratio, self.rope_dim, self.rope_base, self.eps = (
            window, topk, ratio, rope_dim, rope_base, eps)
        dev = torch.device(device)
        bf = torch.bfloat16
        self.state_kv = torch.empty(B, 2 * ratio, 2 * d, dtype=bf, device=dev)
        self.state_score = torch.empty_like(self.state_kv)
        self.idx_state_kv = torch.empty(B, 2 * ratio, 2 * d_I, dtype=bf, device=dev)
        self.idx_state_score = torch.empty_like(self.idx_state_kv)
        state_reset(compressor_cfg(ratio, d, rope_dim, rope_base, eps), self.state_kv, self.state_score)
        state_reset(compressor_cfg(ratio, d_I, rope_dim, rope_base, eps), self.idx_state_kv, self.idx_state_score)
        self.cache = torch.zeros(B, max_entries, d, dtype=bf, device=dev)
        self.idx_cache = torch.zeros(B, max_entries, d_I, dtype=bf, device=dev)
        self.ring = torch.zeros(B, window, d, dtype=bf, device=dev)
        self.topk_idx = torch.empty(B, topk, dtype=torch.int32, device=dev)
        self.ws = workspace(_lib.CSA_WS_DECODE_FUSED, B, 1, max_entries, topk, dev)
        self.gamma = torch.ones(d, dtype=bf, device=dev)
        self.idx_gamma = torch.ones(d_I, dtype=bf, device=dev)

    def step(self, pos, kv, score, idx_kv, idx_score, win_kv, q, q_idx, w, sink, out=None, cache_f32=None,
             stage_events=None):
        """One decode step for every request (csa_decode_fused)."""
        return decode_fused(self, pos, kv, score, idx_kv, idx_score, win_kv, q, q_idx, w, sink, out, cache_f32,
                            stage_events)

    def prepare(self, pos, kv, score, idx_kv, idx_score, win_kv, q, q_idx, w, sink, out=None,
                cache_f32=None) -> "PreparedDecode":
        """Check and pack the arguments of step() once for repeated launches on fixed buffers."""
        a, out = _csa_decode_args(self, pos, kv, score, idx_kv, idx_score, win_kv, q, q_idx, w, sink, out,
                                  cache_f32)
        keep = (self, pos, kv, score, idx_kv, idx_score, win_kv, q, q_idx, w, sink, cache_f32, out)
        return PreparedDecode("csa_decode_fused", 5, a, keep)


def _event_array(events, n: int):
    """ctypes array of the raw cudaEvent_t handles of n recorded torch.cuda.Event objects."""
    if events is None:
        return None
    if len(events) != n:
        raise ValueError(f"stage_events needs {n} events")
    for e in events:
        if not e.cuda_event:      # torch creates the CUDA event on its first record
            e.record()
    return (ctypes.c_void_p * n)(*[e.cuda_event for e in events])


def _csa_decode_args(st: "CsaDecodeState", pos, kv, score, idx_kv, idx_score, win_kv, q, q_idx, w, sink,
                     out: Optional[torch.Tensor], cache_f32: Optional[torch.Tensor]):
    B, H, d, H_I, d_I = st.B, st.H, st.d, st.H_I, st.d_I
    _need(pos, "pos", torch.int32, (B,))
    _need(kv, "kv", torch.bfloat16, (B, 2 * d))
    _need(score, "score", torch.bfloat16, (B, 2 * d))
    _need(idx_kv, "idx_kv", torch.bfloat16, (B, 2 * d_I))
    _need(idx_score, "idx_score", torch.bfloat16, (B, 2 * d_I))
    _need(win_kv, "win_kv", torch.bfloat16, (B, d))
    _need(q, "q", torch.bfloat16, (B, H, d))
    _need(q_idx, "q_idx", torch.bfloat16, (B, H_I, d_I))
    _need(w, "w", torch.float32, (B, H_I))
    _need(sink, "sink", torch.float32, (H,))
    if out is None:
        out = torch.empty(B, H, d, dtype=torch.bfloat16, device=q.device)
    _need(out, "out", out.dtype, (B, H, d))
    if cache_f32 is not None:
        _need(cache_f32, "cache_f32", torch.float32, st.cache.shape)
    a = DecodeArgs()
    a.B, a.H, a.d, a.rope_dim, a.H_I, a.d_I = B, H, d, st.rope_dim, H_I, d_I
    a.ratio, a.window, a.topk = st.ratio, st.window, st.topk
    a.rope_base, a.eps, a.scale = st.rope_base, st.eps, 1.0 / math.sqrt(d)
    a.pos, a.kv, a.score, a.idx_kv, a.idx_score = (pos.data_ptr(), kv.data_ptr(), score.data_ptr(),
                                                   idx_kv.data_ptr(), idx_score.data_ptr())
    a.win_kv, a.q, a.q_idx, a.w, a.sink = win_kv.data_ptr(), q.data_ptr(), q_idx.data_ptr(), w.data_ptr(), sink.data_ptr()
    a.gamma, a.idx_gamma = st.gamma.data_ptr(), st.idx_gamma.data_ptr()
    a.state_kv, a.state_score = st.state_kv.data_ptr(), st.state_score.data_ptr()
    a.idx_state_kv, a.idx_state_score = st.idx_state_kv.data_ptr(), st.idx_state_score.data_ptr()
    a.cache, a.cache_bstride = st.cache.data_ptr(), st.cache.stride(0)
    a.idx_cache, a.idx_bstride = st.idx_cache.data_ptr(), st.idx_cache.stride(0)
    a.max_entries = st.max_entries
    a.ring, a.ring_bstride, a.ring_cap = st.ring.data_ptr(), st.ring.stride(0), st.ring.shape[1]
    a.topk_idx = st.topk_idx.data_ptr()
    a.cache_f32 = _ptr(cache_f32)
    a.out, a.out_is_f32 = out.data_ptr(), int(out.dtype == torch.float32)
    a.ws, a.ws_bytes = st.ws.data_ptr(), st.ws.numel()
    return a, out


class PreparedDecode:
    """One decode step whose arguments were checked and packed once: launch() enqueues it again
    on the current stream with the same buffers (the caller refreshes their contents). It keeps
    the tensors it points to alive."""

    def __init__(self, fn_name: str, n_events: int, args, keep):
        self._fn = getattr(_lib.load(), fn_name)
        self._name = fn_name
        self._n_events = n_events
        self._a = args
        self._keep = keep
        self.out = keep[-1]

    def launch(self, stage_events=None) -> torch.Tensor:
        evs = _event_array(stage_events, self._n_events)
        self._a.stage_events = ctypes.cast(evs, ctypes.c_void_p) if evs is not None else None
        check(self._fn(ctypes.byref(self._a), _stream()), self._name)
        return self.out


def decode_fused(st: "CsaDecodeState", pos, kv, score, idx_kv, idx_score, win_kv, q, q_idx, w, sink,
                 out: Optional[torch.Tensor] = None, cache_f32: Optional[torch.Tensor] = None,
                 stage_events=None) -> torch.Tensor:
    a, out = _csa_decode_args(st, pos, kv, score, idx_kv, idx_score, win_kv, q, q_idx, w, sink, out, cache_f32)
    evs = _event_array(stage_events, 5)
    a.stage_events = ctypes.cast(evs, ctypes.c_void_p) if evs is not None else None
    check(_lib.load().csa_decode_fused(ctypes.byref(a), _stream()), "csa_decode_fused")
    return out


class HcaDecodeState:
    """Device-resident state of one HCA layer for decode (C128A state, cache, window ring)."""

    def __init__(self, B: int, max_entries: int, H: int = 128, d: int = 512, window: int = 128, ratio: int = 128,
                 rope_dim: int = 64, rope_base: float = 10000.0, eps: float = 1e-6, device="cuda"):
        self.B, self.max_entries, self.H, self.d, self.window, self.ratio = B, max_entries, H, d, window, ratio
        self.rope_dim, self.rope_base, self.eps = rope_dim, rope_base, eps
        dev = torch.device(device)
        bf = torch.bfloat16
        self.state_kv = torch.empty(B, ratio, d, dtype=bf, device=dev)
        self.state_score = torch.empty_like(self.state_kv)
        state_reset(compressor_cfg(ratio, d, rope_dim, rope_base, eps), self.state_kv, self.state_score)
        self.cache = torch.zeros(B, max_entries, d, dtype=bf, device=dev)
        self.ring = torch.zeros(B, window, d, dtype=bf, device=dev)
        self.ws = workspace(_lib.CSA_WS_HCA_DECODE_FUSED, B, 1, max_entries, 1, dev)
        self.gamma = torch.ones(d, dtype=bf, device=dev)

    def step(self, pos, kv, score, win_kv, q, sink, out=None, cache_f32=None, stage_events=None):
        return hca_decode_fused(self, pos, kv, score, win_kv, q, sink, out, cache_f32, stage_events)

    def prepare(self, pos, kv, score, win_kv, q, sink, out=None, cache_f32=None) -> "PreparedDecode":
        """Check and pack the arguments of step() once for repeated launches on fixed buffers."""
        a, out = _hca_decode_args(self, pos, kv, score, win_kv, q, sink, out, cache_f32)
        keep = (self, pos, kv, score, win_kv, q, sink, cache_f32, out)
        return PreparedDecode("hca_decode_fused", 3, a, keep)


def _hca_decode_args(st: "HcaDecodeState", pos, kv, score, win_kv, q, sink, out, cache_f32):
    B, H, d = st.B, st.H, st.d
    _need(pos, "pos", torch.int32, (B,))
    _need(kv, "kv", torch.bfloat16, (B, d))
    _need(score, "score", torch.bfloat16, (B, d))
    _need(win_kv, "win_kv", torch.bfloat16, (B, d))
    _need(q, "q", torch.bfloat16, (B, H, d))
    _need(sink, "sink", torch.float32, (H,))
    if out is None:
        out = torch.empty(B, H, d, dtype=torch.bfloat16, device=q.device)
    _need(out, "out", out.dtype, (B, H, d))
    if cache_f32 is not None:
        _need(cache_f32, "cache_f32", torch.float32, st.cache.shape)
    a = HcaDecodeArgs()
    a.B, a.H, a.d, a.rope_dim, a.ratio, a.window = B, H, d, st.rope_dim, st.ratio, st.window
    a.rope_base, a.eps, a.scale = st.rope_base, st.eps, 1.0 / math.sqrt(d)
    a.pos, a.kv, a.score, a.win_kv, a.q, a.sink = (pos.data_ptr(), kv.data_ptr(), score.data_ptr(),
                                                   win_kv.data_ptr(), q.data_ptr(), sink.data_ptr())
    a.gamma, a.state_kv, a.state_score = st.gamma.data_ptr(), st.state_kv.data_ptr(), st.state_score.data_ptr()
    a.cache, a.cache_bstride, a.max_entries = st.cache.data_ptr(), st.cache.stride(0), st.max_entries
    a.ring, a.ring_bstride, a.ring_cap = st.ring.data_ptr(), st.ring.stride(0), st.ring.shape[1]
    a.cache_f32 = _ptr(cache_f32)
    a.out, a.out_is_f32 = out.data_ptr(), int(out.dtype == torch.float32)
    a.ws, a.ws_bytes = st.ws.data_ptr(), st.ws.numel()
    return a, out


def hca_decode_fused(st: "HcaDecodeState", pos, kv, score, win_kv, q, sink, out=None, cache_f32=None,
                     stage_events=None) -> torch.Tensor:
    a, out = _hca_decode_args(st, pos, kv, score, win_kv, q, sink, out, cache_f32)
    evs = _event_array(stage_events, 3)
    a.stage_events = ctypes.cast(evs, ctypes.c_void_p) if evs is not None else None
    check(_lib.load().hca_decode_fused(ctypes.byref(a), _stream()), "hca_decode_fused")
    return out


def output_projection(o: torch.Tensor, wo_a: torch.Tensor, wo_b: torch.Tensor, r: Optional[torch.Tensor] = None,
                      y: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None):
    """Grouped output projection: o holds M rows of G*Kg bf16 values ([B, S, H, d] or [M, G*Kg]),
    wo_a [G, R, Kg] and wo_b [D, G*R] bf16. Returns (r [M, G*R] bf16, y [M, D] fp32)."""
    G, R, Kg = wo_a.shape
    D = wo_b.shape[0]
    _need(wo_a, "wo_a", torch.bfloat16)
    _need(wo_b, "wo_b", torch.bfloat16, (D, G * R))
    _need(o, "o", torch.bfloat16)
    if o.numel() % (G * Kg) != 0:
        raise ValueError("o must hold whole rows of G*Kg values")
    M = o.numel() // (G * Kg)
    if r is None:
        r = torch.empty(M, G * R, dtype=torch.bfloat16, device=o.device)
    if y is None:
        y = torch.empty(M, D, dtype=torch.float32, device=o.device)
    _need(r, "r", torch.bfloat16, (M, G * R))
    _need(y, "y", torch.float32, (M, D))
    if ws is None:
        ws = workspace(_lib.CSA_WS_OUTPUT_PROJ, 1, 1, 1, 1, o.device)
    check(_lib.load().csa_output_projection(M, G, Kg, R, D, o.data_ptr(), wo_a.data_ptr(), wo_b.data_ptr(),
                                            r.data_ptr(), y.data_ptr(), ws.data_ptr(), ws.numel(), _stream()),
          "csa_output_projection")
    return r, y


def linear(x: torch.Tensor, w: torch.Tensor, out_dtype: torch.dtype = torch.bfloat16, y: Optional[torch.Tensor] = None,
           ws: Optional[torch.Tensor] = None) -> torch.Tensor:
    """y = x . w^T for x [M, K], w [N, K] bf16; y bf16 or fp32 [M, N]."""
    M, K = x.shape
    N = w.shape[0]
    _need(x, "x", torch.bfloat16)
    _need(w, "w", torch.bfloat16, (N, K))
    if y is None:
        y = torch.empty(M, N, dtype=out_dtype, device=x.device)
    _need(y, "y", out_dtype, (M, N))
    if out_dtype not in (torch.bfloat16, torch.float32):
        raise TypeError("out_dtype must be bf16 or fp32")
    if ws is None:
        ws = workspace(_lib.CSA_WS_Q_PROJ, 1, 1, 1, 1, x.device)
    check(_lib.load().csa_linear(M, N, K, x.data_ptr(), w.data_ptr(), y.data_ptr(), int(out_dtype == torch.float32),
                                 ws.data_ptr(), ws.numel(), _stream()), "csa_linear")
    return y


def compressor_streams(x: torch.Tensor, w_kv: torch.Tensor, w_score: torch.Tensor):
    """The compressor's per-token states from the hidden states x [M, hidden]: kv = x . w_kv^T and
    score = x . w_score^T (bf16 [M, width]), the inputs of csa_compress."""
    return linear(x, w_kv), linear(x, w_score)


def q_projection(x: torch.Tensor, wq_a: torch.Tensor, gamma: torch.Tensor, wq_b: torch.Tensor, pos: torch.Tensor,
                 H: int = 128, d: int = 512, rope_dim: int = 64, rope_base: float = 10000.0, eps: float = 1e-6,
                 q: Optional[torch.Tensor] = None, ws: Optional[torch.Tensor] = None):
    """Low-rank query path: x [M, hidden], wq_a [q_rank, hidden], gamma [q_rank], wq_b [H*d, q_rank]
    (bf16), pos [M] int32. Returns (qa fp32 [M, q_rank], qr bf16 [M, q_rank], q bf16 [M, H, d])."""
    M, hidden = x.shape
    q_rank = wq_a.shape[0]
    _need(x, "x", torch.bfloat16)
    _need(wq_a, "wq_a", torch.bfloat16, (q_rank, hidden))
    _need(gamma, "gamma", torch.bfloat16, (q_rank,))
    _need(wq_b, "wq_b", torch.bfloat16, (H * d, q_rank))
    _need(pos, "pos", torch.int32, (M,))
    qa = torch.empty(M, q_rank, dtype=torch.float32, device=x.device)
    qr = torch.empty(M, q_rank, dtype=torch.bfloat16, device=x.device)
    if q is None:
        q = torch.empty(M, H, d, dtype=torch.bfloat16, device=x.device)
    _need(q, "q", torch.bfloat16, (M, H, d))
    if ws is None:
        ws = workspace(_lib.CSA_WS_Q_PROJ, 1, 1, 1, 1, x.device)
    check(_lib.load().csa_q_projection(M, hidden, q_rank, H, d, rope_dim, rope_base, eps, pos.data_ptr(),
                                       x.data_ptr(), wq_a.data_ptr(), gamma.data_ptr(), wq_b.data_ptr(),
                                       qa.data_ptr(), qr.data_ptr(), q.data_ptr(), ws.data_ptr(), ws.numel(),
                                       _stream()), "csa_q_projection")
    return qa, qr, q


def window_projection(x: torch.Tensor, wkv: torch.Tensor, pos: torch.Tensor, rope_dim: int = 64,
                      rope_base: float = 10000.0, win: Optional[torch.Tensor] = None,
                      ws: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Window rows: RoPE_pos(x . wkv^T) for x [M, hidden], wkv [d, hidden] bf16; returns bf16 [M, d]."""
    M, hidden = x.shape
    d = wkv.shape[0]
    _need(x, "x", torch.bfloat16)
    _need(wkv, "wkv", torch.bfloat16, (d, hidden))
    _need(pos, "pos", torch.int32, (M,))
    if win is None:
        win = torch.empty(M, d, dtype=torch.bfloat16, device=x.device)
    _need(win, "win", torch.bfloat16, (M, d))
    if ws is None:
        ws = workspace(_lib.CSA_WS_Q_PROJ, 1, 1, 1, 1, x.device)
    check(_lib.load().csa_window_projection(M, hidden, d, rope_dim, rope_base, pos.data_ptr(), x.data_ptr(),
                                            wkv.data_ptr(), win.data_ptr(), ws.data_ptr(), ws.numel(), _stream()),
          "csa_window_projection")
    return win


def device_status(ws: torch.Tensor) -> int:
    """Synchronise the current stream, read and clear the workspace's device status word."""
    st = ctypes.c_int(0)
    check(_lib.load().csa_get_device_status(ws.data_ptr(), _stream(), ctypes.byref(st)), "csa_get_device_status")
    return st.value
