"""CPU oracle for the DeepSeek-V4-Pro compressed-sparse-attention (CSA) layer.

TEST INFRASTRUCTURE ONLY. This module is the slow, obviously-correct reference that
the CUDA path is checked against. Only the test suite, the smoke check and the
benchmark's CPU-baseline / reference leg may import it; the product path never does.
It shares no code with the CUDA path.

Arithmetic is float64 throughout. Inputs arrive as float64 arrays holding bf16 values
(exactly representable). Results that the layer stores in bf16 (compressed cache
entries) are also returned rounded to bf16 by `bf16()`.

Sources (pages are cited by title and section):
  [P1] "DeepSeek-V4-Pro 架构：一个 token 的旅程" (hs-black.github.io/posts/deepseek-v4-pro)
  [P5] "图解DeepSeek V4：详细计算流程解析" (jsqmd.com, news 710938)

Where the pages are silent the oracle takes one reading, named READING-n below:
  R1  "first half / second half": channels [:d] of the previous group's tokens and
      channels [d:] of the current group's tokens ([P5] §2.1, the torch.cat line).
  R2  the previous-group slots of group 0 have gate -inf and weight 0, and are skipped
      (never multiplied), so no 0*NaN can arise ([P1] "一个通道，逐项算出压缩结果").
  R3  RMSNorm: y = gamma * x / sqrt(mean(x^2) + eps) over all d dims, eps = 1e-6.
  R4  RoPE: adjacent pairs (2i, 2i+1) of the last rope_dim dims, theta_i = base^(-2i/rope_dim).
  R5  the RoPE position of compressed entry g is g * ratio (its group's first token).
  R6  the sink is one extra logit per head in the softmax denominator, with no value row;
      the running max includes it.
  R7  the index cache is made by the same C4A compressor at d = 128 (RMSNorm + RoPE).
  R8  C128A: one width-d stream, a state of ratio rows, softmax over all ratio slots.
  R9  one cached 512-dim row serves as both key and value (MQA).
  R10 inverse RoPE on the output uses the query's own position t.
  R11 window = tokens max(0, t-W+1) .. t (the current token included); window rows and
      selected compressed entries are both kept (no de-duplication).
  R12 top-k output is in ascending index order, padded with -1; when k >= visible
      entries, every visible entry is taken.
  R13 ties in the indexer score go to the lower index; -0 equals +0; NaN sorts lowest.
  R14 the compressor scores are used as given (no extra bias).
  R20 output projection: the intermediate r of each group is rounded to bf16 before the second
      product (the pages give the two einsums, not the precision between them).
  R21 query path: qr = rms_norm(x Wq_a^T) uses a weight gamma and eps = 1e-6 (as R3) and is rounded
      to bf16 before the second product; the product qr Wq_b^T is rounded to bf16 before the
      per-head norm; the window row x Wkv^T is rounded to bf16 before its rotation.
"""

from __future__ import annotations

import math
from typing import Dict, List, Optional, Sequence, Tuple

import numpy as np

NEG_INF = -np.inf


# ----------------------------------------------------------------------------- rounding

def bf16(x) -> np.ndarray:
    """Round to the nearest bfloat16 value (ties to even), via float32, returned as float64."""
    f = np.asarray(x, dtype=np.float64).astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + (((u >> np.uint64(16)) & np.uint64(1)) + np.uint64(0x7FFF))) >> np.uint64(16)
    r = (u << np.uint64(16)).astype(np.uint32).view(np.float32).astype(np.float64)
    return np.where(np.isnan(f), np.nan, r)


# ----------------------------------------------------------------------------- norm / rope

def rms_norm(x: np.ndarray, gamma: np.ndarray, eps: float) -> np.ndarray:
    """R3. Normalise by the root-mean-square over the last axis, then scale by gamma.

    [P1] "压缩是逐通道的 learned pooling": pooling is followed by RMSNorm.
    """
    x = np.asarray(x, dtype=np.float64)
    return np.asarray(gamma, dtype=np.float64) * x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)


def rope_angles(pos: float, rope_dim: int, base: float) -> np.ndarray:
    """R4. Angle pos * theta_i for pair i = 0 .. rope_dim/2 - 1, theta_i = base^(-2i/rope_dim)."""
    i = np.arange(rope_dim // 2, dtype=np.float64)
    return float(pos) * np.power(float(base), -2.0 * i / rope_dim)


def rope(x: np.ndarray, pos: float, rope_dim: int, base: float, inverse: bool = False) -> np.ndarray:
    """Rotate the last ``rope_dim`` dims of x (adjacent pairs) by +angle, or -angle if inverse.

    [P1] "低秩 Q": RoPE on the last 64 dims; "输出投影也分组": o = inverse_RoPE(o).
    """
    x = np.asarray(x, dtype=np.float64)
    ang = rope_angles(pos, rope_dim, base)
    if inverse:
        ang = -ang
    c, s = np.cos(ang), np.sin(ang)
    y = x.copy()
    head = x.shape[-1] - rope_dim
    even = x[..., head + 0::2]
    odd = x[..., head + 1::2]
    y[..., head + 0::2] = even * c - odd * s
    y[..., head + 1::2] = even * s + odd * c
    return y


# ----------------------------------------------------------------------------- compressor

def pool_slots(slot_kv: np.ndarray, slot_score: np.ndarray) -> Tuple[np.ndarray, np.ndarray]:
    """Per-channel softmax over the slot axis, then the weighted sum of kv over slots.

    slot_kv, slot_score: [n_slots, d]. A score of -inf marks a missing slot (R2): its
    weight is exactly 0 and its kv is never touched.
    Returns (pooled [d], weights [n_slots, d]).
    [P1] "压缩是逐通道的 learned pooling"; [P5] §2.1 (softmax, multiply, sum over tokens).
    """
    slot_kv = np.asarray(slot_kv, dtype=np.float64)
    slot_score = np.asarray(slot_score, dtype=np.float64)
    valid = ~np.isneginf(slot_score)
    m = np.max(np.where(valid, slot_score, -np.inf), axis=0)          # [d]
    e = np.where(valid, np.exp(np.where(valid, slot_score, 0.0) - m), 0.0)
    wts = e / np.sum(e, axis=0)
    pooled = np.sum(np.where(valid, wts * np.where(valid, slot_kv, 0.0), 0.0), axis=0)
    return pooled, wts


def finish_entry(pooled: np.ndarray, g: int, ratio: int, gamma, eps, rope_dim, rope_base) -> np.ndarray:
    """RMSNorm, then RoPE on the last rope_dim dims at position g*ratio (R5)."""
    return rope(rms_norm(pooled, gamma, eps), g * ratio, rope_dim, rope_base)


class CompressorCfg:
    """ratio 4 + overlap (C4A) or ratio 128 without overlap (C128A)."""

    def __init__(self, ratio: int, d: int, rope_dim: int = 64, rope_base: float = 10000.0,
                 eps: float = 1e-6, overlap: Optional[bool] = None):
        self.ratio = ratio
        self.d = d
        self.rope_dim = rope_dim
        self.rope_base = rope_base
        self.eps = eps
        self.overlap = (ratio == 4) if overlap is None else bool(overlap)

    @property
    def width(self) -> int:          # stream width per token
        return 2 * self.d if self.overlap else self.d

    @property
    def state_rows(self) -> int:
        return 2 * self.ratio if self.overlap else self.ratio


def init_state(cfg: CompressorCfg) -> Tuple[np.ndarray, np.ndarray]:
    """A fresh compressor state: kv rows 0, score rows -inf (R2)."""
    kv = np.zeros((cfg.state_rows, cfg.width))
    sc = np.full((cfg.state_rows, cfg.width), -np.inf)
    return kv, sc


def compressor_step(cfg: CompressorCfg, state_kv: np.ndarray, state_score: np.ndarray, t: int,
                    kv_t: np.ndarray, score_t: np.ndarray, gamma) -> Optional[Tuple[int, np.ndarray]]:
    """Feed token t to the rolling state (in place); return (g, entry) when group g completes.

    C4A ([P5] §2.1): token t writes row ratio + t % ratio. When (t+1) % ratio == 0 the 2*ratio
    slots are [pre rows, channels :d] ++ [cur rows, channels d:] (R1); after compression
    the cur rows are copied over the pre rows.
    C128A ([P5] §3.1, R8): token t writes row t % ratio; when the ratio rows are full
    they are pooled directly (no rotation).
    Visibility ([P1] "压缩条目必须等整组完成后才可见"): entry t // ratio is written only when
    (t + 1) % ratio == 0.
    """
    r, d = cfg.ratio, cfg.d
    if cfg.overlap:
        row = r + t % r
    else:
        row = t % r
    state_kv[row] = kv_t
    state_score[row] = score_t
    if (t + 1) % r != 0:
        return None
    g = t // r
    if cfg.overlap:
        slot_kv = np.concatenate([state_kv[:r, :d], state_kv[r:, d:]], axis=0)
        slot_sc = np.concatenate([state_score[:r, :d], state_score[r:, d:]], axis=0)
    else:
        slot_kv, slot_sc = state_kv, state_score
    pooled, _ = pool_slots(slot_kv, slot_sc)
    entry = finish_entry(pooled, g, r, gamma, cfg.eps, cfg.rope_dim, cfg.rope_base)
    if cfg.overlap:
        state_kv[:r] = state_kv[r:]
        state_score[:r] = state_score[r:]
    return g, entry


def compress_tokens(cfg: CompressorCfg, state_kv, state_score, start_pos: int,
                    kv: np.ndarray, score: np.ndarray, gamma) -> Dict[int, np.ndarray]:
    """Token-by-token state machine over a segment; returns {g: entry (float64)}.

    state_kv / state_score are updated in place. kv, score: [S, width].
    """
    out: Dict[int, np.ndarray] = {}
    for i in range(kv.shape[0]):
        res = compressor_step(cfg, state_kv, state_score, start_pos + i, kv[i], score[i], gamma)
        if res is not None:
            out[res[0]] = res[1]
    return out


def compress_parallel(cfg: CompressorCfg, kv: np.ndarray, score: np.ndarray, gamma) -> np.ndarray:
    """Direct per-group formula over a segment that starts at position 0 ([P1]: prefill
    computes every entry of the segment at once). Returns [S // ratio, d].

    C4A entry g: slots = tokens 4(g-1)..4g-1 at channels [:d] (absent for g = 0) and tokens
    4g..4g+3 at channels [d:]; C128A entry g: tokens 128g..128g+127 at all d channels.
    """
    r, d = cfg.ratio, cfg.d
    n = kv.shape[0] // r
    out = np.zeros((n, d))
    for g in range(n):
        cur = slice(g * r, (g + 1) * r)
        if cfg.overlap:
            if g == 0:
                slot_kv, slot_sc = kv[cur, d:], score[cur, d:]
            else:
                prev = slice((g - 1) * r, g * r)
                slot_kv = np.concatenate([kv[prev, :d], kv[cur, d:]], axis=0)
                slot_sc = np.concatenate([score[prev, :d], score[cur, d:]], axis=0)
        else:
            slot_kv, slot_sc = kv[cur], score[cur]
        pooled, _ = pool_slots(slot_kv, slot_sc)
        out[g] = finish_entry(pooled, g, r, gamma, cfg.eps, cfg.rope_dim, cfg.rope_base)
    return out


def visible_entries(t: int, ratio: int) -> int:
    """[P1] "压缩条目必须等整组完成后才可见": visible = (t + 1) // ratio."""
    return (t + 1) // ratio


# ----------------------------------------------------------------------------- indexer

def indexer_scores(q_idx: np.ndarray, w: np.ndarray, idx_cache: np.ndarray, visible: int) -> np.ndarray:
    """score_s = sum_h w_h * ReLU(q_h . k_s) for s < visible.

    q_idx [H_I, d_I], w [H_I] (may be negative; not a softmax), idx_cache [>= visible, d_I].
    [P1] "少读 KV 之前，Indexer 仍要给历史打分": 64 heads x 128 dims over one shared 128-dim
    compressed index cache; the ReLU is the layer specification's choice.
    """
    k = np.asarray(idx_cache[:visible], dtype=np.float64)
    logits = k @ np.asarray(q_idx, dtype=np.float64).T               # [visible, H_I]
    return np.maximum(logits, 0.0) @ np.asarray(w, dtype=np.float64)


def topk_select(scores: np.ndarray, k: int) -> np.ndarray:
    """Indices of the min(k, n) largest scores, ties to the lower index (R13), returned in
    ascending index order and padded with -1 to length k (R12).

    [P1] "少读 KV 之前…": top-k fixes the main attention reads; [P5] §2 keeps <= topK entries.
    """
    scores = np.asarray(scores, dtype=np.float64)
    n = scores.shape[0]
    key = np.where(np.isnan(scores), -np.inf, scores) + 0.0     # -0 -> +0; NaN lowest
    nan_last = np.isnan(scores).astype(np.int64)
    order = np.lexsort((np.arange(n), -key, nan_last))          # NaN last, then score desc, index asc
    sel = np.sort(order[: min(k, n)])
    out = np.full(k, -1, dtype=np.int64)
    out[: sel.shape[0]] = sel
    return out


# ----------------------------------------------------------------------------- attention

def window_positions(t: int, W: int) -> List[int]:
    """R11: tokens max(0, t - W + 1) .. t."""
    return list(range(max(0, t - W + 1), t + 1))


def gather_candidates(t: int, W: int, ring: np.ndarray, ring_cap: int, cache: np.ndarray,
                      selected: Sequence[int]) -> np.ndarray:
    """The one candidate set: the window rows (ring slot p % ring_cap) followed by the
    selected compressed entries (-1 padding skipped).

    [P1] "局部和压缩记忆，共用一次归一化"; [P5] §2 (concat of the two KV paths; length <=
    window_size + topK).
    """
    rows = [ring[p % ring_cap] for p in window_positions(t, W)]
    rows += [cache[s] for s in selected if s >= 0]
    return np.asarray(rows, dtype=np.float64)


def mqa_with_sink(q: np.ndarray, cand: np.ndarray, sink: np.ndarray, scale: float) -> np.ndarray:
    """Two-pass softmax attention of every head over one shared candidate set (R9), with a
    learned per-head sink in the denominator and no value row for it (R6).

    l_hj = scale * q_h . c_j; m_h = max(max_j l_hj, sink_h);
    o_h = sum_j exp(l_hj - m_h) c_j / (sum_j exp(l_hj - m_h) + exp(sink_h - m_h)).
    [P1] "局部和压缩记忆…" (sink adds to the denominator, no value output); [P5] §2.3 (sink; MQA).
    """
    q = np.asarray(q, dtype=np.float64)
    cand = np.asarray(cand, dtype=np.float64)
    sink = np.asarray(sink, dtype=np.float64)
    logits = scale * (q @ cand.T)                                   # [H, n]
    m = np.maximum(np.max(logits, axis=1), sink)                    # [H]
    e = np.exp(logits - m[:, None])
    denom = np.sum(e, axis=1) + np.exp(sink - m)
    return (e @ cand) / denom[:, None]


def attend_query(q_t: np.ndarray, t: int, W: int, ring, ring_cap, cache, selected, sink,
                 scale: float, rope_dim: int, rope_base: float) -> np.ndarray:
    """Attention of one query over window + selected entries, then inverse RoPE by t (R10)."""
    cand = gather_candidates(t, W, ring, ring_cap, cache, selected)
    o = mqa_with_sink(q_t, cand, sink, scale)
    return rope(o, t, rope_dim, rope_base, inverse=True)


# ----------------------------------------------------------------------------- output projection

def output_projection(o_rows: np.ndarray, wo_a: np.ndarray, wo_b: np.ndarray):
    """[P1] "输出投影也分组，并且降低中间维度": the rows o [M, G*Kg] (the inverse-RoPE'd output of
    groups of 8 heads) are reshaped to [M, G, Kg]; r[m, g, i] = sum_k o[m, g, k] * Wo_a[g, i, k]
    (einsum "bsgd,grd->bsgr"); y = r.flatten(1) @ Wo_b^T. r is rounded to bf16 first (R20).
    Returns (r in float64, r rounded to bf16, y)."""
    M = o_rows.shape[0]
    G, R, Kg = wo_a.shape
    og = o_rows.reshape(M, G, Kg)
    r = np.einsum("mgk,grk->mgr", og, wo_a)
    rb = bf16(r)
    y = rb.reshape(M, G * R) @ wo_b.T
    return r.reshape(M, G * R), rb.reshape(M, G * R), y


# ----------------------------------------------------------------------------- query path

def q_path(x: np.ndarray, wq_a: np.ndarray, gamma: np.ndarray, wq_b: np.ndarray, pos: np.ndarray, H: int,
           d: int = 512, rope_dim: int = 64, rope_base: float = 10000.0, eps: float = 1e-6):
    """[P1] "低秩 Q：两次矩阵乘法接起来": qr = rms_norm(x Wq_a^T); q = (qr Wq_b^T) as [M, H, d];
    q = q / sqrt(mean(q^2 over each head) + eps) (no weight); the last rope_dim dims of each head are
    rotated by the token's position. Precision per R21. Returns (qa, qr rounded to bf16, q)."""
    M = x.shape[0]
    qa = x @ wq_a.T
    qr = bf16(rms_norm(qa, gamma, eps))
    qraw = bf16(qr @ wq_b.T).reshape(M, H, d)
    q = qraw / np.sqrt(np.mean(qraw * qraw, axis=-1, keepdims=True) + eps)
    for m in range(M):
        q[m] = rope(q[m], float(pos[m]), rope_dim, rope_base)
    return qa, qr, q


def window_projection(x: np.ndarray, wkv: np.ndarray, pos: np.ndarray, rope_dim: int = 64,
                      rope_base: float = 10000.0) -> np.ndarray:
    """[P5] §2: the window row of each token is its KV down-projection x Wkv^T ([hidden] -> [d]) with
    the last rope_dim dims rotated by the token's position (R21: rounded to bf16 first; the pages'
    quantisation of the other dims is not applied, R16)."""
    w = bf16(x @ wkv.T)
    return np.stack([rope(w[m], float(pos[m]), rope_dim, rope_base) for m in range(x.shape[0])])


# ----------------------------------------------------------------------------- counters

def reads_per_query(t: int, W: int, ratio: int, topk: Optional[int]) -> int:
    """Rows one query reads: min(W, t+1) window rows + min(k, visible) entries (all visible
    entries when there is no indexer). [P1] "Pro 的 CSA 和 HCA，成本交点在哪里"."""
    vis = visible_entries(t, ratio)
    return min(W, t + 1) + (vis if topk is None else min(topk, vis))


def attention_flops(H: int, reads: int, d: int) -> int:
    """[P1] "Pro 的 CSA 和 HCA…": about 4 x heads x reads x 512 FLOP (dot products + value sum)."""
    return 4 * H * reads * d


# ----------------------------------------------------------------------------- whole layer

def _np(x) -> np.ndarray:
    """torch tensor / array -> float64 numpy (bf16 values are exact in float64)."""
    if hasattr(x, "detach"):
        x = x.detach().to("cpu")
        if x.dtype.is_floating_point:
            x = x.double()
        return x.numpy()
    return np.asarray(x)


def csa_decode_request(inp: Dict[str, np.ndarray], b: int, *, H: int, d: int, W: int, topk: int,
                       d_I: int = 128, rope_dim: int = 64, rope_base: float = 10000.0,
                       eps: float = 1e-6, scale: Optional[float] = None, ratio: int = 4) -> Dict[str, np.ndarray]:
    """One CSA decode step of request b ([P5] §2 order): compressor step for the main
    (d) and index (d_I) streams, window-ring write, indexer, top-k, sparse MQA with sink,
    inverse RoPE. ``inp`` holds float64 numpy arrays shaped as the synthetic decode
    inputs. Returns the new entries, selection, output and updated state/ring.
    """
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    t = int(inp["pos"][b, 0])
    main = CompressorCfg(ratio, d, rope_dim, rope_base, eps)
    index = CompressorCfg(ratio, d_I, rope_dim, rope_base, eps)
    skv, ssc = inp["state_kv"][b].copy(), inp["state_score"][b].copy()
    ikv, isc = inp["idx_state_kv"][b].copy(), inp["idx_state_score"][b].copy()
    cache = inp["cache"][b].copy()
    icache = inp["idx_cache"][b].copy()
    ring = inp["ring"][b].copy()
    res_main = compressor_step(main, skv, ssc, t, inp["kv"][b, 0], inp["score"][b, 0], inp["gamma"])
    res_idx = compressor_step(index, ikv, isc, t, inp["idx_kv"][b, 0], inp["idx_score"][b, 0], inp["idx_gamma"])
    entry = idx_entry = None
    if res_main is not None:
        g, entry = res_main
        cache[g] = bf16(entry)
    if res_idx is not None:
        g, idx_entry = res_idx
        icache[g] = bf16(idx_entry)
    ring_cap = ring.shape[0]
    ring[t % ring_cap] = inp["win_kv"][b, 0]
    vis = visible_entries(t, ratio)
    scores = indexer_scores(inp["q_idx"][b, 0], inp["w"][b, 0], icache, vis)
    sel = topk_select(scores, topk)
    out = attend_query(inp["q"][b, 0], t, W, ring, ring_cap, cache, sel, inp["sink"], scale,
                       rope_dim, rope_base)
    return dict(entry=entry, idx_entry=idx_entry, scores=scores, topk=sel, out=out,
                state_kv=skv, state_score=ssc, idx_state_kv=ikv, idx_state_score=isc,
                cache=cache, idx_cache=icache, ring=ring)


def hca_decode_request(inp: Dict[str, np.ndarray], b: int, *, H: int, d: int, W: int, ratio: int = 128,
                       rope_dim: int = 64, rope_base: float = 10000.0, eps: float = 1e-6,
                       scale: Optional[float] = None) -> Dict[str, np.ndarray]:
    """One HCA decode step of request b ([P5] §3): C128A step, window write, attention over
    the window and every visible entry (no index module), inverse RoPE."""
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    t = int(inp["pos"][b, 0])
    cfg = CompressorCfg(ratio, d, rope_dim, rope_base, eps)
    skv, ssc = inp["state_kv"][b].copy(), inp["state_score"][b].copy()
    cache = inp["cache"][b].copy()
    ring = inp["ring"][b].copy()
    res = compressor_step(cfg, skv, ssc, t, inp["kv"][b, 0], inp["score"][b, 0], inp["gamma"])
    entry = None
    if res is not None:
        g, entry = res
        cache[g] = bf16(entry)
    ring_cap = ring.shape[0]
    ring[t % ring_cap] = inp["win_kv"][b, 0]
    vis = visible_entries(t, ratio)
    out = attend_query(inp["q"][b, 0], t, W, ring, ring_cap, cache, list(range(vis)), inp["sink"],
                       scale, rope_dim, rope_base)
    return dict(entry=entry, out=out, state_kv=skv, state_score=ssc, cache=cache, ring=ring)


def csa_prefill(inp: Dict[str, np.ndarray], b: int, queries: Sequence[int], *, H: int, d: int, W: int,
                topk: int, ratio: int = 4, d_I: int = 128, rope_dim: int = 64, rope_base: float = 10000.0,
                eps: float = 1e-6, scale: Optional[float] = None, with_indexer: bool = True
                ) -> Dict[str, object]:
    """Prefill of request b from an empty cache ([P1] "压缩条目必须等整组完成后才可见": all
    entries at once, each query with its own causal mask). The window rows of the segment
    serve as the ring. Returns the entries (float64 and bf16), and per requested query its
    scores, selection and output."""
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    main = CompressorCfg(ratio, d, rope_dim, rope_base, eps)
    entries = compress_parallel(main, inp["kv"][b], inp["score"][b], inp["gamma"])
    cache = bf16(entries)
    res: Dict[str, object] = dict(entries=entries, cache=cache)
    ring = inp["win_kv"][b]
    S = ring.shape[0]
    if with_indexer:
        index = CompressorCfg(ratio, d_I, rope_dim, rope_base, eps)
        idx_entries = compress_parallel(index, inp["idx_kv"][b], inp["idx_score"][b], inp["idx_gamma"])
        icache = bf16(idx_entries)
        res["idx_entries"] = idx_entries
        res["idx_cache"] = icache
    per_q = {}
    for i in queries:
        t = int(inp["pos"][b, i])
        vis = visible_entries(t, ratio)
        if with_indexer:
            scores = indexer_scores(inp["q_idx"][b, i], inp["w"][b, i], icache, vis)
            sel = topk_select(scores, topk)
        else:
            scores, sel = None, np.arange(vis)
        out = attend_query(inp["q"][b, i], t, W, ring, S, cache, sel, inp["sink"], scale, rope_dim, rope_base)
        per_q[i] = dict(scores=scores, topk=sel, out=out)
    res["queries"] = per_q
    return res


def to_numpy_inputs(inputs: Dict[str, object]) -> Dict[str, np.ndarray]:
    """Convert a dict of tensors (bf16/fp32/int) to float64 / integer numpy arrays."""
    return {k: _np(v) for k, v in inputs.items()}
