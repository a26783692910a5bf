"""Workload table and seeded input generators.

Every tensor is drawn from a torch generator seeded with the workload's seed, in
the fixed order listed in each generator below, so that any consumer (the CUDA
path's tests, the benchmark, the CPU oracle) sees the same values for the same
(workload, device kind). Values follow the workload recipe:

* caches, compressor streams, window rows, q and q_idx: bf16 rounding of N(0, 1);
* q is scaled per head to unit root-mean-square before rounding (the query path
  upstream of the layer RMS-normalises q per head; this only shapes the input
  distribution);
* indexer weights w ~ N(0, 1) / sqrt(d_I) / sqrt(H_I) in fp32 (they may be negative);
* sink ~ N(0, 1) in fp32, one per query head;
* RMSNorm weights (gamma) are all ones.

Nothing here computes a step of the layer.
"""

from __future__ import annotations

import dataclasses
import math
from typing import Dict, Optional

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    kind: str            # "csa_decode" | "hca_decode" | "csa_prefill" | "hca_prefill"
    B: int               # requests
    S: int               # new tokens per request in this call
    ctx: int             # context length per request after this call
    H: int = 128         # query heads
    d: int = 512         # head dim of the shared MQA KV row
    rope_dim: int = 64
    rope_base: float = 10000.0
    eps: float = 1e-6
    W: int = 128         # sliding window (tokens)
    ratio: int = 4       # compression ratio (4: C4A with overlap, 128: C128A)
    H_I: int = 64        # indexer heads
    d_I: int = 128       # indexer head dim (and index-cache width)
    topk: int = 1024
    seed: int = 0

    @property
    def overlap(self) -> int:
        return 1 if self.ratio == 4 else 0

    @property
    def start_pos(self) -> int:
        return self.ctx - self.S

    @property
    def max_entries(self) -> int:
        return self.ctx // self.ratio

    @property
    def ring_cap(self) -> int:
        # Decode keeps a ring of W rows; prefill hands the layer every token's
        # window row, so the "ring" is the whole segment.
        return self.W if self.kind.endswith("decode") else self.S

    @property
    def is_decode(self) -> bool:
        return self.kind.endswith("decode")

    @property
    def has_indexer(self) -> bool:
        return self.kind.startswith("csa")

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS: Dict[str, Workload] = {
    # B=1, S=128, 8 heads x 512, window 16, ratio 4 (32 entries), indexer 4 x 128, top-k 8.
    "tiny_csa_prefill": Workload("tiny_csa_prefill", "csa_prefill", B=1, S=128, ctx=128,
                                 H=8, W=16, H_I=4, topk=8),
    # B=64 requests at position 32767: entry 8191 is completed in-step.
    "pro_csa_decode_32k": Workload("pro_csa_decode_32k", "csa_decode", B=64, S=1, ctx=32768),
    # B=64, ratio 128 without overlap: entry 255 completed in-step, all 256 read.
    "pro_hca_decode_32k": Workload("pro_hca_decode_32k", "hca_decode", B=64, S=1, ctx=32768,
                                   ratio=128, H_I=0, topk=0),
    # B=1, S=8192 new tokens from an empty cache.
    "csa_prefill_8k": Workload("csa_prefill_8k", "csa_prefill", B=1, S=8192, ctx=8192),
    # B=8 requests at position 1048575: 262144 entries per request.
    "long_csa_decode_1m": Workload("long_csa_decode_1m", "csa_decode", B=8, S=1, ctx=1048576),
    # B=1, S=8192 new tokens from an empty cache through the HCA layer: ratio 128 without overlap
    # (64 entries), every visible entry read, no indexer.
    "hca_prefill_8k": Workload("hca_prefill_8k", "hca_prefill", B=1, S=8192, ctx=8192, ratio=128, H_I=0, topk=0),
}


def decode_positions(wl: Workload) -> torch.Tensor:
    """Absolute position of every new token, [B, S] int32."""
    base = torch.arange(wl.start_pos, wl.ctx, dtype=torch.int32)
    return base.unsqueeze(0).repeat(wl.B, 1).contiguous()


_CHUNK = 1 << 24


def _randn(gen: torch.Generator, shape, device, dtype=torch.bfloat16) -> torch.Tensor:
    """N(0,1) draws in chunks (keeps fp32 temporaries small), rounded to dtype."""
    out = torch.empty(shape, dtype=dtype, device=device)
    flat = out.view(-1)
    n = flat.numel()
    for lo in range(0, n, _CHUNK):
        hi = min(n, lo + _CHUNK)
        flat[lo:hi] = torch.randn(hi - lo, generator=gen, device=device, dtype=torch.float32).to(dtype)
    return out


def _unit_rms_rows(gen: torch.Generator, shape, device) -> torch.Tensor:
    """N(0,1) rows scaled to unit root-mean-square along the last axis, bf16."""
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    rows = out.view(-1, shape[-1])
    step = max(1, _CHUNK // shape[-1])
    for lo in range(0, rows.shape[0], step):
        hi = min(rows.shape[0], lo + step)
        x = torch.randn(hi - lo, shape[-1], generator=gen, device=device, dtype=torch.float32)
        x = x * torch.rsqrt(x.square().mean(dim=-1, keepdim=True) + 1e-6)
        rows[lo:hi] = x.to(torch.bfloat16)
    return out


def make_inputs(wl: Workload, device: str = "cpu", seed: Optional[int] = None) -> Dict[str, torch.Tensor]:
    """Draw every input of one call of the layer for workload ``wl``.

    Decode workloads (S=1, every request at position ctx-1):
      cache [B,E,d], idx_cache [B,E,d_I] (entries 0..E-2 hold history; entry E-1 is
      produced in-step), ring [B,W,d], compressor state, the current token's compressor
      streams, its window row, q, q_idx, w, sink.
    Prefill workloads (from an empty cache): compressor streams [B,S,(1+ov)d], window rows
      [B,S,d] (they serve as the ring), q [B,S,H,d], q_idx [B,S,H_I,d_I], w [B,S,H_I], sink.
    Draw order: caches, ring, states, streams, window rows, q, q_idx, w, sink.
    """
    seed = wl.seed if seed is None else seed
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    B, S, d, dI = wl.B, wl.S, wl.d, wl.d_I
    ov = wl.overlap
    width = (1 + ov) * d
    iwidth = 2 * dI
    out: Dict[str, torch.Tensor] = {}
    out["pos"] = decode_positions(wl).to(device)
    E = wl.max_entries

    if wl.is_decode:
        out["cache"] = _randn(gen, (B, E, d), device)
        if wl.has_indexer:
            out["idx_cache"] = _randn(gen, (B, E, dI), device)
        out["ring"] = _randn(gen, (B, wl.W, d), device)
        srows = (1 + ov) * wl.ratio
        out["state_kv"] = _randn(gen, (B, srows, width), device)
        out["state_score"] = _randn(gen, (B, srows, width), device)
        if wl.has_indexer:
            out["idx_state_kv"] = _randn(gen, (B, 2 * wl.ratio, iwidth), device)
            out["idx_state_score"] = _randn(gen, (B, 2 * wl.ratio, iwidth), device)
        out["kv"] = _randn(gen, (B, S, width), device)
        out["score"] = _randn(gen, (B, S, width), device)
        if wl.has_indexer:
            out["idx_kv"] = _randn(gen, (B, S, iwidth), device)
            out["idx_score"] = _randn(gen, (B, S, iwidth), device)
        out["win_kv"] = _randn(gen, (B, S, d), device)
    else:
        out["kv"] = _randn(gen, (B, S, width), device)
        out["score"] = _randn(gen, (B, S, width), device)
        if wl.has_indexer:
            out["idx_kv"] = _randn(gen, (B, S, iwidth), device)
            out["idx_score"] = _randn(gen, (B, S, iwidth), device)
        out["win_kv"] = _randn(gen, (B, S, d), device)

    out["q"] = _unit_rms_rows(gen, (B, S, wl.H, d), device)
    if wl.has_indexer:
        out["q_idx"] = _randn(gen, (B, S, wl.H_I, dI), device)
        out["w"] = (torch.randn(B, S, wl.H_I, generator=gen, device=device, dtype=torch.float32)
                    / math.sqrt(dI) / math.sqrt(wl.H_I))
    out["sink"] = torch.randn(wl.H, generator=gen, device=device, dtype=torch.float32)
    out["gamma"] = torch.ones(d, dtype=torch.bfloat16, device=device)
    if wl.has_indexer:
        out["idx_gamma"] = torch.ones(dI, dtype=torch.bfloat16, device=device)
    return out


# Grouped output projection ([P1] "输出投影也分组"): Pro shapes.
OPROJ_GROUPS, OPROJ_KG, OPROJ_R, OPROJ_D = 16, 4096, 1024, 7168


def make_oproj_inputs(M: int, G: int = OPROJ_GROUPS, Kg: int = OPROJ_KG, R: int = OPROJ_R, D: int = OPROJ_D,
                      seed: int = 0, device: str = "cpu") -> Dict[str, torch.Tensor]:
    """Seeded inputs of the output projection: o [M, G*Kg] ~ bf16 N(0,1) / 4 (the attention output is a
    convex combination of cache rows, smaller than a row), random weights Wo_a [G, R, Kg] ~ N(0,1)/sqrt(Kg)
    and Wo_b [D, G*R] ~ N(0,1)/sqrt(G*R), bf16. Draw order: o, Wo_a, Wo_b."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    o = _randn(gen, (M, G * Kg), device, dtype=torch.float32).mul_(0.25).to(torch.bfloat16)
    wa = _randn(gen, (G, R, Kg), device, dtype=torch.float32).mul_(1.0 / math.sqrt(Kg)).to(torch.bfloat16)
    wb = _randn(gen, (D, G * R), device, dtype=torch.float32).mul_(1.0 / math.sqrt(G * R)).to(torch.bfloat16)
    return {"o": o, "wo_a": wa, "wo_b": wb}


# Low-rank query path ([P1] "低秩 Q") and the window-row projection: Pro shapes.
QPATH_HIDDEN, QPATH_RANK, QPATH_HEADS = 7168, 1536, 128


def make_qpath_inputs(M: int, hidden: int = QPATH_HIDDEN, q_rank: int = QPATH_RANK, H: int = QPATH_HEADS,
                      d: int = 512, start_pos: int = 0, seed: int = 0, device: str = "cpu") -> Dict[str, torch.Tensor]:
    """Seeded inputs of the query path and the window-row projection: x [M, hidden] ~ bf16 N(0,1),
    Wq_a [q_rank, hidden] ~ N(0,1)/sqrt(hidden), gamma = 1, Wq_b [H*d, q_rank] ~ N(0,1)/sqrt(q_rank),
    Wkv [d, hidden] ~ N(0,1)/sqrt(hidden) (bf16), positions start_pos .. start_pos+M-1.
    Draw order: x, Wq_a, Wq_b, Wkv."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    x = _randn(gen, (M, hidden), device)
    wa = _randn(gen, (q_rank, hidden), device, dtype=torch.float32).mul_(1.0 / math.sqrt(hidden)).to(torch.bfloat16)
    wb = _randn(gen, (H * d, q_rank), device, dtype=torch.float32).mul_(1.0 / math.sqrt(q_rank)).to(torch.bfloat16)
    wkv = _randn(gen, (d, hidden), device, dtype=torch.float32).mul_(1.0 / math.sqrt(hidden)).to(torch.bfloat16)
    pos = torch.arange(start_pos, start_pos + M, dtype=torch.int32, device=device)
    return {"x": x, "wq_a": wa, "gamma_q": torch.ones(q_rank, dtype=torch.bfloat16, device=device), "wq_b": wb,
            "wkv": wkv, "pos": pos}
