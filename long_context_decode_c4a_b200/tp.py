"""Tensor-parallel indexer: the indexer heads split over the ranks of a process group.

"DeepSeek-V4-Pro 架构：一个 token 的旅程", section "少读 KV 之前，Indexer 仍要给历史打分": under tensor
parallelism over the indexer heads, each rank scores the history with its own heads, the partial
scores are summed across ranks (an all-reduce), and only then are the top-k entries selected. The
score is a sum over heads of w_h * ReLU(q_h . k), so the partial sums add up to the full score.

Every rank runs csa_indexer_scores on its head shard, torch.distributed sums the score rows (NCCL
on GPUs), and csa_topk selects on every rank (each rank then holds the same selection).
"""

from __future__ import annotations

from typing import Optional, Tuple

import torch
import torch.distributed as dist

from . import ops


def head_shard(H_I: int, rank: int, world: int) -> Tuple[int, int]:
    """Heads [lo, hi) of rank `rank` when H_I heads are split evenly over `world` ranks."""
    if H_I % world != 0:
        raise ValueError(f"{H_I} indexer heads do not split evenly over {world} ranks")
    per = H_I // world
    return rank * per, (rank + 1) * per


def tp_indexer_topk(q_pos: torch.Tensor, q_idx_shard: torch.Tensor, w_shard: torch.Tensor, idx_cache: torch.Tensor,
                    k: int, ratio: int = 4, group: Optional[dist.ProcessGroup] = None,
                    scores: Optional[torch.Tensor] = None) -> torch.Tensor:
    """Top-k selection with the indexer heads sharded over `group`: q_idx_shard [B,S,H_I/N,d_I] and
    w_shard [B,S,H_I/N] hold this rank's heads (see head_shard). Returns topk_idx [B,S,k], the same
    on every rank."""
    scores = ops.indexer_scores(q_pos, q_idx_shard, w_shard, idx_cache, ratio, scores=scores)
    # Columns past a query's visible prefix are not written by the scorer and not read by the
    # selection, so whatever the sum makes of them is never used.
    if dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(scores, op=dist.ReduceOp.SUM, group=group)
    return ops.topk(q_pos, scores, k, ratio)
