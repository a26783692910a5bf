"""The tensor-parallel indexer's two halves on one GPU (csa_indexer_scores, csa_topk).

The ranks of a head split are emulated one after another on the same GPU: each head shard's
partial scores come from csa_indexer_scores, the test adds them (standing in for the all-reduce),
and csa_topk selects. The sum must match the oracle's scores of all heads, and the selection the
oracle's top-k of them (near-tie rule)."""

import numpy as np
import pytest
import torch

from oracle import csa_oracle as O
from synth import WORKLOADS, make_inputs
from tests.parity import check_topk, np64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ops():
    from long_context_decode_c4a_b200 import ops
    return ops


@pytest.mark.parametrize("world", [2, 4])
def test_head_shards_sum_to_the_full_scores_and_select_the_same_entries(ops, world):
    from long_context_decode_c4a_b200.tp import head_shard
    wl = WORKLOADS["pro_csa_decode_32k"].scaled(B=3, ctx=8192)
    inp = make_inputs(wl, device="cuda")
    pos = inp["pos"]
    q_idx, w, icache = inp["q_idx"], inp["w"], inp["idx_cache"]
    B, S, H_I = w.shape
    total = torch.zeros(B, S, wl.max_entries, dtype=torch.float32, device="cuda")
    for r in range(world):
        lo, hi = head_shard(H_I, r, world)
        part = ops.indexer_scores(pos, q_idx[:, :, lo:hi].contiguous(), w[:, :, lo:hi].contiguous(), icache)
        total += part
    sel = ops.topk(pos, total, wl.topk)
    torch.cuda.synchronize()
    for b in range(B):
        t = int(pos[b, 0])
        vis = (t + 1) // wl.ratio
        ref = O.indexer_scores(np64(q_idx[b, 0]), np64(w[b, 0]), O.bf16(np64(icache[b])), vis)
        got = np64(total[b, 0, :vis])
        assert np.max(np.abs(got - ref)) <= 1e-4 * np.max(np.abs(ref)) + 1e-6
        check_topk(np64(sel[b, 0]), ref, wl.topk, f"tp world={world} b={b}")


def test_topk_over_given_scores_matches_the_fused_selection(ops):
    """csa_topk on the scores csa_indexer_topk itself produced selects the same indices."""
    wl = WORKLOADS["pro_csa_decode_32k"].scaled(B=4, ctx=32768)
    inp = make_inputs(wl, device="cuda")
    scores = torch.empty(wl.B, 1, wl.max_entries, dtype=torch.float32, device="cuda")
    fused = ops.indexer_topk(inp["pos"], inp["q_idx"], inp["w"], inp["idx_cache"], wl.topk, scores=scores)
    alone = ops.topk(inp["pos"], scores, wl.topk)
    torch.cuda.synchronize()
    assert torch.equal(fused, alone)
