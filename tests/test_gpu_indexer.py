"""GPU parity of the lightning indexer (tcgen05) and the radix-select top-k (csa_indexer_topk)."""

import math

import numpy as np
import pytest
import torch

from oracle import csa_oracle as O
from tests.parity import check_topk, np64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ops():
    from long_context_decode_c4a_b200 import ops
    return ops


def _inputs(B, S, H_I, E_cap, seed, dup_every=0):
    g = torch.Generator().manual_seed(seed)
    q_idx = torch.randn(B, S, H_I, 128, generator=g).to(torch.bfloat16)
    w = torch.randn(B, S, H_I, generator=g) / math.sqrt(128) / math.sqrt(H_I)
    cache = torch.randn(B, E_cap, 128, generator=g).to(torch.bfloat16)
    if dup_every:
        # repeated entries give exactly equal scores: ties must go to the lower index
        cache = cache[:, (torch.arange(E_cap) // dup_every) * dup_every].contiguous()
    return q_idx, w, cache


def _run(ops, pos, q_idx, w, cache, topk):
    B, S = pos.shape
    scores = torch.full((B, S, cache.shape[1]), float("nan"), dtype=torch.float32, device="cuda")
    idx = ops.indexer_topk(pos.cuda(), q_idx.cuda(), w.cuda(), cache.cuda(), topk, scores=scores)
    torch.cuda.synchronize()
    return np64(scores), np64(idx)


@pytest.mark.parametrize("case", ["decode_ragged", "prefill_groups", "tiny_heads", "ties"])
def test_indexer_scores_and_topk(ops, case):
    if case == "decode_ragged":      # S = 1, E not a multiple of the 128-entry tile, varied positions
        B, S, H_I, E_cap, topk = 3, 1, 64, 1000, 256
        pos = torch.tensor([[3999], [2100], [130]], dtype=torch.int32)
    elif case == "prefill_groups":   # S > 1: 4 queries per tcgen05 tile (N = 256), causal visibility
        B, S, H_I, E_cap, topk = 1, 301, 64, 300, 64
        pos = torch.arange(S, dtype=torch.int32)[None] * 4
    elif case == "tiny_heads":       # 4 indexer heads (the tiny config), 64 queries per tile
        B, S, H_I, E_cap, topk = 1, 128, 4, 32, 8
        pos = torch.arange(S, dtype=torch.int32)[None]
    else:
        B, S, H_I, E_cap, topk = 2, 1, 64, 2000, 300
        pos = torch.tensor([[7999], [6003]], dtype=torch.int32)
    q_idx, w, cache = _inputs(B, S, H_I, E_cap, seed=hash(case) % 1000, dup_every=8 if case == "ties" else 0)
    sc, idx = _run(ops, pos, q_idx, w, cache, topk)
    qn, wn, cn = np64(q_idx), np64(w), np64(cache)
    for b in range(B):
        for i in range(S):
            t = int(pos[b, i])
            E = min((t + 1) // 4, E_cap)
            ref = O.indexer_scores(qn[b, i], wn[b, i], cn[b], E)
            got = sc[b, i, :E]
            scale = max(1e-30, np.max(np.abs(ref))) if E else 1.0
            assert np.max(np.abs(got - ref), initial=0.0) <= 1e-4 * scale, f"scores b={b} i={i}"
            assert np.all(np.isnan(sc[b, i, E:])), "no score beyond the visible entries may be written"
            # Same fp32 scores on both sides: the selection must agree exactly.
            assert np.array_equal(idx[b, i], O.topk_select(got, topk)), f"top-k on GPU scores b={b} i={i}"
            # Against the oracle's fp64 scores: the near-tie rule.
            check_topk(idx[b, i], ref, topk, f"b={b} i={i}")


def test_topk_two_stage_long_rows(ops):
    """E > 16384 entries per query uses chunked selection plus a merge."""
    B, S, H_I, topk = 2, 1, 64, 1024
    E_cap = 40000
    pos = torch.tensor([[4 * 40000 - 1], [4 * 33000 + 2]], dtype=torch.int32)
    q_idx, w, cache = _inputs(B, S, H_I, E_cap, seed=11, dup_every=3)
    sc, idx = _run(ops, pos, q_idx, w, cache, topk)
    for b in range(B):
        E = min((int(pos[b, 0]) + 1) // 4, E_cap)
        got = sc[b, 0, :E]
        assert np.array_equal(idx[b, 0], O.topk_select(got, topk)), f"b={b}"
        ref = O.indexer_scores(np64(q_idx[b, 0]), np64(w[b, 0]), np64(cache[b]), E)
        check_topk(idx[b, 0], ref, topk, f"b={b}")


def test_topk_long_rows_exact(ops):
    """Rows of 262144 entries (chunks of 16384 selected apart, then their lists merged): random
    scores; one value everywhere (the first k indices); two values whose tie at the threshold spans
    chunk boundaries; +-inf and NaN with a shorter visible count; and a row with fewer visible
    entries than k. Exact against the oracle's selection on the same fp32 scores."""
    B, E, k = 5, 262144, 1024
    g = torch.Generator().manual_seed(23)
    sc = torch.randn(B, 1, E, generator=g)
    sc[1] = 0.5
    sc[2] = 0.5
    hot = torch.randperm(E, generator=g)[:500]
    sc[2, 0, hot] = 1.0                                  # 500 above, the first 524 of the 0.5s kept
    sc[3, 0, ::1001] = float("inf")
    sc[3, 0, 7::2003] = float("nan")
    sc[3, 0, 11::3001] = -float("inf")
    pos = torch.full((B, 1), 4 * E - 1, dtype=torch.int32)
    pos[3, 0] = 4 * 100000 - 1                          # 100000 visible entries
    pos[4, 0] = 4 * 900 - 1                             # 900 visible entries < k
    idx = ops.topk(pos.cuda(), sc.cuda(), k)
    torch.cuda.synchronize()
    idx = idx.cpu().numpy()
    for b in range(B):
        Eb = min((int(pos[b, 0]) + 1) // 4, E)
        want = O.topk_select(sc[b, 0, :Eb].double().numpy(), k)
        assert np.array_equal(idx[b, 0], want), f"row {b}"
    assert np.array_equal(idx[1, 0], np.arange(k))
    assert np.array_equal(idx[4, 0], np.r_[np.arange(900), -np.ones(k - 900)])


def test_topk_edge_cases(ops):
    """No visible entry, fewer entries than k, and exactly k entries."""
    B, S, H_I, topk = 1, 4, 64, 16
    pos = torch.tensor([[0, 2, 40, 63]], dtype=torch.int32)      # E = 0, 0, 10, 16
    q_idx, w, cache = _inputs(B, S, H_I, 16, seed=5)
    sc, idx = _run(ops, pos, q_idx, w, cache, topk)
    assert np.all(idx[0, 0] == -1) and np.all(idx[0, 1] == -1)
    assert np.array_equal(idx[0, 2], np.r_[np.arange(10), -np.ones(6)])
    assert np.array_equal(idx[0, 3], np.arange(16))


@pytest.mark.parametrize("case", ["all_equal", "one_outlier", "inf_nan", "wide_range", "two_values"])
def test_topk_adversarial_score_distributions(ops, case):
    """Score rows whose shape stresses the radix select: one value everywhere, a single far
    outlier above a tie, +-inf and NaN scores (NaN ranks last), scores spread over ~2^100, and two
    distinct values. The selection must equal the oracle's order on the very scores the GPU wrote."""
    B, S, H_I, topk = 2, 1, 64, 1024
    E = 6000 if case != "wide_range" else 16000
    q_idx, w, cache = _inputs(B, S, H_I, E, seed=17)
    if case == "all_equal":
        cache[:] = cache[:, :1]
    elif case == "one_outlier":
        cache[:] = cache[:, :1]
        cache[:, 4321] = cache[:, 4321] * 64
    elif case == "inf_nan":
        # q dims 5 and 9 > 0; request 0 weights all < 0, request 1 all > 0: a row with +inf in
        # dim 5 scores -inf (request 0) or +inf (request 1); +inf in 5 with -inf in 9 gives NaN.
        q_idx[..., 5] = q_idx[..., 5].abs() + 0.1
        q_idx[..., 9] = q_idx[..., 9].abs() + 0.1
        w[0] = -w[0].abs()
        w[1] = w[1].abs()
        cache[:, ::97, 5] = float("inf")
        cache[:, 3::89, 5] = float("inf")
        cache[:, 3::89, 9] = -float("inf")
    elif case == "wide_range":
        scale = torch.exp2(torch.randint(-50, 50, (B, E, 1)).float())
        cache = (cache.float() * scale).to(torch.bfloat16)
    elif case == "two_values":
        cache[:] = cache[:, :1]
        cache[:, 1::3] = cache[:, 1::3] * 2
    pos = torch.full((B, S), 4 * E - 1, dtype=torch.int32)
    sc, idx = _run(ops, pos, q_idx, w, cache, topk)
    if case == "inf_nan":
        assert np.isnan(sc[:, 0, :E]).all(axis=0).any()
        assert (sc[0, 0, :E] == -np.inf).any() and (sc[1, 0, :E] == np.inf).any()
    for b in range(B):
        assert np.array_equal(idx[b, 0], O.topk_select(sc[b, 0, :E], topk)), f"b={b}"
