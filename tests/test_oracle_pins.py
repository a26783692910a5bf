"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each test checks the oracle against something other than itself: a hand-derived value
stored under tests/golden/ (with its derivation and page citation), a closed form, an
invariant, a special case that reduces to a textbook routine, or brute force on tiny
inputs.
"""

import itertools
import json
import math
import os

import numpy as np
import pytest
from scipy.special import softmax

from oracle import csa_oracle as O


def _load(golden_dir, name):
    with open(os.path.join(golden_dir, name)) as f:
        return json.load(f)


# ----------------------------------------------------------------------------- rounding

def test_bf16_rounding_matches_known_values():
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7 -> even mantissa (1.0); 1 + 3*2^-8 -> 1 + 2^-6.
    assert O.bf16(1.0 + 2.0 ** -8) == 1.0
    assert O.bf16(1.0 + 3 * 2.0 ** -8) == 1.0 + 2.0 ** -6
    assert O.bf16(-2.0 ** -130) == -2.0 ** -130          # subnormal in bf16 is exact here
    assert O.bf16(np.inf) == np.inf and np.isnan(O.bf16(np.nan))
    # Every bf16 value round-trips.
    bits = np.arange(0, 1 << 16, 7, dtype=np.uint32) << 16
    with np.errstate(invalid="ignore"):          # the NaN patterns among the bits
        vals = bits.view(np.float32).astype(np.float64)
    fin = np.isfinite(vals)
    assert np.array_equal(O.bf16(vals[fin]), vals[fin])


# ----------------------------------------------------------------------------- RoPE (T8)

def test_rope_matches_complex_rotation():
    rng = np.random.default_rng(1)
    x = rng.standard_normal(512)
    pos, base, rd = 32767, 10000.0, 64
    y = O.rope(x, pos, rd, base)
    z = x[-rd:][0::2] + 1j * x[-rd:][1::2]
    theta = np.array([base ** (-(2.0 * i) / rd) for i in range(rd // 2)])
    zr = z * np.exp(1j * pos * theta)
    assert np.allclose(y[-rd:][0::2], zr.real, atol=1e-12)
    assert np.allclose(y[-rd:][1::2], zr.imag, atol=1e-12)
    assert np.array_equal(y[:-rd], x[:-rd])


def test_rope_inverse_identity_norm_and_position_zero():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((3, 512))
    for pos in (0, 1, 127, 32767, 1048575):
        y = O.rope(x, pos, 64, 10000.0)
        assert np.allclose(O.rope(y, pos, 64, 10000.0, inverse=True), x, atol=1e-12)
        assert np.allclose(np.linalg.norm(y[:, -64:], axis=1), np.linalg.norm(x[:, -64:], axis=1))
    assert np.array_equal(O.rope(x, 0, 64, 10000.0), x)
    # pair 0 has theta = 1: rotation by exactly pos radians
    e = np.zeros(512); e[448] = 1.0
    y = O.rope(e, 5, 64, 10000.0)
    assert np.isclose(y[448], math.cos(5)) and np.isclose(y[449], math.sin(5))


def test_entry_norm_rope_golden(golden_dir):
    g = _load(golden_dir, "entry_norm_rope_hand.json")
    y = O.finish_entry(np.array(g["x"]), g["g"], g["ratio"], 1.0, 0.0, 2, 10000.0)
    assert np.allclose(y, g["expected"], atol=1e-12)


# ----------------------------------------------------------------------------- compressor

def test_first_group_hand_example(golden_dir):
    """T2: the first group pools only its 4 current slots; the -inf previous slots have weight 0."""
    g = _load(golden_dir, "compress_first_group_hand.json")
    prev_sc = np.full((4, 1), -np.inf)
    prev_kv = np.full((4, 1), np.nan)          # never touched: skipped, not multiplied by 0
    slot_kv = np.concatenate([prev_kv, np.array(g["cur_kv"])[:, None]])
    slot_sc = np.concatenate([prev_sc, np.array(g["cur_scores"])[:, None]])
    pooled, wts = O.pool_slots(slot_kv, slot_sc)
    assert np.isclose(pooled[0], g["pooled"], atol=1e-12)
    assert np.allclose(wts[4:, 0], g["weights"], atol=1e-12)
    assert np.array_equal(wts[:4, 0], np.zeros(4))


def test_first_group_reduces_to_four_slot_softmax():
    rng = np.random.default_rng(3)
    cfg = O.CompressorCfg(4, 16, rope_dim=8)
    kv = rng.standard_normal((4, 32))
    sc = rng.standard_normal((4, 32)) * 3
    skv, ssc = O.init_state(cfg)
    out = O.compress_tokens(cfg, skv, ssc, 0, kv, sc, np.ones(16))
    w = softmax(sc[:, 16:], axis=0)
    pooled = np.sum(w * kv[:, 16:], axis=0)
    ref = O.rope(O.rms_norm(pooled, 1.0, cfg.eps), 0, 8, 10000.0)
    assert np.allclose(out[0], ref, atol=1e-12)


def test_weights_sum_to_one_and_constant_vector_closed_form():
    """T1: per-channel weights sum to 1, so equal kv slots give RoPE(RMSNorm(v)) for any scores."""
    rng = np.random.default_rng(4)
    d = 512
    v = rng.standard_normal(d)
    gamma = 1 + 0.1 * rng.standard_normal(d)
    cfg = O.CompressorCfg(4, d)
    for trial in range(3):
        sc = rng.standard_normal((8, 2 * d)) * 5
        kv = np.tile(np.concatenate([v, v]), (8, 1))
        out = O.compress_parallel(cfg, kv, sc, gamma)
        _, wts = O.pool_slots(np.concatenate([kv[:4, :d], kv[4:, d:]]), np.concatenate([sc[:4, :d], sc[4:, d:]]))
        assert np.allclose(wts.sum(axis=0), 1.0, atol=1e-12)
        ref = O.rope(gamma * v / math.sqrt(np.mean(v * v) + 1e-6), 4, 64, 10000.0)
        assert np.allclose(out[1], ref, atol=1e-10)


def test_halves_come_from_previous_first_and_current_second():
    """R1 (the torch.cat line of the C4A section): entry g mixes channels [:d] of the previous
    group's tokens with channels [d:] of the current group's. Values placed in the other
    halves must not appear; the result is a closed form in the two constant blocks."""
    d = 8
    cfg = O.CompressorCfg(4, d, rope_dim=2)
    A, Bv, s1, s2 = 2.0, -3.0, 0.7, -0.4
    kv = np.zeros((8, 2 * d)); sc = np.zeros((8, 2 * d))
    kv[:4, :d] = A; kv[:4, d:] = 1e6          # previous group: first half A, second half junk
    kv[4:, d:] = Bv; kv[4:, :d] = -1e6        # current group: second half B, first half junk
    sc[:4, :d] = s1; sc[4:, d:] = s2
    sc[:4, d:] = 50.0; sc[4:, :d] = 50.0      # junk scores must be ignored too
    out = O.compress_parallel(cfg, kv, sc, np.ones(d))
    pooled = (math.exp(s1) * A + math.exp(s2) * Bv) / (math.exp(s1) + math.exp(s2))
    x = np.full(d, pooled)
    ref = O.rope(x / math.sqrt(pooled * pooled + 1e-6), 4, 2, 10000.0)
    assert np.allclose(out[1], ref, atol=1e-9)


@pytest.mark.parametrize("ratio,d", [(4, 64), (4, 128), (128, 64)])
def test_state_machine_equals_parallel_and_chunked(ratio, d):
    """T3: the token-by-token rolling state equals the direct per-group formula, and
    uneven chunks resumed from the state equal one shot."""
    rng = np.random.default_rng(5 + ratio)
    cfg = O.CompressorCfg(ratio, d)
    S = 8 * ratio + 3
    kv = rng.standard_normal((S, cfg.width))
    sc = rng.standard_normal((S, cfg.width)) * 2
    gamma = 1 + 0.1 * rng.standard_normal(d)
    par = O.compress_parallel(cfg, kv, sc, gamma)
    skv, ssc = O.init_state(cfg)
    seq = O.compress_tokens(cfg, skv, ssc, 0, kv, sc, gamma)
    assert sorted(seq) == list(range(S // ratio))
    for g in seq:
        assert np.allclose(seq[g], par[g], atol=1e-12)
    # chunked: uneven splits
    cuts = [0, 1, ratio + 2, 3 * ratio - 1, 5 * ratio, S]
    skv2, ssc2 = O.init_state(cfg)
    got = {}
    for lo, hi in zip(cuts[:-1], cuts[1:]):
        got.update(O.compress_tokens(cfg, skv2, ssc2, lo, kv[lo:hi], sc[lo:hi], gamma))
    assert sorted(got) == sorted(seq)
    for g in got:
        assert np.array_equal(got[g], seq[g])
    assert np.array_equal(skv2, skv) and np.array_equal(ssc2, ssc)


def test_entry_visible_only_when_group_completes():
    """T4 (compressor side): entry g is emitted at t = ratio*g + ratio - 1 and not before."""
    cfg = O.CompressorCfg(4, 16, rope_dim=8)
    rng = np.random.default_rng(6)
    skv, ssc = O.init_state(cfg)
    for t in range(20):
        res = O.compressor_step(cfg, skv, ssc, t, rng.standard_normal(32), rng.standard_normal(32), 1.0)
        if (t + 1) % 4 == 0:
            assert res is not None and res[0] == t // 4
        else:
            assert res is None
        assert O.visible_entries(t, 4) == (t + 1) // 4


# ----------------------------------------------------------------------------- indexer / top-k

def test_indexer_hand_example(golden_dir):
    g = _load(golden_dir, "indexer_hand.json")
    s = O.indexer_scores(np.array(g["q_idx"]), np.array(g["w"]), np.array(g["idx_cache"]), 3)
    assert np.allclose(s, g["expected"], atol=1e-15)
    s2 = O.indexer_scores(np.array(g["q_idx"]), np.array(g["w"]), np.array(g["idx_cache"]), 2)
    assert s2.shape == (2,)


def test_indexer_brute_force_loops():
    rng = np.random.default_rng(7)
    q = rng.standard_normal((3, 5)); w = rng.standard_normal(3); k = rng.standard_normal((6, 5))
    s = O.indexer_scores(q, w, k, 6)
    for j in range(6):
        acc = 0.0
        for h in range(3):
            dot = sum(q[h, c] * k[j, c] for c in range(5))
            acc += w[h] * (dot if dot > 0 else 0.0)
        assert abs(acc - s[j]) < 1e-12


def _beats(a, b, sc):
    """Total order of the selection: higher score first, lower index on ties."""
    return sc[a] > sc[b] or (sc[a] == sc[b] and a < b)


@pytest.mark.parametrize("seed", range(6))
def test_topk_brute_force_over_all_subsets(seed):
    rng = np.random.default_rng(100 + seed)
    n, k = 8, 3
    sc = rng.integers(-3, 4, size=n).astype(np.float64)    # many ties
    if seed == 0:
        sc[:] = 0.0
        sc[[1, 5]] = -0.0
    sel = O.topk_select(sc, k)
    winners = [set(c) for c in itertools.combinations(range(n), k)
               if all(_beats(a, b, sc) for a in c for b in range(n) if b not in c)]
    assert len(winners) == 1
    assert set(sel.tolist()) == winners[0]
    assert list(sel) == sorted(sel)


def test_topk_padding_and_nan():
    sel = O.topk_select(np.array([0.5, 2.0, -1.0]), 5)
    assert sel.tolist() == [0, 1, 2, -1, -1]
    sel = O.topk_select(np.array([np.nan, 1.0, 0.0, np.nan]), 2)
    assert sel.tolist() == [1, 2]
    sel = O.topk_select(np.array([]), 3)
    assert sel.tolist() == [-1, -1, -1]


# ----------------------------------------------------------------------------- attention

def test_sink_softmax_hand_example(golden_dir):
    g = _load(golden_dir, "sink_softmax_hand.json")
    o = O.mqa_with_sink(np.array([g["q"]]), np.array(g["cand"]), np.array([g["sink"]]), 1.0)
    assert np.allclose(o[0], g["expected"], atol=1e-12)


def test_sink_to_minus_infinity_is_plain_softmax():
    """T6."""
    rng = np.random.default_rng(8)
    q = rng.standard_normal((4, 16)); c = rng.standard_normal((9, 16))
    o = O.mqa_with_sink(q, c, np.full(4, -np.inf), 0.25)
    ref = softmax(0.25 * q @ c.T, axis=1) @ c
    assert np.allclose(o, ref, atol=1e-12)


def test_sink_equals_extra_zero_value_column():
    rng = np.random.default_rng(9)
    q = rng.standard_normal((4, 16)); c = rng.standard_normal((9, 16)); sink = rng.standard_normal(4) * 3
    o = O.mqa_with_sink(q, c, sink, 0.25)
    logits = np.concatenate([0.25 * q @ c.T, sink[:, None]], axis=1)
    vals = np.concatenate([c, np.zeros((1, 16))], axis=0)
    assert np.allclose(o, softmax(logits, axis=1) @ vals, atol=1e-12)


def test_window_positions():
    assert O.window_positions(5, 16) == list(range(0, 6))
    assert O.window_positions(100, 16) == list(range(85, 101))
    assert O.window_positions(0, 128) == [0]


def _dense_reference(q, t, W, ring, ring_cap, cache, n_vis, sink, scale, rope_dim, base):
    """Textbook softmax attention over window + every visible entry, with the sink as an
    extra logit carrying a zero value row, then the inverse rotation by t written with
    complex numbers."""
    rows = [ring[p % ring_cap] for p in range(max(0, t - W + 1), t + 1)] + [cache[s] for s in range(n_vis)]
    C = np.array(rows)
    logits = np.concatenate([scale * q @ C.T, sink[:, None]], axis=1)
    o = softmax(logits, axis=1) @ np.concatenate([C, np.zeros((1, C.shape[1]))])
    z = o[:, -rope_dim:][:, 0::2] + 1j * o[:, -rope_dim:][:, 1::2]
    theta = np.array([base ** (-(2.0 * i) / rope_dim) for i in range(rope_dim // 2)])
    z = z * np.exp(-1j * t * theta)
    o[:, -rope_dim:][:, 0::2] = z.real
    o[:, -rope_dim:][:, 1::2] = z.imag
    return o


def test_topk_at_least_visible_reduces_to_dense_attention():
    """T5 on the tiny shape (8 heads x 512, window 16, ratio 4): with k >= visible the CSA
    layer is dense attention over window + all entries."""
    rng = np.random.default_rng(10)
    S, H, d, W = 128, 8, 512, 16
    inp = dict(
        kv=rng.standard_normal((1, S, 2 * d)), score=rng.standard_normal((1, S, 2 * d)),
        idx_kv=rng.standard_normal((1, S, 256)), idx_score=rng.standard_normal((1, S, 256)),
        win_kv=rng.standard_normal((1, S, d)), q=rng.standard_normal((1, S, H, d)) / math.sqrt(d) * 3,
        q_idx=rng.standard_normal((1, S, 4, 128)), w=rng.standard_normal((1, S, 4)),
        sink=rng.standard_normal(H), gamma=np.ones(d), idx_gamma=np.ones(128),
        pos=np.arange(S)[None, :])
    qs = [0, 3, 4, 17, 64, 127]
    res = O.csa_prefill(inp, 0, qs, H=H, d=d, W=W, topk=S // 4)
    for i in qs:
        ref = _dense_reference(inp["q"][0, i], i, W, inp["win_kv"][0], S, res["cache"], (i + 1) // 4,
                               inp["sink"], 1 / math.sqrt(d), 64, 10000.0)
        assert np.allclose(res["queries"][i]["out"], ref, atol=1e-10)


def test_hca_prefill_is_dense_attention_over_every_visible_entry():
    """HCA ([P5] §3, no index module): the prefill path without the indexer (C128A, ratio 128, no
    overlap) equals dense attention over the window and every visible entry, written out
    independently of the oracle's candidate gathering."""
    rng = np.random.default_rng(11)
    S, H, d, W, ratio = 300, 4, 512, 16, 128
    inp = dict(kv=rng.standard_normal((1, S, d)), score=rng.standard_normal((1, S, d)),
               win_kv=rng.standard_normal((1, S, d)), q=rng.standard_normal((1, S, H, d)) / math.sqrt(d) * 3,
               sink=rng.standard_normal(H), gamma=np.ones(d), pos=np.arange(S)[None, :])
    qs = [0, 126, 127, 128, 255, 256, 299]
    res = O.csa_prefill(inp, 0, qs, H=H, d=d, W=W, topk=0, ratio=ratio, with_indexer=False)
    assert res["cache"].shape == (S // ratio, d)
    for i in qs:
        ref = _dense_reference(inp["q"][0, i], i, W, inp["win_kv"][0], S, res["cache"], (i + 1) // ratio,
                               inp["sink"], 1 / math.sqrt(d), 64, 10000.0)
        assert np.allclose(res["queries"][i]["out"], ref, atol=1e-10)


def test_future_group_values_do_not_leak():
    """T4: adversarial values in an incomplete group (and later tokens) do not change the
    output of any query that precedes the group's completion."""
    rng = np.random.default_rng(11)
    S, H, d, W = 64, 4, 512, 16
    base = dict(
        kv=rng.standard_normal((1, S, 2 * d)), score=rng.standard_normal((1, S, 2 * d)),
        idx_kv=rng.standard_normal((1, S, 256)), idx_score=rng.standard_normal((1, S, 256)),
        win_kv=rng.standard_normal((1, S, d)), q=rng.standard_normal((1, S, H, d)) / 8,
        q_idx=rng.standard_normal((1, S, 4, 128)), w=rng.standard_normal((1, S, 4)),
        sink=rng.standard_normal(H), gamma=np.ones(d), idx_gamma=np.ones(128), pos=np.arange(S)[None, :])
    t_query = 41                      # group 10 = tokens 40..43 is incomplete at t = 41
    bad = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in base.items()}
    for key in ("kv", "score", "idx_kv", "idx_score"):
        bad[key][0, 42:] = 1e4
    bad["win_kv"][0, 42:] = 1e4
    a = O.csa_prefill(base, 0, [t_query], H=H, d=d, W=W, topk=4)
    b = O.csa_prefill(bad, 0, [t_query], H=H, d=d, W=W, topk=4)
    assert np.array_equal(a["queries"][t_query]["out"], b["queries"][t_query]["out"])
    # ... while a query after completion does see the change.
    a = O.csa_prefill(base, 0, [47], H=H, d=d, W=W, topk=4)
    b = O.csa_prefill(bad, 0, [47], H=H, d=d, W=W, topk=4)
    assert not np.allclose(a["queries"][47]["out"], b["queries"][47]["out"])


# ----------------------------------------------------------------------------- counters (T7)

def test_flop_ledger_matches_printed_values(golden_dir):
    g = _load(golden_dir, "flop_ledger.json")
    c, h = g["csa"], g["hca"]
    rc = O.reads_per_query(c["t"], c["window"], c["ratio"], c["topk"])
    rh = O.reads_per_query(h["t"], h["window"], h["ratio"], None)
    assert rc == c["reads"] and rh == h["reads"]
    fc = O.attention_flops(g["heads"], rc, g["d"])
    fh = O.attention_flops(g["heads"], rh, g["d"])
    assert fc == c["flops"] and fh == h["flops"]
    assert round(fc / 1e6) == c["printed_mflop"] and round(fh / 1e6) == h["printed_mflop"]


def test_reads_per_query_edge_cases():
    assert O.reads_per_query(0, 128, 4, 1024) == 1          # first token: itself only
    assert O.reads_per_query(3, 128, 4, 1024) == 5          # entry 0 completes at t = 3
    assert O.reads_per_query(8191, 128, 4, 1024) == 128 + 1024
    assert O.reads_per_query(1048575, 128, 4, 1024) == 1152


def test_csa_and_hca_reads_cross_where_the_visible_entries_reach_k():
    """[P1] "Pro 的 CSA 和 HCA，成本交点在哪里": top-k fixes CSA's reads (128 + 1024) while HCA reads
    every visible entry, one per 128 tokens, so the two read counts are equal when (t + 1) / 128 =
    1024, at a 128K context (t = 131071), and HCA reads more beyond it: 128 + 8192 at 1M."""
    csa = lambda t: O.reads_per_query(t, 128, 4, 1024)
    hca = lambda t: O.reads_per_query(t, 128, 128, None)
    assert hca(32767) == 384 and csa(32767) == 1152
    assert hca(131071) == csa(131071) == 1152
    assert hca(131071 - 128) < csa(131071 - 128)
    assert hca(1048575) == 128 + 8192 > csa(1048575)


def test_prefill_totals_match_arithmetic_series():
    """An 8192-token CSA prefill from an empty cache, totalled over its queries and checked against
    sums of arithmetic series rather than a loop. u = t + 1 runs over 1..8192.

    Visible entries: floor(u/4) is k for the four values u = 4k..4k+3, and 2048 at u = 8192. The
    sum is 4 (1 + ... + 2047) + 2048 = 8,386,560 (query, entry) pairs for the indexer.

    Reads: the window part min(128, u) sums to 128 * 129 / 2 + (8192 - 128) * 128 = 1,040,448. The
    selected part min(1024, floor(u/4)) sums to 4 (1 + ... + 1023) over u < 4096, plus 1024 for each
    of the 4097 values u >= 4096, which is 6,290,432. The total is 7,330,880 reads."""
    S = 8192
    assert sum(O.visible_entries(t, 4) for t in range(S)) == 4 * (2047 * 2048 // 2) + 2048 == 8_386_560
    window = 128 * 129 // 2 + (S - 128) * 128
    selected = 4 * (1023 * 1024 // 2) + 4097 * 1024
    assert (window, selected) == (1_040_448, 6_290_432)
    assert sum(O.reads_per_query(t, 128, 4, 1024) for t in range(S)) == window + selected == 7_330_880
    # HCA (ratio 128, every visible entry): floor(u/128) sums to 128 (1 + ... + 63) + 64.
    assert sum(O.reads_per_query(t, 128, 128, None) for t in range(S)) == window + 128 * (63 * 64 // 2) + 64


def test_large_sink_stays_finite():
    """R6: the running max includes the sink, so a sink far above every logit gives an
    output near zero instead of overflowing."""
    q = np.ones((1, 4)); c = np.ones((3, 4)) * 0.1
    o = O.mqa_with_sink(q, c, np.array([1000.0]), 1.0)
    assert np.all(np.isfinite(o)) and np.max(np.abs(o)) < 1e-300
    # A sink 720 above the three equal logits (0.4): exp(720) overflows float64, but with the sink in
    # the max every exponent is <= 0 and the output keeps its closed form 0.1 * 3 e^-720 / (1 + 3 e^-720)
    # = 0.3 e^-720 (a subnormal, about 2e-314), which an overflowed denominator would flush to 0.
    o = O.mqa_with_sink(q, c, np.array([720.4]), 1.0)
    assert np.allclose(o, 0.3 * math.exp(-720.0), rtol=1e-6, atol=0.0) and np.all(o > 0)


def test_heads_have_softmaxes_of_their_own():
    """[P5] §2.3 (MQA): the heads share one candidate set but each normalises its own logits, so a
    head's output does not depend on the other heads, even when their logits lie 800 apart (far
    beyond float64's exp range)."""
    rng = np.random.default_rng(40)
    cand = rng.standard_normal((6, 8))
    cand[:, 0] = 1.0                     # a constant dim: q[h, 0] shifts every logit of head h
    q = rng.standard_normal((3, 8))
    q[1, 0] = 1000.0                     # head 1: logits near +1000
    q[2, 0] = -1000.0                    # head 2: logits near -1000, far below its sink
    sink = np.array([0.3, -1.0, 2.0])
    together = O.mqa_with_sink(q, cand, sink, 1.0)
    assert np.all(np.isfinite(together))
    for h in range(3):
        alone = O.mqa_with_sink(q[h:h + 1], cand, sink[h:h + 1], 1.0)
        assert np.allclose(together[h], alone[0], rtol=1e-12, atol=1e-14)
    assert np.allclose(together[2], 0.0, atol=1e-300)   # head 2: the sink takes all the weight


def test_rmsnorm_eps_matters_for_small_vectors():
    """R3: eps = 1e-6 sits inside the square root. For a constant vector of 1e-4 the
    normalised value is 1e-4 / sqrt(1e-8 + 1e-6); a zero vector stays zero."""
    x = np.full(8, 1e-4)
    y = O.rms_norm(x, 1.0, 1e-6)
    assert np.allclose(y, 1e-4 / math.sqrt(1e-8 + 1e-6), rtol=1e-12)
    assert np.array_equal(O.rms_norm(np.zeros(8), 1.0, 1e-6), np.zeros(8))


# ----------------------------------------------------------------------------- output projection

def test_output_projection_one_hot_weights_select_values():
    """[P1] "输出投影也分组": with Wo_a[g] selecting dims perm_g of its group and Wo_b a permutation,
    y picks single entries of o, so every index of the grouped einsum and the flatten is checked."""
    rng = np.random.default_rng(20)
    M, G, Kg, R = 3, 4, 16, 8
    D = G * R
    o = O.bf16(rng.standard_normal((M, G * Kg)))
    wa = np.zeros((G, R, Kg))
    sel = [rng.choice(Kg, R, replace=False) for _ in range(G)]
    for g in range(G):
        wa[g, np.arange(R), sel[g]] = 1.0
    perm = rng.permutation(G * R)
    wb = np.zeros((D, G * R))
    wb[np.arange(D), perm] = 1.0
    r, rb, y = O.output_projection(o, wa, wb)
    for m in range(M):
        for g in range(G):
            for i in range(R):
                assert r[m, g * R + i] == o[m, g * Kg + sel[g][i]]
        for j in range(D):
            c = perm[j]
            assert y[m, j] == o[m, (c // R) * Kg + sel[c // R][c % R]]


def test_output_projection_groups_are_independent_and_linear():
    """Changing the input of one group changes only that group's block of r; the bf16 rounding of
    r (R20) commutes with a power-of-two scale, so y scales exactly."""
    rng = np.random.default_rng(21)
    M, G, Kg, R, D = 2, 3, 32, 8, 5
    o = O.bf16(rng.standard_normal((M, G * Kg)))
    wa = O.bf16(rng.standard_normal((G, R, Kg)))
    wb = O.bf16(rng.standard_normal((D, G * R)))
    r, rb, y = O.output_projection(o, wa, wb)
    o2 = o.copy()
    o2[:, Kg:2 * Kg] += 1.0
    r2, _, _ = O.output_projection(o2, wa, wb)
    changed = np.any(r2 != r, axis=0)
    assert not changed[:R].any() and changed[R:2 * R].any() and not changed[2 * R:].any()
    _, rb4, y4 = O.output_projection(4.0 * o, wa, wb)
    assert np.array_equal(rb4, 4.0 * rb) and np.allclose(y4, 4.0 * y, rtol=0, atol=1e-12 * np.abs(y).max())
    # r is exactly the per-group matrix product before rounding; y uses the rounded r
    for g in range(G):
        assert np.allclose(r[:, g * R:(g + 1) * R], o[:, g * Kg:(g + 1) * Kg] @ wa[g].T, rtol=1e-14, atol=1e-12)
    assert np.array_equal(rb, O.bf16(r))


def test_output_projection_rounds_r_before_the_second_product():
    """R20 on values fixed by hand: o = [1, 2^-9] summed by Wo_a = [1, 1] gives r = 1 + 2^-9, which
    lies below half a bf16 step above 1, so the rounded r is 1 and y = 1 * 3 = 3 exactly; o = [1,
    3 * 2^-8] gives r = 1 + 3 * 2^-8, half-way between two bf16 values, which rounds to the even
    one, 1 + 2^-6, and y = 3 + 3 * 2^-6."""
    wa = np.ones((1, 1, 2))
    wb = np.array([[3.0]])
    for second, r_exact, y_exact in ((2.0 ** -9, 1.0 + 2.0 ** -9, 3.0),
                                     (3 * 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, 3.0 + 3 * 2.0 ** -6)):
        r, rb, y = O.output_projection(np.array([[1.0, second]]), wa, wb)
        assert r[0, 0] == r_exact and y[0, 0] == y_exact


# ----------------------------------------------------------------------------- query path

def _complex_rotate(v, pos, rope_dim, base):
    """Rotation of the last rope_dim dims as complex multiplication (textbook form)."""
    head = v.shape[-1] - rope_dim
    z = v[..., head::2] + 1j * v[..., head + 1::2]
    theta = base ** (-np.arange(rope_dim // 2) * 2.0 / rope_dim)
    z = z * np.exp(1j * pos * theta)
    out = v.copy()
    out[..., head::2] = z.real
    out[..., head + 1::2] = z.imag
    return out


def test_q_path_one_hot_weights_closed_form():
    """[P1] "低秩 Q": with Wq_a selecting input dims and Wq_b selecting qr dims, every step has a closed
    form: qa = selected x, qr = gamma qa / sqrt(mean(qa^2) + eps), each head of q = its selected qr
    values over their RMS, then the complex rotation of its last 64 dims by the position."""
    rng = np.random.default_rng(30)
    M, hidden, q_rank, H, d, eps = 3, 64, 16, 2, 512, 1e-6
    x = O.bf16(rng.standard_normal((M, hidden)))
    sel_a = rng.choice(hidden, q_rank, replace=False)
    wq_a = np.zeros((q_rank, hidden))
    wq_a[np.arange(q_rank), sel_a] = 1.0
    gamma = O.bf16(rng.uniform(0.5, 1.5, q_rank))
    sel_b = rng.integers(0, q_rank, H * d)
    wq_b = np.zeros((H * d, q_rank))
    wq_b[np.arange(H * d), sel_b] = 1.0
    pos = np.array([0, 7, 123456])
    qa, qr, q = O.q_path(x, wq_a, gamma, wq_b, pos, H, d, eps=eps)
    assert np.array_equal(qa, x[:, sel_a])
    exp_qr = O.bf16(gamma * x[:, sel_a] / np.sqrt(np.mean(x[:, sel_a] ** 2, axis=1, keepdims=True) + eps))
    assert np.array_equal(qr, exp_qr)
    for m in range(M):
        heads = exp_qr[m, sel_b].reshape(H, d)
        heads = heads / np.sqrt(np.mean(heads ** 2, axis=1, keepdims=True) + eps)
        assert np.allclose(q[m], _complex_rotate(heads, pos[m], 64, 10000.0), rtol=0, atol=1e-12)
    # position 0 leaves q unrotated; every head keeps its mean square m / (m + eps)
    assert np.allclose(np.mean(q ** 2, axis=-1), 1.0, atol=1e-4)


def test_window_projection_one_hot_closed_form():
    """[P5] §2: the window row is the down-projected row with its last 64 dims rotated by the position."""
    rng = np.random.default_rng(31)
    M, hidden, d = 2, 1024, 512
    x = O.bf16(rng.standard_normal((M, hidden)))
    sel = rng.choice(hidden, d, replace=False)
    wkv = np.zeros((d, hidden))
    wkv[np.arange(d), sel] = 1.0
    pos = np.array([5, 99999])
    w = O.window_projection(x, wkv, pos)
    for m in range(M):
        assert np.allclose(w[m], _complex_rotate(x[m, sel], pos[m], 64, 10000.0), rtol=0, atol=1e-12)


def test_q_path_rounds_the_product_before_the_head_norm():
    """R21 on values fixed by hand: qa = [1, 1] gives qr = 1 / sqrt(1 + eps), which rounds to 1 in
    bf16; Wq_b row 0 = [1, 2^-9] then gives 1 + 2^-9 in dim 0 of head 0 and every other row [1, 0]
    gives 1. 1 + 2^-9 lies below half a bf16 step above 1, so the rounded product is 1 in every dim,
    and the per-head norm leaves all unrotated dims of the head equal (1 / sqrt(1 + eps))."""
    H, d, eps = 1, 512, 1e-6
    x = np.array([[1.0, 1.0]])
    wq_a = np.eye(2)
    wq_b = np.zeros((H * d, 2))
    wq_b[:, 0] = 1.0
    wq_b[0, 1] = 2.0 ** -9
    qa, qr, q = O.q_path(x, wq_a, np.ones(2), wq_b, np.array([0]), H, d, eps=eps)
    assert np.array_equal(qr, np.ones((1, 2)))
    want = 1.0 / np.sqrt(1.0 + eps)
    assert np.all(q[0, 0, :d - 64] == want)


def test_window_row_rounds_before_its_rotation():
    """R21 on values fixed by hand: a window row whose dims 448 and 449 (the first rotated pair) come
    out of the product as 1 + 2^-9 and 0 rounds to (1, 0) first, so at position 1 the pair is exactly
    (cos theta_0, sin theta_0) = (cos 1, sin 1); an unrounded row would give (1 + 2^-9)(cos 1, sin 1)."""
    d = 512
    x = np.array([[1.0, 2.0 ** -9]])
    wkv = np.zeros((d, 2))
    wkv[448] = [1.0, 1.0]
    w = O.window_projection(x, wkv, np.array([1]))
    assert w[0, 448] == np.cos(1.0) and w[0, 449] == np.sin(1.0)
    assert np.all(w[0, :448] == 0.0)


# ----------------------------------------------------------------------------- decode step composition

def _prefill_inputs(rng, S, H, d, ratio):
    """Random float64 inputs of one request's prefill segment from position 0 (tiny shapes)."""
    ov = ratio == 4
    width = 2 * d if ov else d
    inp = dict(kv=rng.standard_normal((1, S, width)), score=rng.standard_normal((1, S, width)),
               win_kv=rng.standard_normal((1, S, d)), q=rng.standard_normal((1, S, H, d)) / math.sqrt(d) * 3,
               sink=rng.standard_normal(H), gamma=np.ones(d), pos=np.arange(S)[None, :])
    if ov:
        inp.update(idx_kv=rng.standard_normal((1, S, 256)), idx_score=rng.standard_normal((1, S, 256)),
                   q_idx=rng.standard_normal((1, S, 4, 128)), w=rng.standard_normal((1, S, 4)),
                   idx_gamma=np.ones(128))
    return inp


def _decode_inputs_at(pre, t, W, ratio, rng):
    """The decode-step inputs of token t, built from a prefill segment the way a serving loop holds
    them before the step: the compressor states after tokens 0..t-1 (token-by-token machine), the
    cache rows of every group completed before t, a W-slot ring with the window rows of tokens
    t-W+1..t-1 at slot p % W, and token t's own streams. Cache rows not yet written and the ring slot
    token t will take hold stale values (random draws), as pooled memory does."""
    d = pre["win_kv"].shape[2]
    E = pre["win_kv"].shape[1] // ratio
    main = O.CompressorCfg(ratio, d)
    skv, ssc = O.init_state(main)
    done = O.compress_tokens(main, skv, ssc, 0, pre["kv"][0, :t], pre["score"][0, :t], pre["gamma"])
    cache = O.bf16(rng.standard_normal((E, d)))
    for g, e in done.items():
        cache[g] = O.bf16(e)
    ring = O.bf16(rng.standard_normal((W, d)))
    for p in range(max(0, t - W + 1), t):
        ring[p % W] = pre["win_kv"][0, p]
    one = lambda x: x[:, t:t + 1]
    inp = dict(state_kv=skv[None], state_score=ssc[None], cache=cache[None], ring=ring[None],
               kv=one(pre["kv"]), score=one(pre["score"]), win_kv=one(pre["win_kv"]), q=one(pre["q"]),
               sink=pre["sink"], gamma=pre["gamma"], pos=np.array([[t]]))
    if "idx_kv" in pre:
        idx = O.CompressorCfg(ratio, 128)
        ikv, isc = O.init_state(idx)
        idone = O.compress_tokens(idx, ikv, isc, 0, pre["idx_kv"][0, :t], pre["idx_score"][0, :t],
                                  pre["idx_gamma"])
        icache = O.bf16(rng.standard_normal((E, 128)))
        for g, e in idone.items():
            icache[g] = O.bf16(e)
        inp.update(idx_state_kv=ikv[None], idx_state_score=isc[None], idx_cache=icache[None],
                   idx_kv=one(pre["idx_kv"]), idx_score=one(pre["idx_score"]), q_idx=one(pre["q_idx"]),
                   w=one(pre["w"]), idx_gamma=pre["idx_gamma"])
    return inp


@pytest.mark.parametrize("t", [3, 11, 13, 31, 63, 70, 127])
def test_csa_decode_step_equals_prefill_query_at_the_same_position(t):
    """The decode step composes its modules in the pages' order ([P5] §2: compressor, then the index
    module over the index cache, then attention over window + selected entries): the compressor step
    of token t, which completes entry t // 4 when (t + 1) % 4 == 0, lands in both caches before the
    indexer scores and attention reads them, and token t's window row is in the ring before attention.
    A decode step fed the state a serving loop holds after tokens 0..t-1 must therefore reproduce the
    prefill's query t ([P1] "压缩条目必须等整组完成后才可见": every query sees (t + 1) // 4 entries),
    whose parallel compression is pinned against the state machine above. t covers group completion
    and non-completion, all-visible selection (t < 32 with top-k 8) and t below and above the window."""
    S, H, d, W, topk = 128, 8, 512, 16, 8
    rng = np.random.default_rng(20)
    pre = _prefill_inputs(rng, S, H, d, 4)
    dec_in = _decode_inputs_at(pre, t, W, 4, np.random.default_rng(21))
    dec = O.csa_decode_request(dec_in, 0, H=H, d=d, W=W, topk=topk)
    ref = O.csa_prefill(pre, 0, [t], H=H, d=d, W=W, topk=topk)
    q = ref["queries"][t]
    vis = (t + 1) // 4
    assert dec["scores"].shape == (vis,)
    assert np.allclose(dec["scores"], q["scores"], rtol=1e-12, atol=1e-12)
    assert np.array_equal(dec["topk"], q["topk"])
    assert np.allclose(dec["out"], q["out"], rtol=1e-10, atol=1e-12)
    if (t + 1) % 4 == 0:
        g = t // 4
        assert np.allclose(dec["entry"], ref["entries"][g], rtol=1e-12, atol=1e-12)
        assert np.allclose(dec["idx_entry"], ref["idx_entries"][g], rtol=1e-12, atol=1e-12)
        assert np.array_equal(dec["cache"][g], ref["cache"][g])
        assert np.array_equal(dec["idx_cache"][g], ref["idx_cache"][g])
    else:
        assert dec["entry"] is None and dec["idx_entry"] is None
    assert np.array_equal(dec["ring"][t % W], pre["win_kv"][0, t])


@pytest.mark.parametrize("t", [127, 255, 300, 383])
def test_hca_decode_step_equals_prefill_query_at_the_same_position(t):
    """HCA ([P5] §3: C128A, no index module): the C128A step of token t completes entry t // 128 when
    (t + 1) % 128 == 0 and is in the cache before attention reads every visible entry; token t's
    window row is in the ring first. The decode step must reproduce the HCA prefill's query t."""
    S, H, d, W, ratio = 384, 4, 512, 16, 128
    rng = np.random.default_rng(22)
    pre = _prefill_inputs(rng, S, H, d, ratio)
    dec_in = _decode_inputs_at(pre, t, W, ratio, np.random.default_rng(23))
    dec = O.hca_decode_request(dec_in, 0, H=H, d=d, W=W, ratio=ratio)
    ref = O.csa_prefill(pre, 0, [t], H=H, d=d, W=W, topk=0, ratio=ratio, with_indexer=False)
    assert np.allclose(dec["out"], ref["queries"][t]["out"], rtol=1e-10, atol=1e-12)
    if (t + 1) % ratio == 0:
        g = t // ratio
        assert np.allclose(dec["entry"], ref["entries"][g], rtol=1e-12, atol=1e-12)
        assert np.array_equal(dec["cache"][g], ref["cache"][g])
    else:
        assert dec["entry"] is None
    assert np.array_equal(dec["ring"][t % W], pre["win_kv"][0, t])
