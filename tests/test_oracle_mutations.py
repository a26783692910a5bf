"""Mutation check of the oracle's pins.

Each case plants one plausible mistake (a dropped term, a wrong sign, index, axis or operand) in a
copy of the oracle built in memory from its source text, on the CPU; the oracle's file is never
written. The pins of test_oracle_pins.py then run against the mutant, and at least one of them must
fail. A control case runs the same pins against the unmodified source, which must pass them all, so a
broken runner cannot pass for a caught mutant.

Not listed, because no test can tell them apart from the oracle:
- dropping the +0.0 that folds -0 into +0 before the top-k sort (numpy's sort already orders -0 and
  +0 as equal);
- writing C128A token t into state row (t + 1) % 128 instead of t % 128: the entry pools all 128
  rows with one softmax, so any fixed permutation of the rows within a group gives the same entry.
  Which row holds which token is a storage convention of the state (no page fixes it); the GPU
  tests compare the kernels' state rows with the oracle's bit for bit;
- taking the slots' max over every slot instead of the valid ones: a missing slot's score is -inf,
  which no max picks while one slot is valid."""

import itertools
import os
import types

import numpy as np
import pytest

from tests import test_oracle_pins as pins

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ORACLE_SRC = os.path.join(ROOT, "oracle", "csa_oracle.py")

# name -> (text in the oracle, the mistake put in its place)
MUTATIONS = {
    # compressor
    "state_machine_wrong_halves": (
        "slot_kv = np.concatenate([state_kv[:r, :d], state_kv[r:, d:]], axis=0)",
        "slot_kv = np.concatenate([state_kv[:r, d:], state_kv[r:, :d]], axis=0)"),
    "direct_formula_wrong_half": (
        "slot_kv = np.concatenate([kv[prev, :d], kv[cur, d:]], axis=0)",
        "slot_kv = np.concatenate([kv[prev, d:], kv[cur, d:]], axis=0)"),
    "first_group_takes_the_pre_channels": ("                slot_kv, slot_sc = kv[cur, d:], score[cur, d:]",
                                           "                slot_kv, slot_sc = kv[cur, :d], score[cur, :d]"),
    "fresh_state_scores_zero": ("    sc = np.full((cfg.state_rows, cfg.width), -np.inf)",
                                "    sc = np.zeros((cfg.state_rows, cfg.width))"),
    "pool_weights_from_kv": ("    e = np.where(valid, np.exp(np.where(valid, slot_score, 0.0) - m), 0.0)",
                             "    e = np.where(valid, np.exp(np.where(valid, slot_kv, 0.0) - m), 0.0)"),
    "segment_restarts_at_position_zero": (
        "res = compressor_step(cfg, state_kv, state_score, start_pos + i, kv[i], score[i], gamma)",
        "res = compressor_step(cfg, state_kv, state_score, i, kv[i], score[i], gamma)"),
    "state_not_rolled": ("        state_kv[:r] = state_kv[r:]\n", "        pass\n"),
    "softmax_over_channels": ("wts = e / np.sum(e, axis=0)", "wts = e / np.sum(e, axis=1, keepdims=True)"),
    "entry_position_off_by_one": ("rope(rms_norm(pooled, gamma, eps), g * ratio,",
                                  "rope(rms_norm(pooled, gamma, eps), g * ratio + 1,"),
    "rmsnorm_without_eps": ("/ np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)",
                            "/ np.sqrt(np.mean(x * x, axis=-1, keepdims=True))"),
    "entry_visible_one_early": ("return (t + 1) // ratio", "return t // ratio + 1"),
    "c4a_token_into_pre_rows": ("        row = r + t % r\n", "        row = t % r\n"),
    "state_scores_not_rolled": ("        state_score[:r] = state_score[r:]\n", "        pass\n"),
    "rmsnorm_without_gamma": ("return np.asarray(gamma, dtype=np.float64) * x / np.sqrt", "return x / np.sqrt"),
    # rounding
    "bf16_round_half_up": ("(((u >> np.uint64(16)) & np.uint64(1)) + np.uint64(0x7FFF))", "(np.uint64(0x8000))"),
    "bf16_truncates": ("u = (u + (((u >> np.uint64(16)) & np.uint64(1)) + np.uint64(0x7FFF))) >> np.uint64(16)",
                       "u = u >> np.uint64(16)"),
    # RoPE
    "rope_wrong_sign": ("y[..., head + 1::2] = even * s + odd * c", "y[..., head + 1::2] = -even * s + odd * c"),
    "rope_inverse_ignored": ("    if inverse:\n        ang = -ang\n", "    if inverse:\n        pass\n"),
    "rope_cos_sin_swapped": ("    c, s = np.cos(ang), np.sin(ang)", "    s, c = np.cos(ang), np.sin(ang)"),
    "rope_frequency_exponent_halved": ("return float(pos) * np.power(float(base), -2.0 * i / rope_dim)",
                                       "return float(pos) * np.power(float(base), -1.0 * i / rope_dim)"),
    "rope_on_the_first_dims": ("    head = x.shape[-1] - rope_dim\n", "    head = 0\n"),
    # indexer and top-k
    "indexer_without_relu": ("return np.maximum(logits, 0.0) @", "return logits @"),
    "indexer_relu_after_weighting": (
        "return np.maximum(logits, 0.0) @ np.asarray(w, dtype=np.float64)",
        "return np.maximum(logits @ np.asarray(w, dtype=np.float64), 0.0)"),
    "ties_to_higher_index": ("order = np.lexsort((np.arange(n), -key, nan_last))",
                             "order = np.lexsort((-np.arange(n), -key, nan_last))"),
    "selection_in_score_order": ("sel = np.sort(order[: min(k, n)])", "sel = order[: min(k, n)]"),
    "topk_takes_the_smallest": ("order = np.lexsort((np.arange(n), -key, nan_last))",
                                "order = np.lexsort((np.arange(n), key, nan_last))"),
    "nan_sorts_highest": ("order = np.lexsort((np.arange(n), -key, nan_last))",
                          "order = np.lexsort((np.arange(n), -key, -nan_last))"),
    "indexer_scores_one_entry_too_many": ("k = np.asarray(idx_cache[:visible], dtype=np.float64)",
                                          "k = np.asarray(idx_cache[:visible + 1], dtype=np.float64)"),
    # attention
    "window_shifted": ("return list(range(max(0, t - W + 1), t + 1))", "return list(range(max(0, t - W), t))"),
    "window_ring_slot_off_by_one": ("rows = [ring[p % ring_cap] for p in window_positions(t, W)]",
                                    "rows = [ring[(p + 1) % ring_cap] for p in window_positions(t, W)]"),
    "padding_rows_gathered": ("rows += [cache[s] for s in selected if s >= 0]",
                              "rows += [cache[s] for s in selected]"),
    "one_max_over_all_heads": ("    m = np.maximum(np.max(logits, axis=1), sink)",
                               "    m = np.maximum(np.max(logits, axis=0).max(), sink)"),
    "hca_reads_capped_like_csa": ("return min(W, t + 1) + (vis if topk is None else min(topk, vis))",
                                  "return min(W, t + 1) + (min(1024, vis) if topk is None else min(topk, vis))"),
    "sink_scaled_like_the_logits": ("m = np.maximum(np.max(logits, axis=1), sink)",
                                    "sink = scale * sink\n    m = np.maximum(np.max(logits, axis=1), sink)"),
    "sink_left_out_of_the_max": ("m = np.maximum(np.max(logits, axis=1), sink)", "m = np.max(logits, axis=1)"),
    "sink_not_in_denominator": ("denom = np.sum(e, axis=1) + np.exp(sink - m)", "denom = np.sum(e, axis=1)"),
    "logits_unscaled": ("logits = scale * (q @ cand.T)", "logits = (q @ cand.T)"),
    "output_rotated_forward": ("return rope(o, t, rope_dim, rope_base, inverse=True)",
                               "return rope(o, t, rope_dim, rope_base)"),
    # output projection
    "projection_wrong_group_weights": ('r = np.einsum("mgk,grk->mgr", og, wo_a)',
                                       'r = np.einsum("mgk,grk->mgr", og, wo_a[::-1])'),
    "projection_groups_interleaved": ("    og = o_rows.reshape(M, G, Kg)\n",
                                      "    og = o_rows.reshape(M, Kg, G).transpose(0, 2, 1)\n"),
    "projection_r_not_rounded": ("y = rb.reshape(M, G * R) @ wo_b.T", "y = r.reshape(M, G * R) @ wo_b.T"),
    # query path and window rows
    "q_without_gamma": ("qr = bf16(rms_norm(qa, gamma, eps))", "qr = bf16(rms_norm(qa, 1.0, eps))"),
    "q_norm_over_all_heads": ("q = qraw / np.sqrt(np.mean(qraw * qraw, axis=-1, keepdims=True) + eps)",
                              "q = qraw / np.sqrt(np.mean(qraw * qraw, axis=(-2, -1), keepdims=True) + eps)"),
    "q_heads_split_wrong": ("qraw = bf16(qr @ wq_b.T).reshape(M, H, d)",
                            "qraw = bf16(qr @ wq_b.T).reshape(M, d, H).transpose(0, 2, 1)"),
    "q_head_norm_without_eps": ("q = qraw / np.sqrt(np.mean(qraw * qraw, axis=-1, keepdims=True) + eps)",
                                "q = qraw / np.sqrt(np.mean(qraw * qraw, axis=-1, keepdims=True))"),
    "window_row_rotated_at_next_position": ("rope(w[m], float(pos[m]), rope_dim, rope_base)",
                                            "rope(w[m], float(pos[m]) + 1.0, rope_dim, rope_base)"),
    "q_rotated_at_next_position": ("q[m] = rope(q[m], float(pos[m]), rope_dim, rope_base)",
                                   "q[m] = rope(q[m], float(pos[m]) + 1.0, rope_dim, rope_base)"),
    "q_product_not_rounded": ("qraw = bf16(qr @ wq_b.T).reshape(M, H, d)", "qraw = (qr @ wq_b.T).reshape(M, H, d)"),
    "window_row_not_rounded": ("w = bf16(x @ wkv.T)", "w = x @ wkv.T"),
    "window_row_not_rotated": (
        "return np.stack([rope(w[m], float(pos[m]), rope_dim, rope_base) for m in range(x.shape[0])])",
        "return w.copy()"),
    # order of the modules in one decode step
    "indexer_scored_before_the_in_step_index_entry": (
        'scores = indexer_scores(inp["q_idx"][b, 0], inp["w"][b, 0], icache, vis)',
        'scores = indexer_scores(inp["q_idx"][b, 0], inp["w"][b, 0], inp["idx_cache"][b], vis)'),
    "ring_written_after_attention": (
        'out = attend_query(inp["q"][b, 0], t, W, ring, ring_cap, cache, sel,',
        'out = attend_query(inp["q"][b, 0], t, W, inp["ring"][b], ring_cap, cache, sel,'),
    "entry_written_after_attention": (
        'out = attend_query(inp["q"][b, 0], t, W, ring, ring_cap, cache, sel,',
        'out = attend_query(inp["q"][b, 0], t, W, ring, ring_cap, inp["cache"][b], sel,'),
    "hca_ring_written_after_attention": (
        'out = attend_query(inp["q"][b, 0], t, W, ring, ring_cap, cache, list(range(vis)),',
        'out = attend_query(inp["q"][b, 0], t, W, inp["ring"][b], ring_cap, cache, list(range(vis)),'),
    "decode_ring_slot_of_the_next_token": (
        '    ring[t % ring_cap] = inp["win_kv"][b, 0]\n    vis = visible_entries(t, ratio)\n    scores',
        '    ring[(t + 1) % ring_cap] = inp["win_kv"][b, 0]\n    vis = visible_entries(t, ratio)\n    scores'),
    "decode_scaled_by_the_index_width": (
        '    scale = 1.0 / math.sqrt(d) if scale is None else scale\n    t = int(inp["pos"][b, 0])\n    main',
        '    scale = 1.0 / math.sqrt(d_I) if scale is None else scale\n    t = int(inp["pos"][b, 0])\n    main'),
    "hca_prefill_drops_the_last_entry": ("            scores, sel = None, np.arange(vis)",
                                         "            scores, sel = None, np.arange(max(vis - 1, 0))"),
    "decode_entry_not_rounded": ("        cache[g] = bf16(entry)\n    if res_idx", "        cache[g] = entry\n    if res_idx"),
    "decode_index_stream_with_the_main_gamma": ('inp["idx_score"][b, 0], inp["idx_gamma"])',
                                                'inp["idx_score"][b, 0], inp["gamma"])'),
    "decode_in_step_entry_not_visible": ("    vis = visible_entries(t, ratio)\n    scores",
                                         "    vis = visible_entries(t - 1, ratio)\n    scores"),
    "hca_in_step_entry_not_visible": ("    vis = visible_entries(t, ratio)\n    out = attend_query",
                                      "    vis = visible_entries(t - 1, ratio)\n    out = attend_query"),
    "prefill_entries_not_rounded": ("    cache = bf16(entries)\n", "    cache = entries\n"),
    "hca_entry_written_after_attention": (
        'out = attend_query(inp["q"][b, 0], t, W, ring, ring_cap, cache, list(range(vis)),',
        'out = attend_query(inp["q"][b, 0], t, W, ring, ring_cap, inp["cache"][b], list(range(vis)),'),
}


def _oracle_from(source: str) -> types.ModuleType:
    mod = types.ModuleType("csa_oracle_mutant")
    mod.__file__ = ORACLE_SRC
    exec(compile(source, ORACLE_SRC, "exec"), mod.__dict__)
    return mod


def _pin_calls(golden_dir):
    """Every pin of test_oracle_pins.py with each of its parameter sets, in file order."""
    calls = []
    for name, fn in vars(pins).items():
        if not (name.startswith("test_") and callable(fn)):
            continue
        axes = []
        for mark in getattr(fn, "pytestmark", []):
            if mark.name != "parametrize":
                continue
            argnames, values = mark.args[0], mark.args[1]
            argnames = [a.strip() for a in argnames.split(",")] if isinstance(argnames, str) else list(argnames)
            axes.append([dict(zip(argnames, v if len(argnames) > 1 else (v,))) for v in values])
        for combo in itertools.product(*axes) if axes else [()]:
            kwargs = {}
            for part in combo:
                kwargs.update(part)
            if "golden_dir" in fn.__code__.co_varnames[:fn.__code__.co_argcount]:
                kwargs["golden_dir"] = golden_dir
            calls.append((name, fn, kwargs))
    return calls


def _first_failing_pin(monkeypatch, module, golden_dir):
    monkeypatch.setattr(pins, "O", module)
    for name, fn, kwargs in _pin_calls(golden_dir):
        try:
            with np.errstate(all="ignore"):
                fn(**kwargs)
        except Exception as exc:          # an assertion, or the mutant breaking a shape
            return f"{name}{kwargs or ''}: {type(exc).__name__}"
    return None


def _source():
    with open(ORACLE_SRC) as f:
        return f.read()


def test_control_unmodified_oracle_passes_every_pin(monkeypatch, golden_dir):
    assert len(_pin_calls(golden_dir)) >= 30
    assert _first_failing_pin(monkeypatch, _oracle_from(_source()), golden_dir) is None


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_fails_a_pin(monkeypatch, golden_dir, name):
    before, after = MUTATIONS[name]
    src = _source()
    assert src.count(before) == 1, f"{name}: the text to mutate must occur exactly once"
    caught = _first_failing_pin(monkeypatch, _oracle_from(src.replace(before, after)), golden_dir)
    assert caught is not None, f"{name}: no pin fails"
