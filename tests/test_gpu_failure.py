"""Failure detection on the device, in forms that fault, trap or hang no GPU, and the hand-off from a
prefill segment to decode steps.

* A bounded wait that runs out: the library's mbarrier wait, run on a phase nothing completes with a
  short limit, records CSA_ERR_TIMEOUT and its site in the status word and returns; the context stays
  usable for the next call.
* An out-of-range selection: a top-k list naming an entry at or past the query's visible count (memory
  that exists, so nothing can fault) is reported as CSA_ERR_BOUNDS, the entry is skipped, and the output
  is the attention over the rest of the list.
* The hand-off ([P5] §2.1: the compressor's rolling state carries over between calls): a prefill segment
  through csa_compress, its last window rows placed in the ring, then several csa_decode_fused steps,
  each checked against the oracle's query at the same position over the whole token stream.
"""

import math

import numpy as np
import pytest
import torch

from oracle import csa_oracle as O
from synth import WORKLOADS, make_inputs
from tests.parity import assert_attn_close, check_topk, np64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ops():
    from long_context_decode_c4a_b200 import ops
    return ops


def test_bounded_wait_runs_out_reports_timeout_and_context_stays_usable(ops):
    from long_context_decode_c4a_b200 import _lib
    lib = _lib.load()
    ws = ops.workspace(_lib.CSA_WS_SPARSE_ATTN, 1, 1, 1, 1, "cuda")
    ws.zero_()
    rc = lib.csa_watchdog_selftest(ws.data_ptr(), ws.numel(), 200_000, torch.cuda.current_stream().cuda_stream)
    assert rc == _lib.CSA_OK
    torch.cuda.synchronize()
    site = int(ws.view(torch.int32)[1])
    assert ops.device_status(ws) == _lib.CSA_ERR_TIMEOUT
    assert site == 900
    # Refused before any launch.
    assert lib.csa_watchdog_selftest(ws.data_ptr(), ws.numel(), 0, None) == _lib.CSA_ERR_INVALID_ARG
    assert lib.csa_watchdog_selftest(ws.data_ptr(), ws.numel(), 1 << 31, None) == _lib.CSA_ERR_INVALID_ARG
    assert lib.csa_watchdog_selftest(None, 256, 1000, None) == _lib.CSA_ERR_WORKSPACE
    # The context still runs a normal call, whose status word reads clean.
    wl = WORKLOADS["tiny_csa_prefill"]
    inp = {k: v.cuda() for k, v in make_inputs(wl).items()}
    cache = torch.zeros(1, wl.max_entries, wl.d, dtype=torch.bfloat16, device="cuda")
    out = torch.empty(1, wl.S, wl.H, wl.d, dtype=torch.float32, device="cuda")
    ws2 = ops.workspace(_lib.CSA_WS_HCA_ATTN, 1, wl.S, 1, 1, "cuda")
    ops.hca_attn(inp["pos"], inp["q"], inp["win_kv"], cache, inp["sink"], wl.W, ratio=4, out=out, ws=ws2)
    torch.cuda.synchronize()
    assert ops.device_status(ws2) == _lib.CSA_OK
    assert torch.isfinite(out).all()


def test_selection_past_the_visible_entries_is_reported_and_skipped(ops):
    """csa_sparse_attn given a list whose last entries lie in [visible, max_entries): CSA_ERR_BOUNDS, and
    the output equals the attention over the in-range entries alone."""
    from long_context_decode_c4a_b200 import _lib
    wl = WORKLOADS["pro_csa_decode_32k"].scaled(B=2, ctx=4096, topk=64)
    inp = make_inputs(wl)
    inp_np = O.to_numpy_inputs(inp)
    t = 2000                                  # 500 entries visible out of max_entries = 1024
    vis = (t + 1) // 4
    pos = torch.full((wl.B, 1), t, dtype=torch.int32)
    rng = np.random.default_rng(5)
    good = np.sort(rng.choice(vis, size=60, replace=False))
    bad = np.array([vis, vis + 3, 700, wl.max_entries - 1])         # entries not yet visible at t
    lists = [np.concatenate([good, bad]), np.concatenate([good[:30], bad[:1], np.full(33, -1)])]
    topk = torch.tensor(np.stack(lists)[:, None, :], dtype=torch.int32)
    q = inp["q"].cuda()
    ring = inp["ring"].cuda()
    cache = inp["cache"].cuda()
    out = torch.empty(wl.B, 1, wl.H, wl.d, dtype=torch.float32, device="cuda")
    ws = ops.workspace(_lib.CSA_WS_SPARSE_ATTN, wl.B, 1, 1, 1, "cuda")
    ws.zero_()
    ops.sparse_attn(pos.cuda(), q, ring, cache, topk.cuda(), inp["sink"].cuda(), wl.W, out=out, ws=ws)
    torch.cuda.synchronize()
    assert ops.device_status(ws) == _lib.CSA_ERR_BOUNDS
    assert torch.isfinite(out).all()
    for b in range(wl.B):
        sel = [int(s) for s in lists[b] if 0 <= s < vis]
        ref = O.attend_query(inp_np["q"][b, 0], t, wl.W, inp_np["ring"][b], wl.W, inp_np["cache"][b], sel,
                             inp_np["sink"], 1 / math.sqrt(wl.d), wl.rope_dim, wl.rope_base)
        assert_attn_close(out[b, 0], ref, f"bounds b={b}")


def test_prefill_segment_then_decode_steps_match_the_oracle(ops):
    """S = 600 tokens of prefill through csa_compress (both streams), then six fused decode steps at
    t = 600..605 (t = 603 completes entry 150 in-step); every step's selection and output are checked
    against the oracle's query t over the whole 606-token stream."""
    S, N = 600, 6
    wl = WORKLOADS["csa_prefill_8k"].scaled(S=S + N, ctx=S + N, topk=64)
    inp = make_inputs(wl)
    inp_np = O.to_numpy_inputs(inp)
    d, dI, W = wl.d, wl.d_I, wl.W
    E = 256                                          # cache capacity: entries 0..255
    dev = "cuda"
    st = ops.CsaDecodeState(1, E, H=wl.H, d=d, H_I=wl.H_I, d_I=dI, window=W, topk=wl.topk, device=dev)
    x = {k: v.cuda() for k, v in inp.items()}
    start = torch.zeros(1, dtype=torch.int32, device=dev)
    # Prefill: the segment's tokens 0..S-1 through both compressors, into the decode state's caches.
    ops.compress(ops.compressor_cfg(4, d), start, x["kv"][:, :S].contiguous(), x["score"][:, :S].contiguous(),
                 x["gamma"], st.state_kv, st.state_score, st.cache)
    ops.compress(ops.compressor_cfg(4, dI), start, x["idx_kv"][:, :S].contiguous(),
                 x["idx_score"][:, :S].contiguous(), x["idx_gamma"], st.idx_state_kv, st.idx_state_score,
                 st.idx_cache)
    # The ring: window rows of tokens S-W..S-1 at slot p % W.
    for p in range(S - W, S):
        st.ring[0, p % W].copy_(x["win_kv"][0, p])
    full = O.csa_prefill(inp_np, 0, list(range(S, S + N)), H=wl.H, d=d, W=W, topk=wl.topk)
    out = torch.empty(1, wl.H, d, dtype=torch.float32, device=dev)
    for t in range(S, S + N):
        tok = lambda k: x[k][:, t].contiguous()
        st.step(torch.tensor([t], dtype=torch.int32, device=dev), tok("kv"), tok("score"), tok("idx_kv"),
                tok("idx_score"), tok("win_kv"), tok("q"), tok("q_idx"), tok("w"), x["sink"], out=out)
        torch.cuda.synchronize()
        assert ops.device_status(st.ws) == 0
        q = full["queries"][t]
        sel = check_topk(np64(st.topk_idx[0]), q["scores"], wl.topk, f"t={t}")
        if np.array_equal(sel, q["topk"][: len(sel)]):
            ref = q["out"]
        else:
            ref = O.attend_query(inp_np["q"][0, t], t, W, inp_np["win_kv"][0], S + N, full["cache"], sel.tolist(),
                                 inp_np["sink"], 1 / math.sqrt(d), wl.rope_dim, wl.rope_base)
        assert_attn_close(out[0], ref, f"decode t={t} after a {S}-token prefill")
    # Entry 150 (tokens 600..603, completed at t = 603) equals the prefill formula's.
    g = 603 // 4
    e = np64(st.cache[0, g])
    assert np.max(np.abs(e - full["entries"][g])) <= 5e-3 + 2 ** -8 * np.max(np.abs(full["entries"][g]))
