"""GPU parity of the whole layer: fused CSA / HCA decode steps and the CSA prefill pipeline, on the
workload shapes (small batches in full, the full-size workloads on sampled requests/queries)."""

import math

import numpy as np
import pytest
import torch

from oracle import csa_oracle as O
from synth import WORKLOADS, make_inputs
from tests.parity import assert_attn_close, assert_compress_close, check_topk, np64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ops():
    from long_context_decode_c4a_b200 import ops
    return ops


def csa_state_from(ops, wl, inp):
    st = ops.CsaDecodeState(wl.B, wl.max_entries, H=wl.H, d=wl.d, H_I=wl.H_I, d_I=wl.d_I, window=wl.W,
                            topk=wl.topk, device="cuda")
    for name in ("state_kv", "state_score", "idx_state_kv", "idx_state_score", "cache", "idx_cache", "ring"):
        getattr(st, name).copy_(inp[name])
    return st


def run_csa_decode(ops, wl, inp, out_dtype=torch.float32):
    st = csa_state_from(ops, wl, inp)
    out = torch.empty(wl.B, wl.H, wl.d, dtype=out_dtype, device="cuda")
    cache32 = torch.zeros(st.cache.shape, dtype=torch.float32, device="cuda")
    st.step(inp["pos"][:, 0].contiguous(), inp["kv"][:, 0].contiguous(), inp["score"][:, 0].contiguous(),
            inp["idx_kv"][:, 0].contiguous(), inp["idx_score"][:, 0].contiguous(), inp["win_kv"][:, 0].contiguous(),
            inp["q"][:, 0].contiguous(), inp["q_idx"][:, 0].contiguous(), inp["w"][:, 0].contiguous(), inp["sink"],
            out=out, cache_f32=cache32)
    torch.cuda.synchronize()
    assert ops.device_status(st.ws) == 0
    return st, out, cache32


def check_csa_request(wl, inp_np, st, out, cache32, b):
    ref = O.csa_decode_request(inp_np, b, H=wl.H, d=wl.d, W=wl.W, topk=wl.topk)
    t = int(inp_np["pos"][b, 0])
    g = t // wl.ratio
    assert_compress_close(cache32[b, g:g + 1], st.cache[b, g:g + 1], ref["entry"][None], f"main entry b={b}")
    assert np.array_equal(np64(st.state_kv[b]), ref["state_kv"])
    assert np.array_equal(np64(st.state_score[b]), ref["state_score"])
    assert np.array_equal(np64(st.idx_state_kv[b]), ref["idx_state_kv"])
    assert np.array_equal(np64(st.ring[b]), ref["ring"])
    # The index entry feeds the indexer: check it against the oracle's float64 value.
    gi = np64(st.idx_cache[b, g])
    assert np.max(np.abs(gi - ref["idx_entry"])) <= 5e-3 + np.max(np.abs(ref["idx_entry"])) * 2 ** -8
    sel = check_topk(np64(st.topk_idx[b]), ref["scores"], wl.topk, f"b={b}")
    if not np.array_equal(np.sort(sel), ref["topk"][: len(sel)]):
        # Near-tie swap: check the attention on the GPU's own selection.
        ref_out = O.attend_query(inp_np["q"][b, 0], t, wl.W, ref["ring"], wl.W, ref["cache"], sel.tolist(),
                                 inp_np["sink"], 1 / math.sqrt(wl.d), wl.rope_dim, wl.rope_base)
    else:
        ref_out = ref["out"]
    return assert_attn_close(out[b], ref_out, f"csa decode b={b}")


def test_csa_decode_fused_small_batch(ops):
    wl = WORKLOADS["pro_csa_decode_32k"].scaled(B=3)
    inp = make_inputs(wl)
    inp_np = O.to_numpy_inputs(inp)
    st, out, cache32 = run_csa_decode(ops, wl, {k: v.cuda() for k, v in inp.items()})
    for b in range(wl.B):
        check_csa_request(wl, inp_np, st, out, cache32, b)


def test_csa_decode_fused_ragged_positions(ops):
    """Requests at different positions: some complete a group in-step, some do not."""
    wl = WORKLOADS["pro_csa_decode_32k"].scaled(B=4, ctx=8192)
    inp = make_inputs(wl)
    inp["pos"] = torch.tensor([[8191], [8190], [4096], [1001]], dtype=torch.int32)
    inp_np = O.to_numpy_inputs(inp)
    st, out, cache32 = run_csa_decode(ops, wl, {k: v.cuda() for k, v in inp.items()})
    for b in range(wl.B):
        t = int(inp_np["pos"][b, 0])
        ref = O.csa_decode_request(inp_np, b, H=wl.H, d=wl.d, W=wl.W, topk=wl.topk)
        if (t + 1) % 4 == 0:
            g = t // 4
            assert_compress_close(cache32[b, g:g + 1], st.cache[b, g:g + 1], ref["entry"][None], f"b={b}")
        assert np.array_equal(np64(st.state_kv[b]), ref["state_kv"])
        assert np.array_equal(np64(st.ring[b]), ref["ring"])
        sel = check_topk(np64(st.topk_idx[b]), ref["scores"], wl.topk, f"b={b}")
        ref_out = O.attend_query(inp_np["q"][b, 0], t, wl.W, ref["ring"], wl.W, ref["cache"], sel.tolist(),
                                 inp_np["sink"], 1 / math.sqrt(wl.d), 64, 10000.0)
        assert_attn_close(out[b], ref_out, f"b={b}")


def test_csa_decode_is_deterministic(ops):
    wl = WORKLOADS["pro_csa_decode_32k"].scaled(B=2)
    inp = {k: v.cuda() for k, v in make_inputs(wl).items()}
    _, o1, _ = run_csa_decode(ops, wl, inp, torch.bfloat16)
    _, o2, _ = run_csa_decode(ops, wl, inp, torch.bfloat16)
    assert torch.equal(o1, o2)


def test_hca_decode_fused_small_batch(ops):
    wl = WORKLOADS["pro_hca_decode_32k"].scaled(B=3)
    inp = make_inputs(wl)
    inp_np = O.to_numpy_inputs(inp)
    dinp = {k: v.cuda() for k, v in inp.items()}
    st = ops.HcaDecodeState(wl.B, wl.max_entries, H=wl.H, d=wl.d, window=wl.W)
    for name in ("state_kv", "state_score", "cache", "ring"):
        getattr(st, name).copy_(dinp[name])
    out = torch.empty(wl.B, wl.H, wl.d, dtype=torch.float32, device="cuda")
    cache32 = torch.zeros(st.cache.shape, dtype=torch.float32, device="cuda")
    st.step(dinp["pos"][:, 0].contiguous(), dinp["kv"][:, 0].contiguous(), dinp["score"][:, 0].contiguous(),
            dinp["win_kv"][:, 0].contiguous(), dinp["q"][:, 0].contiguous(), dinp["sink"], out=out,
            cache_f32=cache32)
    torch.cuda.synchronize()
    assert ops.device_status(st.ws) == 0
    for b in range(wl.B):
        ref = O.hca_decode_request(inp_np, b, H=wl.H, d=wl.d, W=wl.W, ratio=wl.ratio)
        g = 32767 // 128
        assert_compress_close(cache32[b, g:g + 1], st.cache[b, g:g + 1], ref["entry"][None], f"hca entry b={b}")
        assert np.array_equal(np64(st.state_kv[b]), ref["state_kv"])
        assert np.array_equal(np64(st.ring[b]), ref["ring"])
        assert_attn_close(out[b], ref["out"], f"hca decode b={b}")


def run_csa_prefill(ops, wl, inp):
    """Prefill through the C ABI: compress (main and index), indexer + top-k, sparse attention."""
    B, S, d, dI = wl.B, wl.S, wl.d, wl.d_I
    dev = "cuda"
    E = wl.max_entries
    main_cfg, idx_cfg = ops.compressor_cfg(4, d), ops.compressor_cfg(4, dI)
    skv = torch.empty(B, 8, 2 * d, dtype=torch.bfloat16, device=dev)
    ssc = torch.empty_like(skv)
    ikv = torch.empty(B, 8, 2 * dI, dtype=torch.bfloat16, device=dev)
    isc = torch.empty_like(ikv)
    ops.state_reset(main_cfg, skv, ssc)
    ops.state_reset(idx_cfg, ikv, isc)
    cache = torch.zeros(B, E, d, dtype=torch.bfloat16, device=dev)
    cache32 = torch.zeros(B, E, d, dtype=torch.float32, device=dev)
    icache = torch.zeros(B, E, dI, dtype=torch.bfloat16, device=dev)
    start = torch.zeros(B, dtype=torch.int32, device=dev)
    ops.compress(main_cfg, start, inp["kv"], inp["score"], inp["gamma"], skv, ssc, cache, cache32)
    ops.compress(idx_cfg, start, inp["idx_kv"], inp["idx_score"], inp["idx_gamma"], ikv, isc, icache)
    scores = torch.zeros(B, S, E, dtype=torch.float32, device=dev)
    topk = ops.indexer_topk(inp["pos"], inp["q_idx"], inp["w"], icache, wl.topk, scores=scores)
    out = torch.empty(B, S, wl.H, d, dtype=torch.float32, device=dev)
    ops.sparse_attn(inp["pos"], inp["q"], inp["win_kv"], cache, topk, inp["sink"], wl.W, out=out)
    torch.cuda.synchronize()
    return dict(cache=cache, cache32=cache32, icache=icache, scores=scores, topk=topk, out=out)


def check_prefill_queries(wl, inp_np, res, queries):
    ref = O.csa_prefill(inp_np, 0, queries, H=wl.H, d=wl.d, W=wl.W, topk=wl.topk)
    assert_compress_close(res["cache32"][0], res["cache"][0], ref["entries"], "prefill main entries")
    gi = np64(res["icache"][0])
    assert np.max(np.abs(gi - ref["idx_entries"])) <= 5e-3 + 2 ** -8 * np.max(np.abs(ref["idx_entries"]))
    worst = 0.0
    for i in queries:
        t = int(inp_np["pos"][0, i])
        q = ref["queries"][i]
        sel = check_topk(np64(res["topk"][0, i]), q["scores"], wl.topk, f"query {i}")
        if not np.array_equal(sel, q["topk"][: len(sel)]):
            ref_out = O.attend_query(inp_np["q"][0, i], t, wl.W, inp_np["win_kv"][0], wl.S, ref["cache"],
                                     sel.tolist(), inp_np["sink"], 1 / math.sqrt(wl.d), 64, 10000.0)
        else:
            ref_out = q["out"]
        worst = max(worst, assert_attn_close(res["out"][0, i], ref_out, f"prefill query {i}"))
    return worst


def test_tiny_prefill_end_to_end(ops):
    """The tiny workload (B=1, S=128, 8 heads, window 16, 4 indexer heads, top-k 8), every query."""
    wl = WORKLOADS["tiny_csa_prefill"]
    inp = make_inputs(wl)
    res = run_csa_prefill(ops, wl, {k: v.cuda() for k, v in inp.items()})
    check_prefill_queries(wl, O.to_numpy_inputs(inp), res, list(range(wl.S)))


def test_prefill_medium_end_to_end(ops):
    """S = 1000 tokens (250 entries, several indexer tiles and a ragged tail), sampled queries."""
    wl = WORKLOADS["csa_prefill_8k"].scaled(S=1000, ctx=1000, topk=64)
    inp = make_inputs(wl)
    res = run_csa_prefill(ops, wl, {k: v.cuda() for k, v in inp.items()})
    check_prefill_queries(wl, O.to_numpy_inputs(inp), res, [0, 2, 3, 4, 63, 127, 128, 255, 256, 511, 998, 999])


def run_hca_prefill(ops, wl, inp):
    """HCA prefill through the C ABI: the C128A stream over the segment, then attention over the
    window and every visible entry."""
    B, S, d = wl.B, wl.S, wl.d
    dev = "cuda"
    E = wl.max_entries
    cfg = ops.compressor_cfg(wl.ratio, d)
    skv = torch.empty(B, wl.ratio, d, dtype=torch.bfloat16, device=dev)
    ssc = torch.empty_like(skv)
    ops.state_reset(cfg, skv, ssc)
    cache = torch.zeros(B, E, d, dtype=torch.bfloat16, device=dev)
    cache32 = torch.zeros(B, E, d, dtype=torch.float32, device=dev)
    start = torch.zeros(B, dtype=torch.int32, device=dev)
    ops.compress(cfg, start, inp["kv"], inp["score"], inp["gamma"], skv, ssc, cache, cache32)
    out = torch.empty(B, S, wl.H, d, dtype=torch.float32, device=dev)
    ops.hca_attn(inp["pos"], inp["q"], inp["win_kv"], cache, inp["sink"], wl.W, ratio=wl.ratio, out=out)
    torch.cuda.synchronize()
    return dict(cache=cache, cache32=cache32, out=out, state_kv=skv)


def check_hca_prefill_queries(wl, inp_np, res, queries):
    ref = O.csa_prefill(inp_np, 0, queries, H=wl.H, d=wl.d, W=wl.W, topk=0, ratio=wl.ratio, with_indexer=False)
    assert_compress_close(res["cache32"][0], res["cache"][0], ref["entries"], "hca prefill entries")
    for i in queries:
        assert_attn_close(res["out"][0, i], ref["queries"][i]["out"], f"hca prefill query {i}")


def test_hca_prefill_medium_end_to_end(ops):
    """S = 1000 tokens through the HCA layer (ratio 128: 7 entries, a ragged last group), queries at
    every point where an entry becomes visible and at the window edges."""
    wl = WORKLOADS["hca_prefill_8k"].scaled(S=1000, ctx=1000)
    inp = make_inputs(wl)
    res = run_hca_prefill(ops, wl, {k: v.cuda() for k, v in inp.items()})
    queries = [0, 1, 126, 127, 128, 129, 255, 256, 383, 384, 511, 639, 640, 767, 895, 896, 998, 999]
    check_hca_prefill_queries(wl, O.to_numpy_inputs(inp), res, queries)
