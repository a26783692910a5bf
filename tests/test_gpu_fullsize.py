"""Parity at the full workload sizes, in the launch configuration the benchmark times, on sampled
requests / queries that the oracle computes one by one."""

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


class RowSource:
    """Read-only view of selected rows of a device tensor [E, d] (fetched on demand, float64)."""

    def __init__(self, t):
        self.t = t
        self.cache = {}

    def __getitem__(self, s):
        s = int(s)
        if s not in self.cache:
            self.cache[s] = self.t[s].double().cpu().numpy()
        return self.cache[s]


def _sub(inp, b):
    """Request b's decode inputs as float64 numpy arrays with a leading batch of 1."""
    return {k: (np64(v[b:b + 1]) if v.dim() > 1 and k not in ("sink", "gamma", "idx_gamma") else np64(v))
            for k, v in inp.items() if k not in ("cache", "idx_cache")}


def test_pro_csa_decode_full_batch_sampled(ops):
    """B = 64 requests at 32K context (the benchmark's workload), requests 0, 37 and 63."""
    wl = WORKLOADS["pro_csa_decode_32k"]
    inp = make_inputs(wl, device="cuda")
    st = ops.CsaDecodeState(wl.B, wl.max_entries, device="cuda")
    for n in ("state_kv", "state_score", "idx_state_kv", "idx_state_score", "cache", "idx_cache", "ring"):
        getattr(st, n).copy_(inp[n])
    out = torch.empty(wl.B, wl.H, wl.d, dtype=torch.float32, device="cuda")
    cache32 = torch.zeros(st.cache.shape, dtype=torch.float32, device="cuda")
    x = {k: inp[k][:, 0].contiguous() for k in ("pos", "kv", "score", "idx_kv", "idx_score", "win_kv", "q", "q_idx", "w")}
    st.step(x["pos"], x["kv"], x["score"], x["idx_kv"], x["idx_score"], x["win_kv"], x["q"], x["q_idx"], x["w"],
            inp["sink"], out=out, cache_f32=cache32)
    torch.cuda.synchronize()
    assert ops.device_status(st.ws) == 0
    for b in (0, 37, 63):
        sub = _sub(inp, b)
        sub["cache"] = np64(inp["cache"][b:b + 1])
        sub["idx_cache"] = np64(inp["idx_cache"][b:b + 1])
        ref = O.csa_decode_request(sub, 0, H=wl.H, d=wl.d, W=wl.W, topk=wl.topk)
        g = wl.max_entries - 1
        assert_compress_close(cache32[b, g:g + 1], st.cache[b, g:g + 1], ref["entry"][None], f"b={b}")
        assert np.array_equal(np64(st.state_kv[b]), ref["state_kv"])
        assert np.array_equal(np64(st.ring[b]), ref["ring"])
        sel = check_topk(np64(st.topk_idx[b]), ref["scores"], wl.topk, f"b={b}")
        ref_out = O.attend_query(sub["q"][0, 0], int(sub["pos"][0, 0]), wl.W, ref["ring"], wl.W, ref["cache"],
                                 sel.tolist(), sub["sink"], 1 / math.sqrt(wl.d), 64, 10000.0)
        assert_attn_close(out[b], ref_out, f"b={b}")


def test_pro_hca_decode_full_batch_sampled(ops):
    wl = WORKLOADS["pro_hca_decode_32k"]
    inp = make_inputs(wl, device="cuda")
    st = ops.HcaDecodeState(wl.B, wl.max_entries, device="cuda")
    for n in ("state_kv", "state_score", "cache", "ring"):
        getattr(st, n).copy_(inp[n])
    out = torch.empty(wl.B, wl.H, wl.d, dtype=torch.float32, device="cuda")
    x = {k: inp[k][:, 0].contiguous() for k in ("pos", "kv", "score", "win_kv", "q")}
    st.step(x["pos"], x["kv"], x["score"], x["win_kv"], x["q"], inp["sink"], out=out)
    torch.cuda.synchronize()
    assert ops.device_status(st.ws) == 0
    for b in (0, 21, 63):
        sub = _sub(inp, b)
        sub["cache"] = np64(inp["cache"][b:b + 1])
        ref = O.hca_decode_request(sub, 0, H=wl.H, d=wl.d, W=wl.W, ratio=wl.ratio)
        assert np.array_equal(np64(st.state_kv[b]), ref["state_kv"])
        assert_attn_close(out[b], ref["out"], f"hca b={b}")


def test_csa_prefill_8k_sampled(ops):
    """S = 8192 tokens from an empty cache: every compressed entry, and sampled queries."""
    from tests.test_gpu_layer import run_csa_prefill
    wl = WORKLOADS["csa_prefill_8k"]
    inp = make_inputs(wl, device="cuda")
    res = run_csa_prefill(ops, wl, inp)
    main = O.CompressorCfg(4, wl.d)
    index = O.CompressorCfg(4, wl.d_I)
    ent = O.compress_parallel(main, np64(inp["kv"][0]), np64(inp["score"][0]), np64(inp["gamma"]))
    ient = O.compress_parallel(index, np64(inp["idx_kv"][0]), np64(inp["idx_score"][0]), np64(inp["idx_gamma"]))
    assert_compress_close(res["cache32"][0], res["cache"][0], ent, "prefill main entries")
    icache = O.bf16(ient)
    cache = O.bf16(ent)
    gi = np64(res["icache"][0])
    assert np.max(np.abs(gi - ient)) <= 5e-3 + 2 ** -8 * np.max(np.abs(ient))
    ring = RowSource(inp["win_kv"][0])
    sink = np64(inp["sink"])
    for i in (0, 3, 4, 511, 512, 4095, 4096, 6000, 8190, 8191):
        t = i
        vis = (t + 1) // 4
        sc = O.indexer_scores(np64(inp["q_idx"][0, i]), np64(inp["w"][0, i]), icache, vis)
        sel = check_topk(np64(res["topk"][0, i]), sc, wl.topk, f"query {i}")
        ref_out = O.attend_query(np64(inp["q"][0, i]), t, wl.W, ring, wl.S, cache, sel.tolist(), sink,
                                 1 / math.sqrt(wl.d), 64, 10000.0)
        assert_attn_close(res["out"][0, i], ref_out, f"prefill query {i}")


def test_hca_prefill_8k_sampled(ops):
    """S = 8192 tokens through the HCA layer from an empty cache: all 64 entries, sampled queries."""
    from tests.test_gpu_layer import run_hca_prefill
    wl = WORKLOADS["hca_prefill_8k"]
    inp = make_inputs(wl, device="cuda")
    res = run_hca_prefill(ops, wl, inp)
    cfg = O.CompressorCfg(wl.ratio, wl.d)
    ent = O.compress_parallel(cfg, np64(inp["kv"][0]), np64(inp["score"][0]), np64(inp["gamma"]))
    assert_compress_close(res["cache32"][0], res["cache"][0], ent, "hca prefill entries")
    cache = O.bf16(ent)
    ring = RowSource(inp["win_kv"][0])
    sink = np64(inp["sink"])
    for i in (0, 127, 128, 4095, 4096, 6000, 8190, 8191):
        t = i
        ref_out = O.attend_query(np64(inp["q"][0, i]), t, wl.W, ring, wl.S, cache, list(range((t + 1) // wl.ratio)),
                                 sink, 1 / math.sqrt(wl.d), 64, 10000.0)
        assert_attn_close(res["out"][0, i], ref_out, f"hca prefill query {i}")


def test_long_context_decode_sampled(ops):
    """B = 8 requests at position 1,048,575 (262,144 entries each): the chunked top-k path."""
    wl = WORKLOADS["long_csa_decode_1m"]
    inp = make_inputs(wl, device="cuda")
    st = ops.CsaDecodeState(wl.B, wl.max_entries, device="cuda")
    for n in ("state_kv", "state_score", "idx_state_kv", "idx_state_score", "cache", "idx_cache", "ring"):
        getattr(st, n).copy_(inp[n])
    out = torch.empty(wl.B, wl.H, wl.d, dtype=torch.float32, device="cuda")
    x = {k: inp[k][:, 0].contiguous() for k in ("pos", "kv", "score", "idx_kv", "idx_score", "win_kv", "q", "q_idx", "w")}
    st.step(x["pos"], x["kv"], x["score"], x["idx_kv"], x["idx_score"], x["win_kv"], x["q"], x["q_idx"], x["w"],
            inp["sink"], out=out)
    torch.cuda.synchronize()
    assert ops.device_status(st.ws) == 0
    b = 5
    t = int(inp["pos"][b, 0])
    g = t // 4
    # the oracle's compressor step for this request (both streams)
    icfg = O.CompressorCfg(4, wl.d_I)
    ikv, isc = np64(inp["idx_state_kv"][b]), np64(inp["idx_state_score"][b])
    _, ientry = O.compressor_step(icfg, ikv, isc, t, np64(inp["idx_kv"][b, 0]), np64(inp["idx_score"][b, 0]),
                                  np64(inp["idx_gamma"]))
    mcfg = O.CompressorCfg(4, wl.d)
    mkv, msc = np64(inp["state_kv"][b]), np64(inp["state_score"][b])
    _, mentry = O.compressor_step(mcfg, mkv, msc, t, np64(inp["kv"][b, 0]), np64(inp["score"][b, 0]),
                                  np64(inp["gamma"]))
    icache = np64(inp["idx_cache"][b])
    icache[g] = O.bf16(ientry)
    sc = O.indexer_scores(np64(inp["q_idx"][b, 0]), np64(inp["w"][b, 0]), icache, (t + 1) // 4)
    sel = check_topk(np64(st.topk_idx[b]), sc, wl.topk, "long decode")
    ring = np64(inp["ring"][b])
    ring[t % wl.W] = np64(inp["win_kv"][b, 0])
    cache = RowSource(inp["cache"][b])      # the input cache, with the oracle's own new entry g
    cache.cache[g] = O.bf16(mentry)
    ref_out = O.attend_query(np64(inp["q"][b, 0]), t, wl.W, ring, wl.W, cache, sel.tolist(), np64(inp["sink"]),
                             1 / math.sqrt(wl.d), 64, 10000.0)
    assert np.max(np.abs(np64(st.cache[b, g]) - mentry)) <= 5e-3 + 2 ** -8 * np.max(np.abs(mentry))
    assert_attn_close(out[b], ref_out, "long decode")
