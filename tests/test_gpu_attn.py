"""GPU parity of sparse MQA with sink + inverse RoPE (csa_sparse_attn) and HCA attention (hca_attn)."""

import math

import numpy as np
import pytest
import torch

from oracle import csa_oracle as O
from tests.parity import assert_attn_close, np64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ops():
    from long_context_decode_c4a_b200 import ops
    return ops


def _q(B, S, H, d, g):
    x = torch.randn(B, S, H, d, generator=g)
    return (x * torch.rsqrt(x.square().mean(-1, keepdim=True) + 1e-6)).to(torch.bfloat16)


def _random_topk(B, S, pos, k, ratio, g):
    out = torch.full((B, S, k), -1, dtype=torch.int32)
    for b in range(B):
        for i in range(S):
            E = (int(pos[b, i]) + 1) // ratio
            n = min(k, E)
            if n:
                sel = torch.randperm(E, generator=g)[:n].sort().values
                out[b, i, :n] = sel.to(torch.int32)
    return out


@pytest.mark.parametrize("case", ["decode", "early_positions", "tiny_heads", "bf16_out"])
def test_sparse_attn(ops, case):
    g = torch.Generator().manual_seed(hash(case) % 997)
    d = 512
    if case == "decode":
        B, S, H, W, k, E_cap = 3, 1, 128, 128, 1024, 8192
        pos = torch.tensor([[32767], [20001], [4200]], dtype=torch.int32)
        ring_cap = W
    elif case == "early_positions":   # t < window and t < 3: partial window, no or few entries
        B, S, H, W, k, E_cap = 1, 6, 128, 128, 64, 64
        pos = torch.tensor([[0, 1, 3, 5, 100, 255]], dtype=torch.int32)
        ring_cap = 256
    elif case == "tiny_heads":
        B, S, H, W, k, E_cap = 1, 4, 8, 16, 8, 32
        pos = torch.tensor([[17, 64, 100, 127]], dtype=torch.int32)
        ring_cap = 128
    else:
        B, S, H, W, k, E_cap = 2, 1, 128, 128, 200, 1000
        pos = torch.tensor([[3999], [777]], dtype=torch.int32)
        ring_cap = W
    q = _q(B, S, H, d, g)
    ring = torch.randn(B, ring_cap, d, generator=g).to(torch.bfloat16)
    cache = torch.randn(B, E_cap, d, generator=g).to(torch.bfloat16)
    sink = torch.randn(H, generator=g)
    topk = _random_topk(B, S, pos, k, 4, g)
    out_dtype = torch.bfloat16 if case == "bf16_out" else torch.float32
    out = torch.empty(B, S, H, d, dtype=out_dtype, device="cuda")
    ops.sparse_attn(pos.cuda(), q.cuda(), ring.cuda(), cache.cuda(), topk.cuda(), sink.cuda(), W, out=out)
    torch.cuda.synchronize()
    for b in range(B):
        for i in range(S):
            t = int(pos[b, i])
            ref = O.attend_query(np64(q[b, i]), t, W, np64(ring[b]), ring_cap, np64(cache[b]),
                                 np64(topk[b, i]).tolist(), np64(sink), 1 / math.sqrt(d), 64, 10000.0)
            assert_attn_close(out[b, i], ref, f"{case} b={b} i={i} t={t}", bf16_out=out_dtype == torch.bfloat16)


def test_sink_minus_infinity_is_plain_softmax(ops):
    """T6 on the GPU: a sink of -inf removes the sink term."""
    g = torch.Generator().manual_seed(3)
    B, S, H, d, W = 1, 1, 128, 512, 128
    pos = torch.tensor([[999]], dtype=torch.int32)
    q = _q(B, S, H, d, g)
    ring = torch.randn(B, W, d, generator=g).to(torch.bfloat16)
    cache = torch.randn(B, 250, d, generator=g).to(torch.bfloat16)
    topk = _random_topk(B, S, pos, 100, 4, g)
    sink = torch.full((H,), float("-inf"))
    out = torch.empty(B, S, H, d, dtype=torch.float32, device="cuda")
    ops.sparse_attn(pos.cuda(), q.cuda(), ring.cuda(), cache.cuda(), topk.cuda(), sink.cuda(), W, out=out)
    torch.cuda.synchronize()
    ref = O.attend_query(np64(q[0, 0]), 999, W, np64(ring[0]), W, np64(cache[0]), np64(topk[0, 0]).tolist(),
                         np64(sink), 1 / math.sqrt(d), 64, 10000.0)
    assert np.all(np.isfinite(ref))
    assert_attn_close(out[0, 0], ref, "sink -inf")


def test_large_logits_rescale(ops):
    """Candidates whose logits jump far above the running max force the O rescale path."""
    g = torch.Generator().manual_seed(4)
    B, S, H, d, W = 1, 1, 128, 512, 128
    pos = torch.tensor([[4095]], dtype=torch.int32)
    q = _q(B, S, H, d, g)
    ring = torch.randn(B, W, d, generator=g).to(torch.bfloat16)
    cache = torch.randn(B, 1024, d, generator=g).to(torch.bfloat16)
    # late entries aligned with q (per head 0 direction) produce logits ~ +20 in later tiles
    cache[0, 900:] = (q[0, 0, 0].float() * 6).to(torch.bfloat16)
    topk = torch.arange(1024, dtype=torch.int32).reshape(1, 1, 1024)
    sink = torch.zeros(H)
    out = torch.empty(B, S, H, d, dtype=torch.float32, device="cuda")
    ops.sparse_attn(pos.cuda(), q.cuda(), ring.cuda(), cache.cuda(), topk.cuda(), sink.cuda(), W, out=out)
    torch.cuda.synchronize()
    ref = O.attend_query(np64(q[0, 0]), 4095, W, np64(ring[0]), W, np64(cache[0]), list(range(1024)), np64(sink),
                         1 / math.sqrt(d), 64, 10000.0)
    assert_attn_close(out[0, 0], ref, "rescale")


@pytest.mark.parametrize("ratio,E_cap,pos_list", [(128, 256, [32767, 20000, 127, 5000]), (4, 600, [2399, 130])])
def test_hca_attn(ops, ratio, E_cap, pos_list):
    g = torch.Generator().manual_seed(ratio)
    B, S, H, d, W = len(pos_list), 1, 128, 512, 128
    pos = torch.tensor(pos_list, dtype=torch.int32)[:, None]
    q = _q(B, S, H, d, g)
    ring = torch.randn(B, W, d, generator=g).to(torch.bfloat16)
    cache = torch.randn(B, E_cap, d, generator=g).to(torch.bfloat16)
    sink = torch.randn(H, generator=g)
    out = torch.empty(B, S, H, d, dtype=torch.float32, device="cuda")
    ops.hca_attn(pos.cuda(), q.cuda(), ring.cuda(), cache.cuda(), sink.cuda(), W, ratio=ratio, out=out)
    torch.cuda.synchronize()
    for b in range(B):
        t = pos_list[b]
        vis = min((t + 1) // ratio, E_cap)
        ref = O.attend_query(np64(q[b, 0]), t, W, np64(ring[b]), W, np64(cache[b]), list(range(vis)), np64(sink),
                             1 / math.sqrt(d), 64, 10000.0)
        assert_attn_close(out[b, 0], ref, f"hca b={b} t={t}")


def test_csa_with_all_entries_equals_hca(ops):
    """T5 on the GPU: top-k covering every visible entry gives the HCA (dense) result."""
    g = torch.Generator().manual_seed(9)
    B, S, H, d, W = 2, 1, 128, 512, 128
    pos = torch.tensor([[1023], [555]], dtype=torch.int32)
    q = _q(B, S, H, d, g)
    ring = torch.randn(B, W, d, generator=g).to(torch.bfloat16)
    cache = torch.randn(B, 256, d, generator=g).to(torch.bfloat16)
    sink = torch.randn(H, generator=g)
    topk = torch.full((B, S, 300), -1, dtype=torch.int32)
    for b in range(B):
        E = (int(pos[b, 0]) + 1) // 4
        topk[b, 0, :E] = torch.arange(E, dtype=torch.int32)
    o1 = torch.empty(B, S, H, d, dtype=torch.float32, device="cuda")
    o2 = torch.empty_like(o1)
    # Status-only workspaces: one CTA pair per query in both calls, so the arithmetic is the same.
    ws1 = torch.zeros(256, dtype=torch.uint8, device="cuda")
    ws2 = torch.zeros(256, dtype=torch.uint8, device="cuda")
    ops.sparse_attn(pos.cuda(), q.cuda(), ring.cuda(), cache.cuda(), topk.cuda(), sink.cuda(), W, out=o1, ws=ws1)
    ops.hca_attn(pos.cuda(), q.cuda(), ring.cuda(), cache.cuda(), sink.cuda(), W, ratio=4, out=o2, ws=ws2)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)


@pytest.mark.parametrize("mode,out_dtype", [("csa", torch.float32), ("hca", torch.float32), ("csa", torch.bfloat16)])
def test_split_candidates_match_one_pair_per_query(ops, mode, out_dtype):
    """Split-candidate mode (a query's tiles spread over several CTA pairs, partials merged by
    log-sum-exp) against one pair per query (a status-only workspace) and against the oracle. Query
    0 sits at t = 0 (one candidate: most splits are empty, split 0 holds the sink), query 3 at a
    position with a ragged last tile."""
    g = torch.Generator().manual_seed(21)
    B, S, H, d, W = 4, 1, 128, 512, 128
    pos = torch.tensor([[0], [32767], [1500], [4242]], dtype=torch.int32)
    E_cap = 8192 if mode == "csa" else 256
    q = _q(B, S, H, d, g)
    ring = torch.randn(B, W, d, generator=g).to(torch.bfloat16)
    cache = torch.randn(B, E_cap, d, generator=g).to(torch.bfloat16)
    sink = torch.randn(H, generator=g)
    args = [pos.cuda(), q.cuda(), ring.cuda(), cache.cuda()]
    topk = _random_topk(B, S, pos, 1024, 4, g) if mode == "csa" else None
    kind = ops._lib.CSA_WS_SPARSE_ATTN if mode == "csa" else ops._lib.CSA_WS_HCA_ATTN
    ws_split = ops.workspace(kind, B, S, 1, 1, "cuda")
    assert ws_split.numel() > 256          # the workspace holds the partials of several splits per query
    outs = []
    for ws in (ws_split, torch.zeros(256, dtype=torch.uint8, device="cuda")):
        out = torch.empty(B, S, H, d, dtype=out_dtype, device="cuda")
        if mode == "csa":
            ops.sparse_attn(*args, topk.cuda(), sink.cuda(), W, out=out, ws=ws)
        else:
            ops.hca_attn(*args, sink.cuda(), W, ratio=128, out=out, ws=ws)
        torch.cuda.synchronize()
        assert ops.device_status(ws) == 0
        outs.append(out)
    split, single = outs
    for b in range(B):
        t = int(pos[b, 0])
        sel = np64(topk[b, 0]).tolist() if mode == "csa" else list(range(min((t + 1) // 128, E_cap)))
        ref = O.attend_query(np64(q[b, 0]), t, W, np64(ring[b]), W, np64(cache[b]), sel, np64(sink),
                             1 / math.sqrt(d), 64, 10000.0)
        bf = out_dtype == torch.bfloat16
        tag = f"{mode} {'bf16' if bf else 'fp32'} out"
        assert_attn_close(split[b, 0], ref, f"{tag} split b={b} t={t}", bf16_out=bf)
        assert_attn_close(single[b, 0], ref, f"{tag} one pair b={b} t={t}", bf16_out=bf)
    # The two differ only by rounding (other running maxima for P's bf16 parts, another order of the
    # same sums, and for bf16 output one rounding step): far below what a dropped or misweighted split
    # would leave.
    rms = single.float().square().mean().sqrt()
    bound = 2e-3 * float(rms) + (float(single.float().abs().max()) * 2.0 ** -8 if out_dtype == torch.bfloat16 else 0.0)
    assert float((split.float() - single.float()).abs().max()) <= bound


@pytest.mark.parametrize("mode", ["csa", "hca"])
def test_largest_candidate_sets(ops, mode):
    """The largest candidate set the attention takes: a window of 1024 rows plus 2048 selected (CSA)
    or 2048 visible (HCA) entries, 96 tiles per query. Run with one CTA pair per query (the whole
    list in one pair's shared memory) and with the tiles split over pairs; both match the oracle and
    report no device error."""
    from long_context_decode_c4a_b200 import _lib
    g = torch.Generator().manual_seed(31)
    B, S, H, d, W = 2, 1, 128, 512, 1024
    if mode == "csa":
        ratio, E_cap = 4, 12000
        pos = torch.tensor([[40000], [8195]], dtype=torch.int32)   # 10000 and 2049 entries visible
        topk = _random_topk(B, S, pos, 2048, ratio, g)
    else:
        ratio, E_cap = 128, 2048
        pos = torch.tensor([[2048 * 128 + 100], [2048 * 128 - 1]], dtype=torch.int32)  # 2048 visible
        topk = None
    q = _q(B, S, H, d, g)
    ring = torch.randn(B, W, d, generator=g).to(torch.bfloat16)
    cache = torch.randn(B, E_cap, d, generator=g).to(torch.bfloat16)
    sink = torch.randn(H, generator=g)
    kind = _lib.CSA_WS_SPARSE_ATTN if mode == "csa" else _lib.CSA_WS_HCA_ATTN
    refs = []
    for b in range(B):
        t = int(pos[b, 0])
        sel = [int(s) for s in topk[b, 0] if s >= 0] if mode == "csa" else list(range(min((t + 1) // ratio, E_cap)))
        assert len(sel) == 2048
        refs.append(O.attend_query(np64(q[b, 0]), t, W, np64(ring[b]), W, np64(cache[b]), sel, np64(sink),
                                   1 / math.sqrt(d), 64, 10000.0))
    args = [x.cuda() for x in (pos, q, ring, cache)]
    for label, ws in (("one pair", torch.zeros(256, dtype=torch.uint8, device="cuda")),
                      ("split", ops.workspace(kind, B, S, 1, 1, "cuda"))):
        out = torch.empty(B, S, H, d, dtype=torch.float32, device="cuda")
        if mode == "csa":
            ops.sparse_attn(*args, topk.cuda(), sink.cuda(), W, out=out, ws=ws)
        else:
            ops.hca_attn(*args, sink.cuda(), W, ratio=ratio, out=out, ws=ws)
        torch.cuda.synchronize()
        assert ops.device_status(ws) == _lib.CSA_OK, label
        for b in range(B):
            assert_attn_close(out[b, 0], refs[b], f"{mode} {label} b={b}")
