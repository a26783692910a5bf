"""GPU parity of the C4A / C128A compressor (csa_compress, csa_state_reset) against the oracle."""

import numpy as np
import pytest
import torch

from oracle import csa_oracle as O
from tests.parity import assert_compress_close, np64

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ops():
    from long_context_decode_c4a_b200 import ops
    return ops


def _streams(B, S, width, seed, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    kv = torch.randn(B, S, width, generator=g).to(torch.bfloat16)
    sc = (torch.randn(B, S, width, generator=g) * scale).to(torch.bfloat16)
    return kv, sc


@pytest.mark.parametrize("ratio,d", [(4, 512), (4, 128), (128, 512)])
def test_compress_segments_vs_state_machine(ops, ratio, d):
    """Uneven segments per call, per-request data; entries match the oracle's rolling state and
    the GPU state after every call equals the oracle's state bit for bit."""
    torch.manual_seed(0)
    overlap = 1 if ratio == 4 else 0
    width = (1 + overlap) * d
    B = 3
    S_total = 3 * ratio + 7 if ratio == 128 else 45
    cuts = [0, 1, 2, ratio + 1, 2 * ratio + 3, S_total] if ratio == 128 else [0, 1, 5, 6, 20, 33, 45]
    kv, sc = _streams(B, S_total, width, seed=ratio + d, scale=2.0)
    gamma = (1 + 0.1 * torch.randn(d)).to(torch.bfloat16)
    cfg = ops.compressor_cfg(ratio, d)
    E = S_total // ratio
    dev = "cuda"
    rows = (1 + overlap) * ratio
    skv = torch.empty(B, rows, width, dtype=torch.bfloat16, device=dev)
    ssc = torch.empty_like(skv)
    ops.state_reset(cfg, skv, ssc)
    cache = torch.zeros(B, E, d, dtype=torch.bfloat16, device=dev)
    cache32 = torch.zeros(B, E, d, dtype=torch.float32, device=dev)
    ocfg = O.CompressorCfg(ratio, d)
    o_states = [O.init_state(ocfg) for _ in range(B)]
    o_entries = [{} for _ in range(B)]
    gnp = np64(gamma)
    for lo, hi in zip(cuts[:-1], cuts[1:]):
        start = torch.full((B,), lo, dtype=torch.int32, device=dev)
        ops.compress(cfg, start, kv[:, lo:hi].contiguous().to(dev), sc[:, lo:hi].contiguous().to(dev),
                     gamma.to(dev), skv, ssc, cache, cache32)
        torch.cuda.synchronize()
        for b in range(B):
            o_entries[b].update(O.compress_tokens(ocfg, o_states[b][0], o_states[b][1], lo, np64(kv[b, lo:hi]),
                                                  np64(sc[b, lo:hi]), gnp))
            gk, gs = np64(skv[b]), np64(ssc[b])
            assert np.array_equal(gk, o_states[b][0]), f"state kv differs after segment [{lo},{hi}) b={b}"
            assert np.array_equal(gs, o_states[b][1]), f"state score differs after segment [{lo},{hi}) b={b}"
    for b in range(B):
        ref = np.stack([o_entries[b][g] for g in range(E)])
        assert_compress_close(cache32[b], cache[b], ref, f"ratio {ratio} d {d} b {b}")


def test_prefill_parallel_matches_direct_formula(ops):
    """One-shot prefill of 128 tokens (tiny config streams) against the per-group formula."""
    d, S, B = 512, 128, 2
    kv, sc = _streams(B, S, 2 * d, seed=7)
    gamma = torch.ones(d, dtype=torch.bfloat16)
    cfg = ops.compressor_cfg(4, d)
    skv = torch.empty(B, 8, 2 * d, dtype=torch.bfloat16, device="cuda")
    ssc = torch.empty_like(skv)
    ops.state_reset(cfg, skv, ssc)
    cache = torch.zeros(B, S // 4, d, dtype=torch.bfloat16, device="cuda")
    cache32 = torch.zeros(B, S // 4, d, dtype=torch.float32, device="cuda")
    ops.compress(cfg, torch.zeros(B, dtype=torch.int32, device="cuda"), kv.cuda(), sc.cuda(), gamma.cuda(), skv, ssc,
                 cache, cache32)
    torch.cuda.synchronize()
    ocfg = O.CompressorCfg(4, d)
    for b in range(B):
        ref = O.compress_parallel(ocfg, np64(kv[b]), np64(sc[b]), np64(gamma))
        assert_compress_close(cache32[b], cache[b], ref, f"b {b}")


def test_decode_step_at_32k(ops):
    """S = 1 at t = 32767 from a random state (the decode workload's compressor step)."""
    for ratio, d in ((4, 512), (4, 128), (128, 512)):
        overlap = 1 if ratio == 4 else 0
        width = (1 + overlap) * d
        rows = (1 + overlap) * ratio
        B = 4
        g = torch.Generator().manual_seed(ratio * 7 + d)
        skv0 = torch.randn(B, rows, width, generator=g).to(torch.bfloat16)
        ssc0 = torch.randn(B, rows, width, generator=g).to(torch.bfloat16)
        kv = torch.randn(B, 1, width, generator=g).to(torch.bfloat16)
        sc = torch.randn(B, 1, width, generator=g).to(torch.bfloat16)
        E = 32768 // ratio
        cache = torch.zeros(B, E, d, dtype=torch.bfloat16, device="cuda")
        cache32 = torch.zeros(B, E, d, dtype=torch.float32, device="cuda")
        skv, ssc = skv0.cuda(), ssc0.cuda()
        ops.compress(ops.compressor_cfg(ratio, d), torch.full((B,), 32767, dtype=torch.int32, device="cuda"),
                     kv.cuda(), sc.cuda(), torch.ones(d, dtype=torch.bfloat16, device="cuda"), skv, ssc, cache,
                     cache32)
        torch.cuda.synchronize()
        ocfg = O.CompressorCfg(ratio, d)
        for b in range(B):
            okv, osc = np64(skv0[b]).copy(), np64(ssc0[b]).copy()
            g_, entry = O.compressor_step(ocfg, okv, osc, 32767, np64(kv[b, 0]), np64(sc[b, 0]), np.ones(d))
            assert g_ == E - 1
            assert_compress_close(cache32[b, E - 1:E], cache[b, E - 1:E], entry[None], f"ratio {ratio} d {d}")
            assert np.array_equal(np64(skv[b]), okv) and np.array_equal(np64(ssc[b]), osc)
            # nothing else in the cache was touched
            assert torch.count_nonzero(cache[b, :E - 1]) == 0


@pytest.mark.parametrize("ratio", [4, 128])
def test_decode_step_mixed_positions(ops, ratio):
    """One decode step for requests at different positions: some complete a group in the step
    (C128A: group 0 too), some do not; each request's entry and state against the oracle, and no
    other cache row touched."""
    d = 512
    overlap = 1 if ratio == 4 else 0
    width = (1 + overlap) * d
    rows = (1 + overlap) * ratio
    # C4A's group 0 has no previous group (its slots are the reset state's, weight 0), so a random
    # state is a valid input there only for C128A.
    pos = [32767, 32766, 127 if ratio == 128 else 7, 5000, 2 * ratio - 1]
    B = len(pos)
    g = torch.Generator().manual_seed(31 + ratio)
    skv0 = torch.randn(B, rows, width, generator=g).to(torch.bfloat16)
    ssc0 = torch.randn(B, rows, width, generator=g).to(torch.bfloat16)
    kv = torch.randn(B, 1, width, generator=g).to(torch.bfloat16)
    sc = torch.randn(B, 1, width, generator=g).to(torch.bfloat16)
    gamma = (1 + 0.1 * torch.randn(d, generator=g)).to(torch.bfloat16)
    E = 32768 // ratio
    cache = torch.zeros(B, E, d, dtype=torch.bfloat16, device="cuda")
    cache32 = torch.zeros(B, E, d, dtype=torch.float32, device="cuda")
    skv, ssc = skv0.cuda(), ssc0.cuda()
    ops.compress(ops.compressor_cfg(ratio, d), torch.tensor(pos, dtype=torch.int32, device="cuda"), kv.cuda(),
                 sc.cuda(), gamma.cuda(), skv, ssc, cache, cache32)
    torch.cuda.synchronize()
    ocfg = O.CompressorCfg(ratio, d)
    for b, t in enumerate(pos):
        okv, osc = np64(skv0[b]).copy(), np64(ssc0[b]).copy()
        res = O.compressor_step(ocfg, okv, osc, t, np64(kv[b, 0]), np64(sc[b, 0]), np64(gamma))
        assert np.array_equal(np64(skv[b]), okv) and np.array_equal(np64(ssc[b]), osc), f"state b={b} t={t}"
        touched = torch.nonzero(cache[b].abs().sum(-1)).flatten().tolist()
        if (t + 1) % ratio == 0:
            gi, entry = res
            assert gi == t // ratio and touched == [gi], f"b={b} t={t}"
            assert_compress_close(cache32[b, gi:gi + 1], cache[b, gi:gi + 1], entry[None], f"ratio {ratio} b={b} t={t}")
        else:
            assert res is None and touched == [], f"b={b} t={t}"


def test_state_reset_values(ops):
    cfg = ops.compressor_cfg(4, 128)
    skv = torch.full((2, 8, 256), 3.0, dtype=torch.bfloat16, device="cuda")
    ssc = torch.full_like(skv, 3.0)
    ops.state_reset(cfg, skv, ssc)
    assert torch.all(skv == 0) and torch.all(torch.isneginf(ssc.float()))
