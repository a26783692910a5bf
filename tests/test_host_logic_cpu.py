"""Host-side logic that needs no GPU: the benchmark's algorithmic ledgers, the tensor-parallel head
split, and the bindings' refusal of tensors that are not on a CUDA device (the layer has no CPU
path)."""

import math

import pytest
import torch

import bench
from oracle import csa_oracle as O
from synth import WORKLOADS
from synth.workloads import OPROJ_D, OPROJ_GROUPS, OPROJ_KG, OPROJ_R, QPATH_HIDDEN, QPATH_RANK


def test_prefill_ledgers_match_per_query_reads():
    """The bench's FLOP count of a prefill pass is the pages' 4 x heads x reads x 512 per query
    ([P1] "Pro 的 CSA 和 HCA，成本交点在哪里"), with reads from the oracle's own counter, plus for CSA
    the indexer's 2 x H_I x d_I per (query, visible entry)."""
    for name in ("csa_prefill_8k", "hca_prefill_8k", "tiny_csa_prefill"):
        wl = WORKLOADS[name]
        attn, idx = bench.prefill_ledger(wl)
        want_attn = sum(O.attention_flops(wl.H, O.reads_per_query(t, wl.W, wl.ratio,
                                                                   wl.topk if wl.has_indexer else None), wl.d)
                        for t in range(wl.S))
        assert attn == want_attn, name
        if wl.has_indexer:
            assert idx == sum(2 * wl.H_I * wl.d_I * O.visible_entries(t, wl.ratio) for t in range(wl.S))
        else:
            assert idx == 0


def test_projection_shapes_follow_the_printed_parameter_counts():
    """[P1]: the query path holds 7168 x 1536 + 1536 x 65536 = 106.5 Mi weights; the output
    projection 64 Mi + 112 Mi = 176 Mi."""
    mi = 1 << 20
    assert QPATH_HIDDEN * QPATH_RANK + QPATH_RANK * 128 * 512 == int(106.5 * mi)
    assert OPROJ_GROUPS * OPROJ_R * OPROJ_KG == 64 * mi
    assert OPROJ_D * OPROJ_GROUPS * OPROJ_R == 112 * mi


def test_head_shard_covers_every_head_once():
    from long_context_decode_c4a_b200.tp import head_shard
    for world in (1, 2, 4, 8):
        spans = [head_shard(64, r, world) for r in range(world)]
        assert spans[0][0] == 0 and spans[-1][1] == 64
        assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
    with pytest.raises(ValueError):
        head_shard(64, 0, 3)


def test_bindings_refuse_host_tensors():
    """Every entry of the binding takes device tensors only: a CPU tensor is refused before the
    library is called (there is no CPU fallback)."""
    from long_context_decode_c4a_b200 import ops
    x = torch.zeros(4, 128, dtype=torch.bfloat16)
    w = torch.zeros(128, 128, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="CUDA"):
        ops.linear(x, w)
    with pytest.raises(ValueError, match="CUDA"):
        ops.output_projection(torch.zeros(1, 64, dtype=torch.bfloat16), torch.zeros(1, 128, 64, dtype=torch.bfloat16),
                              torch.zeros(128, 128, dtype=torch.bfloat16))
    with pytest.raises(ValueError, match="CUDA"):
        ops.topk(torch.zeros(1, 1, dtype=torch.int32), torch.zeros(1, 1, 8), 4)


def test_decode_bytes_ledger():
    """The bench's bytes per decode query: attention reads 1152 rows of 1 KB plus q and output; the
    indexer launch the visible index entries plus q_idx, w and the score row, plus the compressor
    step it runs (both streams' states and token rows, the entries and the window row)."""
    wl = WORKLOADS["pro_csa_decode_32k"]
    per_q, reads = bench.decode_bytes(wl)
    assert reads == O.reads_per_query(wl.ctx - 1, wl.W, wl.ratio, wl.topk) == 1152
    assert per_q["attention"] == reads * wl.d * 2 + 2 * wl.H * wl.d * 2 + wl.topk * 4
    E = wl.max_entries
    comp_main = 2 * 8 * 1024 * 2 + 2 * 1024 * 2 + 512 * 2 + 2 * 512 * 2
    comp_idx = 2 * 8 * 2 * 128 * 2 + 2 * 2 * 128 * 2 + 128 * 2
    assert per_q["compress"] == 0
    assert per_q["indexer"] == E * wl.d_I * 2 + wl.H_I * wl.d_I * 2 + wl.H_I * 4 + E * 4 + comp_main + comp_idx
    assert math.isclose(per_q["attention"] / 1e6, 1.44, rel_tol=0.01)
    # HCA keeps the compressor launch of its own.
    per_h, _ = bench.decode_bytes(WORKLOADS["pro_hca_decode_32k"])
    assert per_h["compress"] > 0 and "indexer" not in per_h


def test_graph_rounds_fit_the_timed_steps():
    """The CUDA graph of the timed loop holds whole rounds of the input-set sequence and never more
    steps than the run times (the rest are launched directly)."""
    assert bench.graph_rounds(10, 200, 4) == 10
    assert bench.graph_rounds(10, 12, 4) == 3
    assert bench.graph_rounds(10, 3, 4) == 1
    assert bench.graph_rounds(1, 200, 4) == 1
    assert bench.graph_rounds(10, 20, 2) == 10
    for steps in range(1, 60):
        r = bench.graph_rounds(10, steps, 4)
        assert r >= 1 and (r * 4 <= steps or steps < 4)


def test_decode_launch_counts_follow_the_library_rules():
    """gpu_launches claims: CSA 32K = indexer (compressor step inside) + top-k + attention; 1M
    context = indexer + top-k chunks + merge + attention split over 9 pairs per query + combine; HCA
    = C128A step + attention; a small CSA batch splits its attention (combine added)."""
    import bench
    assert bench.decode_launches(WORKLOADS["pro_csa_decode_32k"]) == 3
    assert bench.decode_launches(WORKLOADS["long_csa_decode_1m"]) == 5
    assert bench.decode_launches(WORKLOADS["pro_hca_decode_32k"]) == 2
    assert bench.decode_launches(WORKLOADS["pro_csa_decode_32k"].scaled(B=8)) == 4


def test_packed_inputs_round_trip_every_tensor():
    """The end-to-end timing copies a step's inputs in one buffer: every tensor of a decode step gets
    its own 256-byte aligned, non-overlapping slot, and the views give back the same values."""
    g = torch.Generator().manual_seed(5)
    inputs = {
        "pos": torch.randint(0, 1 << 20, (3,), dtype=torch.int32, generator=g),
        "kv": torch.randn(3, 2, 512, generator=g),
        "win_kv": torch.randn(3, 512, generator=g).to(torch.bfloat16),
        "q": torch.randn(3, 5, 512, generator=g).to(torch.bfloat16),
        "w": torch.randn(3, 7, generator=g),
    }
    offs, total = bench.packed_layout(inputs)
    spans = sorted((offs[k], offs[k] + v.numel() * v.element_size()) for k, v in inputs.items())
    assert all(o % 256 == 0 for o in offs.values())
    assert all(a[1] <= b[0] for a, b in zip(spans, spans[1:]))
    assert total % 256 == 0 and spans[-1][1] <= total
    flat = torch.zeros(total, dtype=torch.uint8)
    views = bench.packed_views(flat, inputs, offs)
    for k, v in views.items():
        v.copy_(inputs[k])
    again = bench.packed_views(flat.clone(), inputs, offs)
    for k, v in inputs.items():
        assert again[k].dtype == v.dtype and again[k].shape == v.shape
        assert torch.equal(again[k], v), k
