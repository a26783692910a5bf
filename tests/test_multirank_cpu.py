"""The multi-process path of bench.py on CPU: two gloo ranks, as torchrun would start them.

Requests are sharded over ranks (every rank owns its own B requests, no data-path collective);
the only collectives are the barrier around the timed region and the max over ranks of the step
time. The reference arm runs on rank 0 alone.
"""

import argparse
import contextlib
import io
import os
import socket

import pytest
import torch
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank: int, world: int, port: int, q) -> None:
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    try:
        import bench
        from synth import WORKLOADS, make_inputs

        w, r, _ = bench.dist_setup(world)
        bench.barrier(w)
        # The max over ranks of a per-rank time.
        m = bench.max_over_ranks(1.5 * (rank + 1), w)
        # Each rank draws its own requests: the shard seeds differ by rank.
        wl = WORKLOADS["pro_csa_decode_32k"].scaled(B=1)
        x = make_inputs(wl, seed=wl.seed + 1000 * rank)
        digest = float(x["q"].float().sum())
        # The reference arm: rank 0 prints one JSON line, the others return without output.
        args = argparse.Namespace(warmup=3, steps=1)
        out = io.StringIO()
        with contextlib.redirect_stdout(out):
            rc = bench.run_reference(wl, args)
        bench.barrier(w)
        import torch.distributed as dist
        dist.destroy_process_group()
        q.put((rank, w, r, m, digest, rc, out.getvalue()))
    except Exception as e:  # noqa: BLE001
        q.put((rank, "error", repr(e)))


@pytest.mark.timeout(600)
def test_two_gloo_ranks_shard_requests_and_reduce_time():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        item = q.get(timeout=500)
        res[item[0]] = item
    for p in procs:
        p.join(timeout=60)
    for r in range(world):
        assert res[r][1] != "error", res[r]
        _, w, rr, m, digest, rc, out = res[r]
        assert (w, rr, rc) == (world, r, 0)
        assert m == pytest.approx(3.0)                     # max over ranks of 1.5 * (rank + 1)
    assert res[0][4] != res[1][4], "the two ranks drew the same requests"
    line = res[0][6].strip().splitlines()
    assert len(line) == 1 and '"impl": "reference"' in line[0]
    assert res[1][6].strip() == ""


def _tp_worker(rank: int, world: int, port: int, q) -> None:
    """One rank of the tensor-parallel indexer over gloo, with the kernels replaced by the oracle."""
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank), MASTER_ADDR="127.0.0.1",
                      MASTER_PORT=str(port))
    try:
        import types

        import numpy as np
        import torch.distributed as dist

        import long_context_decode_c4a_b200.tp as tp
        from oracle import csa_oracle as O
        from synth import WORKLOADS, make_inputs

        def fake_scores(q_pos, q_idx, w, idx_cache, ratio, scores=None):
            B, S, H, _ = q_idx.shape
            E = idx_cache.shape[1]
            out = torch.zeros(B, S, E, dtype=torch.float64)
            for b in range(B):
                for i in range(S):
                    vis = min((int(q_pos[b, i]) + 1) // ratio, E)
                    out[b, i, :vis] = torch.from_numpy(O.indexer_scores(
                        q_idx[b, i].double().numpy(), w[b, i].double().numpy(), idx_cache[b].double().numpy(), vis))
            return out

        def fake_topk(q_pos, scores, k, ratio):
            B, S, E = scores.shape
            out = torch.full((B, S, k), -1, dtype=torch.int32)
            for b in range(B):
                for i in range(S):
                    vis = min((int(q_pos[b, i]) + 1) // ratio, E)
                    sel = O.topk_select(scores[b, i, :vis].numpy(), k)
                    out[b, i, :len(sel)] = torch.from_numpy(np.asarray(sel, dtype=np.int32))
            return out

        tp.ops = types.SimpleNamespace(indexer_scores=fake_scores, topk=fake_topk)
        dist.init_process_group("gloo", rank=rank, world_size=world)
        wl = WORKLOADS["pro_csa_decode_32k"].scaled(B=2, ctx=2048, topk=64)
        inp = make_inputs(wl, seed=3)  # the same inputs on every rank
        lo, hi = tp.head_shard(wl.H_I, rank, world)
        sel = tp.tp_indexer_topk(inp["pos"], inp["q_idx"][:, :, lo:hi], inp["w"][:, :, lo:hi], inp["idx_cache"],
                                 wl.topk)
        full = fake_topk(inp["pos"], fake_scores(inp["pos"], inp["q_idx"], inp["w"], inp["idx_cache"], 4), wl.topk, 4)
        dist.destroy_process_group()
        q.put((rank, bool(torch.equal(sel, full)), (lo, hi)))
    except Exception as e:  # noqa: BLE001
        q.put((rank, "error", repr(e)))


@pytest.mark.timeout(600)
def test_tensor_parallel_indexer_over_two_gloo_ranks():
    """[P1] "少读 KV 之前，Indexer 仍要给历史打分": each rank scores with half of the indexer heads, the
    partial scores are summed by an all-reduce, and every rank selects the same entries as the
    unsplit indexer."""
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_tp_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        item = q.get(timeout=500)
        res[item[0]] = item
    for p in procs:
        p.join(timeout=60)
    assert res[0][1] != "error", res[0]
    assert res[1][1] != "error", res[1]
    assert res[0][1] is True and res[1][1] is True
    assert res[0][2] == (0, 32) and res[1][2] == (32, 64)


@pytest.mark.timeout(600)
def test_bench_starts_its_own_ranks_without_a_launcher():
    """`python bench.py --gpus 2` without torchrun starts two ranks itself (RANK / WORLD_SIZE set as
    torchrun sets them); rank 0 alone prints one line, which reports both GPUs. The reference arm runs
    here, on the CPU."""
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = {k: v for k, v in os.environ.items() if k not in ("RANK", "WORLD_SIZE", "LOCAL_RANK", "MASTER_PORT")}
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--gpus", "2",
                        "--workload", "pro_hca_decode_32k", "--batch", "2", "--steps", "1", "--warmup", "3"],
                       capture_output=True, text=True, env=env, timeout=500, cwd=root)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [x for x in r.stdout.splitlines() if x.strip()]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["cpu_baseline"]["cores"] >= 1 and line["value"] > 0
