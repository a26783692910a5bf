#!/usr/bin/env python
"""Benchmark of the CSA layer on B200: prints ONE JSON line on rank 0.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Default workload: Pro CSA decode, B=64 requests per GPU at 32K context (8192 compressed entries,
128-token window, 128 heads x 512, indexer 64 x 128, top-k 1024). A step is one fused decode
step of every request through the C ABI (compressor step of the main and index streams + window
write, indexer, top-k, sparse MQA with sink, inverse RoPE). Inputs are synthetic, resident in
HBM, and rotate over several sets whose per-step footprint exceeds the 126 MB L2, so no step is
served from data the previous step left in L2. Multi-GPU runs shard requests (each rank owns its
own B requests; no collective on the data path) and report the whole-job aggregate.

--impl reference times the CPU oracle (the plain float64 reference of the layer) on the host
cores, on a bounded sample of the same workload, as the reference arm.
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

from synth import WORKLOADS, make_inputs  # noqa: E402

METRIC = "CSA decode queries/s @32K ctx B=64; achieved HBM GB/s as % of B200 peak"


# ------------------------------------------------------------------------------ helpers

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return dict(hbm_gbs=float(d["hbm_gbs"]), bf16_tflops=float(d["bf16_tflops"]),
                    bf16_tflops_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0, source="fallback")


def kernel_hash(files):
    """Hash of the kernel's sources with comments and blank space removed: a recorded ncu capture
    stays valid across comment edits and is invalidated by any change to the code."""
    import re
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, "long_context_decode_c4a_b200", "csrc", f), encoding="utf-8") as fh:
            src = fh.read()
        src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
        src = re.sub(r"//[^\n]*", " ", src)
        h.update(" ".join(src.split()).encode())
    return h.hexdigest()[:16]


def traffic_for(kernel: str, workload: str, files):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on the current source."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(f"{kernel}@{workload}")
    if not e or e.get("source_hash") != kernel_hash(files):
        return None
    return e.get("bytes_per_launch")


class ClockSampler:
    """SM clock and clock-event-reason samples taken through NVML (read-only queries) while the
    timed steps run on the device: `poll_until(event)` samples every millisecond until the event
    that closes the timed region has completed."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown", 0x8),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown", 0x40),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown", 0x20),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap", 0x4),
               ("hw_power_brake_slowdown", "nvmlClocksEventReasonHwPowerBrakeSlowdown", 0x80))

    def __init__(self, device_index: int):
        self.nv = None
        self.handle = None
        self.rows = []
        try:
            import pynvml as nv
            nv.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            try:
                self.handle = nv.nvmlDeviceGetHandleByUUID("GPU-" + uuid)
            except Exception:  # noqa: BLE001
                self.handle = nv.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(self.handle, nv.NVML_CLOCK_SM)
            self.nv = nv
        except Exception:  # noqa: BLE001
            self.nv = None

    def sample(self):
        if self.nv is None:
            return
        try:
            mhz = self.nv.nvmlDeviceGetClockInfo(self.handle, self.nv.NVML_CLOCK_SM)
            mask = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
            self.rows.append((mhz, mask))
        except Exception:  # noqa: BLE001
            pass

    def poll_until(self, event, period_s: float = 0.001):
        self.sample()
        while not event.query():
            time.sleep(period_s)
            self.sample()

    def result(self):
        if not self.rows:
            return None
        names = [n for n, attr, bit in self.REASONS
                 if any(m & getattr(self.nv, attr, bit) for _, m in self.rows)]
        return {"sm_mhz": statistics.median(r[0] for r in self.rows), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(names), "samples": len(self.rows), "source": "nvml"}


def dist_setup(n_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------------------ per-step byte / flop ledgers

def graph_rounds(requested: int, steps: int, sets: int) -> int:
    """Rounds of the input-set sequence per CUDA graph: as many as requested, but no more than the
    timed steps hold, so that a graph always serves when there are at least `sets` steps."""
    return max(1, min(requested, steps // max(1, sets)))


def decode_launches(wl) -> int:
    """Kernels one decode step launches, by the library's rules: CSA = indexer (with the compressor
    step) + top-k (one launch up to 16384 entries per row, chunks + merge beyond) + attention; HCA =
    the C128A step + attention; plus the combine kernel when the attention splits each query's
    candidates over several CTA pairs (at most 16, 74 // queries and half the longest list's tiles)."""
    cands = wl.W + (wl.topk if wl.has_indexer else min(wl.max_entries, 2048))
    splits = max(1, min(16, 74 // max(1, wl.B * wl.S), ((cands + 31) // 32) // 2))
    n = 2 + (1 if splits > 1 else 0)
    if wl.has_indexer:
        n += 1 if wl.max_entries <= 16384 else 2
    return n


def decode_bytes(wl):
    """Algorithmic HBM bytes per query of each kernel of one CSA/HCA decode step."""
    E = wl.max_entries
    reads = wl.W + (min(wl.topk, E) if wl.has_indexer else E)
    width = (1 + wl.overlap) * wl.d
    rows = (1 + wl.overlap) * wl.ratio
    out = {}
    # compressor step: state rows (kv + score) read, the token's streams read, state row(s) written,
    # the entry written; window row read + written.
    comp = 2 * rows * width * 2 + 2 * width * 2 + wl.d * 2 + 2 * wl.d * 2
    if wl.has_indexer:
        comp += 2 * 8 * 2 * wl.d_I * 2 + 2 * 2 * wl.d_I * 2 + wl.d_I * 2
        out["indexer"] = E * wl.d_I * 2 + wl.H_I * wl.d_I * 2 + wl.H_I * 4 + E * 4
        out["topk"] = E * 4 + wl.topk * 4
    if wl.has_indexer:
        # The CSA decode step runs the compressor inside the indexer launch: its bytes belong to that launch.
        out["indexer"] += comp
        out["compress"] = 0
    else:
        out["compress"] = comp
    out["attention"] = reads * wl.d * 2 + 2 * wl.H * wl.d * 2 + (wl.topk * 4 if wl.has_indexer else 0)
    return out, reads


# ------------------------------------------------------------------------------ our arm

def step_inputs(inp):
    keys = ["pos", "kv", "score", "idx_kv", "idx_score", "win_kv", "q", "q_idx", "w"]
    return {k: inp[k][:, 0].contiguous() for k in keys if k in inp}


def packed_layout(tensors, align: int = 256):
    """Byte offsets of `tensors` laid end to end, each at a multiple of `align`, and the total size."""
    offs, total = {}, 0
    for k, v in tensors.items():
        offs[k] = total
        total += -(-v.numel() * v.element_size() // align) * align
    return offs, total


def packed_views(flat, tensors, offs):
    """Views of the uint8 buffer `flat` with the dtype and shape of each of `tensors`."""
    return {k: flat[offs[k]:offs[k] + v.numel() * v.element_size()].view(v.dtype).view(v.shape)
            for k, v in tensors.items()}


def run_ours_decode(wl, args, world, rank, light: bool = False):
    from long_context_decode_c4a_b200 import ops
    dev = torch.device("cuda")
    csa = wl.has_indexer
    sets = []
    for s in range(args.sets):
        inp = make_inputs(wl, device="cuda", seed=wl.seed + 1000 * rank + s)
        if csa:
            st = ops.CsaDecodeState(wl.B, wl.max_entries, H=wl.H, d=wl.d, H_I=wl.H_I, d_I=wl.d_I, window=wl.W,
                                    topk=wl.topk, device=dev)
            names = ("state_kv", "state_score", "idx_state_kv", "idx_state_score", "cache", "idx_cache", "ring")
        else:
            st = ops.HcaDecodeState(wl.B, wl.max_entries, H=wl.H, d=wl.d, window=wl.W, ratio=wl.ratio, device=dev)
            names = ("state_kv", "state_score", "cache", "ring")
        for n in names:
            getattr(st, n).copy_(inp[n])
        x = step_inputs(inp)
        x["sink"] = inp["sink"]
        x["out"] = torch.empty(wl.B, wl.H, wl.d, dtype=torch.bfloat16, device=dev)
        sets.append((st, x))
        del inp
    torch.cuda.synchronize()

    preps = []
    for st, x in sets:
        if csa:
            preps.append(st.prepare(x["pos"], x["kv"], x["score"], x["idx_kv"], x["idx_score"], x["win_kv"], x["q"],
                                    x["q_idx"], x["w"], x["sink"], out=x["out"]))
        else:
            preps.append(st.prepare(x["pos"], x["kv"], x["score"], x["win_kv"], x["q"], x["sink"], out=x["out"]))

    def call(i, evs=None):
        preps[i % len(preps)].launch(stage_events=evs)

    nstage = 5 if csa else 3
    # NVML is opened before the warm-up: its start-up (tens of ms) must not leave the GPU idle, and
    # its clocks low, just before the timed region.
    clocks = ClockSampler(torch.cuda.current_device())
    for i in range(args.warmup):
        call(i)
    torch.cuda.synchronize()
    # One CUDA graph holds `reps` rounds of one step of every input set (the launches keep their
    # programmatic dependencies, which a graph boundary ends); the timed region replays it and
    # launches any remaining steps directly.
    graph = None
    reps = graph_rounds(getattr(args, "graph_reps", 1), args.steps, len(preps))
    per_graph = reps * len(preps)
    if args.graph:
        side = torch.cuda.Stream()
        side.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(side):
            for i in range(len(preps)):
                call(i)
        torch.cuda.current_stream().wait_stream(side)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for i in range(per_graph):
                call(i % len(preps))
        torch.cuda.synchronize()
        # Warm replays right before the timed region (at least 2, and at least `warmup` steps), so the
        # timed steps start on a busy GPU at its running clocks.
        for _ in range(max(2, -(-args.warmup // per_graph))):
            graph.replay()
    else:
        for i in range(args.warmup):
            call(i)
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    # Every timed step is enqueued before the first clock sample: an NVML query takes milliseconds
    # of host time, and one taken between launches would leave the device idle inside the timed
    # region. The samples are taken while the queued steps drain.
    t0.record()
    k = 0
    if graph is not None:
        while k + per_graph <= args.steps:
            graph.replay()
            k += per_graph
    for kk in range(k, args.steps):
        call(kk)
    t1.record()
    clocks.poll_until(t1)
    torch.cuda.synchronize()
    barrier(world)
    clk = clocks.result()
    ms = t0.elapsed_time(t1) / args.steps
    ms = max_over_ranks(ms, world)
    del graph
    for st, _ in sets:
        status = ops.device_status(st.ws)
        if status != 0:
            raise RuntimeError(f"device status {status} after the timed steps")

    # ---- per-kernel durations: the same steps again with CUDA events recorded between the kernels
    # on the launching stream (an event between two kernels also ends their launch overlap, so
    # these steps run separately from the timed ones above)
    stage_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(nstage)] for _ in range(args.steps)]
    for row in stage_ev:       # create the underlying events before the loop
        for e in row:
            e.record()
    torch.cuda.synchronize()
    for k in range(args.steps):
        call(k, evs=stage_ev[k])
    torch.cuda.synchronize()
    stage_names = ["compress", "indexer", "topk", "attention"] if csa else ["compress", "attention"]
    stage_ms = {n: statistics.mean(stage_ev[k][i].elapsed_time(stage_ev[k][i + 1]) for k in range(args.steps))
                for i, n in enumerate(stage_names)}

    launches_per_step = decode_launches(wl)
    # ---- single-step latency: one step per replay of a one-step CUDA graph, the device idle before
    # it (synchronised between steps), events on the launching stream. This is what one decode step
    # of this layer costs on its own, without the overlap of consecutive steps' launches.
    one = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        call(0)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    with torch.cuda.graph(one):
        call(0)
    lat = []
    for k in range(max(8, min(args.steps, 50)) + 3):
        torch.cuda.synchronize()
        a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        one.replay()
        z.record()
        torch.cuda.synchronize()
        if k >= 3:
            lat.append(a.elapsed_time(z))
    single_ms = max_over_ranks(statistics.median(lat), world)
    del one
    if light:
        return dict(ms=ms, stage_ms=stage_ms, clocks=clk, launches=launches_per_step * args.steps,
                    single_ms=single_ms)
    # ---- end-to-end through the public API with host buffers: every step copies its inputs from
    # pinned host memory, runs, and copies its output back. Copies run on their own streams and
    # overlap the neighbouring steps' compute (two device buffer sets, events between streams).
    # A step's inputs sit in one pinned host buffer (each at a 256-byte offset) and reach the device
    # in one copy, into views of one device buffer that the prepared step reads.
    st, x = sets[0]
    inputs = {k: v for k, v in x.items() if k not in ("out", "sink")}
    offs, total = packed_layout(inputs)
    host_flat = torch.empty(total, dtype=torch.uint8).pin_memory()
    for k, v in packed_views(host_flat, inputs, offs).items():
        v.copy_(inputs[k])
    out_host = [torch.empty(x["out"].shape, dtype=x["out"].dtype).pin_memory() for _ in range(2)]
    h2d = total
    d2h = out_host[0].numel() * out_host[0].element_size()
    dev_flat = [torch.empty(total, dtype=torch.uint8, device=dev) for _ in range(2)]
    dev_in = [packed_views(f, inputs, offs) for f in dev_flat]
    dev_out = [torch.empty_like(x["out"]) for _ in range(2)]
    e2e_preps = []   # [buffer][input set]
    for buf in range(2):
        row = []
        for stt, xx in sets:
            xin = dict(xx)
            xin.update(dev_in[buf])
            if csa:
                row.append(stt.prepare(xin["pos"], xin["kv"], xin["score"], xin["idx_kv"], xin["idx_score"],
                                       xin["win_kv"], xin["q"], xin["q_idx"], xin["w"], xin["sink"],
                                       out=dev_out[buf]))
            else:
                row.append(stt.prepare(xin["pos"], xin["kv"], xin["score"], xin["win_kv"], xin["q"], xin["sink"],
                                       out=dev_out[buf]))
        e2e_preps.append(row)
    comp = torch.cuda.current_stream()
    s_h2d, s_d2h = torch.cuda.Stream(), torch.cuda.Stream()
    h2d_done = [torch.cuda.Event() for _ in range(2)]
    comp_done = [torch.cuda.Event() for _ in range(2)]
    d2h_done = [torch.cuda.Event() for _ in range(2)]
    for e in comp_done + d2h_done:
        e.record(comp)

    def e2e_step(i):
        buf = i % 2
        s_h2d.wait_event(comp_done[buf])          # step i-2 finished reading dev_in[buf]
        with torch.cuda.stream(s_h2d):
            dev_flat[buf].copy_(host_flat, non_blocking=True)
            h2d_done[buf].record(s_h2d)
        comp.wait_event(h2d_done[buf])
        comp.wait_event(d2h_done[buf])             # step i-2's output was copied out of dev_out[buf]
        e2e_preps[buf][i % len(sets)].launch()
        comp_done[buf].record(comp)
        s_d2h.wait_event(comp_done[buf])
        with torch.cuda.stream(s_d2h):
            out_host[buf].copy_(dev_out[buf], non_blocking=True)
            d2h_done[buf].record(s_d2h)

    for i in range(args.warmup):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_h2d)
    for k in range(args.steps):
        e2e_step(k)
    s_h2d.wait_stream(s_d2h)
    e1.record(s_h2d)
    torch.cuda.synchronize()
    barrier(world)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / args.steps, world)
    return dict(ms=ms, stage_ms=stage_ms, clocks=clk, e2e_ms=e2e_ms, h2d=h2d, d2h=d2h,
                launches=launches_per_step * args.steps, single_ms=single_ms)


def prefill_ledger(wl):
    """Algorithmic tensor FLOPs of one prefill pass: attention 4*H*reads*d per query (the pages'
    analytic count) plus, for CSA, the indexer's 2*H_I*d_I per (query, visible entry). HCA reads
    every visible entry and has no indexer."""
    attn = idx = 0
    for t in range(wl.S):
        vis = min((t + 1) // wl.ratio, wl.max_entries)   # entries visible to query t
        sel = min(wl.topk, vis) if wl.has_indexer else vis
        reads = min(wl.W, t + 1) + sel                    # window rows + selected (or all visible) entries
        attn += 4 * wl.H * reads * wl.d
        if wl.has_indexer:
            idx += 2 * wl.H_I * wl.d_I * vis
    return attn, idx


def run_prefill(wl, steps: int, warmup: int):
    """One prefill pass over S tokens from an empty cache, through the C ABI. CSA: both compressor
    streams (C4A), indexer + top-k, sparse attention. HCA: the C128A stream and attention over every
    visible entry. Returns ms per pass and per stage."""
    from long_context_decode_c4a_b200 import ops
    dev = "cuda"
    inp = make_inputs(wl, device=dev)
    B, S, d, dI, E = wl.B, wl.S, wl.d, wl.d_I, wl.max_entries
    csa = wl.has_indexer
    rows = (1 + wl.overlap) * wl.ratio
    main_cfg = ops.compressor_cfg(wl.ratio, d)
    skv = torch.empty(B, rows, (1 + wl.overlap) * d, dtype=torch.bfloat16, device=dev)
    ssc = torch.empty_like(skv)
    cache = torch.zeros(B, E, d, dtype=torch.bfloat16, device=dev)
    start = torch.zeros(B, dtype=torch.int32, device=dev)
    out = torch.empty(B, S, wl.H, d, dtype=torch.bfloat16, device=dev)
    if csa:
        idx_cfg = ops.compressor_cfg(4, dI)
        ikv = torch.empty(B, 8, 2 * dI, dtype=torch.bfloat16, device=dev)
        isc = torch.empty_like(ikv)
        icache = torch.zeros(B, E, dI, dtype=torch.bfloat16, device=dev)
        topk = torch.empty(B, S, wl.topk, dtype=torch.int32, device=dev)
        ws_i = ops.workspace(ops._lib.CSA_WS_INDEXER_TOPK, B, S, E, wl.topk, dev)
        ws_a = ops.workspace(ops._lib.CSA_WS_SPARSE_ATTN, B, S, E, wl.topk, dev)
        wss = (ws_i, ws_a)
    else:
        ws_a = ops.workspace(ops._lib.CSA_WS_HCA_ATTN, B, S, 1, 1, dev)
        wss = (ws_a,)

    def one(evs=None):
        if evs:
            evs[0].record()
        ops.state_reset(main_cfg, skv, ssc)
        ops.compress(main_cfg, start, inp["kv"], inp["score"], inp["gamma"], skv, ssc, cache)
        if csa:
            ops.state_reset(idx_cfg, ikv, isc)
            ops.compress(idx_cfg, start, inp["idx_kv"], inp["idx_score"], inp["idx_gamma"], ikv, isc, icache)
        if evs:
            evs[1].record()
        if csa:
            ops.indexer_topk(inp["pos"], inp["q_idx"], inp["w"], icache, wl.topk, topk_idx=topk, ws=ws_i)
        if evs:
            evs[2].record()
        if csa:
            ops.sparse_attn(inp["pos"], inp["q"], inp["win_kv"], cache, topk, inp["sink"], wl.W, out=out, ws=ws_a)
        else:
            ops.hca_attn(inp["pos"], inp["q"], inp["win_kv"], cache, inp["sink"], wl.W, ratio=wl.ratio, out=out, ws=ws_a)
        if evs:
            evs[3].record()

    for _ in range(warmup):
        one()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(steps)]
    for k in range(steps):
        one(evs[k])
    torch.cuda.synchronize()
    for w in wss:
        if ops.device_status(w) != 0:
            raise RuntimeError("device status after the prefill passes")
    per = lambda i, j: statistics.mean(e[i].elapsed_time(e[j]) for e in evs)
    stages = {"compress": per(0, 1), "attention": per(2, 3)}
    if csa:
        stages["indexer_topk"] = per(1, 2)
    return dict(ms=per(0, 3), stage_ms=stages)


def run_output_projection(M: int, steps: int, warmup: int):
    """The grouped output projection on M rows of the Pro shapes through the C ABI (two GEMM launches,
    plus a zeroing launch when the second contraction is split over K). Returns ms per call."""
    from long_context_decode_c4a_b200 import ops
    from synth.workloads import make_oproj_inputs
    inp = make_oproj_inputs(M, device="cuda")
    G, R, Kg = inp["wo_a"].shape
    D = inp["wo_b"].shape[0]
    r = torch.empty(M, G * R, dtype=torch.bfloat16, device="cuda")
    y = torch.empty(M, D, dtype=torch.float32, device="cuda")
    ws = ops.workspace(ops._lib.CSA_WS_OUTPUT_PROJ, 1, 1, 1, 1, "cuda")
    for _ in range(warmup):
        ops.output_projection(inp["o"], inp["wo_a"], inp["wo_b"], r, y, ws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        ops.output_projection(inp["o"], inp["wo_a"], inp["wo_b"], r, y, ws)
    e1.record()
    torch.cuda.synchronize()
    if ops.device_status(ws) != 0:
        raise RuntimeError("device status after the output projection")
    ms = e0.elapsed_time(e1) / steps
    weights = (G * R * Kg + D * G * R) * 2
    traffic = weights + M * G * Kg * 2 + 2 * M * G * R * 2 + M * D * 4
    flops = 2 * M * (G * R * Kg + D * G * R)
    del inp, r, y
    return ms, traffic, flops


def run_q_path(M: int, steps: int, warmup: int):
    """The low-rank query path on M tokens of the Pro shapes through the C ABI (two GEMMs, the row
    RMSNorm and the per-head norm with RoPE). Returns ms per call, algorithmic bytes and FLOPs."""
    from long_context_decode_c4a_b200 import ops
    from synth.workloads import make_qpath_inputs
    inp = make_qpath_inputs(M, device="cuda")
    hidden, q_rank, H = inp["x"].shape[1], inp["wq_a"].shape[0], inp["wq_b"].shape[0] // 512
    q = torch.empty(M, H, 512, dtype=torch.bfloat16, device="cuda")
    ws = ops.workspace(ops._lib.CSA_WS_Q_PROJ, 1, 1, 1, 1, "cuda")
    call = lambda: ops.q_projection(inp["x"], inp["wq_a"], inp["gamma_q"], inp["wq_b"], inp["pos"], H=H, q=q, ws=ws)
    for _ in range(warmup):
        call()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        call()
    e1.record()
    torch.cuda.synchronize()
    if ops.device_status(ws) != 0:
        raise RuntimeError("device status after the query path")
    ms = e0.elapsed_time(e1) / steps
    weights = (q_rank * hidden + H * 512 * q_rank) * 2
    traffic = weights + M * hidden * 2 + 2 * M * q_rank * (4 + 2) + 2 * M * H * 512 * 2
    flops = 2 * M * (q_rank * hidden + H * 512 * q_rank)
    del inp, q
    return ms, traffic, flops


def extra_workloads(args, peaks):
    """Short measurements of the other synthetic configurations (one GPU, same process)."""
    res = {}
    for name in ("pro_hca_decode_32k", "long_csa_decode_1m"):
        wl = WORKLOADS[name]
        a = argparse.Namespace(**vars(args))
        a.steps, a.warmup, a.sets = 20, 3, 2 if name == "long_csa_decode_1m" else args.sets
        r = run_ours_decode(wl, a, 1, 0, light=True)
        per_q, reads = decode_bytes(wl)
        total = sum(per_q.values()) * wl.B
        res[name] = {"value": wl.B * 1000.0 / r["ms"], "unit": "queries/s", "tokens_per_s": wl.B * 1000.0 / r["ms"],
                     "ms_per_step": r["ms"], "single_step_latency_us": r["single_ms"] * 1e3,
                     "kernels_ms": r["stage_ms"], "reads_per_query": reads,
                     "roofline": {"bound": "hbm", "achieved": total / (r["ms"] * 1e-3) / 1e9, "peak": peaks["hbm_gbs"],
                                  "unit": "GB/s", "frac": total / (r["ms"] * 1e-3) / 1e9 / peaks["hbm_gbs"],
                                  "scope": "whole step, algorithmic bytes"}}
        torch.cuda.empty_cache()
    for name, steps in (("csa_prefill_8k", 3), ("hca_prefill_8k", 3), ("tiny_csa_prefill", 20)):
        wl = WORKLOADS[name]
        r = run_prefill(wl, steps, 3)
        attn_f, idx_f = prefill_ledger(wl)
        tf = (attn_f + idx_f) / (r["ms"] * 1e-3) / 1e12
        res[name] = {"value": wl.B * wl.S * 1000.0 / r["ms"], "unit": "tokens/s", "ms_per_step": r["ms"],
                     "kernels_ms": r["stage_ms"],
                     "roofline": {"bound": "tensor", "achieved": tf, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                                  "frac": tf / peaks["bf16_tflops"], "flops_per_pass": attn_f + idx_f,
                                  "scope": "whole pass, algorithmic FLOPs (attention 4*H*reads*d + CSA indexer)"}}
        torch.cuda.empty_cache()
    # The projections around the path: the low-rank query path before it ([P1] "低秩 Q", 106.5 Mi
    # weights) and the grouped output projection after it ([P1] "输出投影也分组", 176 Mi). Decode rows
    # stream the weights (HBM-bound); prefill rows are dense contractions (tensor-bound).
    for name, M, steps, fn in (("q_path_decode_b64", 64, 20, run_q_path), ("q_path_prefill_8k", 8192, 3, run_q_path),
                               ("output_projection_decode_b64", 64, 20, run_output_projection),
                               ("output_projection_prefill_8k", 8192, 3, run_output_projection)):
        ms, traffic, flops = fn(M, steps, 3)
        if M <= 256:
            ach = traffic / (ms * 1e-3) / 1e9
            roof = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                    "frac": ach / peaks["hbm_gbs"], "bytes_per_call": traffic,
                    "scope": "weights + inputs + intermediates (written and read) + outputs, algorithmic bytes"}
        else:
            ach = flops / (ms * 1e-3) / 1e12
            roof = {"bound": "tensor", "achieved": ach, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                    "frac": ach / peaks["bf16_tflops"], "flops_per_call": flops,
                    "scope": "2 x rows x weights (both contractions)"}
        shape = ("hidden 7168 -> q_rank 1536 -> 128 heads x 512" if fn is run_q_path
                 else "G=16 groups x Kg=4096 -> R=1024, then 16384 -> D=7168")
        res[name] = {"value": M * 1000.0 / ms, "unit": "rows/s", "ms_per_step": ms, "rows": M, "shape": shape,
                     "roofline": roof}
        torch.cuda.empty_cache()
    return res


def _oracle_requests(job):
    """One worker of the CPU oracle's timing (a spawned process with one BLAS thread): draws each
    request of its seed list untimed, then times the oracle's decode step on it. Returns the summed
    seconds of the timed steps."""
    wl, seeds = job
    from threadpoolctl import threadpool_limits

    from oracle import csa_oracle as O
    secs = 0.0
    with threadpool_limits(1):
        for s in seeds:
            inp = O.to_numpy_inputs(make_inputs(wl, seed=s))
            t = time.perf_counter()
            if wl.has_indexer:
                O.csa_decode_request(inp, 0, H=wl.H, d=wl.d, W=wl.W, topk=wl.topk)
            else:
                O.hca_decode_request(inp, 0, H=wl.H, d=wl.d, W=wl.W, ratio=wl.ratio)
            secs += time.perf_counter() - t
    return secs


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # not every platform has an affinity mask
        return os.cpu_count() or 1


class OracleTimer:
    """The CPU oracle timed on the host cores: independent requests (each drawn with its own seed at
    the workload's shapes) are spread over one spawned worker process per core, each with one BLAS
    thread. A batch's time is its makespan: the largest of the workers' summed oracle seconds (the
    draws of the inputs are not timed)."""

    def __init__(self, wl, cores: int):
        import multiprocessing
        self.wl = wl.scaled(B=1)
        self.cores = max(1, cores)
        self.pool = multiprocessing.get_context("spawn").Pool(self.cores)

    def time_requests(self, seeds) -> float:
        jobs = [(self.wl, list(seeds[i::self.cores])) for i in range(self.cores) if seeds[i::self.cores]]
        return max(self.pool.map(_oracle_requests, jobs, chunksize=1))

    def close(self):
        self.pool.terminate()
        self.pool.join()


def cpu_baseline_decode(wl, budget_s: float = 12.0):
    """The oracle on a bounded sample of the workload: whole batches of wl.B requests, as many as fit
    in about budget_s seconds of CPU work spread over the host cores."""
    cores = min(host_cores(), wl.B)
    timer = OracleTimer(wl, cores)
    try:
        one = timer.time_requests([1])
        rounds = int(max(1, min(8, budget_s / max(one * wl.B, 1e-3))))
        seeds = list(range(10, 10 + rounds * wl.B))
        secs = timer.time_requests(seeds)
    finally:
        timer.close()
    return {"value": len(seeds) / secs, "unit": "queries/s", "cores": cores, "kind": "oracle",
            "sample": f"{rounds} x {wl.B} requests of {wl.name} (each drawn with its own seed), float64 numpy "
                      f"oracle, one worker process per core with one BLAS thread; makespan of the oracle's time"}


# ------------------------------------------------------------------------------ main

def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default="pro_csa_decode_32k", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--sets", type=int, default=4, help="rotating input sets")
    ap.add_argument("--batch", type=int, default=0, help="requests per GPU (default: the workload's)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="skip the short runs of the other configurations")
    ap.add_argument("--graph-reps", type=int, default=10,
                    help="rounds of the input-set sequence captured in one CUDA graph (a graph boundary "
                         "ends the programmatic overlap of consecutive launches)")
    ap.add_argument("--no-graph", dest="graph", action="store_false",
                    help="launch every timed step from the host instead of replaying a CUDA graph")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    wl = WORKLOADS[args.workload]
    if args.batch:
        wl = wl.scaled(B=args.batch)
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # Started without a launcher: start the N ranks here, as torchrun would.
        return spawn_ranks(args.gpus, sys.argv[1:] if argv is None else list(argv))
    if args.impl == "reference":
        if not wl.is_decode:
            ap.error("the reference arm times the decode workloads")
        return run_reference(wl, args)

    world, rank, local = dist_setup(args.gpus)
    if not wl.is_decode:
        return run_prefill_line(wl, args, world, rank)
    r = run_ours_decode(wl, args, world, rank)
    peaks = load_peaks()
    per_q, reads = decode_bytes(wl)
    B_total = wl.B * world
    value = B_total * 1000.0 / r["ms"]
    # dominant kernel (largest share of the step) and its roofline
    dom = max(("indexer", "attention") if wl.has_indexer else ("attention",), key=lambda n: r["stage_ms"][n])
    bytes_launch = per_q[dom] * wl.B
    achieved = bytes_launch / (r["stage_ms"][dom] * 1e-3) / 1e9
    files = {"indexer": ["indexer.cu", "compress_decode.cuh", "ptx.cuh", "kernels.cuh"],
             "attention": ["attn.cu", "ptx.cuh", "kernels.cuh", "rope.cuh"]}[dom]
    total_bytes = sum(per_q.values()) * wl.B
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "queries/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": r["ms"],
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": wl.name, "global_batch": B_total, "requests_per_gpu": wl.B, "context": wl.ctx,
                   "compressed_entries": wl.max_entries, "window": wl.W, "heads": wl.H, "head_dim": wl.d,
                   "indexer_heads": wl.H_I, "topk": wl.topk, "reads_per_query": reads,
                   "parallelism": f"requests sharded over {world} GPU(s), no data-path collective",
                   "l2": f"{args.sets} rotating input sets, each step reads {total_bytes / 1e6:.0f} MB > 126 MB L2",
                   "launch": ("CUDA graph of one step per input set, replayed" if args.graph
                              else "every step launched from the host")},
        "tokens_per_s": value,
        "step_hbm_gbs": total_bytes / (r["ms"] * 1e-3) / 1e9,
        "step_hbm_frac": total_bytes / (r["ms"] * 1e-3) / 1e9 / peaks["hbm_gbs"],
        "kernels_ms": r["stage_ms"],
        "roofline": {"kernel": dom, "bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "peak_source": peaks["source"],
                     "traffic": traffic_for(dom, wl.name, files),
                     "algorithmic_bytes_per_launch": bytes_launch},
        "e2e": {"value": B_total * 1000.0 / r["e2e_ms"], "unit": "queries/s", "h2d_bytes_per_step": r["h2d"],
                "d2h_bytes_per_step": r["d2h"]},
        "gpu_launches": r["launches"],
        "single_step": {"latency_us": r["single_ms"] * 1e3,
                        "how": "one step per replay of a one-step CUDA graph, synchronised between steps "
                               "(no overlap with neighbouring steps); median, CUDA events on the launching stream"},
        "clocks": r["clocks"],
    }
    if world == 1 and not args.no_extra:
        line["workloads"] = extra_workloads(args, peaks)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline_decode(wl)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def spawn_ranks(n: int, argv) -> int:
    """Run this script as n ranks on this node (RANK, LOCAL_RANK, WORLD_SIZE and the rendezvous address
    set as torchrun sets them); rank 0 prints the JSON line. Returns the largest exit code."""
    import socket
    import subprocess
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    procs = []
    for r in range(n):
        env = dict(os.environ, RANK=str(r), LOCAL_RANK=str(r), WORLD_SIZE=str(n), LOCAL_WORLD_SIZE=str(n),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        procs.append(subprocess.Popen([sys.executable, os.path.abspath(__file__)] + list(argv), env=env))
    return max(p.wait() for p in procs)


def run_prefill_line(wl, args, world, rank) -> int:
    """A prefill workload: every rank runs the whole pass on its own GPU (replicas, no collective); the
    line reports tokens/s over all ranks and the pass's algorithmic tensor FLOPs against the measured
    dense bf16 peak."""
    peaks = load_peaks()
    r = run_prefill(wl, args.steps, args.warmup)
    ms = max_over_ranks(r["ms"], world)
    attn_f, idx_f = prefill_ledger(wl)
    tf = (attn_f + idx_f) / (ms * 1e-3) / 1e12
    line = {
        "metric": f"{'CSA' if wl.has_indexer else 'HCA'} prefill tokens/s @{wl.S} tokens; achieved TFLOP/s as % of "
                  f"B200 dense bf16 peak",
        "value": world * wl.B * wl.S * 1000.0 / ms, "unit": "tokens/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": wl.name, "requests_per_gpu": wl.B, "tokens": wl.S, "heads": wl.H, "head_dim": wl.d,
                   "window": wl.W, "topk": wl.topk, "parallelism": f"{world} replica(s), no data-path collective"},
        "kernels_ms": r["stage_ms"],
        "roofline": {"bound": "tensor", "achieved": tf, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": tf / peaks["bf16_tflops"], "peak_source": peaks["source"],
                     "flops_per_pass": attn_f + idx_f},
    }
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def run_reference(wl, args):
    """The reference arm: the CPU oracle as it stands, rank 0 only, on the host cores; every step is a
    bounded sample of the workload's requests."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if rank != 0:
        return 0
    cores = min(host_cores(), wl.B)
    timer = OracleTimer(wl, cores)
    try:
        one = timer.time_requests([1])
        per_step = max(1, min(wl.B, int(cores * 2.0 / max(one, 1e-3))))
        total_steps = args.warmup + args.steps
        while per_step > 1 and total_steps * per_step * one / cores > 150:
            per_step //= 2
        for i in range(args.warmup):
            timer.time_requests(list(range(1000 + i * per_step, 1000 + (i + 1) * per_step)))
        secs = [timer.time_requests(list(range(5000 + k * per_step, 5000 + (k + 1) * per_step)))
                for k in range(args.steps)]
    finally:
        timer.close()
    value = per_step * args.steps / sum(secs)
    line = {
        "metric": METRIC, "value": value, "unit": "queries/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": 1000.0 * sum(secs) / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
        "config": {"workload": wl.name, "global_batch": wl.B, "requests_per_gpu": wl.B, "context": wl.ctx,
                   "sample_requests_per_step": per_step},
        "cpu_baseline": {"value": value, "unit": "queries/s", "cores": cores, "kind": "oracle",
                         "sample": f"{per_step} requests of {wl.name} per step (each drawn with its own seed), "
                                   f"float64 numpy oracle, one worker process per core with one BLAS thread"},
        "e2e": {"value": value, "unit": "queries/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
