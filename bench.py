"""Benchmark of the paged decode-attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

One step is one layer's decode step of the named workload, through the
library's C ABI: copy-on-write block copies (workloads that have them), the
cache write of each sequence's new token, then paged decode attention.
Inputs are seeded synthetic tensors resident in HBM; L2 is flushed before
every timed step, outside the step's events: a 256 MiB write, then a 256 MiB
read of another buffer, so that the write's dirty lines are written back
during the flush (the decode after a write-only flush is reported too).

Printed (rank 0, one JSON line): KV-read GB/s of the whole step (``value``),
% of the measured HBM peak, sequences/s, the decode launch's roofline
fraction, the end-to-end figure through the same API with host buffers, the
fp64 CPU oracle's throughput on a bounded sample, SM clocks sampled during the
timed region, and a few secondary workloads.

N > 1 (torchrun, one process per GPU): every rank runs its own replica of the
workload (weak scaling, no collective on the data path); timings are the max
over ranks.  ``--impl reference`` times the CPU oracle instead (rank 0 only).
"""

from __future__ import annotations

import argparse
import json
import os
import shutil
import statistics
import subprocess
import tempfile
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged decode attention: achieved KV-read HBM GB/s (% of peak), seq/s"
# Layers of one model step in the layer rotation: the decode's plan is made once per this many layers
# (the first runs pa_decode, the others pa_decode_planned), as a serving engine plans once per step.  28 is the layer count
# of Qwen2.5-7B, whose attention shape (28 query heads, 4 KV heads, head_dim 128) the workloads use.
MODEL_LAYERS = 28
FALLBACK_HBM_GBS = 6650.0


def kernel_source_hash() -> str:
    """Hash of the device code the profiles were taken on.

    The device part of csrc/decode.cu (up to its host-side section) and
    csrc/pa_common.cuh: host-side launch choices do not change the kernels.
    """
    import hashlib

    csrc = os.path.join(ROOT, "paged_kv_cache_362_b200", "csrc")
    dec = open(os.path.join(csrc, "decode.cu"), "rb").read()
    dec = dec.split(b"\n// host side\n")[0]
    common = open(os.path.join(csrc, "pa_common.cuh"), "rb").read()
    return hashlib.sha256(dec + common).hexdigest()[:16]


def profiled_traffic(workload: str):
    """DRAM bytes per launch of the attention kernel from the committed ncu capture.

    profiles/traffic.json records the capture together with a hash of the
    device code it was taken on; a changed kernel gets null, not a stale number.
    """
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            t = json.load(f)
        if kernel_source_hash() != t["source_sha256_16"]:
            return None
        return t[workload]["decode_tc_kernel_bytes"]
    except Exception:
        return None


def measured_hbm_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------
def dist_setup(n_gpus):
    import torch

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return rank, world


def dist_max(x: float) -> float:
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()):
        return x
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def aggregate(kv_bytes_local: int, ms_local: float):
    """Whole-job KV GB/s of a weak-scaling replica run and the max-over-ranks step time (ms).

    Every rank processes its own replica; the job's throughput is the bytes all
    ranks read divided by the slowest rank's step time.
    """
    import torch.distributed as dist

    world = dist.get_world_size() if (dist.is_available() and dist.is_initialized()) else 1
    ms = dist_max(ms_local)
    total = dist_sum(float(kv_bytes_local))
    return total / (ms * 1e-3) / 1e9, ms, world


def dist_sum(x: float) -> float:
    import torch
    import torch.distributed as dist

    if not (dist.is_available() and dist.is_initialized()):
        return x
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def dist_barrier():
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized():
        dist.barrier()


def dist_done():
    import torch.distributed as dist

    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.proc = None
        self.path = os.path.join(tempfile.gettempdir(), f"pa_bench_clocks_gpu{gpu_index}_{os.getpid()}.csv")
        exe = shutil.which("nvidia-smi")
        if exe is None:
            return
        self.f = open(self.path, "w")
        self.proc = subprocess.Popen([exe, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                      "-i", str(gpu_index), "-lms", "50"], stdout=self.f,
                                     stderr=subprocess.DEVNULL)

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        try:
            os.remove(self.path)
        except OSError:
            pass
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
# workload on the device
# ---------------------------------------------------------------------------
class DeviceWorkload:
    def __init__(self, name: str, seed: int, partition_size: int | None = None, placement: str | None = None,
                 block_size: int | None = None, layers: int = 1):
        import torch

        import paged_kv_cache_362_b200 as pa
        from workloads import build_workload, device_values, get_config

        self.pa = pa
        self.cfg = get_config(name)
        if block_size is not None and block_size != self.cfg.block_size:
            # the same sequences in blocks of another size; the pool keeps its token capacity
            self.cfg = get_config(name, block_size=block_size,
                                  num_blocks=self.cfg.num_blocks * self.cfg.block_size // block_size)
        self.wl = build_workload(self.cfg, seed=seed, placement=placement)
        self.P = self.cfg.partition_size if partition_size is None else partition_size
        dev = torch.device("cuda")
        v = device_values(self.wl, dev)
        self.q, self.key, self.value = v["q"], v["key"], v["value"]
        self.kc, self.vc = v["key_cache"], v["value_cache"]
        # one K/V pool per model layer; block tables, context lengths and q are
        # shared by the layers of a step, as in a serving engine
        self.kcs = [self.kc] + [self.kc.clone() for _ in range(layers - 1)]
        self.vcs = [self.vc] + [self.vc.clone() for _ in range(layers - 1)]
        self.layers = layers
        wl = self.wl
        self.bt = torch.from_numpy(wl.block_tables).to(dev)
        self.cl = torch.from_numpy(wl.context_lens).to(dev)
        self.slots = torch.from_numpy(wl.slot_mapping).to(dev)
        self.pairs = torch.from_numpy(np.ascontiguousarray(wl.copy_pairs)).to(dev)
        self.has_copy = wl.copy_pairs.shape[0] > 0
        c = self.cfg
        self.max_ctx = wl.max_context_len
        self.ws = pa.make_workspace(wl.num_seqs, c.num_heads, c.num_kv_heads, c.head_dim, self.max_ctx, self.P)
        self.out = torch.empty_like(self.q)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.kv_bytes = wl.kv_bytes()
        # copy_blocks (when the step forks), reshape_and_cache, and the kernels pa_decode enqueues
        self.decode_launches = pa.decode_launch_count(wl.num_seqs, c.num_heads, c.num_kv_heads, c.head_dim,
                                                      self.max_ctx, self.P, c.dtype)
        self.launches_per_step = (1 if self.has_copy else 0) + 1 + self.decode_launches
        # with a plan made once per step of the model (pa_decode_plan) and one planned decode per layer
        self.planned_launches = pa.decode_launch_count(wl.num_seqs, c.num_heads, c.num_kv_heads, c.head_dim,
                                                       self.max_ctx, self.P, c.dtype, planned=True)

    def pre(self, layer: int = 0):
        kc, vc = self.kcs[layer], self.vcs[layer]
        if self.has_copy:
            self.pa.copy_blocks(kc, vc, self.pairs, status=self.status)
        self.pa.reshape_and_cache(self.key, self.value, kc, vc, self.slots, status=self.status)

    def decode(self, layer: int = 0, planned: bool = False):
        c = self.cfg
        self.pa.decode(self.out, self.q, self.kcs[layer], self.vcs[layer], self.bt, self.cl, c.scale, self.max_ctx,
                       self.ws, partition_size=self.P, status=self.status, planned=planned)

    def layer_decode(self, layer: int):
        """Decode of model layer ``layer`` (on pool layer mod the pools): the step's first layer runs pa_decode,
        which leaves its plan in the workspace, and the step's other layers decode with that plan."""
        self.decode(layer % self.layers, planned=layer % MODEL_LAYERS != 0)


def unique_kv_bytes(wl) -> int:
    """K/V bytes of the distinct physical blocks a decode step reads (shared blocks once)."""
    c = wl.cfg
    bs = c.block_size
    seen = {}
    for b in range(wl.num_seqs):
        n = int(wl.context_lens[b])
        for j in range(-(-n // bs)):
            blk = int(wl.block_tables[b, j])
            seen[blk] = max(seen.get(blk, 0), min(bs, n - bs * j))
    elt = {"f32": 4, "f16": 2, "bf16": 2}[c.dtype]
    return sum(seen.values()) * c.num_kv_heads * c.head_dim * 2 * elt


def pct3(xs):
    return [round(float(v), 5) for v in np.percentile(np.asarray(xs), [10, 50, 90])]


def time_steps(w: DeviceWorkload, steps: int, warmup: int, flush, use_graph: bool):
    """Per-step CUDA-event times (ms): the whole step, and the decode alone.

    With graphs, a step is one CUDA graph (the block copies and the append,
    then the decode, chained by programmatic dependent launch), as a serving
    loop captures it.  The decode alone is timed in a second pass: its own
    graph, after an untimed append.  Each pass times ``steps`` steps with an
    L2 flush before each, bracketed by a synchronize and a barrier.
    """
    import torch

    stream = torch.cuda.current_stream()
    graph_step = graph_pre = graph_dec = None
    if use_graph:
        for _ in range(3):
            w.pre()
            w.decode()
        torch.cuda.synchronize()
        s = torch.cuda.Stream()
        s.wait_stream(stream)
        with torch.cuda.stream(s):
            graph_step = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph_step, stream=s):
                w.pre()
                w.decode()
            graph_pre = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph_pre, stream=s):
                w.pre()
            graph_dec = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph_dec, stream=s):
                w.decode()
        stream.wait_stream(s)
        torch.cuda.synchronize()

    def run_step():
        if graph_step is not None:
            graph_step.replay()
        else:
            w.pre()
            w.decode()

    def run_pre():
        graph_pre.replay() if graph_pre is not None else w.pre()

    def run_dec():
        graph_dec.replay() if graph_dec is not None else w.decode()

    for _ in range(max(warmup, 3)):
        flush()
        run_step()
    torch.cuda.synchronize()
    dist_barrier()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for e0, e1 in ev:
        flush()
        e0.record(stream)
        run_step()
        e1.record(stream)
    torch.cuda.synchronize()
    dist_barrier()
    step_ms = [e0.elapsed_time(e1) for e0, e1 in ev]
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for e0, e1 in ev:
        flush()
        run_pre()
        e0.record(stream)
        run_dec()
        e1.record(stream)
    torch.cuda.synchronize()
    dist_barrier()
    dec_ms = [e0.elapsed_time(e1) for e0, e1 in ev]
    return step_ms, dec_ms


def time_steps_layers(w: DeviceWorkload, steps: int, warmup: int, plan_every_call: bool = False):
    """Per-step CUDA-event times (ms) of consecutive steps that go to different layers' K/V pools.

    A serving engine runs the decode once per layer, each layer on its own
    pool, while block tables, context lengths and the kernels' code stay hot.
    Step k here is layer k mod L of the workload (L pools of the workload's
    size each, together far larger than L2), so no step finds in L2 the K/V
    it reads: the step two layers back read other data of the same size.  No
    flush runs between steps.  Whole steps (graphs of copy + append + decode)
    and the decode alone (after an untimed append) are timed in two passes.
    As in a serving engine, the decode's work list depends only on the context
    lengths, which the layers of a model step share: the first layer of every
    MODEL_LAYERS makes it (pa_decode, which leaves it in the workspace) and the
    others decode with it (pa_decode_planned), so planning is in the timed
    steps once per model step.  Layer m decodes pool m mod L.  With
    plan_every_call, every layer runs pa_decode instead (a plan in every call).
    """
    import torch

    stream = torch.cuda.current_stream()
    L = MODEL_LAYERS   # graphs per model step; layer m uses pool m mod w.layers
    layer_decode = (lambda l: w.decode(l % w.layers)) if plan_every_call else w.layer_decode
    for l in range(L):
        for _ in range(2):
            w.pre(l % w.layers)
            layer_decode(l)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    s.wait_stream(stream)
    g_step, g_pre, g_dec = [], [], []
    with torch.cuda.stream(s):
        for l in range(L):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                w.pre(l % w.layers)
                layer_decode(l)
            g_step.append(g)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                w.pre(l % w.layers)
            g_pre.append(g)
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                layer_decode(l)
            g_dec.append(g)
    stream.wait_stream(s)
    torch.cuda.synchronize()
    for k in range(max(warmup, 3) * w.layers):
        g_step[k % L].replay()
    torch.cuda.synchronize()
    dist_barrier()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for k, (e0, e1) in enumerate(ev):
        e0.record(stream)
        g_step[k % L].replay()
        e1.record(stream)
    torch.cuda.synchronize()
    dist_barrier()
    step_ms = [e0.elapsed_time(e1) for e0, e1 in ev]
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for k, (e0, e1) in enumerate(ev):
        g_pre[k % L].replay()
        e0.record(stream)
        g_dec[k % L].replay()
        e1.record(stream)
    torch.cuda.synchronize()
    dist_barrier()
    dec_ms = [e0.elapsed_time(e1) for e0, e1 in ev]
    return step_ms, dec_ms


def time_e2e(w: DeviceWorkload, steps: int, warmup: int, flush):
    """The same step through the public API from pinned host buffers: H2D inputs, step, D2H output."""
    import torch

    host = {}
    for name in ("q", "key", "value", "slots", "bt", "cl") + (("pairs",) if w.has_copy else ()):
        t = getattr(w, name)
        h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
        h.copy_(t)
        host[name] = h
    out_h = torch.empty(w.out.shape, dtype=w.out.dtype, pin_memory=True)
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out_h.numel() * out_h.element_size()
    stream = torch.cuda.current_stream()

    def one():
        for name, h in host.items():
            getattr(w, name).copy_(h, non_blocking=True)
        w.pre()
        w.decode()
        out_h.copy_(w.out, non_blocking=True)

    for _ in range(max(warmup, 3)):
        flush()
        one()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for e0, e1 in ev:
        flush()
        e0.record(stream)
        one()
        e1.record(stream)
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in ev], h2d, d2h


# ---------------------------------------------------------------------------
# CPU oracle timing (reported baseline; also the --impl reference arm)
# ---------------------------------------------------------------------------
def _oracle_subproblem(name: str, seed: int, nseq: int, sample_seed: int):
    """Host pools holding only ``nseq`` sampled sequences' blocks, values drawn on the host."""
    from workloads import Workload, build_workload, get_config, host_values

    cfg = get_config(name)
    wl = build_workload(cfg, seed=seed)
    rng = np.random.default_rng(sample_seed)
    seqs = np.sort(rng.choice(wl.num_seqs, size=min(nseq, wl.num_seqs), replace=False))
    nblk = [-(-int(wl.context_lens[b]) // 16) for b in seqs]
    ids = sorted({int(x) for b, n in zip(seqs, nblk) for x in wl.block_tables[b, :n]})
    remap = {o: i for i, o in enumerate(ids)}
    bt = np.full((len(seqs), max(1, max(nblk))), -1, np.int32)
    for i, (b, n) in enumerate(zip(seqs, nblk)):
        bt[i, :n] = [remap[int(x)] for x in wl.block_tables[b, :n]]
    sub = Workload(cfg=cfg, seed=sample_seed, context_lens=wl.context_lens[seqs].copy(), block_tables=bt,
                   slot_mapping=np.zeros(0, np.int64), copy_pairs=np.zeros((0, 2), np.int64),
                   num_blocks=max(1, len(ids)))
    return cfg, sub, host_values(sub), wl.num_seqs


def _oracle_run(cfg, sub, v, threads):
    from oracle import c_oracle

    c_oracle.decode(v["q"], v["key_cache"], v["value_cache"], sub.block_tables, sub.context_lens, cfg.scale,
                    cfg.dtype, cfg.num_kv_heads, num_threads=threads)


def block_manager_step(name: str, seed: int, steps: int = 200):
    """Host time of the block manager's part of a decode step for the workload's batch.

    The workload's sequences are added to a C++ block manager (pa_block_manager.h)
    with their context lengths; a quarter of them are then forked (shared
    prefixes), and each step appends one token to every sequence and reads the
    block tables for pa_decode.  Returns a dict for the JSON line.
    """
    import paged_kv_cache_362_b200 as pa
    from workloads import build_workload, get_config

    cfg = get_config(name)
    wl = build_workload(cfg, seed=seed)
    nseq = wl.num_seqs
    ctx = wl.context_lens.astype(int)
    need = int(sum(-(-c // 16) + (steps + 15) // 16 + 1 for c in ctx)) * 2
    bm = pa.BlockManager(need, 16)
    for i, c in enumerate(ctx):
        bm.add_sequence(i, int(c))
    forks = list(range(nseq, nseq + nseq // 4))
    for j, child in enumerate(forks):
        bm.fork(j, child)
    ids = np.arange(nseq + len(forks), dtype=np.int64)
    mb = -(-(int(ctx.max()) + steps + 16) // 16)
    copies = 0
    t0 = time.perf_counter()
    for _ in range(steps):
        _, pairs = bm.append_tokens(ids)
        copies += len(pairs)
        bm.block_tables(ids, mb)
    per = (time.perf_counter() - t0) / steps
    return {"workload": name, "sequences": int(ids.size), "forked": len(forks), "steps": steps,
            "us_per_step": round(per * 1e6, 1), "copy_pairs_total": copies,
            "what": "append one token per sequence (slot mapping, copy-on-write pairs) + block tables, host C++"}


def swap_bandwidth(w, nblocks: int = 4096, reps: int = 5):
    """pa_swap_blocks between the workload's device pools and pinned host pools, both ways (GB/s)."""
    import torch

    pa = w.pa
    shape = (nblocks,) + tuple(w.kc.shape[1:])
    hk = torch.empty(shape, dtype=w.kc.dtype).pin_memory()
    hv = torch.empty(shape, dtype=w.kc.dtype).pin_memory()
    rng = np.random.default_rng(3)
    dev_ids = rng.choice(w.kc.shape[0], size=nblocks, replace=False)
    out_pairs = torch.from_numpy(np.stack([dev_ids, np.arange(nblocks)], 1).astype(np.int64)).cuda()
    in_pairs = torch.from_numpy(np.stack([np.arange(nblocks), dev_ids], 1).astype(np.int64)).cuda()
    nbytes = 2 * hk.numel() * hk.element_size()
    res = {"blocks": nblocks, "bytes": nbytes}
    for name, args in (("device_to_host_gbs", (w.kc, w.vc, hk, hv, out_pairs)),
                       ("host_to_device_gbs", (hk, hv, w.kc, w.vc, in_pairs))):
        pa.swap_blocks(*args)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(reps):
            pa.swap_blocks(*args)
        e1.record()
        torch.cuda.synchronize()
        res[name] = round(nbytes * reps / (e0.elapsed_time(e1) * 1e-3) / 1e9, 1)
    return res


def prefill_throughput(seed: int, reps: int = 20):
    """pa_prefill on chunked prompts (4 sequences: 512 new tokens on 3,584 cached ones, Qwen-shaped
    heads, bf16): causal attention TFLOP/s against the measured bf16 tensor peak.  Each timed call
    follows an L2 flush (the 34 MB of K/V would otherwise stay L2-resident between calls) and is
    timed alone with CUDA events; the median is reported."""
    import torch

    import paged_kv_cache_362_b200 as pa

    B, past, chunk, Hq, Hkv, D = 4, 3584, 512, 28, 4, 128
    ctx = past + chunk
    nbps = ctx // 16
    g = torch.Generator(device="cuda").manual_seed(seed)
    kc = torch.randn((B * nbps, Hkv, 16, D), generator=g, device="cuda").to(torch.bfloat16)
    vc = torch.randn((B * nbps, Hkv, 16, D), generator=g, device="cuda").to(torch.bfloat16)
    perm = np.random.default_rng(seed).permutation(B * nbps).astype(np.int32)
    bt = torch.from_numpy(perm.reshape(B, nbps)).cuda()
    q = torch.randn((B * chunk, Hq, D), generator=g, device="cuda").to(torch.bfloat16)
    out = torch.empty_like(q)
    qs = torch.arange(0, B * chunk + 1, chunk, dtype=torch.int32, device="cuda")
    cl = torch.full((B,), ctx, dtype=torch.int32, device="cuda")
    args = (out, q, kc, vc, bt, qs, cl, 1 / D ** 0.5, chunk)
    # pa_prefill_ws: the workspace (scratch) lets the kernel split its last, partial wave
    ws_bytes = pa.prefill_workspace_size(B, Hq, Hkv, D, chunk, "bf16")
    ws = torch.zeros(max(ws_bytes, 16), dtype=torch.uint8, device="cuda")
    flush_w = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    for _ in range(3):
        pa.prefill(*args, workspace=ws)
    torch.cuda.synchronize()
    times = []
    for _ in range(reps):
        flush_w.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        pa.prefill(*args, workspace=ws)
        e1.record()
        torch.cuda.synchronize()
        times.append(e0.elapsed_time(e1))
    ms = float(np.median(times))
    flops = 4 * Hq * D * B * sum(past + i + 1 for i in range(chunk))
    tf = flops / (ms * 1e-3) / 1e12
    peak, peak_kind = measured_bf16_peak()
    tc = chunk * (Hq // Hkv) >= 32
    kernel = "tcgen05 (prefill_tc_kernel)" if tc else "mma.sync (prefill_kernel)"
    # tensor-core work issued per 128-key step of a 128-row tile: QK^T (K = D) and, for bf16, PV
    # twice (P's hi and lo parts); the useful flops count each PV once
    issued = 1.5 if tc else 1.0
    return {"workload": f"{B} sequences x ({chunk} new on {past} cached tokens), 28/4 heads, D 128, bf16",
            "kernel": kernel, "ms": round(ms, 4), "ms_p10_p50_p90": pct3(times), "tflops": round(tf, 1),
            "peak_tflops": peak, "peak_kind": peak_kind, "frac": round(tf / peak, 4),
            "roofline": {"bound": "tensor", "achieved": round(tf, 1), "peak": peak, "unit": "TFLOP/s",
                         "frac": round(tf / peak, 4),
                         "issued_tflops": round(tf * issued, 1),
                         "note": "achieved counts causal attention flops (4 x D per query-key pair); the "
                                 "kernel issues 1.5x that on the tensor cores (bf16 P as hi + lo)"},
            "l2": "flushed before every timed call (256 MiB write), each call timed alone; median of "
                  f"{reps}",
            "call": f"pa_prefill_ws ({ws_bytes} B workspace: the last partial wave split by key range, "
                    "then merged by a second kernel)"}


def measured_bf16_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            v = json.load(f).get("bf16_tflops")
        if v:
            return float(v), "measured"
    except Exception:
        pass
    return 1590.0, "fallback"


def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def oracle_sample_throughput(name: str, seed: int, budget_s: float, max_seqs: int, threads: int | None = None):
    """fp64 C oracle on a bounded sample of the workload: (KV GB/s, seq/s, threads, sample text)."""
    cfg, sub, v, total = _oracle_subproblem(name, seed, max_seqs, seed + 7)
    threads = threads or os.cpu_count() or 1
    reps, t0 = 0, time.perf_counter()
    while True:
        _oracle_run(cfg, sub, v, threads)
        reps += 1
        el = time.perf_counter() - t0
        if el >= budget_s or reps >= 50:
            break
    per = el / reps
    sample = (f"{sub.num_seqs} of {total} sequences of {name} (seed {seed}), {reps} run(s), "
              f"fp64 C oracle with OpenMP on {threads} thread(s)")
    return sub.kv_bytes() / per / 1e9, sub.num_seqs / per, threads, sample, per


def run_reference(args):
    """The CPU oracle as the reference arm: W + K steps, each a bounded sample of the workload."""
    threads = os.cpu_count() or 1
    cfg, sub, v, total = _oracle_subproblem(args.workload, args.seed, 8, args.seed + 1)
    t0 = time.perf_counter()
    _oracle_run(cfg, sub, v, threads)
    per8 = max(time.perf_counter() - t0, 1e-4)
    steps, warm = args.steps, args.warmup
    per_step_budget = args.ref_total_s / max(1, steps + warm)
    nseq = int(max(1, min(total, 8 * per_step_budget / per8)))
    subs = [_oracle_subproblem(args.workload, args.seed, nseq, args.seed + 100 + i) for i in range(4)]
    for i in range(warm):
        c, s_, v_, _ = subs[i % 4]
        _oracle_run(c, s_, v_, threads)
    times, kv, seqs = [], 0, 0
    for i in range(steps):
        c, s_, v_, _ = subs[i % 4]
        t0 = time.perf_counter()
        _oracle_run(c, s_, v_, threads)
        times.append(time.perf_counter() - t0)
        kv += s_.kv_bytes()
        seqs += s_.num_seqs
    el = sum(times)
    gbs = kv / el / 1e9
    sample = (f"each step: {nseq} of {total} sequences of {args.workload} (4 rotating seeded samples), "
              f"fp64 C oracle with OpenMP on {threads} threads")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": steps, "warmup": warm, "ms_per_step": round(1e3 * el / steps, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": args.workload, "seed": args.seed,
                                        "sample_seqs_per_step": nseq},
        "seq_per_s": round(seqs / el, 3),
        "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default="churned256")
    ap.add_argument("--partition-size", type=int, default=None)
    ap.add_argument("--block-size", type=int, default=None, choices=[8, 16, 32],
                    help="pool block size (default: the workload's, 16); the pool keeps its token capacity")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-graph", action="store_true", help="launch every step from the host (no CUDA graph)")
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=10.0, help="seconds of CPU oracle timing")
    ap.add_argument("--cpu-seqs", type=int, default=64)
    ap.add_argument("--ref-total-s", type=float, default=90.0, help="CPU seconds the reference arm may take")
    ap.add_argument("--layers", type=int, default=4,
                    help="K/V pools (model layers) the layer-rotation measurement cycles through")
    ap.add_argument("--prefill-only", action="store_true",
                    help="time pa_prefill on its chunked-prompt workload, print its JSON line and exit")
    args = ap.parse_args()

    if args.impl == "reference":
        if int(os.environ.get("RANK", "0")) == 0:
            run_reference(args)
        return
    rank, world = dist_setup(args.gpus)

    import torch

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    if args.prefill_only:
        if rank == 0:
            print(json.dumps(prefill_throughput(args.seed)), flush=True)
        dist_done()
        return
    peak, peak_kind = measured_hbm_peak()
    # L2 flush before every timed step: write 256 MiB (twice the L2), then read
    # another 256 MiB so that the write's dirty lines are written back during
    # the flush rather than during the step that follows
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")
    flush_rd = torch.ones(64 << 20, dtype=torch.float32, device="cuda")
    flush_acc = torch.zeros((), dtype=torch.float32, device="cuda")

    def flush():
        flush_buf.zero_()
        torch.sum(flush_rd, dim=0, out=flush_acc)

    flush_write_only = lambda: flush_buf.zero_()
    use_graph = not args.no_graph

    w = DeviceWorkload(args.workload, args.seed + rank, args.partition_size, block_size=args.block_size,
                       layers=args.layers)
    # Timed steps: consecutive steps decode different layers' K/V pools (the
    # layer rotation of a serving engine: K/V cold, block tables and code hot);
    # without graphs or with one layer, an L2 flush before every step instead
    rotation = use_graph and w.layers > 1
    clocks = ClockSampler(torch.cuda.current_device())
    if rotation:
        step_ms, dec_ms = time_steps_layers(w, args.steps, args.warmup)
    else:
        step_ms, dec_ms = time_steps(w, args.steps, args.warmup, flush, use_graph)
    clk = clocks.stop()
    torch.cuda.synchronize()
    status = int(w.status.item())
    if status != 0:
        raise SystemExit(f"device status {status}: {w.pa.error_string(status)}")

    value, ms, _ = aggregate(w.kv_bytes, float(np.mean(step_ms)))
    total_bytes = dist_sum(float(w.kv_bytes))
    dec = dist_max(float(np.mean(dec_ms)))
    achieved = w.kv_bytes / (dec * 1e-3) / 1e9
    # the same rotation with pa_decode in every layer (a plan in every call)
    every = None
    if rotation:
        _, e_dec = time_steps_layers(w, max(200, args.steps // 4), args.warmup, plan_every_call=True)
        ed = dist_max(float(np.mean(e_dec)))
        every = {"decode_ms": round(ed, 5), "achieved": round(w.kv_bytes / (ed * 1e-3) / 1e9, 1),
                 "frac": round(w.kv_bytes / (ed * 1e-3) / 1e9 / peak, 4)}
    # the same steps after an L2 flush each (K/V, tables and the kernels' code all cold)
    f_step, f_dec = time_steps(w, args.steps, args.warmup, flush, use_graph) if rotation else (step_ms, dec_ms)
    f_s, f_d = dist_max(float(np.mean(f_step))), dist_max(float(np.mean(f_dec)))

    e2e_ms, h2d, d2h = time_e2e(w, max(50, args.steps // 10), args.warmup, flush)
    e2e = dist_max(float(np.mean(e2e_ms)))
    # the same decode after a write-only flush: the step then also pays for
    # writing back up to an L2 of the flush's dirty lines
    _, wo_dec = time_steps(w, max(50, args.steps // 10), args.warmup, flush_write_only, use_graph)
    wo = dist_max(float(np.mean(wo_dec)))
    flushed = {"step_ms": round(f_s, 5), "decode_ms": round(f_d, 5),
               "step_kv_gbs": round(w.kv_bytes / (f_s * 1e-3) / 1e9, 1),
               "achieved": round(w.kv_bytes / (f_d * 1e-3) / 1e9, 1),
               "frac": round(w.kv_bytes / (f_d * 1e-3) / 1e9 / peak, 4),
               "decode_ms_p10_p50_p90": pct3(f_dec)}

    secondary = {}
    placement = {}
    if not args.no_secondary:
        for name in ("long32k", "qwen_layer", "shared_prefix"):
            if name == args.workload:
                continue
            sw = DeviceWorkload(name, args.seed + rank, layers=args.layers if rotation else 1)
            if rotation:
                s_step, s_dec = time_steps_layers(sw, max(50, args.steps // 10), args.warmup)
            else:
                s_step, s_dec = time_steps(sw, max(50, args.steps // 10), args.warmup, flush, use_graph)
            _, sf_dec = time_steps(sw, max(50, args.steps // 10), args.warmup, flush, use_graph)
            sd = dist_max(float(np.mean(s_dec)))
            ss = dist_max(float(np.mean(s_step)))
            sfd = dist_max(float(np.mean(sf_dec)))
            if name == "shared_prefix":
                ub = unique_kv_bytes(sw.wl)
                unique_note = {"unique_kv_bytes": ub, "decode_unique_gbs": round(ub / (sd * 1e-3) / 1e9, 1)}
            else:
                unique_note = {}
            secondary[name] = {"decode_ms_p10_p50_p90": pct3(s_dec), **unique_note,
                "decode_ms": round(sd, 5), "step_ms": round(ss, 5),
                "decode_kv_gbs": round(sw.kv_bytes / (sd * 1e-3) / 1e9, 1),
                "decode_frac_of_peak": round(sw.kv_bytes / (sd * 1e-3) / 1e9 / peak, 4),
                "decode_kv_gbs_flushed_every_step": round(sw.kv_bytes / (sfd * 1e-3) / 1e9, 1),
                "kv_bytes": sw.kv_bytes, "seq_per_s": round(sw.wl.num_seqs / (ss * 1e-3), 1),
                "decode_launches": (f"{sw.planned_launches} per planned layer, {sw.decode_launches} in the first "
                                    f"of every {MODEL_LAYERS}" if rotation else sw.decode_launches),
            }
            del sw
            torch.cuda.empty_cache()
        # cost of scattered blocks: the same sequences with contiguous (identity) placement
        for name in ("churned256", "long32k"):
            res = {}
            for pl in (None, "identity"):
                pw = DeviceWorkload(name, args.seed + rank, placement=pl)
                _, p_dec = time_steps(pw, max(50, args.steps // 10), args.warmup, flush, use_graph)
                res[pl or pw.cfg.placement] = dist_max(float(np.mean(p_dec)))
                del pw
                torch.cuda.empty_cache()
            (shuf, ms_s), (_, ms_i) = list(res.items())
            placement[name] = {f"decode_ms_{shuf}": round(ms_s, 5), "decode_ms_identity": round(ms_i, 5),
                               "overhead_pct": round(100 * (ms_s / ms_i - 1), 2)}

    # the block-size trade-off: the same sequences in 8-, 16- and 32-token blocks
    sweep = {}
    if not args.no_secondary:
        for name in ("churned256", "long32k"):
            rows = {}
            for bs in (8, 16, 32):
                bw = DeviceWorkload(name, args.seed + rank, block_size=bs)
                _, b_dec = time_steps(bw, max(50, args.steps // 10), args.warmup, flush, use_graph)
                bd = dist_max(float(np.mean(b_dec)))
                cl = bw.wl.context_lens.astype(np.int64)
                nblk = -(-cl // bs)
                rows[str(bs)] = {
                    "decode_ms": round(bd, 5), "decode_ms_p10_p50_p90": pct3(b_dec),
                    "decode_kv_gbs": round(bw.kv_bytes / (bd * 1e-3) / 1e9, 1),
                    "decode_frac_of_peak": round(bw.kv_bytes / (bd * 1e-3) / 1e9 / peak, 4),
                    "blocks": int(nblk.sum()), "block_table_bytes": int(nblk.sum()) * 4,
                    "wasted_slots": int((nblk * bs - cl).sum()),
                    "wasted_pct": round(100 * float((nblk * bs - cl).sum()) / float((nblk * bs).sum()), 2),
                    "decode_launches": bw.decode_launches,
                }
                if int(bw.status.item()) != 0:
                    raise SystemExit(f"device status {int(bw.status.item())} at block size {bs}")
                del bw
                torch.cuda.empty_cache()
            sweep[name] = rows

    cpu = None
    if rank == 0 and world == 1:
        gbs, sps, threads, sample, _ = oracle_sample_throughput(args.workload, args.seed, args.cpu_budget,
                                                                args.cpu_seqs)
        gbs1, _, _, sample1, _ = oracle_sample_throughput(args.workload, args.seed, args.cpu_budget / 4,
                                                          max(1, args.cpu_seqs // 8), threads=1)
        cpu = {"value": round(gbs, 4), "unit": "GB/s", "cores": threads, "kind": "oracle", "sample": sample,
               "value_1_thread": round(gbs1, 4), "sample_1_thread": sample1, "cpu_model": cpu_model()}

    bm_step = block_manager_step(args.workload, args.seed) if rank == 0 else None
    swap = swap_bandwidth(w) if rank == 0 and not args.no_secondary else None
    prefill_res = prefill_throughput(args.seed) if rank == 0 and not args.no_secondary else None

    if rank == 0:
        c = w.cfg
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms, 5), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": c.dtype, "data": "synthetic",
            "config": {"workload": c.name, "num_seqs": w.wl.num_seqs, "num_heads": c.num_heads,
                       "num_kv_heads": c.num_kv_heads, "head_dim": c.head_dim, "block_size": c.block_size,
                       "num_blocks": c.num_blocks, "mean_context": float(np.mean(w.wl.context_lens)),
                       "max_context": w.max_ctx, "partition_size": w.P or "auto",
                       "parallelism": f"replicas x{world}",
                       "l2": (f"no flush: consecutive timed steps decode {w.layers} different layers' K/V pools "
                              "(each larger than L2, so no step finds the K/V it reads in L2), while block tables, "
                              "context lengths, q and the kernels' code stay L2-resident as in a serving engine; "
                              "roofline.flushed_every_step repeats the steps after a 256 MiB write + 256 MiB read "
                              "flush each") if rotation else
                             ("flushed before every timed step, outside its events: a 256 MiB write, then a "
                              "256 MiB read of another buffer (so the flush's dirty lines are written back before "
                              "the step)"),
                       "cuda_graph": ("one graph per step (copy + append + decode, PDL-chained); the decode "
                                      "alone timed as its own graph") if use_graph else False,
                       "step": ("copy_blocks + " if w.has_copy else "") + "reshape_and_cache + decode" + (
                           f" (the first of every {MODEL_LAYERS} layers, one model step of a 28-layer model, "
                           "pa_decode, which leaves the step's plan in the workspace; the others "
                           "pa_decode_planned)" if rotation else " (pa_decode)")},
            "pct_of_peak": round(100 * value / world / peak, 2),
            "seq_per_s": round(w.wl.num_seqs * world / (ms * 1e-3), 1),
            "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                         "frac": round(achieved / peak, 4), "traffic": profiled_traffic(c.name if c.block_size == 16 else f"{c.name}_bs{c.block_size}"),
                         "algorithmic_bytes": w.kv_bytes,
                         "kernel": ((f"per layer: pa_decode_planned ({w.planned_launches} launch(es): attention "
                                     f"[+ reduce]), and in the first of every {MODEL_LAYERS} layers (a model step) "
                                     f"pa_decode ({w.decode_launches} launch(es), planning included): the mean per "
                                     f"layer over consecutive timed steps")
                                    if rotation else
                                    f"pa_decode call ({w.decode_launches} launch(es): [plan +] attention "
                                    "[+ reduce]), timed together") +
                                   "; traffic = DRAM bytes of the attention kernel from profiles/traffic.json; "
                                   "plan_in_every_call is the same rotation with pa_decode in every layer; "
                                   "flushed_every_step and after_write_only_flush time pa_decode (a plan in "
                                   "every call)",
                         "peak_kind": peak_kind,
                         "flushed_every_step": flushed,
                         "plan_in_every_call": every,
                         "after_write_only_flush": {"decode_ms": round(wo, 5),
                                                    "achieved": round(w.kv_bytes / (wo * 1e-3) / 1e9, 1),
                                                    "frac": round(w.kv_bytes / (wo * 1e-3) / 1e9 / peak, 4)}},
            "cpu_baseline": cpu,
            "e2e": {"value": round(total_bytes / (e2e * 1e-3) / 1e9, 2), "unit": "GB/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": round(e2e, 5)},
            "step_ms_p10_p50_p90": pct3(step_ms), "decode_ms_p10_p50_p90": pct3(dec_ms),
            "placement_overhead": placement,
            "block_size_sweep": sweep,
            "block_manager": bm_step,
            "swap": swap,
            "prefill": prefill_res,
            "gpu_launches": ((w.launches_per_step - w.decode_launches + w.planned_launches) * args.steps
                             + (w.decode_launches - w.planned_launches) * -(-args.steps // MODEL_LAYERS))
                            if rotation else w.launches_per_step * args.steps,
            "clocks": clk,
            "secondary": secondary,
        }
        print(json.dumps(line), flush=True)
    dist_done()


if __name__ == "__main__":
    main()
