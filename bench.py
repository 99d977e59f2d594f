#!/usr/bin/env python
"""Benchmark: batch-1 packed SAGE GEMV over a Qwen3-4B-shaped decoder layer on B200.

A step is one Qwen3-4B-shaped decoder layer at batch 1 (hidden 2560): its
seven projections (q, k, v, o, gate, up, down) computed straight from 2.25-bit
codes, with the operations between them fused (RMSNorm, attention over one
cached position, residual adds, SiLU * up), in ONE launch of the libsage engine
(sage_decoder_layer_forward).  Every step reads a different copy of the layer's
packed planes, so the working set (> 4 x the 126 MB L2) comes from HBM.
Reported alongside (under "extra"): the seven projections as one grouped launch
with independent inputs, the four dependency stages as four launches, the
4096 -> 12288 batch sweep through the GEMV and tcgen05 paths, the grouped-expert
MoE GEMV, and the encoder / blockwise-optimisation kernels.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Prints ONE JSON line (rank 0).  ``value`` is the whole-job throughput in GB/s
of packed bytes (codes + mu/delta + codebooks + x + y) per layer; ``us_per_layer``
is the device time of one layer.  ``--impl reference`` times the CPU oracle on
a bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import json
import os
import platform
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "batch-1 packed VQ GEMV µs/layer and achieved HBM GB/s vs B200 peak"
LAYER_SHAPES = "q 2560->4096, k/v 2560->1024, o 4096->2560, gate/up 2560->9728, down 9728->2560"


def workload(mode: str) -> str:
    how = {"fused": "the decoder layer in one launch", "stages": "its four dependency stages as four launches",
           "grouped7": "the seven projections in one grouped launch"}[mode]
    return f"Qwen3-4B-shaped decoder layer at batch 1, 7 packed linears ({LAYER_SHAPES}), {how}"
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0
L2_BYTES = 126 * 1024 * 1024
KERNEL = "engine_kernel<1> (libsage packed GEMV engine, sm_100a)"


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as fh:
            d = json.load(fh)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def _peak_tflops():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as fh:
            d = json.load(fh)
        return float(d["bf16_tflops"]), "measured (bf16 burst; fp16 dense has the same nominal rate)"
    except Exception:
        return 1590.0, "fallback"


def max_over_ranks(ms: float, dist, device) -> float:
    """The job's time is its slowest rank's: all-reduce MAX of a per-rank time
    (no-op on one process)."""
    if dist is None:
        return float(ms)
    import torch
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(world: int, bytes_per_step: int, steps: int, ms: float) -> float:
    """Whole-job throughput: every rank runs its own replica of the step."""
    return world * bytes_per_step * steps / (ms * 1e-3) / 1e9


def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except Exception:
        pass
    return platform.processor() or "unknown"


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.proc = None
        d = os.environ.get("SAGE_CLOCKS_DIR")  # keeps the raw samples (one CSV per rank)
        self.path = (os.path.join(d, f"clocks_rank{gpu_index}.csv") if d and os.path.isdir(d)
                     else os.path.join(tempfile.gettempdir(), f"sage_clocks_{os.getpid()}_{gpu_index}.csv"))
        self.gpu = gpu_index

    def start(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.fh, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.fh.close()
        sm, mx, power, reasons = [], None, [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            p = [x.strip() for x in line.split(",")]
            if len(p) < 9:
                continue
            try:
                sm.append(float(p[1]))
                mx = float(p[2])
                power.append(float(p[3]))
            except ValueError:
                continue
            for nm, v in zip(names, p[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx, "samples": len(sm),
                "power_w": statistics.median(power) if power else None, "reasons": sorted(reasons)}


def kernel_source_hash() -> str:
    """sha256 over the engine's sources: DRAM counters taken on other sources are stale."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "bit_vector_quantized_sage_b200", "csrc")
    for n in ("sage_gemv.cu", "sage_device.cuh", "sage_engine.h", "sage_layer.cpp"):
        h.update(open(os.path.join(csrc, n), "rb").read())
    return h.hexdigest()


def traffic_for(mode: str):
    """DRAM bytes (read + write) per launch of the timed kernel from the committed ncu
    summary, or None when the summary was taken on other kernel sources."""
    p = os.path.join(ROOT, "profiles", "engine_traffic.json")
    try:
        d = json.load(open(p))
    except Exception:
        return None, "no committed ncu DRAM capture"
    if d.get("source_sha256") != kernel_source_hash():
        return None, "ncu DRAM capture taken on other kernel sources"
    e = d.get("modes", {}).get(mode)
    if not e:
        return None, f"no ncu DRAM capture for mode {mode}"
    return e["dram_bytes_per_launch"], e.get("note", "")


def dist_summary(samples_us):
    a = np.asarray(samples_us, dtype=np.float64)
    return {"median": round(float(np.median(a)), 3), "p10": round(float(np.percentile(a, 10)), 3),
            "p90": round(float(np.percentile(a, 90)), 3), "n": int(a.size)}


# ---------------------------------------------------------------------------
# The CPU oracle as a timed baseline: unpack of the packed planes, fp32
# reconstruction and fp64 matvec (oracle/), one process per core, each on its
# own share of 256-row blocks.  The planes come from the oracle's own packer,
# so nothing here runs the library.
# ---------------------------------------------------------------------------

_ORACLE_DATA = {}


def _oracle_source(kind: str, name: str):
    """(code fields, x) of one matrix of a workload, built once per process."""
    key = (kind, name)
    if key in _ORACLE_DATA:
        return _ORACLE_DATA[key]
    import oracle
    import synth
    if kind == "layer":
        if "layer" not in _ORACLE_DATA:
            L = synth.config1()
            for f in L.mats:
                f.perm = oracle.esg_perm(L.energies[f.name])
            _ORACLE_DATA["layer"] = L
        L = _ORACLE_DATA["layer"]
        f = next(m for m in L.mats if m.name == name)
        x = L.xs[[s for s in synth.QWEN3_4B_STAGES if name in s][0][0]]
    elif kind == "up8b":
        f, x = synth.config3(1)
    else:  # "moe:<proj>:<expert>", T = 1 token
        _, proj, e = name.split(":")
        spec = synth.config4(1)
        f = spec.expert(int(e), int(proj))
        x = spec.x if int(proj) < 2 else spec.x_down[:1]
    _ORACLE_DATA[key] = (f, x)
    return f, x


def _oracle_prepare(task):
    import oracle
    import synth
    kind, name, r0, r1 = task
    f, x = _oracle_source(kind, name)
    R = r1 - r0
    main, meta = oracle.pack(R, f.d_in, f.log2K, f.signs[r0:r1], f.idx[r0:r1], f.q[r0:r1], f.mu[r0:r1],
                             f.delta[r0:r1])
    nbytes = main.nbytes + meta.nbytes + (1 << f.log2K) * 16 + x.nbytes + x.shape[0] * R * 2
    return (f, x, R, main, meta, nbytes)


def _oracle_run(prep):
    import oracle
    import synth
    f, x, R, main, meta, _ = prep
    u = oracle.unpack(R, f.d_in, f.log2K, main, meta)
    g = synth.Fields(R, f.d_in, f.log2K, u["signs"], u["idx"], u["q"], u["mu"], u["delta"], f.codebook, f.perm)
    return oracle.gemv(g, x)


def _oracle_worker(inq, outq):
    sys.path.insert(0, ROOT)
    while True:
        tasks = inq.get()
        if tasks is None:
            return
        preps = [_oracle_prepare(t) for t in tasks]
        outq.put(("ready", None))
        inq.get()  # go
        t0 = time.perf_counter()
        for p in preps:
            _oracle_run(p)
        t1 = time.perf_counter()
        outq.put(("done", (sum(p[-1] for p in preps), t0, t1)))


class OraclePool:
    """Persistent spawn-context worker processes (safe next to a CUDA context)."""

    def __init__(self, n: int):
        import multiprocessing as mp
        ctx = mp.get_context("spawn")
        self.n = n
        self.inq = [ctx.Queue() for _ in range(n)]
        self.outq = ctx.Queue()
        self.procs = [ctx.Process(target=_oracle_worker, args=(self.inq[i], self.outq), daemon=True)
                      for i in range(n)]
        for p in self.procs:
            p.start()

    def run(self, shards):
        """shards: one task list per worker.  Returns (bytes, wall seconds from the first
        worker's start to the last one's end)."""
        active = [i for i in range(self.n) if shards[i]]
        for i in active:
            self.inq[i].put(shards[i])
        for _ in active:
            self.outq.get()
        for i in active:
            self.inq[i].put("go")
        res = [self.outq.get()[1] for _ in active]
        nbytes = sum(r[0] for r in res)
        return nbytes, max(r[2] for r in res) - min(r[1] for r in res)

    def close(self):
        for q in self.inq:
            q.put(None)
        for p in self.procs:
            p.join(timeout=10)


def layer_block_tasks():
    """(kind, matrix, r0, r1) for every 256-row block of the seven layer matrices, with its
    weight count as cost."""
    import synth
    out = []
    for name, d_out, d_in in synth.QWEN3_4B_LAYER:
        for r0 in range(0, d_out, 256):
            r1 = min(d_out, r0 + 256)
            out.append((("layer", name, r0, r1), (r1 - r0) * d_in))
    return out


def shard(tasks_with_cost, n):
    """Longest-processing-time split of the tasks over n workers."""
    loads = [0] * n
    shards = [[] for _ in range(n)]
    for t, c in sorted(tasks_with_cost, key=lambda tc: -tc[1]):
        i = int(np.argmin(loads))
        shards[i].append(t)
        loads[i] += c
    return shards


def oracle_layer_baseline(pool_1, pool_n, fraction: float = 1.0, offset: int = 0):
    """Oracle GB/s on `fraction` of the layer's blocks (every 1/fraction-th block from
    `offset`): once on one core, once on all of pool_n's cores."""
    tasks = layer_block_tasks()
    if fraction < 1.0:
        step = max(1, int(round(1.0 / fraction)))
        tasks = tasks[offset % step::step]
    out = {}
    for label, pool in (("1", pool_1), ("n", pool_n)):
        if pool is None:
            continue
        b, s = pool.run(shard(tasks, pool.n))
        out[label] = (b / s / 1e9, s, pool.n)
    return out, len(tasks)


# ---------------------------------------------------------------------------
# Workload construction (product path: synth + libsage)
# ---------------------------------------------------------------------------

def clone_matrix(m):
    import bit_vector_quantized_sage_b200 as sage
    return sage.PackedMatrix(m.d_out, m.d_in, m.log2K, m.main.clone(), m.meta.clone(), m.codebook.clone(),
                             m.perm.clone() if m.perm is not None else None, m.name)


def layer_bytes(mats, M=1):
    """Algorithmic bytes of one layer: packed planes + codebooks + x + y (perm excluded)."""
    tot = perm = 0
    for m in mats.values():
        tot += m.packed_bytes + (1 << m.log2K) * 16 + M * m.d_in * 2 + M * m.d_out * 2
        perm += m.d_in * 4 if m.perm is not None else 0
    return tot, perm


def build_layers():
    """Seeded Qwen3-4B-shaped layer (ESG permutations from its channel energies) and
    enough device copies of its packed planes that rotating through them streams
    more than 4 x L2 from HBM."""
    import synth
    import bit_vector_quantized_sage_b200 as sage
    L = synth.config1()
    base = {}
    for f in L.mats:
        f.perm = sage.sage_esg_permutation(L.energies[f.name])
        base[f.name] = sage.PackedMatrix.from_fields(f)
    nbytes, _ = layer_bytes(base)
    replicas = max(2, int(np.ceil(4 * L2_BYTES / nbytes)) + 1)
    layers = [base] + [{n: clone_matrix(m) for n, m in base.items()} for _ in range(replicas - 1)]
    return L, layers


class LayerStages:
    """The layer's four dependency stages (q|k|v, o, gate|up, down) as four grouped
    launches chained with programmatic dependent launch; synthetic stage inputs."""
    launches = 4

    def __init__(self, lay, xs, ys, ws):
        import synth
        import bit_vector_quantized_sage_b200 as sage
        self.calls = [sage.GroupedCall([lay[n] for n in st], [xs[st[0]]] * len(st), [ys[n] for n in st], 1, ws)
                      for st in synth.QWEN3_4B_STAGES]

    def __call__(self, stream=None):
        for c in self.calls:
            c(stream)


class LayerGrouped7:
    """All seven projections in one grouped launch, each on its own synthetic input (no
    dependencies between them)."""
    launches = 1

    def __init__(self, lay, xs, ys, ws):
        import synth
        import bit_vector_quantized_sage_b200 as sage
        xmap = {n: xs[[st for st in synth.QWEN3_4B_STAGES if n in st][0][0]] for n in lay}
        names = list(lay)
        self.call = sage.GroupedCall([lay[n] for n in names], [xmap[n] for n in names], [ys[n] for n in names], 1, ws)

    def __call__(self, stream=None):
        self.call(stream)


def make_runners(mode, layers, L):
    """Per-replica callables for one layer mode, plus their shared device inputs/outputs,
    workspace and the host-visible input/output tensors of an end-to-end step."""
    import torch
    import synth
    import bit_vector_quantized_sage_b200 as sage
    base = layers[0]
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()
    if mode == "fused":
        inp = synth.decoder_inputs(1, 1, 2560)
        h = dev(inp.h)
        outs = {n: torch.zeros((1, m.d_out), dtype=torch.int16, device="cuda") for n, m in base.items()}
        outs["h_out"] = torch.zeros((1, 2560), dtype=torch.int16, device="cuda")
        nh, nkv, hd = synth.QWEN3_4B_HEADS
        an, mn = dev(inp.attn_norm), dev(inp.mlp_norm)
        runs = [sage.DecoderLayer(lay, an, mn, nh, nkv, hd, inp.eps, outs, 1) for lay in layers]
        ws = runs[0].ws
        for r in runs:
            r.ws = ws
        fns = [lambda st, r=r: r(h, st) for r in runs]
        return fns, ws, {"h": (h, inp.h)}, {"h_out": outs["h_out"]}, 1
    xs = {k: dev(v) for k, v in L.xs.items()}
    ys = {n: torch.zeros((1, m.d_out), dtype=torch.int16, device="cuda") for n, m in base.items()}
    if mode == "stages":
        ws = sage.Workspace(max(sage.sage_workspace_size(sage.SAGE_OP_GROUPED, [base[n] for n in st], 1)
                                for st in synth.QWEN3_4B_STAGES))
        runs = [LayerStages(lay, xs, ys, ws) for lay in layers]
    else:
        ws = sage.Workspace(sage.sage_workspace_size(sage.SAGE_OP_GROUPED, list(base.values()), 1))
        runs = [LayerGrouped7(lay, xs, ys, ws) for lay in layers]
    fns = [lambda st, r=r: r(st) for r in runs]
    return fns, ws, {k: (xs[k], L.xs[k]) for k in xs}, ys, runs[0].launches


# ---------------------------------------------------------------------------
# Device timing
# ---------------------------------------------------------------------------

def capture(fn, stream):
    import torch
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn(torch.cuda.current_stream())
    return g


def per_call_us(fns, stream, rounds=12):
    """Device time per call: one CUDA graph holds the calls back to back (they rotate
    over copies of the data larger than L2, chained by programmatic dependent launch
    as a stream of layers is), replayed `rounds` times with events around each
    replay.  Returns one per-call average per replay (us)."""
    import torch
    g = capture(lambda st: [f(st) for f in fns], stream)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(rounds + 1)]
    ev[0].record(stream)
    for k in range(rounds):
        g.replay()
        ev[k + 1].record(stream)
    torch.cuda.synchronize()
    out = [ev[i].elapsed_time(ev[i + 1]) * 1e3 / len(fns) for i in range(rounds)]
    del g
    return out


def bench_gemm(stream):
    """4096 -> 12288 up-projection, (K,V) = (32,5): batch 1-8 through the GEMV engine,
    16-128 through the tcgen05 path (sage_gemm dispatches).  Per batch: device us
    (median, p10, p90 over replays of the copies of the planes), TFLOP/s against the
    dense fp16 tensor peak and GB/s of packed bytes against HBM."""
    import torch
    import synth
    import bit_vector_quantized_sage_b200 as sage
    f, _ = synth.config3(1)
    A0 = sage.PackedMatrix.from_fields(f)
    As = [A0] + [clone_matrix(A0) for _ in range(int(np.ceil(2 * L2_BYTES / A0.packed_bytes)))]
    peak, kind = _peak_tflops()
    hbm, _ = _peaks()
    out = []
    for M in (1, 2, 4, 8, 16, 32, 64, 128):
        _, xb = synth.config3(M)
        x = torch.from_numpy(xb.view(np.int16)).cuda()
        y = torch.zeros((M, f.d_out), dtype=torch.int16, device="cuda")
        ws = sage.Workspace(sage.sage_workspace_size(sage.SAGE_OP_GEMM, A0, M))
        fns = [lambda st, A=A: sage.sage_gemm(A, x, M, y, ws, st) for A in As]
        for fn in fns[:3]:
            fn(stream)
        t = per_call_us(fns, stream)
        assert sage.sage_query_status(ws) == sage.SAGE_OK
        us = float(np.median(t))
        flops = 2.0 * M * f.d_out * f.d_in
        nbytes = A0.packed_bytes + 32 * 16 + M * f.d_in * 2 + M * f.d_out * 2
        tf = flops / (us * 1e-6) / 1e12
        out.append({"M": M, "path": "gemv" if M <= 8 else "tcgen05", "us": dist_summary(t),
                    "tflops": round(tf, 1), "tensor_frac": round(tf / peak, 4),
                    "gbs": round(nbytes / (us * 1e-6) / 1e9, 1), "hbm_frac": round(nbytes / (us * 1e-6) / 1e9 / hbm, 4)})
    return {"workload": "4096->12288 up-projection, (K,V)=(32,5), planes rotated over copies > 2 x L2",
            "peak_tflops": peak, "peak_kind": kind, "points": out}


def bench_moe(stream, reps=20):
    """128 experts (gate/up 2048 -> 768, down 768 -> 2048), top-8 routing, T tokens; one
    sage_moe_gemv call per projection.  Two timings per point:
      - `us`: calls back to back over four copies of the expert set (252 MB > L2), one
        CUDA graph, as a stream of MoE layers runs (median/p10/p90 over 12 replays);
      - `us_cold`: a single call after L2 is flushed by reading a buffer twice its size
        (a read leaves clean lines: a write-based flush would leave the call to write
        back ~126 MB of dirty lines), launch latency included."""
    import torch
    import synth
    import bit_vector_quantized_sage_b200 as sage
    hbm, _ = _peaks()
    flush = torch.ones(2 * L2_BYTES // 4, dtype=torch.float32, device="cuda")
    out = []
    for proj in (0, 2):
        packed = None
        for T in (1, 4, 16):
            spec = synth.config4(T)
            if packed is None:
                packed = [sage.PackedMatrix.from_fields(spec.expert(e, proj)) for e in range(synth.MOE_EXPERTS)]
                sets = [packed] + [[clone_matrix(m) for m in packed] for _ in range(3)]
            n_pairs = T * synth.MOE_TOPK
            pe = torch.from_numpy(spec.routes.reshape(-1).astype(np.int32)).cuda()
            if proj < 2:
                xb, xrow = spec.x, np.repeat(np.arange(T, dtype=np.int32), synth.MOE_TOPK)
            else:
                xb, xrow = spec.x_down, np.arange(n_pairs, dtype=np.int32)
            x = torch.from_numpy(xb.view(np.int16)).cuda()
            xr = torch.from_numpy(xrow).cuda()
            d_out = synth.MOE_PROJ[proj][1]
            y = torch.zeros((n_pairs, d_out), dtype=torch.int16, device="cuda")
            ws = sage.Workspace(sage.sage_workspace_size(sage.SAGE_OP_MOE, packed, n_pairs))
            fns = [lambda st, E=E: sage.sage_moe_gemv(E, pe, xr, n_pairs, x, y, ws, st) for E in sets]
            for fn in fns:
                fn(stream)
            t = per_call_us(fns, stream)
            g = capture(fns[0], stream)
            tc = []
            for _ in range(reps):
                sink = flush.sum()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                g.replay()
                e1.record(stream)
                e1.synchronize()
                tc.append(e0.elapsed_time(e1) * 1e3)
            del g, sink
            assert sage.sage_query_status(ws) == sage.SAGE_OK
            active = np.unique(spec.routes)
            nbytes = sum(packed[e].packed_bytes + (1 << packed[e].log2K) * 16 for e in active)
            nbytes += xb.nbytes + n_pairs * d_out * 2
            us = float(np.median(t))
            pt = {"proj": synth.MOE_PROJ[proj][0], "T": T, "experts": int(active.size), "us": dist_summary(t),
                  "gbs": round(nbytes / (us * 1e-6) / 1e9, 1), "hbm_frac": round(nbytes / (us * 1e-6) / 1e9 / hbm, 4),
                  "us_cold": dist_summary(tc)}
            if proj == 2:  # the down projection followed by the router-weighted combine
                wr = torch.from_numpy(np.random.default_rng(T).dirichlet(np.ones(synth.MOE_TOPK), size=T)
                                      .astype(np.float32)).cuda()
                yt = torch.zeros((T, d_out), dtype=torch.int16, device="cuda")
                fc = [lambda st, E=E: (sage.sage_moe_gemv(E, pe, xr, n_pairs, x, y, ws, st),
                                       sage.sage_moe_combine(T, synth.MOE_TOPK, y, wr, yt, st)) for E in sets]
                for fn in fc:
                    fn(stream)
                pt["us_with_combine"] = dist_summary(per_call_us(fc, stream))
                assert sage.sage_query_status(ws) == sage.SAGE_OK
            out.append(pt)
        del sets
    del flush
    return {"workload": "128 experts, top-8, one projection per call (in-kernel routing + grouped GEMV)",
            "points": out}


def bench_qdq(stream):
    """The continuous-parameter decode (blockwise optimisation forward) of a
    4096 x 4096 matrix at (K, V) = (64, 4): per subvector it reads rho, the
    sign byte and the index (7 B) and writes 8 fp32 weights and the radius code
    (33 B); reported as GB/s of those bytes against the HBM copy rate."""
    import torch
    import synth
    import bit_vector_quantized_sage_b200 as sage
    f = synth.qdq_inputs(7, 4096, 4096, 6)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    alpha, rho, signs, idx = dev(f.alpha), dev(f.rho), dev(f.signs), dev(f.idx.view(np.int16))
    Ws = [torch.empty((4096, 4096), dtype=torch.float32, device="cuda") for _ in range(3)]
    q = torch.empty((4096, 512), dtype=torch.uint8, device="cuda")
    fns = [lambda st, W=W: sage.sage_qdq_forward(4096, 4096, 6, alpha, rho, signs, idx, W, q, None, st) for W in Ws]
    for fn in fns:
        fn(stream)
    t = per_call_us(fns, stream)
    us = float(np.median(t))
    nsv = 4096 * 512
    nbytes = nsv * (4 + 1 + 2) + nsv * (32 + 1) + 64 * 7 * 4
    hbm, _ = _peaks()
    del Ws
    return {"workload": "continuous-parameter decode (QDQ forward), 4096 x 4096, (K,V)=(64,4), fp32 W out",
            "us": dist_summary(t), "gbs": round(nbytes / (us * 1e-6) / 1e9, 1),
            "hbm_frac": round(nbytes / (us * 1e-6) / 1e9 / hbm, 4), "bytes_per_call": nbytes}


def bench_abs(stream, reps=10):
    """Adaptive bit splitting on the weight-derived 4096 x 4096 layer: Eq. 8 of
    each of the five split encodings (the library's CPU encoder, outside the
    timing) against W, and the Eq. 9 choice.  Per candidate the score reads the
    packed planes, the permutation, W (fp32, 64 MB) and the energies."""
    import torch
    import synth
    import bit_vector_quantized_sage_b200 as sage
    packed = []
    inits = {}
    t_cpu_enc = 0.0
    for log2K in (4, 5, 6, 7, 8):
        inp, _ = synth.config2(d_out=4096, d_in=4096, n_samples=65536, iters=10, log2K=log2K)
        inits[log2K] = inp.init
        t0 = time.perf_counter()
        r = sage.sage_encode(inp.W, inp.energies, log2K, inp.gamma, inp.sample, inp.init, inp.iters)
        t_cpu_enc += time.perf_counter() - t0
        f = synth.Fields(4096, 4096, log2K, r["signs"], r["idx"], r["q"], r["mu"], r["delta"], r["codebook"],
                         r["perm"], f"K=2^{log2K}")
        packed.append(sage.PackedMatrix.from_fields(f))
    W = torch.from_numpy(inp.W.astype(np.float32)).cuda()
    e = torch.from_numpy(inp.energies.astype(np.float32)).cuda()
    ws = sage.Workspace(sage.sage_workspace_size(sage.SAGE_OP_ABS, packed, 1))  # all five: one sync
    best, errs = sage.sage_abs_select(packed, W, e, ws, stream)
    t = []
    for _ in range(reps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        sage.sage_abs_select(packed, W, e, ws, stream)
        e1.record(stream)
        e1.synchronize()
        t.append(e0.elapsed_time(e1) * 1e3 / 5)
    us = float(np.median(t))
    nbytes = packed[0].packed_bytes + 4096 * 4 + 4096 * 4096 * 4 + 4096 * 4
    hbm, _ = _peaks()
    # the same selection with the five encodings made on the GPU (k-means, row
    # stage, device packer), from the host-side inputs (permutation, Eq. 4 weights,
    # samples), which are computed once per matrix
    t0 = time.perf_counter()
    x = sage.sage_encode_inputs(inp.W, inp.energies, inp.gamma, inp.sample)
    t_inputs = time.perf_counter() - t0
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    Wd, Pd, Wtd, permd, omd = dev(inp.W), dev(x["P"]), dev(x["Wt"]), dev(x["perm"]), dev(x["omega"])
    initd = {k: dev(v) for k, v in inits.items()}
    kws = sage.Workspace(sage.sage_kmeans_workspace_size(Pd.shape[0]))
    fl = [torch.empty((4096, 512), dtype=torch.uint8, device="cuda"), torch.empty((4096, 512), dtype=torch.int16, device="cuda"),
          torch.empty((4096, 512), dtype=torch.uint8, device="cuda"), torch.empty((4096, 32), dtype=torch.int16, device="cuda"),
          torch.empty((4096, 32), dtype=torch.int16, device="cuda")]

    def gpu_abs():
        cands = []
        for log2K in (4, 5, 6, 7, 8):
            _, cb16, _ = sage.sage_kmeans(Pd, Wtd, log2K, initd[log2K], 10, kws, stream)
            sage.sage_encode_rows(4096, 4096, log2K, Wd, permd, omd, cb16, *fl, stream)
            main, meta = sage.sage_pack_device(4096, 4096, log2K, *fl, stream)
            cands.append(sage.PackedMatrix(4096, 4096, log2K, main, meta, cb16.reshape(-1), permd))
        return sage.sage_abs_select(cands, W, e, ws, stream)

    g_best, g_errs = gpu_abs()
    tg = []
    for _ in range(3):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        gpu_abs()
        e1.record(stream)
        e1.synchronize()
        tg.append(e0.elapsed_time(e1) * 1e3)
    assert sage.sage_query_status(kws) == 0
    return {"workload": "Eq. 8 score of the five split encodings of the weight-derived 4096 x 4096 layer, Eq. 9 choice",
            "best_log2K": 4 + best, "errors": [round(x, 6) for x in errs],
            "us_per_candidate": dist_summary(t), "gbs": round(nbytes / (us * 1e-6) / 1e9, 1),
            "hbm_frac": round(nbytes / (us * 1e-6) / 1e9 / hbm, 4),
            "note": "one synchronous sage_abs_select over the five candidates (the host adds each one's CTA partials)",
            "gpu_encoder_end_to_end": {
                "what": "the five encodings on the GPU (sage_kmeans 10 rounds, sage_encode_rows, sage_pack_device) "
                        "and the Eq. 8 scores / Eq. 9 choice",
                "us": dist_summary(tg), "best_log2K": 4 + g_best, "same_errors_as_cpu_encoder": g_errs == errs,
                "host_inputs_s": round(t_inputs, 3),
                "cpu_encoder_s": round(t_cpu_enc, 3), "cpu_encoder_cores": host_cores(),
                "cpu_encoder_what": "the five sage_encode calls (all host cores), packing excluded"}}


def bench_encode_rows(stream, reps=10):
    """The encoder's per-row stage (Eq. 6 over K codewords in fp64, Eq. 14, Eq. 2)
    on the weight-derived 4096 x 4096 layer at (K, V) = (64, 4), with the CPU
    encoder's codebook and permutation; the oracle's same stage on one host core
    beside it."""
    import torch
    import oracle
    import synth
    import bit_vector_quantized_sage_b200 as sage
    inp, _ = synth.config2()
    r = sage.sage_encode(inp.W, inp.energies, inp.log2K, inp.gamma, inp.sample, inp.init, inp.iters)
    om = oracle.omega_columns(inp.energies, r["perm"], inp.gamma)
    dev = lambda a: torch.from_numpy(np.ascontiguousarray(a)).cuda()
    W, perm, omd, cb = dev(inp.W), dev(r["perm"].astype(np.int32)), dev(om), dev(r["codebook"].view(np.int16))
    S, G = 512, 32
    outs = [torch.empty((4096, S), dtype=torch.uint8, device="cuda"), torch.empty((4096, S), dtype=torch.int16, device="cuda"),
            torch.empty((4096, S), dtype=torch.uint8, device="cuda"), torch.empty((4096, G), dtype=torch.int16, device="cuda"),
            torch.empty((4096, G), dtype=torch.int16, device="cuda")]
    fn = lambda st: sage.sage_encode_rows(4096, 4096, inp.log2K, W, perm, omd, cb, *outs, st)
    fn(stream)
    t = per_call_us([fn], stream)
    t0 = time.perf_counter()
    oracle.encode_rows(inp.W[:256], r["perm"], om, r["codebook"], inp.log2K)
    cpu_s = (time.perf_counter() - t0) * 16  # 256 of 4096 rows
    us = float(np.median(t))
    # the weighted spherical k-means on the same layer's 65,536 samples
    S_ = inp.W.shape[1] // 8
    o_, j_ = inp.sample // S_, inp.sample % S_
    P = np.ascontiguousarray(np.abs(inp.W[o_[:, None], r["perm"].reshape(S_, 8)[j_]]))
    Wt = np.ascontiguousarray(om.reshape(S_, 8)[j_])
    Pd, Wd, initd = dev(P), dev(Wt), dev(inp.init)
    _, _, kws = sage.sage_kmeans(Pd, Wd, inp.log2K, initd, inp.iters, stream=stream)
    km = []
    for _ in range(5):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        sage.sage_kmeans(Pd, Wd, inp.log2K, initd, inp.iters, kws, stream)
        b.record(stream)
        b.synchronize()
        km.append(a.elapsed_time(b) * 1e3)
    t0 = time.perf_counter()
    oracle.kmeans(P, Wt, 1 << inp.log2K, inp.init, 1)
    km_cpu_s = (time.perf_counter() - t0) * inp.iters  # one round, scaled by the rounds
    return {"workload": "encoder row stage (Eq. 6 over 64 codewords in fp64, Eq. 14, Eq. 2), 4096 x 4096",
            "us": dist_summary(t), "subvectors_per_s": round(4096 * 512 / (us * 1e-6) / 1e9, 3),
            "unit": "G subvectors/s", "oracle_one_core_s_extrapolated": round(cpu_s, 3),
            "oracle_sample": "rows 0-255, scaled by 16",
            "kmeans": {"workload": f"weighted spherical k-means, {len(inp.sample)} samples, K = {1 << inp.log2K}, "
                                   f"{inp.iters} rounds",
                       "us": dist_summary(km), "oracle_one_core_s_extrapolated": round(km_cpu_s, 3),
                       "oracle_sample": f"one round, scaled by {inp.iters}"}}


def oracle_beside(pool_1):
    """The oracle on one core beside the up-projection and MoE workloads (GB/s of packed
    bytes on a sample: two 256-row blocks of the up-projection; the gate and down
    matrices of the first four experts routed for one token)."""
    import synth
    out = {}
    b, s = pool_1.run([[("up8b", "up8b", 0, 256), ("up8b", "up8b", 6144, 6400)]])
    out["up8b_4096x12288"] = {"gbs": round(b / s / 1e9, 4), "seconds": round(s, 3), "cores": 1,
                              "sample": "rows 0-255 and 6144-6399"}
    routes = synth.config4(1).routes[0][:4]
    tasks = []
    for proj, d_out in ((0, 768), (2, 2048)):
        for e in routes:
            tasks.append(("moe", f"moe:{proj}:{int(e)}", 0, d_out))
    b, s = pool_1.run([tasks])
    out["moe_T1"] = {"gbs": round(b / s / 1e9, 4), "seconds": round(s, 3), "cores": 1,
                     "sample": "gate and down of 4 of the 8 routed experts, T = 1"}
    return out


# ---------------------------------------------------------------------------
# Arms
# ---------------------------------------------------------------------------

def run_reference(args):
    """The CPU oracle on the same workload: each step is a bounded sample of the layer
    (every 8th 256-row block, rotating the offset so that 8 steps cover the layer) on
    all host cores."""
    world, rank, _ = _dist()
    if rank != 0:
        return 0
    cores = host_cores()
    pool = OraclePool(cores)
    try:
        for i in range(args.warmup):
            oracle_layer_baseline(None, pool, fraction=1 / 8, offset=i)
        vals, secs, nb = [], 0.0, 0
        for i in range(args.steps):
            r, nb = oracle_layer_baseline(None, pool, fraction=1 / 8, offset=i)
            vals.append(r["n"][0])
            secs += r["n"][1]
    finally:
        pool.close()
    value = statistics.median(vals)
    desc = (f"1/8 of the layer per step ({nb} of its 120 256-row blocks, offset rotating), "
            f"oracle unpack + fp32 reconstruction + fp64 matvec, {cores} processes on {cpu_model()}")
    layer_b = 31_664_896
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / max(1, args.steps) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded; synth.config1)",
        "config": {"workload": workload(args.layer), "batch": 1, "layer_mode": args.layer, "sample": desc},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": desc,
                         "cpu_model": cpu_model()},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "us_per_layer_extrapolated": layer_b / (value * 1e9) * 1e6,
    }
    print(json.dumps(line))
    return 0


EXTRAS = {
    "gemm": ("up_proj_4096x12288_batch_sweep", lambda st: bench_gemm(st)),
    "moe": ("moe_128_experts", lambda st: bench_moe(st)),
    "qdq": ("qdq_forward_4096x4096", lambda st: bench_qdq(st)),
    "abs": ("abs_select_4096x4096", lambda st: bench_abs(st)),
    "encoder": ("encode_rows_4096x4096", lambda st: bench_encode_rows(st)),
}


def run_extras(names):
    """The listed extra measurements alone, on one GPU (one JSON line)."""
    import torch
    import bit_vector_quantized_sage_b200 as sage
    from bit_vector_quantized_sage_b200 import build as sage_build
    sage_build.build()
    sage.load()
    stream = torch.cuda.Stream()
    out = {}
    with torch.cuda.stream(stream):
        for n in names:
            key, fn = EXTRAS[n]
            out[key] = fn(stream)
    print(json.dumps({"extra": out}))
    return 0


def run_gpu(args):
    import torch
    import bit_vector_quantized_sage_b200 as sage
    from bit_vector_quantized_sage_b200 import build as sage_build
    world, rank, local = _dist()
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    if rank == 0 or not os.path.exists(sage_build.LIB):
        sage_build.build()
    if dist is not None:
        dist.barrier()
    sage.load()

    L, layers = build_layers()
    replicas = len(layers)
    one_layer_bytes, perm_bytes = layer_bytes(layers[0])
    stream = torch.cuda.Stream()
    torch.cuda.set_stream(stream)
    modes = {}
    for mode in ("fused", "stages", "grouped7"):
        modes[mode] = make_runners(mode, layers, L)
    fns, ws, inputs, outputs, launches = modes[args.layer]

    # ---- warm-up (eager, through the public API) ----
    with torch.cuda.stream(stream):
        for i in range(max(3, args.warmup)):
            fns[i % replicas](stream)
        torch.cuda.synchronize()
    assert sage.sage_query_status(ws) == sage.SAGE_OK

    # ---- timed region: one CUDA graph of K layers over rotating replicas ----
    with torch.cuda.stream(stream):
        g_all = capture(lambda st: [fns[k % replicas](st) for k in range(args.steps)], stream)
        g_all.replay()
        torch.cuda.synchronize()
    clocks = Clocks(local)
    clocks.start()
    time.sleep(0.3)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(stream)
    g_all.replay()
    end.record(stream)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    clk = clocks.stop()
    ms = max_over_ranks(start.elapsed_time(end), dist, "cuda")
    assert sage.sage_query_status(ws) == sage.SAGE_OK
    del g_all
    us_per_layer = ms * 1e3 / args.steps
    value = whole_job_gbs(world, one_layer_bytes, args.steps, ms)

    # ---- per-layer distribution of every layer mode (one graph per layer) ----
    layer_modes = {}
    with torch.cuda.stream(stream):
        for mode, (mf, mws, _, _, ml) in modes.items():
            t = per_call_us(mf, stream)
            assert sage.sage_query_status(mws) == sage.SAGE_OK
            med = float(np.median(t))
            layer_modes[mode] = {"launches_per_layer": ml, "us_per_layer": dist_summary(t),
                                 "gbs": round(one_layer_bytes / (med * 1e-6) / 1e9, 1),
                                 "hbm_frac": round(one_layer_bytes / (med * 1e-6) / 1e9 / _peaks()[0], 4)}
    for m in layer_modes.values():
        m["timing"] = "per layer: one CUDA graph over the rotating copies, median/p10/p90 over 12 replays"
    layer_modes["fused"]["what"] = ("the decoder layer as one launch: RMSNorm -> q|k|v, attention over one cached "
                                    "position -> o, residual + RMSNorm -> gate|up, SiLU * up -> down + residual")
    layer_modes["stages"]["what"] = "the four stages as four grouped launches (PDL-chained), synthetic stage inputs"
    layer_modes["grouped7"]["what"] = "the seven projections in one grouped launch, independent synthetic inputs"

    # ---- end to end through the public API with host buffers ----
    h_in = {k: torch.from_numpy(np.ascontiguousarray(v[1]).view(np.int16)).pin_memory() for k, v in inputs.items()}
    h_out = {k: torch.zeros(tuple(v.shape), dtype=torch.int16).pin_memory() for k, v in outputs.items()}
    h2d = sum(v.numel() * 2 for v in h_in.values())
    d2h = sum(v.numel() * 2 for v in h_out.values())
    e2e_steps = max(20, min(args.steps, 200))
    with torch.cuda.stream(stream):
        for k in range(3):
            fns[k % replicas](stream)
        torch.cuda.synchronize()
        e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e_start.record(stream)
        for k in range(e2e_steps):
            for n, hx in h_in.items():
                inputs[n][0].copy_(hx, non_blocking=True)
            fns[k % replicas](stream)
            for n, hy in h_out.items():
                hy.copy_(outputs[n], non_blocking=True)
            stream.synchronize()  # the host reads the step's result
        e_end.record(stream)
        torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e_start.elapsed_time(e_end) / e2e_steps, dist, "cuda")
    e2e_value = whole_job_gbs(world, one_layer_bytes, 1, e2e_ms)
    assert sage.sage_query_status(ws) == sage.SAGE_OK

    extra = {"layer_modes": layer_modes}
    if rank == 0 and world == 1 and not args.no_extra:
        with torch.cuda.stream(stream):
            for key, fn in EXTRAS.values():
                extra[key] = fn(stream)

    peak, peak_kind = _peaks()
    traffic, traffic_note = traffic_for(args.layer)
    achieved = one_layer_bytes / (us_per_layer * 1e-6) / 1e9
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        torch.cuda.synchronize()
        cores = host_cores()
        pool_1, pool_n = OraclePool(1), OraclePool(cores)
        try:
            r, nblk = oracle_layer_baseline(pool_1, pool_n)
            beside = oracle_beside(pool_1)
        finally:
            pool_1.close()
            pool_n.close()
        desc = (f"the whole layer ({nblk} 256-row blocks of the seven matrices): oracle unpack + fp32 reconstruction "
                f"+ fp64 matvec, one process per core on {cpu_model()}")
        cpu = {"value": r["n"][0], "unit": "GB/s", "cores": r["n"][2], "kind": "oracle", "sample": desc,
               "seconds": round(r["n"][1], 3), "cpu_model": cpu_model(),
               "single_core": {"value": r["1"][0], "unit": "GB/s", "cores": 1, "seconds": round(r["1"][1], 3)},
               "beside_other_workloads": beside}
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16",
        "data": "synthetic (seeded; synth.config1)",
        "config": {"workload": workload(args.layer),
                   "batch": 1, "layer_mode": args.layer, "what": layer_modes[args.layer]["what"],
                   "packed_bytes_per_layer": one_layer_bytes, "perm_bytes_per_layer": perm_bytes,
                   "l2": f"inputs larger than L2: {replicas} rotating copies of the packed layer "
                         f"({replicas * one_layer_bytes / 2**20:.0f} MiB)",
                   "parallelism": f"replicas x{world}"},
        "us_per_layer": us_per_layer,
        "us_per_layer_dist": layer_modes[args.layer]["us_per_layer"],
        "hbm_fraction": value / world / peak,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "peak_kind": peak_kind,
                     "frac_nominal": achieved / NOMINAL_HBM_GBS, "nominal_peak": NOMINAL_HBM_GBS,
                     "traffic": traffic, "traffic_note": traffic_note, "kernel": KERNEL,
                     "launches_per_step": launches,
                     "algorithmic_bytes_per_step": one_layer_bytes},
        "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "us_per_layer": e2e_ms * 1e3, "api": "public Python binding over the C ABI, eager calls"},
        "gpu_launches": args.steps * launches,
        "clocks": clk,
        "cpu_baseline": cpu,
        "extra": extra,
    }
    if rank == 0:
        print(json.dumps(line))
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="sage", choices=["sage", "reference"])
    ap.add_argument("--layer", default="fused", choices=["fused", "stages", "grouped7"],
                    help="how the layer's seven projections are launched (default: the fused decoder layer)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="skip the batch sweep and MoE measurements")
    ap.add_argument("--only-extra", default="",
                    help="comma list of extras to run alone (gemm, moe, qdq, abs, encoder), without the layer "
                         "measurement; prints {\"extra\": ...} (for profiling those kernels)")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    if args.only_extra:
        return run_extras(args.only_extra.split(","))
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
