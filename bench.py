#!/usr/bin/env python
"""Benchmark: batch-1 packed SAGE GEMV over a Qwen3-4B-shaped decoder layer on B200.

A step is one decoder layer's seven packed linears at batch 1, launched as its
four dependency stages (q|k|v, o, gate|up, down; one grouped GEMV launch each,
chained with programmatic dependent launch).  Inputs are synthetic (seeded, see
synth/), resident in HBM; every step reads a different copy of the layer's
packed planes so the working set (>= 4 x the 126 MB L2) comes from HBM.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Prints ONE JSON line (rank 0).  ``value`` is the whole-job throughput in GB/s of
packed bytes (codes + mu/delta + codebooks + x + y) per layer; ``us_per_layer``
is the device time of one layer.  ``--impl reference`` times the CPU oracle on a
bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "batch-1 packed VQ GEMV µs/layer and achieved HBM GB/s vs B200 peak"
WORKLOAD = "Qwen3-4B-shaped decoder layer, 7 packed linears (q,k,v,o,gate,up,down), hidden 2560, batch 1"
FALLBACK_HBM_GBS = 6650.0
L2_BYTES = 126 * 1024 * 1024


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as fh:
            d = json.load(fh)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


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


# ---------------------------------------------------------------------------
# Workload construction (product path only: synth + libsage)
# ---------------------------------------------------------------------------

def build_layer(replicas: int):
    import torch
    import synth
    import bit_vector_quantized_sage_b200 as sage
    L = synth.config1()
    base = {}
    for f in L.mats:
        f.perm = sage.sage_esg_permutation(L.energies[f.name])
        base[f.name] = sage.PackedMatrix.from_fields(f)
    layers = []
    for r in range(replicas):
        if r == 0:
            layers.append(base)
            continue
        layers.append({n: sage.PackedMatrix(m.d_out, m.d_in, m.log2K, m.main.clone(), m.meta.clone(),
                                            m.codebook.clone(), m.perm.clone() if m.perm is not None else None, n)
                       for n, m in base.items()})
    xs = {s[0]: torch.from_numpy(L.xs[s[0]].view(np.int16)).cuda() for s in synth.QWEN3_4B_STAGES}
    return L, layers, xs


def layer_bytes(mats, M=1):
    """Algorithmic bytes of one layer: packed planes + codebooks + x + y (perm excluded)."""
    tot = 0
    perm = 0
    for m in mats.values():
        tot += m.packed_bytes + (1 << m.log2K) * 16 + M * m.d_in * 2 + M * m.d_out * 2
        perm += m.d_in * 4 if m.perm is not None else 0
    return tot, perm


class LayerRunner:
    """Pre-marshalled grouped launches for one layer replica."""

    def __init__(self, mats, xs, ys, ws):
        import synth
        import bit_vector_quantized_sage_b200 as sage
        self.calls = []
        for stage in synth.QWEN3_4B_STAGES:
            ms = [mats[n] for n in stage]
            self.calls.append(sage.GroupedCall(ms, [xs[stage[0]]] * len(stage), [ys[n] for n in stage], 1, ws))

    def __call__(self, stream=None):
        for c in self.calls:
            c(stream)


class Clocks:
    """nvidia-smi sampling during the timed region."""

    def __init__(self, gpu_index: int):
        self.proc = None
        # SAGE_CLOCKS_DIR keeps the raw samples (one CSV per rank); default: a temp file
        d = os.environ.get("SAGE_CLOCKS_DIR")
        self.path = (os.path.join(d, f"clocks_rank{gpu_index}.csv") if d and os.path.isdir(d)
                     else os.path.join(tempfile.gettempdir(), f"sage_clocks_{os.getpid()}_{gpu_index}.csv"))
        self.gpu = gpu_index

    def start(self):
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={q}",
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
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            p = [x.strip() for x in line.split(",")]
            if len(p) < 9:
                continue
            try:
                sm.append(float(p[1]))
                mx = float(p[2])
            except ValueError:
                continue
            for nm, v in zip(names, p[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": mx,
                "samples": len(sm), "reasons": sorted(reasons)}


def _traffic_for(kernel_src_hash: str):
    p = os.path.join(ROOT, "profiles", "gemv_traffic.json")
    try:
        d = json.load(open(p))
    except Exception:
        return None, None
    if d.get("source_sha256") != kernel_src_hash:
        return None, d.get("source_sha256")
    return d.get("traffic_bytes_per_launch"), d.get("source_sha256")


def _kernel_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "bit_vector_quantized_sage_b200", "csrc")
    for n in ("sage_gemv.cu", "sage_device.cuh"):
        h.update(open(os.path.join(csrc, n), "rb").read())
    return h.hexdigest()


def cpu_oracle_sample(rows_per_matrix: int = 256, seconds_cap: float = 60.0):
    """Times the CPU oracle (unpack + fp32 reconstruction + fp64 matvec) on the first
    ``rows_per_matrix`` rows of each of the layer's seven matrices, single-threaded.
    Returns (GB/s of packed bytes, sample description, cores used)."""
    import oracle
    import synth
    import bit_vector_quantized_sage_b200 as sage
    L = synth.config1()
    tot_bytes, tot_s = 0, 0.0
    for f in L.mats:
        f.perm = sage.sage_esg_permutation(L.energies[f.name])
        x = L.xs[[s for s in synth.QWEN3_4B_STAGES if f.name in s][0][0]]
        R = min(rows_per_matrix, f.d_out)
        # row-octet slice of the planes for the first R rows
        sub = synth.Fields(R, f.d_in, f.log2K, f.signs[:R], f.idx[:R], f.q[:R], f.mu[:R], f.delta[:R],
                           f.codebook, f.perm, f.name)
        m_sub, t_sub = sage.sage_pack(R, f.d_in, f.log2K, sub.signs, sub.idx, sub.q, sub.mu, sub.delta)
        t0 = time.perf_counter()
        u = oracle.unpack(R, f.d_in, f.log2K, m_sub, t_sub)
        g = synth.Fields(R, f.d_in, f.log2K, u["signs"], u["idx"], u["q"], u["mu"], u["delta"], f.codebook, f.perm)
        oracle.gemv(g, x)
        tot_s += time.perf_counter() - t0
        mb, tb = sage.sage_packed_sizes(R, f.d_in, f.log2K)
        tot_bytes += mb + tb + (1 << f.log2K) * 16 + f.d_in * 2 + R * 2
        if tot_s > seconds_cap:
            break
    desc = (f"first {rows_per_matrix} rows of each of the 7 layer matrices" if rows_per_matrix < 9728
            else "the whole layer, all 7 matrices") + " (unpack + reconstruct + fp64 matvec, single thread)"
    return tot_bytes / tot_s / 1e9, desc, 1, tot_s


def _peak_tflops():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as fh:
            d = json.load(fh)
        return float(d["bf16_tflops"]), "measured (bf16 burst; fp16 dense has the same nominal rate)"
    except Exception:
        return 1590.0, "fallback"


def _timed_calls(fn, stream, reps, flush):
    """Median device time (ms) of one fn call with L2 flushed before each call.
    The call is captured once in a CUDA graph; the flush is enqueued first, so
    the host side of the replay overlaps it and the events bracket device work
    only."""
    import torch
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        fn(torch.cuda.current_stream())
    g.replay()
    times = []
    for _ in range(reps):
        flush.fill_(1)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        g.replay()
        e1.record(stream)
        e1.synchronize()
        times.append(e0.elapsed_time(e1))
    del g
    return statistics.median(times)


def bench_gemm(stream, flush, reps=20):
    """Config 3: 4096 -> 12288, (K,V) = (32,5); batch 1-8 through the GEMV
    kernel, 16-128 through the tcgen05 path (sage_gemm).  Per batch: device us,
    TFLOP/s against the measured dense fp16 peak and GB/s of packed bytes."""
    import torch
    import synth
    import bit_vector_quantized_sage_b200 as sage
    f, _ = synth.config3(1)
    A = sage.PackedMatrix.from_fields(f)
    peak, kind = _peak_tflops()
    hbm, _ = _peaks()
    out = []
    for M in (1, 2, 4, 8, 16, 32, 64, 128):
        _, xb = synth.config3(M)
        x = torch.from_numpy(xb.view(np.int16)).cuda()
        y = torch.zeros((M, f.d_out), dtype=torch.int16, device="cuda")
        ws = sage.Workspace(sage.sage_workspace_size(sage.SAGE_OP_GEMM, A, M))
        fn = lambda st: sage.sage_gemm(A, x, M, y, ws, st)
        for _ in range(3):
            fn(stream)
        ms = _timed_calls(fn, stream, reps, flush)
        assert sage.sage_query_status(ws) == sage.SAGE_OK
        flops = 2.0 * M * f.d_out * f.d_in
        nbytes = A.packed_bytes + 32 * 16 + M * f.d_in * 2 + M * f.d_out * 2
        tf = flops / (ms * 1e-3) / 1e12
        out.append({"M": M, "path": "gemv" if M <= 8 else "tcgen05", "us": round(ms * 1e3, 2),
                    "tflops": round(tf, 1), "tensor_frac": round(tf / peak, 4),
                    "gbs": round(nbytes / (ms * 1e-3) / 1e9, 1), "hbm_frac": round(nbytes / (ms * 1e-3) / 1e9 / hbm, 4)})
    return {"workload": "4096->12288 up-projection, (K,V)=(32,5), L2 flushed before each call",
            "peak_tflops": peak, "peak_kind": kind, "points": out}


def bench_moe(stream, flush, reps=20):
    """Config 4: 128 experts, gate 2048 -> 768 and down 768 -> 2048, top-8,
    T tokens; one sage_moe_gemv call per projection."""
    import torch
    import synth
    import bit_vector_quantized_sage_b200 as sage
    hbm, _ = _peaks()
    out = []
    for proj in (0, 2):
        packed = None
        for T in (1, 4, 16):
            spec = synth.config4(T)
            if packed is None:
                packed = [sage.PackedMatrix.from_fields(spec.expert(e, proj)) for e in range(synth.MOE_EXPERTS)]
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
            fn = lambda st: sage.sage_moe_gemv(packed, pe, xr, n_pairs, x, y, ws, st)
            for _ in range(3):
                fn(stream)
            ms = _timed_calls(fn, stream, reps, flush)
            assert sage.sage_query_status(ws) == sage.SAGE_OK
            active = np.unique(spec.routes)
            nbytes = sum(packed[e].packed_bytes + (1 << packed[e].log2K) * 16 for e in active)
            nbytes += xb.nbytes + n_pairs * d_out * 2
            out.append({"proj": synth.MOE_PROJ[proj][0], "T": T, "experts": int(active.size),
                        "us": round(ms * 1e3, 2), "gbs": round(nbytes / (ms * 1e-3) / 1e9, 1),
                        "hbm_frac": round(nbytes / (ms * 1e-3) / 1e9 / hbm, 4)})
    return {"workload": "128 experts, top-8, one projection per call, L2 flushed before each call", "points": out}


def run_reference(args):
    ws, rank, _ = _dist()
    if rank != 0:
        return 0
    for _ in range(args.warmup):
        cpu_oracle_sample(rows_per_matrix=32)
    vals, secs = [], 0.0
    for _ in range(args.steps):
        v, desc, cores, s = cpu_oracle_sample(rows_per_matrix=256)
        vals.append(v)
        secs += s
    value = statistics.median(vals)
    layer_b = 31_682_560  # packed layer bytes scale: reported per-layer time from the GB/s
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": ws,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": secs / max(1, args.steps) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded; see synth/config1)",
        "config": {"workload": WORKLOAD, "batch": 1, "sample": desc},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "us_per_layer_extrapolated": layer_b / (value * 1e9) * 1e6,
    }
    print(json.dumps(line))
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

    L, layers1, xs = build_layer(1)
    one_layer_bytes, perm_bytes = layer_bytes(layers1[0])
    replicas = max(2, int(np.ceil(4 * L2_BYTES / one_layer_bytes)) + 1)
    _, layers, xs = build_layer(replicas)
    ys = {f.name: torch.zeros((1, f.d_out), dtype=torch.int16, device="cuda") for f in L.mats}
    ws = sage.Workspace(max(sage.sage_workspace_size(sage.SAGE_OP_GROUPED, [layers[0][n] for n in st], 1)
                            for st in __import__("synth").QWEN3_4B_STAGES))
    runners = [LayerRunner(lay, xs, ys, ws) for lay in layers]
    stream = torch.cuda.Stream()
    torch.cuda.set_stream(stream)

    # ---- warm-up (eager) ----
    for i in range(max(3, args.warmup)):
        runners[i % replicas](stream)
    torch.cuda.synchronize()
    assert sage.sage_query_status(ws) == sage.SAGE_OK

    def capture(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            fn(torch.cuda.current_stream())
        return g

    def time_graph(g, reps=1):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1)

    import synth
    n_stage = len(synth.QWEN3_4B_STAGES)
    stage_bytes = []
    for stage in synth.QWEN3_4B_STAGES:
        stage_bytes.append(sum(layers[0][n].packed_bytes + (1 << layers[0][n].log2K) * 16 +
                               layers[0][n].d_in * 2 + layers[0][n].d_out * 2 for n in stage))

    # ---- per-stage kernel time: one graph = the stage launched once per replica ----
    stage_avg = []
    with torch.cuda.stream(stream):
        for s_i in range(n_stage):
            g = capture(lambda st: [runners[r].calls[s_i](st) for r in range(replicas)])
            for _ in range(3):
                g.replay()
            ms_s = time_graph(g, reps=max(1, 200 // replicas))
            stage_avg.append(ms_s / (max(1, 200 // replicas) * replicas))
            del g

    # ---- timed region: one graph holding K layers back to back (rotating replicas) ----
    with torch.cuda.stream(stream):
        g_all = capture(lambda st: [runners[k % replicas](st) for k in range(args.steps)])
        for _ in range(max(3, args.warmup // max(1, args.steps) + 1)):
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
    us_per_layer = ms * 1e3 / args.steps
    value = whole_job_gbs(world, one_layer_bytes, args.steps, ms)
    del g_all

    # ---- end to end through the public API with host buffers (graph per step) ----
    h_x = {k: torch.from_numpy(L.xs[k].view(np.int16)).pin_memory() for k in xs}
    h_y = {n: torch.zeros(tuple(ys[n].shape), dtype=torch.int16).pin_memory() for n in ys}
    h2d = sum(v.numel() * 2 for v in h_x.values())
    d2h = sum(v.numel() * 2 for v in h_y.values())
    e2e_steps = max(20, args.steps // 2)

    def e2e_step(st, r):
        for n, hx in h_x.items():
            xs[n].copy_(hx, non_blocking=True)
        runners[r](st)
        for n, hy in h_y.items():
            hy.copy_(ys[n], non_blocking=True)

    with torch.cuda.stream(stream):
        g_e2e = [capture(lambda st, r=r: e2e_step(st, r)) for r in range(replicas)]
        for r in range(replicas):
            g_e2e[r].replay()
        torch.cuda.synchronize()
        e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e_start.record(stream)
        for k in range(e2e_steps):
            g_e2e[k % replicas].replay()
            stream.synchronize()          # the host reads the step's result
        e_end.record(stream)
        torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e_start.elapsed_time(e_end) / e2e_steps, dist, "cuda")
    e2e_value = whole_job_gbs(world, one_layer_bytes, 1, e2e_ms)
    del g_e2e

    extra = {}
    if rank == 0 and not args.no_extra:
        flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device="cuda")
        with torch.cuda.stream(stream):
            extra["gemm_config3"] = bench_gemm(stream, flush)
            extra["moe_config4"] = bench_moe(stream, flush)
        del flush

    peak, peak_kind = _peaks()
    achieved = sum(stage_bytes) / (sum(stage_avg) * 1e-3) / 1e9
    traffic, _ = _traffic_for(_kernel_hash())
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, desc, cores, secs = cpu_oracle_sample(rows_per_matrix=args.cpu_rows)
        cpu = {"value": v, "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": desc,
               "seconds": round(secs, 2)}
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16",
        "data": "synthetic (seeded; see synth/config1)",
        "config": {"workload": WORKLOAD, "batch": 1, "stages": "q|k|v, o, gate|up, down (4 grouped launches)",
                   "packed_bytes_per_layer": one_layer_bytes, "perm_bytes_per_layer": perm_bytes,
                   "l2": f"inputs larger than L2: {replicas} rotating copies of the packed layer "
                         f"({replicas * one_layer_bytes / 2**20:.0f} MiB)",
                   "parallelism": f"replicas x{world}"},
        "us_per_layer": us_per_layer,
        "hbm_fraction": value / world / peak,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic, "peak_kind": peak_kind,
                     "kernel": "gemv_kernel<1> (grouped packed GEMV)",
                     "stage_us": [round(s * 1e3, 3) for s in stage_avg],
                     "stage_bytes": stage_bytes},
        "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "us_per_layer": e2e_ms * 1e3},
        "gpu_launches": args.steps * n_stage,
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
    ap.add_argument("--cpu-rows", type=int, default=1 << 30,
                    help="rows per matrix in the CPU-oracle baseline sample (default: the whole layer)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="skip the batch sweep and MoE measurements")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)
    return run_gpu(args)


if __name__ == "__main__":
    sys.exit(main())
