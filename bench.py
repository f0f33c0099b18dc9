#!/usr/bin/env python
"""Benchmark of the fused QK-RMSNorm + causal 3D RoPE + KV-cache append step on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload chunk720p|chunk480p|longhorizon] [--trig table|onthefly]
                    [--eager] [--path auto|registers|tma]

One step is the whole 720P sequence of a Wan-14B-shaped backbone (21 latent frames of
45x80, 40 heads of 128, bf16) in seven chunk calls of 10800 tokens, start frames 0, 3,
..., 18, appended into a 75600-token KV cache -- the Self-Forcing chunk loop of
"Accelerating Video Generation Inference with Sequential-Parallel 3D Positional Encoding
Using a Global Time Index" (Section 3.3.2), at the 720P size.  Inputs are seeded
synthetic tensors (N(0,1) rounded to bf16; RMSNorm weights U(0.5, 1.5)); every chunk has
its own buffers and each launch streams 663.6 MB, well above the 126 MB L2, so no L2
flush is needed between launches.

One step's seven launches are captured once in a CUDA graph and replayed (the chunk loop
of an inference server); --eager launches them one by one instead.

Under torchrun every rank runs the same job on its own GPU with its own seed (weak
scaling, no collective on the data path); the reported time is the maximum over ranks.
Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import csv
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time
from concurrent.futures import ThreadPoolExecutor

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from rotary_position_encoding_b200 import workloads as wl  # noqa: E402

WORKLOADS = {
    "chunk720p": wl.chunk_720p,
    "chunk480p": wl.chunk_480p,
    "longhorizon": wl.long_horizon,
}
METRIC = "fused norm+3D-RoPE+KV-append tokens/s and HBM GB/s (% of B200 peak), 1 GPU"
# the step kernels' sources and their launch planning (the per-launch traffic recorded in
# profiles/traffic.json holds for these only)
KERNEL_SOURCES = [os.path.join(ROOT, "rotary_position_encoding_b200", "csrc", f)
                  for f in ("rope3d_kernels.cuh", "rope3d_tma.cuh", "rope3d.cu")]
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "traffic.json")


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="chunk720p")
    ap.add_argument("--trig", choices=["table", "onthefly"], default="table")
    ap.add_argument("--pairing", choices=["adjacent", "half"], default="adjacent",
                    help="pairing of a head's elements (half: rotate_half, as in M-RoPE)")
    ap.add_argument("--cache-layout", choices=["token", "head"], default="token",
                    help="KV cache [B][C][N][D] (token) or [B][N][C][D] (head)")
    ap.add_argument("--cache-dtype", choices=["same", "fp8", "nvfp4"], default="same",
                    help="KV cache in the input dtype or FP8 E4M3 codes with per-head scales")
    ap.add_argument("--path", choices=["auto", "registers", "tma"], default="auto",
                    help="kernel path of the fused step (auto: the bulk-copy ring when it "
                         "fits in shared memory)")
    ap.add_argument("--sp", type=int, default=0,
                    help="sequence-parallel step with the all-to-all folded in: each chunk is "
                         "cut into SP even token slices (the ranks of one node, emulated on "
                         "this GPU as SP launches) whose heads go to SP destination buffers")
    ap.add_argument("--qkv", action="store_true",
                    help="the QKV-projection-fed step: token rows x [n, N*128] through the "
                         "tcgen05 projection (V appended by its epilogue), then the step")
    ap.add_argument("--gemm-form", type=int, choices=[0, 1, 2], default=0,
                    help="--qkv: projection kernel form (1: one CTA per tile, 2: 2-CTA pairs, "
                         "0: the library default, 2)")
    ap.add_argument("--eager", action="store_true",
                    help="launch every chunk call from Python and time each launch with its "
                         "own CUDA event pair (default: capture one step -- all its chunk "
                         "calls -- in a CUDA graph and replay it; the per-launch time is then "
                         "the step time over its launches)")
    ap.add_argument("--chunks", type=int, default=0,
                    help="use only the first CHUNKS chunk calls per step (profiling captures "
                         "of a smaller case; 0 = the whole step)")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the other workloads measured after the default 720P headline "
                         "(480P chunk and its 4-rank slices, whole 480P vs 8 slices, long "
                         "horizon, FP8 and NVFP4 caches, 8-rank sequence-parallel step and "
                         "the exchange after attention, the rotation alone, QKV projection "
                         "and the step it feeds)")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="upper bound on the oracle's timed CPU work")
    return ap.parse_args(argv)


def workload_for(args) -> wl.Workload:
    w = WORKLOADS[args.workload]()
    if args.chunks:
        w.chunks = w.chunks[: args.chunks]
        w.name += f"_first{len(w.chunks)}chunks"
    return w


# ---------------------------------------------------------------- distributed plumbing

class Dist:
    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local_rank = int(os.environ.get("LOCAL_RANK", "0"))
        self.pg = None
        self.backend = None

    def init(self, backend: str):
        self.backend = backend
        if self.world > 1:
            import datetime

            import torch.distributed as dist
            kw = {}
            if backend == "nccl":
                import torch
                kw["device_id"] = torch.device("cuda", self.local_rank)
            dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120),
                                    **kw)
            self.pg = dist

    def barrier(self):
        if self.pg is not None:
            if self.backend == "nccl":
                self.pg.barrier(device_ids=[self.local_rank])
            else:
                self.pg.barrier()

    def max(self, x: float, device) -> float:
        if self.pg is None:
            return x
        import torch
        t = torch.tensor([x], dtype=torch.float64, device=device)
        self.pg.all_reduce(t, op=self.pg.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.pg is not None:
            self.pg.destroy_process_group()


# ---------------------------------------------------------------- inputs

def make_inputs(w: wl.Workload, seed_offset: int):
    """Host tensors of every chunk call of one step (bf16 bit patterns), generated in
    parallel threads (each tensor has its own seeded generator)."""
    n = w.tokens_per_chunk
    shape = (w.B, n, w.N, wl.HEAD_DIM)
    jobs = [(ci, t) for ci in range(len(w.chunks)) for t in range(3)]

    def gen(job):
        ci, t = job
        rng = wl.rng_for(w.seed + seed_offset, ci, t)
        return wl.normal_tensor(rng, shape, w.dtype)

    with ThreadPoolExecutor(max_workers=min(len(jobs), os.cpu_count() or 1)) as ex:
        arrays = list(ex.map(gen, jobs))
    return [tuple(arrays[3 * ci + t] for t in range(3)) for ci in range(len(w.chunks))]


# ---------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons for one GPU."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None
        self.rows = None
        self.t_start = self.t_end = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu=timestamp,{self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50", "-f", self.path],
                stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def mark(self, which: str):
        setattr(self, "t_" + which, time.time())

    def stop(self):
        """Stop sampling; the clock record of the timed region (marks "start" and "end")."""
        if self.proc is None:
            self.rows = None
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.1)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.rows = []
        with open(self.path) as f:
            for rec in csv.reader(f):
                if len(rec) >= 10:
                    self.rows.append([x.strip() for x in rec])
        os.unlink(self.path)
        return self.window(self.t_start, self.t_end, "timed region")

    @staticmethod
    def _stamp(r):
        try:
            return time.mktime(time.strptime(r[0].split(".")[0], "%Y/%m/%d %H:%M:%S")) + \
                float("0." + r[0].split(".")[1]) if "." in r[0] else 0.0
        except ValueError:
            return None

    def window(self, t0, t1, name="window"):
        """Median SM clock, maximum clock and throttle reasons of the samples taken between
        host times t0 and t1 (all samples if none fall inside)."""
        if self.rows is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = self.rows
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        window = "whole run"
        if t0 is not None and t1 is not None:
            inside = [r for r in rows if (self._stamp(r) is not None
                                          and t0 - 0.06 <= self._stamp(r) <= t1 + 0.06)]
            window = name
            if not inside:
                inside, window = rows, f"whole run ({name} shorter than the sampling period)"
            rows = inside
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        sm = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        mx = [float(r[3]) for r in rows if r[3].replace(".", "").isdigit()]
        reasons = sorted({names[j] for r in rows for j in range(4)
                          if r[6 + j].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows), "window": window}


# ---------------------------------------------------------------- the GPU arm

def kernel_source_hash() -> str:
    import hashlib
    h = hashlib.sha256()
    for p in KERNEL_SOURCES:
        with open(p, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def recorded_traffic(workload_name: str, trig: str):
    """Per-launch DRAM bytes from the committed ncu summary, if it was taken on the
    current kernel source; else None."""
    try:
        with open(PROFILE_TRAFFIC) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    entry = rec.get(workload_name if trig is None else f"{workload_name}/{trig}")
    if not entry or entry.get("kernel_source_sha256_16") != kernel_source_hash():
        return None
    return entry.get("dram_bytes_per_launch")


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": 6650.0}, "fallback"


def run_ours(args, dist: Dist):
    import torch

    from rotary_position_encoding_b200 import rope3d

    torch.cuda.set_device(dist.local_rank)
    device = torch.device("cuda", dist.local_rank)
    dist.init("nccl")
    w = workload_for(args)
    trig = rope3d.ROPE3D_TRIG_TABLE if args.trig == "table" else rope3d.ROPE3D_TRIG_ONTHEFLY
    n = w.tokens_per_chunk
    tokens_per_step = w.B * n * len(w.chunks)
    bytes_per_launch = w.algorithmic_bytes(n)
    if args.cache_dtype == "fp8":
        # q, k, v read and q_out written in the input dtype; K and V cache rows one byte per
        # element plus one fp32 scale per head each
        e = w.elem_bytes
        bytes_per_launch = w.B * n * (w.dim * (4 * e + 2) + 2 * 4 * w.N)
    elif args.cache_dtype == "nvfp4":
        # K and V cache rows half a byte per element plus one E4M3 byte per 16 elements
        e = w.elem_bytes
        bytes_per_launch = w.B * n * (w.dim * 4 * e + 2 * (w.dim // 2 + w.dim // 16))

    host = make_inputs(w, seed_offset=dist.rank)
    wq, wk = wl.norm_weights(w.seed, w.dim)
    wq_d = torch.from_numpy(wq).to(device)
    wk_d = torch.from_numpy(wk).to(device)
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32

    def dev_tensor(a):
        if w.dtype == "bf16":
            return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)
        return torch.from_numpy(a).to(device)

    inputs = [tuple(dev_tensor(a) for a in chunk) for chunk in host]
    q_out = [torch.empty_like(c[0]) for c in inputs]
    pairing = rope3d.ROPE3D_PAIRING_HALF if args.pairing == "half" else rope3d.ROPE3D_PAIRING_ADJACENT
    layout = rope3d.ROPE3D_CACHE_HEAD_MAJOR if args.cache_layout == "head" else rope3d.ROPE3D_CACHE_TOKEN_MAJOR
    cache_shape = ((w.B, w.cache_tokens, w.N, wl.HEAD_DIM) if args.cache_layout == "token"
                   else (w.B, w.N, w.cache_tokens, wl.HEAD_DIM))
    fp8 = args.cache_dtype == "fp8"
    fp4 = args.cache_dtype == "nvfp4"
    if fp4:
        cache_shape = cache_shape[:3] + (wl.HEAD_DIM // 2,)
    quant = fp8 or fp4
    k_cache = torch.zeros(cache_shape, dtype=torch.uint8 if quant else tdt, device=device)
    v_cache = torch.zeros(cache_shape, dtype=torch.uint8 if quant else tdt, device=device)
    sshape = cache_shape[:3] + ((wl.HEAD_DIM // 16,) if fp4 else ())
    sdtype = torch.uint8 if fp4 else torch.float32
    k_scale = torch.zeros(sshape, dtype=sdtype, device=device) if quant else None
    v_scale = torch.zeros(sshape, dtype=sdtype, device=device) if quant else None
    max_t = max(c.frame_offset for c in w.chunks) + w.T
    tables = rope3d.rope3d_tables_init(max_t=max_t, max_h=w.H, max_w=w.W)
    stream = torch.cuda.current_stream(device)
    rope3d.rope3d_testing_force_path({"auto": rope3d.ROPE3D_PATH_AUTO,
                                      "registers": rope3d.ROPE3D_PATH_REGISTERS,
                                      "tma": rope3d.ROPE3D_PATH_TMA}[args.path])

    P = args.sp
    if P:
        if w.N % P or n % P or quant or args.pairing != "adjacent":
            raise SystemExit("--sp needs heads and tokens divisible by SP, adjacent pairing "
                             "and a same-dtype cache")
        hl = w.N // P
        dshape = ((w.B, w.cache_tokens, hl, wl.HEAD_DIM) if args.cache_layout == "token"
                  else (w.B, hl, w.cache_tokens, wl.HEAD_DIM))
        sp_q = [torch.empty((w.B, n, hl, wl.HEAD_DIM), dtype=tdt, device=device)
                for _ in range(P)]
        sp_k = [torch.zeros(dshape, dtype=tdt, device=device) for _ in range(P)]
        sp_v = [torch.zeros(dshape, dtype=tdt, device=device) for _ in range(P)]
        k_cache = v_cache = None
        # each emulated rank reads its own slice of the chunk's rows
        sp_inputs = [[tuple(x[:, r * (n // P):(r + 1) * (n // P)].contiguous() for x in c)
                      for r in range(P)] for c in inputs]
        inputs = None

    def step(events=None):
        j = 0
        for ci, chunk in enumerate(w.chunks):
            for r in range(max(P, 1)):
                if events is not None:
                    events[2 * j].record(stream)
                if P:
                    q, k, v = sp_inputs[ci][r]
                    a = chunk.token_begin + r * (n // P)
                    rope3d.rope3d_qk_norm_rope_append_sp(
                        q, k, v, a, a + n // P, chunk.frame_offset, w.T, w.H, w.W, wq_d, wk_d,
                        w.eps, sp_q, sp_k, sp_v, chunk.slot, tables, trig, layout,
                        q_row0=chunk.token_begin, stream=stream)
                else:
                    q, k, v = inputs[ci]
                    rope3d.rope3d_qk_norm_rope_append_ex(
                        q, k, v, q_out[ci], chunk.token_begin, chunk.token_end,
                        chunk.frame_offset, w.T, w.H, w.W, wq_d, wk_d, w.eps, k_cache, v_cache,
                        chunk.slot, tables, trig, pairing, layout, k_scale, v_scale, stream=stream)
                if events is not None:
                    events[2 * j + 1].record(stream)
                j += 1

    clocks = ClockSampler(dist.local_rank) if dist.rank == 0 else None
    if clocks:
        clocks.start()
        time.sleep(0.3)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    # per-launch events of every timed launch (the kernel's own duration) and the region
    n_launch = len(w.chunks) * max(P, 1)
    if P:
        bytes_per_launch //= P
    graph = None
    if (not args.eager):
        side = torch.cuda.Stream(device)
        side.wait_stream(stream)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.stream(side):
            with torch.cuda.graph(graph, stream=side):
                stream = torch.cuda.current_stream(device)
                step()
        stream = torch.cuda.current_stream(device)
        graph.replay()
        torch.cuda.synchronize()
        per_step_events = []
    else:
        per_step_events = [[torch.cuda.Event(enable_timing=True) for _ in range(2 * n_launch)]
                           for _ in range(args.steps)]
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize()
    if clocks:
        clocks.mark("start")
    start.record(stream)
    for s in range(args.steps):
        if graph is not None:
            graph.replay()
        else:
            step(per_step_events[s])
    end.record(stream)
    torch.cuda.synchronize()
    if clocks:
        clocks.mark("end")
    dist.barrier()
    elapsed_ms = start.elapsed_time(end)
    if graph is not None:
        launch_ms = [elapsed_ms / (args.steps * n_launch)]
    else:
        launch_ms = [ev[2 * j].elapsed_time(ev[2 * j + 1]) for ev in per_step_events
                     for j in range(n_launch)]
    headline_path = rope3d.rope3d_testing_last_path()
    configs = None
    if (not args.no_configs and dist.world == 1 and graph is not None and not P
            and args.workload == "chunk720p" and not args.chunks
            and (args.trig, args.pairing, args.cache_layout, args.cache_dtype, args.path)
            == ("table", "adjacent", "token", "same", "auto")):
        graph = None
        configs = run_configs(torch, rope3d, device, stream, clocks, measured_peaks()[0],
                              (w, inputs, q_out, wq_d, wk_d, tables))
    clock_info = clocks.stop() if clocks else None
    if configs is not None:
        # each workload's clock record, from the samples inside its own timed replays
        for entry in [e for e in configs.values()] + [e["whole"] for e in configs.values()
                                                       if "whole" in e]:
            w_ = entry.get("clocks")
            if isinstance(w_, dict) and "window" in w_:
                entry["clocks"] = (clocks.window(*w_["window"], name=w_["name"]) if clocks
                                   else None)

    elapsed_ms = dist.max(elapsed_ms, device)
    avg_launch_ms = dist.max(statistics.fmean(launch_ms), device)
    total_tokens = tokens_per_step * args.steps * dist.world
    value = total_tokens / (elapsed_ms / 1e3)

    kernel_used = {rope3d.ROPE3D_PATH_TMA: "rope3d::qk_norm_rope_tma_kernel",
                   rope3d.ROPE3D_PATH_REGISTERS: "rope3d::qk_norm_rope_kernel"}.get(
        headline_path, "unknown")
    if P:
        kernel_used += " (head-scatter stores)"
    device_status = rope3d.rope3d_check_device_status(tables)
    if device_status != rope3d.ROPE3D_OK:
        raise RuntimeError("a kernel wait timed out during the benchmark")
    e2e = None
    if not args.no_e2e and ((args.pairing, args.cache_layout, args.cache_dtype) != (
            "adjacent", "token", "same") or P):
        args.no_e2e = True  # the e2e leg runs the default layout only
    if not args.no_e2e:
        e2e = run_e2e(args, w, host, wq_d, wk_d, tables, trig, device, dist, rope3d, torch)

    del per_step_events
    graph = None
    tables.close()
    dist.close()
    if dist.rank != 0:
        return None

    peaks, peak_kind = measured_peaks()
    achieved_gbs = bytes_per_launch / (avg_launch_ms / 1e3) / 1e9
    roofline = {
        "bound": "hbm",
        "achieved": round(achieved_gbs, 1),
        "peak": peaks["hbm_gbs"],
        "unit": "GB/s",
        "frac": round(achieved_gbs / peaks["hbm_gbs"], 4),
        "traffic": recorded_traffic(w.name + (f"/{args.trig}/sp{P}" if P else ""),
                                    args.trig if not P else None),
        "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured"
        else "fallback 6.65 TB/s",
        "kernel": kernel_used,
        "algorithmic_bytes_per_launch": bytes_per_launch,
        "avg_launch_us": round(avg_launch_ms * 1e3, 2),
        "launch_timing": "step time / launches (graph replay)" if (not args.eager)
        else "CUDA event pair around every timed launch",
    }
    line = {
        "metric": METRIC,
        "value": round(value, 1),
        "unit": "tokens/s",
        "n_gpus": dist.world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(elapsed_ms / args.steps, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": w.dtype,
        "data": "synthetic (seeded N(0,1) bf16 q/k/v, U(0.5,1.5) fp32 norm weights)",
        "config": {
            "workload": w.name,
            "grid_per_chunk": [w.T, w.H, w.W],
            "chunks_per_step": len(w.chunks),
            "tokens_per_step": tokens_per_step,
            "batch": w.B,
            "heads": w.N,
            "head_dim": wl.HEAD_DIM,
            "cache_tokens": w.cache_tokens,
            "trig": args.trig,
            "kernel_path": args.path,
            "pairing": args.pairing,
            "cache_layout": args.cache_layout,
            "cache_dtype": args.cache_dtype,
            "launch": "CUDA graph of one step, replayed" if (not args.eager)
            else "eager, one C-ABI call per chunk",
            "l2": "no flush: inputs larger than L2 (each launch streams "
                  f"{bytes_per_launch / 1e6:.1f} MB from its own buffers)",
            "parallelism": f"replicas x{dist.world} (independent streams, no collective)",
            "sequence_parallel": (f"{P} ranks emulated on one GPU: {P} launches per chunk over "
                                  f"even token slices, heads stored to {P} local destination "
                                  f"buffers ({w.N // P} heads each)") if P else None,
        },
        "hbm_gbs": round(bytes_per_launch * n_launch * args.steps * dist.world
                         / (elapsed_ms / 1e3) / 1e9, 1),
        "roofline": roofline,
        "gpu_launches": n_launch * args.steps,
        "clocks": clock_info,
        "e2e": e2e,
    }
    if configs is not None:
        line["configs"] = configs
    if not args.no_cpu_baseline and dist.world == 1:
        line["cpu_baseline"] = cpu_baseline(w, host, args.cpu_seconds)
    return line


def graph_launch_us(torch, step, n_launch, stream, budget_ms=250.0):
    """Capture step() (n_launch kernel launches) in a CUDA graph, replay it for about
    budget_ms after warm-up, and return (mean device time per launch in us, host start and
    end time of the timed replays)."""
    step()
    torch.cuda.synchronize()
    side = torch.cuda.Stream(stream.device)
    side.wait_stream(stream)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(graph, stream=side):
            step()
    torch.cuda.synchronize()
    a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    for _ in range(3):
        graph.replay()
    a.record(stream)
    graph.replay()
    e.record(stream)
    torch.cuda.synchronize()
    reps = max(5, int(budget_ms / max(a.elapsed_time(e), 1e-3)))
    t0 = time.time()
    a.record(stream)
    for _ in range(reps):
        graph.replay()
    e.record(stream)
    torch.cuda.synchronize()
    t1 = time.time()
    us = a.elapsed_time(e) * 1e3 / (reps * n_launch)
    del graph
    return us, (t0, t1)


def run_configs(torch, rope3d, device, stream, clocks, peaks, headline):
    """The other workloads of the step, each measured like the headline (graph replay of
    one step, device time per launch, clocks of its own window): the 480P chunk loop and
    its 4-rank sequence-parallel slices, the whole 480P sequence against its 8 slices
    (with a bit-identity check), the batch-2 long-horizon rollout with table and
    on-the-fly cos/sin, the 720P step with FP8 and NVFP4 caches (on the headline's
    inputs), its 8-rank sequence-parallel slices and the exchange after attention, the
    rotation alone, the QKV projection on the tensor cores with cuBLAS on the same GEMM
    beside it, and the step fed by the projection.  Inputs of the extra workloads are drawn on
    the device (torch.randn with a fixed seed, rounded to bf16; norm weights U(0.5, 1.5))."""
    hbm = peaks["hbm_gbs"]
    out = {}
    gen = torch.Generator(device=device)

    def randn_bf16(shape, seed):
        gen.manual_seed(seed)
        return torch.randn(shape, generator=gen, device=device).to(torch.bfloat16)

    def weights(dim, seed):
        gen.manual_seed(seed)
        return (torch.rand(dim, generator=gen, device=device) + 0.5,
                torch.rand(dim, generator=gen, device=device) + 0.5)

    def entry(name, us, nbytes, window, **extra):
        gbs = nbytes / (us * 1e-6) / 1e9
        d = {"avg_launch_us": round(us, 2), "algorithmic_bytes_per_launch": nbytes,
             "achieved_gbs": round(gbs, 1), "frac": round(gbs / hbm, 4),
             "kernel": {rope3d.ROPE3D_PATH_TMA: "rope3d::qk_norm_rope_tma_kernel",
                        rope3d.ROPE3D_PATH_REGISTERS: "rope3d::qk_norm_rope_kernel"}.get(
                 rope3d.rope3d_testing_last_path(), "unknown"),
             "clocks": {"window": window, "name": name}}
        d.update(extra)
        out[name] = d

    def plain_step(w, ins, q_out, kc, vc, tables, trig=rope3d.ROPE3D_TRIG_TABLE, chunks=None):
        chunks = w.chunks if chunks is None else chunks

        def step():
            for j, c in enumerate(chunks):
                q, k, v = ins[j % len(ins)]
                rope3d.rope3d_qk_norm_rope_append(
                    q, k, v, q_out[j % len(q_out)], c.token_begin, c.token_end, c.frame_offset,
                    w.T, w.H, w.W, ins_w[0], ins_w[1], w.eps, kc, vc, c.slot, tables, trig)
        return step

    # 480P chunk loop: 7 calls of 4680 tokens x 12 heads
    w = wl.chunk_480p()
    n = w.tokens_per_chunk
    shape = (w.B, n, w.N, wl.HEAD_DIM)
    ins = [tuple(randn_bf16(shape, 100 + 3 * j + t) for t in range(3)) for j in range(len(w.chunks))]
    ins_w = weights(w.dim, 99)
    q_out = [torch.empty(shape, dtype=torch.bfloat16, device=device) for _ in w.chunks]
    cshape = (w.B, w.cache_tokens, w.N, wl.HEAD_DIM)
    kc = torch.zeros(cshape, dtype=torch.bfloat16, device=device)
    vc = torch.zeros_like(kc)
    tables = rope3d.rope3d_tables_init(max_t=21, max_h=w.H, max_w=w.W)
    us, win = graph_launch_us(torch, plain_step(w, ins, q_out, kc, vc, tables), len(w.chunks), stream)
    entry("chunk480p_3x30x52_h12_bf16", us, w.algorithmic_bytes(n), win,
          launches_per_step=len(w.chunks),
          note="7 chunk calls (start frames 0..18) into a 32760-token cache, graph replay; "
               "inputs 604 MB per step, above L2")

    # the 4-rank sequence-parallel step at 480P emulated on this GPU: each chunk's 4 token
    # slices (1170 tokens, all 12 heads) store each head's q, K and V at the rank that owns
    # it (3 heads each)
    P4 = 4
    hl4, sl4 = w.N // P4, n // P4
    sp_q = [torch.empty((w.B, n, hl4, wl.HEAD_DIM), dtype=torch.bfloat16, device=device)
            for _ in range(P4)]
    sp_k = [torch.zeros((w.B, w.cache_tokens, hl4, wl.HEAD_DIM), dtype=torch.bfloat16,
                        device=device) for _ in range(P4)]
    sp_v = [torch.zeros_like(sp_k[0]) for _ in range(P4)]
    sp_in = [[tuple(x[:, r * sl4:(r + 1) * sl4].contiguous() for x in c) for r in range(P4)]
             for c in ins]

    def sp4_step():
        for j, c in enumerate(w.chunks):
            for r in range(P4):
                q, k, v = sp_in[j][r]
                a = c.token_begin + r * sl4
                rope3d.rope3d_qk_norm_rope_append_sp(
                    q, k, v, a, a + sl4, c.frame_offset, w.T, w.H, w.W, ins_w[0], ins_w[1],
                    w.eps, sp_q, sp_k, sp_v, c.slot, tables, q_row0=c.token_begin)
    us, win = graph_launch_us(torch, sp4_step, P4 * len(w.chunks), stream)
    entry("chunk480p_3x30x52_h12_bf16/sp4", us, w.algorithmic_bytes(sl4), win,
          launches_per_step=P4 * len(w.chunks),
          note="4 ranks emulated as 4 launches per chunk over 1170-token slices; every head "
               "stored to its owner's buffers (3 heads each, all on this GPU)")
    del sp_q, sp_k, sp_v, sp_in, ins, q_out

    # whole 480P sequence (one call of 32760 tokens) against 8 slices of 4095 tokens
    w = wl.full_480p()
    n = w.tokens_per_chunk
    shape = (w.B, n, w.N, wl.HEAD_DIM)
    q, k, v = (randn_bf16(shape, 200 + t) for t in range(3))
    qo_whole, qo_sl = torch.empty_like(q), torch.empty_like(q)
    kw_, vw_ = torch.zeros_like(q), torch.zeros_like(q)
    ks_, vs_ = torch.zeros_like(q), torch.zeros_like(q)

    def whole():
        rope3d.rope3d_qk_norm_rope_append(q, k, v, qo_whole, 0, n, 0, w.T, w.H, w.W, ins_w[0],
                                          ins_w[1], w.eps, kw_, vw_, 0, tables)
    parts = wl.slices(n, 8)

    def sliced():
        for a, b in parts:
            rope3d.rope3d_qk_norm_rope_append(
                q[:, a:b], k[:, a:b], v[:, a:b], qo_sl[:, a:b], a, b, 0, w.T, w.H, w.W,
                ins_w[0], ins_w[1], w.eps, ks_, vs_, 0, tables)
    us_w, win_w = graph_launch_us(torch, whole, 1, stream)
    kern_w = rope3d.rope3d_testing_last_path()
    us_s, win_s = graph_launch_us(torch, sliced, len(parts), stream)
    torch.cuda.synchronize()
    same = all(torch.equal(a.view(torch.int16), b.view(torch.int16))
               for a, b in ((qo_whole, qo_sl), (kw_, ks_), (vw_, vs_)))
    nbytes = w.algorithmic_bytes(n)
    entry("full480p_21x30x52_h12_bf16/8slices", us_s, nbytes // len(parts), win_s,
          slice_tokens=[b - a for a, b in parts], slices_bit_identical_to_whole=same,
          whole={"avg_launch_us": round(us_w, 2), "algorithmic_bytes_per_launch": nbytes,
                 "frac": round(nbytes / (us_w * 1e-6) / 1e9 / hbm, 4),
                 "kernel": {rope3d.ROPE3D_PATH_TMA: "rope3d::qk_norm_rope_tma_kernel",
                            rope3d.ROPE3D_PATH_REGISTERS: "rope3d::qk_norm_rope_kernel"}.get(
                     kern_w, "unknown"),
                 "clocks": {"window": win_w, "name": "whole"}},
          note="slices: 8 calls of 4095 tokens cutting through frames and rows; each call is "
               "a separate launch (one graph of 8 launches)")
    del q, k, v, qo_whole, qo_sl, kw_, vw_, ks_, vs_
    tables.close()

    # long-horizon rollout: batch 2, 80 chunks (global frames 0..239), rolling 21-frame cache
    w = wl.long_horizon()
    n = w.tokens_per_chunk
    shape = (w.B, n, w.N, wl.HEAD_DIM)
    nsets = 8  # input sets cycled over the 80 calls: 1.4 GB, so every launch reads HBM
    ins = [tuple(randn_bf16(shape, 300 + 3 * j + t) for t in range(3)) for j in range(nsets)]
    q_out = [torch.empty(shape, dtype=torch.bfloat16, device=device) for _ in range(nsets)]
    cshape = (w.B, w.cache_tokens, w.N, wl.HEAD_DIM)
    kc = torch.zeros(cshape, dtype=torch.bfloat16, device=device)
    vc = torch.zeros_like(kc)
    tables = rope3d.rope3d_tables_init(max_t=240, max_h=w.H, max_w=w.W)
    for trig, tname in ((rope3d.ROPE3D_TRIG_TABLE, "table"),
                        (rope3d.ROPE3D_TRIG_ONTHEFLY, "onthefly")):
        us, win = graph_launch_us(torch, plain_step(w, ins, q_out, kc, vc, tables, trig),
                                  len(w.chunks), stream)
        entry(f"longhorizon_b2_3x30x52_h12_bf16/{tname}", us, w.algorithmic_bytes(n), win,
              launches_per_step=len(w.chunks),
              note="80 chunk calls of 2 x 4680 tokens, start frames 0..237, cache slots "
                   "wrapping every 21 frames; 8 input sets cycled")
    del ins, q_out, kc, vc
    tables.close()

    # the 720P step with quantized caches, on the headline's inputs
    w, ins, q_out, wq_d, wk_d, tables = headline
    n = w.tokens_per_chunk
    ins_w = (wq_d, wk_d)
    for fmt in ("fp8", "nvfp4"):
        fp4 = fmt == "nvfp4"
        cshape = (w.B, w.cache_tokens, w.N, wl.HEAD_DIM // 2 if fp4 else wl.HEAD_DIM)
        kc = torch.zeros(cshape, dtype=torch.uint8, device=device)
        vc = torch.zeros_like(kc)
        sshape = cshape[:3] + ((wl.HEAD_DIM // 16,) if fp4 else ())
        sdt = torch.uint8 if fp4 else torch.float32
        ks_, vs_ = (torch.zeros(sshape, dtype=sdt, device=device) for _ in range(2))
        e = w.elem_bytes
        nbytes = (w.B * n * (w.dim * 4 * e + 2 * (w.dim // 2 + w.dim // 16)) if fp4
                  else w.B * n * (w.dim * (4 * e + 2) + 2 * 4 * w.N))

        def qstep():
            for j, c in enumerate(w.chunks):
                q, k, v = ins[j]
                rope3d.rope3d_qk_norm_rope_append_ex(
                    q, k, v, q_out[j], c.token_begin, c.token_end, c.frame_offset, w.T, w.H,
                    w.W, wq_d, wk_d, w.eps, kc, vc, c.slot, tables, k_scale=ks_, v_scale=vs_,
                    k_global=0.5 if fp4 else 0.0, v_global=0.25 if fp4 else 0.0)
        us, win = graph_launch_us(torch, qstep, len(w.chunks), stream)
        entry(f"{w.name}/{fmt}_cache", us, nbytes, win, launches_per_step=len(w.chunks),
              note="q, k, v read and q_out written in bf16; K and V cache rows as "
                   + ("E2M1 codes with E4M3 scales per 16 elements" if fp4
                      else "E4M3 codes with an fp32 scale per head"))
        del kc, vc, ks_, vs_

    # the 8-rank sequence-parallel step emulated on this GPU: each chunk's 8 token slices
    # (1350 tokens, all 40 heads) store each head's q, K and V at the rank that owns it
    P = 8
    hl = w.N // P
    sp_q = [torch.empty((w.B, n, hl, wl.HEAD_DIM), dtype=torch.bfloat16, device=device)
            for _ in range(P)]
    sp_k = [torch.zeros((w.B, w.cache_tokens, hl, wl.HEAD_DIM), dtype=torch.bfloat16,
                        device=device) for _ in range(P)]
    sp_v = [torch.zeros_like(sp_k[0]) for _ in range(P)]
    sl = n // P
    sp_in = [[tuple(x[:, r * sl:(r + 1) * sl].contiguous() for x in c) for r in range(P)]
             for c in ins]

    def sp_step():
        for j, c in enumerate(w.chunks):
            for r in range(P):
                q, k, v = sp_in[j][r]
                a = c.token_begin + r * sl
                rope3d.rope3d_qk_norm_rope_append_sp(
                    q, k, v, a, a + sl, c.frame_offset, w.T, w.H, w.W, wq_d, wk_d, w.eps, sp_q,
                    sp_k, sp_v, c.slot, tables, q_row0=c.token_begin)
    us, win = graph_launch_us(torch, sp_step, P * len(w.chunks), stream)
    entry(f"{w.name}/sp8", us, w.algorithmic_bytes(sl), win, launches_per_step=P * len(w.chunks),
          note="8 ranks emulated as 8 launches per chunk over 1350-token slices; every head "
               "stored to its owner's buffers (5 heads each, all on this GPU)")
    del sp_q, sp_k, sp_v, sp_in

    # the exchange back after attention for the same 8 ranks: each rank's o [1, 10800, 5,
    # 128] (every token, its heads) goes to the 8 ranks' [1, 1350, 40, 128] slices; three
    # chunks' worth of buffers (331 MB of o) so that every launch reads HBM
    o_sets = [[randn_bf16((w.B, n, hl, wl.HEAD_DIM), 500 + 8 * c + r) for r in range(P)]
              for c in range(3)]
    o_out = [[torch.empty((w.B, sl, w.N, wl.HEAD_DIM), dtype=torch.bfloat16, device=device)
              for _ in range(P)] for _ in range(3)]

    def out_step():
        for c in range(3):
            for r in range(P):
                rope3d.rope3d_sp_output_all_to_all(o_sets[c][r], o_out[c], r)
    us, win = graph_launch_us(torch, out_step, 3 * P, stream)
    out_bytes = 2 * w.B * n * hl * wl.HEAD_DIM * 2  # read o, write it out
    entry(f"{w.name}/sp8_output_all_to_all", us, out_bytes, win, launches_per_step=3 * P,
          kernel="rope3d::sp_output_all_to_all_kernel",
          note="Algorithm 3's last step for 8 emulated ranks: each launch moves one rank's "
               "13.8 MB of o (every token, 5 heads) to the 8 ranks' token slices")
    del o_sets, o_out

    # RoPE alone (rope3d_apply) on the headline's q rows: read x, write the rotated rows
    def apply_step():
        for j, c in enumerate(w.chunks):
            rope3d.rope3d_apply(ins[j][0], q_out[j], c.token_begin, c.token_end,
                                c.frame_offset, w.T, w.H, w.W, tables)
    us, win = graph_launch_us(torch, apply_step, len(w.chunks), stream)
    entry(f"{w.name}/apply_rotation_only", us, 2 * w.B * n * w.dim * 2, win,
          launches_per_step=len(w.chunks),
          note="rope3d_apply: the 3D rotation alone (no norm, no cache), x read and the "
               "rotated rows written, 221 MB per call")

    # the QKV projection on the tensor cores (timed alone: the burst peak applies)
    K = w.dim
    xs = [randn_bf16((w.B * n, K), 400 + j) for j in range(3)]
    gen.manual_seed(499)
    wt = (torch.randn((3 * w.dim, K), generator=gen, device=device) * (2.0 / K ** 0.5)).to(
        torch.bfloat16)
    bt = torch.zeros(3 * w.dim, device=device)
    outs = [torch.empty((w.B, n, w.N, wl.HEAD_DIM), dtype=torch.bfloat16, device=device)
            for _ in range(3)]

    def proj():
        for j in range(3):
            rope3d.rope3d_qkv_project(xs[j], wt, bt, *outs)
    us, win = graph_launch_us(torch, proj, 3, stream)
    y = torch.empty((w.B * n, 3 * w.dim), dtype=torch.bfloat16, device=device)

    def cublas():
        for j in range(3):
            torch.matmul(xs[j], wt.t(), out=y)
    us_cb, _ = graph_launch_us(torch, cublas, 3, stream)
    flops = 2.0 * w.B * n * K * 3 * w.dim
    burst = peaks.get("bf16_tflops", 1590.0)
    tf = flops / (us * 1e-6) / 1e12
    out[f"{w.name}/qkv_projection"] = {
        "bound": "tensor", "avg_launch_us": round(us, 2), "algorithmic_flops_per_launch": flops,
        "achieved_tflops": round(tf, 1), "peak_tflops": burst,
        "peak_source": "MEASURED_PEAKS.json bf16_tflops (burst: the kernel is timed alone)",
        "frac": round(tf / burst, 4), "kernel": "rope3d::qkv_proj_kernel<2>",
        "cublas_same_gemm_us": round(us_cb, 2),
        "cublas_tflops": round(flops / (us_cb * 1e-6) / 1e12, 1),
        "clocks": {"window": win, "name": "projection"},
        "note": "x [10800, 5120] bf16 times W^T, W [15360, 5120] bf16, fp32 accumulate, bf16 "
                "out; 3 input sets, graph replay"}
    del outs, y

    # the step fed by the projection (rope3d_qkv_norm_rope_append): the 7 chunk calls of
    # the 720P step from hidden states, 3 input sets cycled
    xs3 = [x.view(w.B, n, K) for x in xs]
    ws = torch.zeros(rope3d.rope3d_qkv_workspace_bytes(w.B, n, w.N), dtype=torch.uint8,
                     device=device)
    kcf = torch.zeros((w.B, w.cache_tokens, w.N, wl.HEAD_DIM), dtype=torch.bfloat16,
                      device=device)
    vcf = torch.zeros_like(kcf)

    def fused():
        for j, c in enumerate(w.chunks):
            rope3d.rope3d_qkv_norm_rope_append(
                xs3[j % 3], wt, bt, q_out[j], ws, c.token_begin, c.token_end, c.frame_offset,
                w.T, w.H, w.W, wq_d, wk_d, w.eps, kcf, vcf, c.slot, tables)
    us, win = graph_launch_us(torch, fused, len(w.chunks), stream)
    tf = flops / (us * 1e-6) / 1e12
    out[f"{w.name}/qkv_fused_step"] = {
        "bound": "tensor", "avg_call_us": round(us, 2), "algorithmic_flops_per_call": flops,
        "achieved_tflops": round(tf, 1), "peak_tflops": burst,
        "peak_source": "MEASURED_PEAKS.json bf16_tflops (burst, as for the projection alone)",
        "frac": round(tf / burst, 4), "tokens_per_s": round(w.B * n / (us * 1e-6), 1),
        "kernel": "rope3d::qkv_proj_kernel<2> (norm-weight, RoPE and V-append epilogue) + "
                  "rope3d::qk_row_scale_kernel",
        "projection_alone_us": out[f"{w.name}/qkv_projection"]["avg_launch_us"],
        "clocks": {"window": win, "name": "projection-fed step"},
        "note": "7 chunk calls of rope3d_qkv_norm_rope_append from x [1, 10800, 5120] bf16 "
                "(3 input sets cycled): the projection GEMM with its epilogue, then the "
                "per-row RMSNorm scale of q and K; graph replay, time per call"}
    del xs, xs3, wt, ws, kcf, vcf

    torch.cuda.empty_cache()
    return out


def run_qkv(args, dist: Dist):
    """The step fed by the QKV projection: every chunk's token rows x [1, n, K] (K = N*128)
    go through rope3d_qkv_norm_rope_append.  The roofline is the projection kernel's, on
    the tensor cores: 2 n K (3 N 128) flops per launch over its own launch time, measured
    by timing rope3d_qkv_project alone on the same shapes; cuBLAS (torch.matmul) on the
    same GEMM is timed beside it for context.  The denominator is the measured burst bf16
    rate, the one for a kernel timed by itself."""
    import torch

    from rotary_position_encoding_b200 import rope3d

    torch.cuda.set_device(dist.local_rank)
    device = torch.device("cuda", dist.local_rank)
    dist.init("nccl")
    w = workload_for(args)
    if w.dtype != "bf16":
        raise SystemExit("--qkv runs bf16 workloads")
    K = w.dim
    n = w.tokens_per_chunk
    trig = rope3d.ROPE3D_TRIG_TABLE if args.trig == "table" else rope3d.ROPE3D_TRIG_ONTHEFLY

    def dev_bf16(a):
        return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)

    xs = [dev_bf16(wl.hidden_states(w, ci, K)) for ci in range(len(w.chunks))]
    w_bits, b = wl.projection_weights(w.seed, w.dim, K)
    wt = dev_bf16(w_bits)
    bt = torch.from_numpy(b).to(device)
    wq, wk = (torch.from_numpy(a).to(device) for a in wl.norm_weights(w.seed, w.dim))
    q_out = [torch.empty((w.B, n, w.N, wl.HEAD_DIM), dtype=torch.bfloat16, device=device)
             for _ in w.chunks]
    workspace = torch.zeros(rope3d.rope3d_qkv_workspace_bytes(w.B, n, w.N), dtype=torch.uint8,
                            device=device)
    shape = (w.B, w.cache_tokens, w.N, wl.HEAD_DIM)
    k_cache = torch.zeros(shape, dtype=torch.bfloat16, device=device)
    v_cache = torch.zeros(shape, dtype=torch.bfloat16, device=device)
    tables = rope3d.rope3d_tables_init(max_t=max(c.frame_offset for c in w.chunks) + w.T,
                                       max_h=w.H, max_w=w.W)
    stream = torch.cuda.current_stream(device)
    rope3d.rope3d_testing_gemm_cta_group(args.gemm_form)

    def step():
        for ci, c in enumerate(w.chunks):
            rope3d.rope3d_qkv_norm_rope_append(
                xs[ci], wt, bt, q_out[ci], workspace, c.token_begin, c.token_end, c.frame_offset,
                w.T, w.H, w.W, wq, wk, w.eps, k_cache, v_cache, c.slot, tables, trig,
                stream=stream)

    clocks = ClockSampler(dist.local_rank) if dist.rank == 0 else None
    if clocks:
        clocks.start()
        time.sleep(0.3)
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize()
    if clocks:
        clocks.mark("start")
    start.record(stream)
    for _ in range(args.steps):
        step()
    end.record(stream)
    torch.cuda.synchronize()
    if clocks:
        clocks.mark("end")
    dist.barrier()
    elapsed_ms = dist.max(start.elapsed_time(end), device)
    clock_info = clocks.stop() if clocks else None

    # the projection kernel alone, and cuBLAS on the same GEMM
    outs = [torch.empty_like(q_out[0]) for _ in range(3)]
    reps = max(3, min(args.steps, 20)) * len(w.chunks)

    def timed(fn):
        for _ in range(3):
            fn(0)
        torch.cuda.synchronize()
        a, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for r in range(reps):
            fn(r % len(w.chunks))
        e.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(e) / reps

    gemm_ms = timed(lambda ci: rope3d.rope3d_qkv_project(xs[ci], wt, bt, *outs, stream=stream))
    y = torch.empty((n, 3 * w.dim), dtype=torch.bfloat16, device=device)
    cublas_ms = timed(lambda ci: torch.matmul(xs[ci].view(n, K), wt.t(), out=y))
    tables.close()
    dist.close()
    if dist.rank != 0:
        return None
    peaks, peak_kind = measured_peaks()
    flops = 2.0 * w.B * n * K * 3 * w.dim
    achieved = flops / (gemm_ms / 1e3) / 1e12
    peak = peaks.get("bf16_tflops", 1590.0)  # burst: the projection is timed by itself
    tokens_per_step = w.B * n * len(w.chunks)
    return {
        "metric": "QKV projection + QK-RMSNorm + 3D RoPE + KV append tokens/s, 1 GPU",
        "value": round(tokens_per_step * args.steps * dist.world / (elapsed_ms / 1e3), 1),
        "unit": "tokens/s",
        "n_gpus": dist.world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(elapsed_ms / args.steps, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) token rows, N(0,4/K) projection weights, N(0,0.01) "
                "bias, U(0.5,1.5) norm weights)",
        "config": {"workload": w.name + "+qkv", "K": K, "heads": w.N,
                   "chunks_per_step": len(w.chunks), "tokens_per_step": tokens_per_step,
                   "launch": "eager, one C-ABI call per chunk (one launch: the projection "
                             "with the norm, rotation and append in its epilogue)",
                   "l2": "no flush: each chunk's x (110 MB) and the weight (157 MB) exceed L2 "
                         "together"},
        "roofline": {"bound": "tensor", "achieved": round(achieved, 1), "peak": peak,
                     "unit": "TFLOP/s", "frac": round(achieved / peak, 4), "traffic": None,
                     "peak_source": f"{peak_kind} bf16_tflops (burst; the projection is timed "
                                    "by itself, about 0.2 s of back-to-back launches)",
                     "kernel": "rope3d::qkv_proj_kernel<%d>" % (args.gemm_form or 2),
                     "algorithmic_flops_per_launch": flops,
                     "avg_launch_ms": round(gemm_ms, 4),
                     "cublas_same_gemm_ms": round(cublas_ms, 4),
                     "cublas_tflops": round(flops / (cublas_ms / 1e3) / 1e12, 1)},
        "gpu_launches": 2 * len(w.chunks) * args.steps,  # projection + row scale (or step)
        "clocks": clock_info,
    }


def run_e2e(args, w, host, wq_d, wk_d, tables, trig, device, dist, rope3d, torch):
    """Same workload through the public call, with the step's inputs copied in from pinned
    host memory and its results (q_out and the appended K/V rows) copied back every step,
    inside the timed region.  The copies run on two side streams, one per direction, so
    chunk c+1's upload and chunk c-1's download overlap chunk c's kernel.  Two device
    slots double-buffer the inputs and q_out; events order each slot's reuse and keep
    the download of a cache range ahead of its next overwrite."""
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    n = w.tokens_per_chunk

    def pinned_from(a):
        t = torch.from_numpy(a.view(np.int16) if w.dtype == "bf16" else a)
        t = t.view(torch.bfloat16) if w.dtype == "bf16" else t
        return t.pin_memory()

    h_in = [tuple(pinned_from(a) for a in chunk) for chunk in host]
    shape = (w.B, n, w.N, wl.HEAD_DIM)
    h_out = [tuple(torch.empty(shape, dtype=tdt).pin_memory() for _ in range(3))
             for _ in w.chunks]
    slots = 2
    d_in = [tuple(torch.empty(shape, dtype=tdt, device=device) for _ in range(3))
            for _ in range(slots)]
    d_qo = [torch.empty(shape, dtype=tdt, device=device) for _ in range(slots)]
    cache_shape = (w.B, w.cache_tokens, w.N, wl.HEAD_DIM)
    k_cache = torch.zeros(cache_shape, dtype=tdt, device=device)
    v_cache = torch.zeros(cache_shape, dtype=tdt, device=device)
    comp = torch.cuda.current_stream(device)
    up = torch.cuda.Stream(device)
    down = torch.cuda.Stream(device)
    ev_comp, ev_out = {}, {}
    counter = [0]
    h2d = d2h = 0

    def step():
        nonlocal h2d, d2h
        h2d = d2h = 0
        for ci, chunk in enumerate(w.chunks):
            g = counter[0]
            j = g % slots
            with torch.cuda.stream(up):
                if g - slots in ev_comp:            # the slot's last reader is done
                    up.wait_event(ev_comp[g - slots])
                for dst, src in zip(d_in[j], h_in[ci]):
                    dst.copy_(src, non_blocking=True)
                    h2d += src.numel() * src.element_size()
                ev_in = torch.cuda.Event()
                ev_in.record(up)
            comp.wait_event(ev_in)
            if g - slots in ev_out:                 # q_out slot and cache rows downloaded
                comp.wait_event(ev_out[g - slots])
            q, k, v = d_in[j]
            rope3d.rope3d_qk_norm_rope_append(
                q, k, v, d_qo[j], chunk.token_begin, chunk.token_end, chunk.frame_offset,
                w.T, w.H, w.W, wq_d, wk_d, w.eps, k_cache, v_cache, chunk.slot, tables, trig,
                comp)
            ev_comp[g] = torch.cuda.Event()
            ev_comp[g].record(comp)
            with torch.cuda.stream(down):
                down.wait_event(ev_comp[g])
                rows = slice(chunk.slot, chunk.slot + n)  # no wrap inside a chunk here
                for dst, src in zip(h_out[ci], (d_qo[j], k_cache[:, rows], v_cache[:, rows])):
                    dst.copy_(src, non_blocking=True)
                    d2h += dst.numel() * dst.element_size()
                ev_out[g] = torch.cuda.Event()
                ev_out[g].record(down)
            ev_comp.pop(g - slots, None)
            ev_out.pop(g - slots, None)
            counter[0] += 1

    steps = max(1, min(args.e2e_steps, args.steps))
    step()
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize()
    start.record(comp)
    up.wait_stream(comp)
    down.wait_stream(comp)
    for _ in range(steps):
        step()
    comp.wait_stream(up)
    comp.wait_stream(down)
    end.record(comp)
    torch.cuda.synchronize()
    dist.barrier()
    ms = dist.max(start.elapsed_time(end), device)
    tokens = w.B * n * len(w.chunks) * steps * dist.world
    return {"value": round(tokens / (ms / 1e3), 1), "unit": "tokens/s",
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "ms_per_step": round(ms / steps, 3),
            "path": "pinned host -> cudaMemcpyAsync (upload stream) -> "
                    "rope3d_qk_norm_rope_append -> cudaMemcpyAsync (download stream) -> "
                    "pinned host, double-buffered, copies overlapping kernels"}


# ---------------------------------------------------------------- the oracle on the host

class OracleSample:
    """The fp64 oracle on a bounded sample of the step: the first chunk calls' tokens in
    512-token sub-batches (at most ``prepared_tokens`` of them, widened to float64 once),
    run over and over until a time budget or a token count is reached.  The oracle's
    work per token does not depend on the token's values, so cycling through a prefix
    times the same work as walking the whole step."""

    SUB = 512

    def __init__(self, w, host, prepared_tokens=4096):
        import oracle
        self.orc = oracle.default()
        self.w = w
        wq, wk = wl.norm_weights(w.seed, w.dim)
        self.wq64, self.wk64 = wq.astype(np.float64), wk.astype(np.float64)
        n = w.tokens_per_chunk
        self.batches = []
        have = 0
        for ci, chunk in enumerate(w.chunks):
            for a in range(0, n, self.SUB):
                if have >= prepared_tokens:
                    break
                e = min(n, a + self.SUB)
                f = [wl.to_f64(x[:, a:e], w.dtype) for x in host[ci]]
                self.batches.append((chunk, a, e, f))
                have += w.B * (e - a)
        self.prepared = have

    def run(self, budget_s: float, max_tokens=None, nthreads=0):
        """Returns (tokens, oracle seconds, threads); nthreads 0 means every core."""
        w = self.w
        done, spent, i = 0, 0.0, 0
        while True:
            chunk, a, e, f = self.batches[i % len(self.batches)]
            i += 1
            m = e - a
            # a cache of m rows placed so the sub-batch fills it exactly; the per-token
            # work is that of the real cache placement
            kc = np.zeros((w.B, m, w.N, wl.HEAD_DIM))
            vc = np.zeros_like(kc)
            t0 = time.perf_counter()
            self.orc.qk_norm_rope_append(f[0], f[1], f[2], a, e, chunk.frame_offset, w.T, w.H,
                                         w.W, self.wq64, self.wk64, w.eps, kc, vc, (-a) % m,
                                         nthreads=nthreads)
            spent += time.perf_counter() - t0
            done += w.B * m
            if spent >= budget_s or (max_tokens is not None and done >= max_tokens):
                return done, spent, nthreads or self.orc.max_threads()


def cpu_baseline(w, host, budget_s):
    """The oracle on every host core for budget_s seconds, then on one core for a third of
    that."""
    sampler = OracleSample(w, host)
    tokens, secs, threads = sampler.run(budget_s)
    tok1, secs1, _ = sampler.run(budget_s / 3.0, nthreads=1)
    return {"value": round(tokens / secs, 1), "unit": "tokens/s", "cores": threads,
            "kind": "oracle",
            "sample": f"{tokens} tokens: the first {sampler.prepared} tokens of the step "
                      f"({w.name}) in 512-token sub-batches, cycled for {secs:.1f} s of fp64 "
                      f"oracle time on {threads} OpenMP threads",
            "single_thread": {"value": round(tok1 / secs1, 1), "unit": "tokens/s",
                              "sample": f"{tok1} tokens of the same sample in {secs1:.1f} s "
                                        f"on one thread"}}


def run_reference(args, dist: Dist):
    """The oracle as it stands on the host cores, on this benchmark's workload; each step
    is a bounded sample sized so the whole run stays within a few minutes."""
    if dist.rank != 0:
        return None
    w = workload_for(args)
    host = make_inputs(w, seed_offset=0)
    sampler = OracleSample(w, host)
    # calibrate: tokens per second of the oracle on this host
    tok, secs, threads = sampler.run(1.0)
    rate = tok / secs
    total_budget = 150.0
    per_step = int(max(1, min(w.B * w.tokens_per_chunk * len(w.chunks),
                              rate * total_budget / max(1, args.steps + args.warmup))))
    for _ in range(args.warmup):
        sampler.run(1e9, max_tokens=per_step)
    total_tok, total_s = 0, 0.0
    for _ in range(args.steps):
        t, s, threads = sampler.run(1e9, max_tokens=per_step)
        total_tok += t
        total_s += s
    value = total_tok / total_s
    sample = (f"{per_step} tokens per step, cycling through the first {sampler.prepared} "
              f"tokens of the {w.name} step in 512-token sub-batches, fp64 oracle, "
              f"{threads} OpenMP threads")
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": round(value, 1),
        "unit": "tokens/s",
        "n_gpus": dist.world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(total_s / args.steps * 1e3, 3),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded N(0,1) bf16 q/k/v, U(0.5,1.5) fp32 norm weights)",
        "config": {"workload": w.name, "tokens_per_step_sampled": per_step,
                   "heads": w.N, "head_dim": wl.HEAD_DIM, "trig": "fp64 libm"},
        "cpu_baseline": {"value": round(value, 1), "unit": "tokens/s", "cores": threads,
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(value, 1), "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    args = parse_args(argv)
    dist = Dist()
    if args.impl == "reference":
        line = run_reference(args, dist)
    elif args.qkv:
        line = run_qkv(args, dist)
    else:
        line = run_ours(args, dist)
    if line is not None and dist.rank == 0:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
