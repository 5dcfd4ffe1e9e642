"""Benchmark of the weight-only skinny GEMM on B200.

One step = one decoder layer's weight-only GEMMs (three 5120x5120 NVFP4
attention projections, the 34816x5120 NVFP4 gate+up and the 5120x17408 FP8
down projection) at M = 1 (one decode token) and then at M = 8 (a k=7
speculative-verify round plus its base token): ten kernel launches.  Weights
rotate through three device copies (702 MB, over 5x the 126 MB L2), so no
launch finds its weights in L2.

Metric: effective HBM GB/s = (packed weight bytes + scale bytes + activation
bytes + output bytes) / device time, with the fraction of the measured HBM
copy bandwidth.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Under torchrun (N > 1) every rank runs the same workload on its own GPU
(replicas: the GEMMs of different requests shard with no exchange); rank 0
prints one JSON line with the max-over-ranks time.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import re
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import synthetic_inputs as si  # noqa: E402

METRIC = "NVFP4/FP8 skinny-GEMM effective HBM GB/s & % of B200 peak at M=1 and M=8"
WORKLOAD = "decoder_layer_m1_m8"
PASSES = (1, 8)          # M of the two passes of a step
COPIES = 3               # weight copies in rotation
FALLBACK_HBM_GBS = 6650.0
KERNEL_SOURCES = ("skinny.cu", "ptx.cuh", "layout.h")


# ---------------------------------------------------------------------------
# Byte accounting (algorithmic bytes: what the operation must move at least)
# ---------------------------------------------------------------------------

def out_bytes(spec) -> int:
    return 4 if spec.out == "f32" else 2


def weight_bytes(spec) -> int:
    if spec.fmt == "nvfp4":
        return spec.N * spec.K // 2 + spec.N * spec.K // 16 + 4
    return spec.N * spec.K + 4 * spec.N


def gemm_bytes(spec, M: int) -> int:
    return weight_bytes(spec) + M * spec.K * 2 + M * spec.N * out_bytes(spec)


def step_bytes() -> int:
    return sum(gemm_bytes(s, M) for M in PASSES for s in si.MIXED_LAYER)


def max_over_ranks(value: float, world: int, device=None) -> float:
    """The largest `value` over all ranks (each rank times its own replica; the
    job takes as long as the slowest one)."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist

    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(world: int, bytes_per_step: int, steps: int, ms: float) -> float:
    """Aggregate effective GB/s of `world` replicas that each ran `steps` steps in `ms`."""
    return world * bytes_per_step * steps / (ms * 1e-3) / 1e9


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def kernel_source_hash() -> str:
    """Hash of the kernel sources' code: comments and whitespace are dropped,
    so a comment edit keeps a traffic record taken on the same code valid."""
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "fp8_weight_only_w4a16_b200", "csrc", name), encoding="utf-8") as f:
            text = f.read()
        text = re.sub(r"//[^\n]*|/\*.*?\*/", "", text, flags=re.S)
        h.update("".join(text.split()).encode())
    return h.hexdigest()[:16]


def recorded_traffic(avg_alg_bytes: float):
    """DRAM bytes per launch of the NVFP4 kernel from the committed ncu summary,
    if it was taken on the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", "nvfp4_gemm_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
    except (OSError, ValueError):
        return None
    if d.get("source_sha") != kernel_source_hash():
        return None
    return float(d["dram_bytes_per_alg_byte"]) * avg_alg_bytes


# ---------------------------------------------------------------------------
# Clock sampling during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.t0 = self.t1 = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(device_index), "--query-gpu=timestamp," + self.FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons = [], [], set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in out.splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for name, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# Workload on the device
# ---------------------------------------------------------------------------

def build_device_workload(dev):
    import torch

    import fp8_weight_only_w4a16_b200 as sk

    weights = [[] for _ in range(COPIES)]
    for i, spec in enumerate(si.MIXED_LAYER):
        logical = si.weights_for(spec, seed=0, cfg_id=si.MIXED_CFG_ID, tensor_id=10 * i)
        if spec.fmt == "nvfp4":
            base = torch.from_numpy(sk.pack_nvfp4(*logical)).to(dev)
            for c in range(COPIES):
                weights[c].append(sk.PackedNVFP4(base if c == 0 else base.clone(), spec.global_scale, spec.N, spec.K))
        else:
            pc = torch.from_numpy(sk.pack_fp8(logical[0])).to(dev)
            s = torch.from_numpy(logical[1]).to(dev)
            for c in range(COPIES):
                weights[c].append(sk.PackedFP8(pc if c == 0 else pc.clone(), s if c == 0 else s.clone(),
                                               spec.N, spec.K))
    xs, ys = make_io_buffers(dev)
    need = max(sk.workspace_bytes(w.fmt, M, w.N, w.K) for w in weights[0] for M in PASSES)
    ws = torch.zeros(need, dtype=torch.uint8, device=dev)
    return weights, xs, ys, ws


def make_io_buffers(dev):
    """Every activation and every output of a step in one contiguous device
    buffer each (views per GEMM, 256-byte aligned), so that the end-to-end pass
    moves a step's inputs and results with one copy each way."""
    import torch

    xs, ys = {}, {}
    x_parts = [(M, i, si.activations(M, spec.K, seed=0, cfg_id=si.MIXED_CFG_ID, tensor_id=100 + i))
               for M in PASSES for i, spec in enumerate(si.MIXED_LAYER)]
    x_buf = torch.zeros(sum(_padded(a.nbytes) for _, _, a in x_parts), dtype=torch.uint8, device=dev)
    off = 0
    for M, i, a in x_parts:
        view = x_buf[off:off + a.nbytes].view(torch.float16).view(a.shape)
        view.copy_(torch.from_numpy(a))
        xs.setdefault(M, []).append(view)
        off += _padded(a.nbytes)
    y_shapes = [(M, spec) for M in PASSES for spec in si.MIXED_LAYER]
    y_bytes = [M * spec.N * (4 if spec.out == "f32" else 2) for M, spec in y_shapes]
    y_buf = torch.zeros(sum(_padded(b) for b in y_bytes), dtype=torch.uint8, device=dev)
    off = 0
    for (M, spec), b in zip(y_shapes, y_bytes):
        dt = torch.float32 if spec.out == "f32" else torch.float16
        ys.setdefault(M, []).append(y_buf[off:off + b].view(dt).view(M, spec.N))
        off += _padded(b)
    xs["buffer"], ys["buffer"] = x_buf, y_buf
    return xs, ys


def _padded(nbytes: int) -> int:
    return (nbytes + 255) // 256 * 256


def bench_config(world: int) -> dict:
    """The workload description both arms print (the reference arm times the
    same workload on a row sample, which its cpu_baseline.sample states)."""
    return {"workload": WORKLOAD,
            "gemms": ["%s %s %dx%d" % (s.name, s.fmt, s.N, s.K) for s in si.MIXED_LAYER],
            "M": list(PASSES), "operands": "NVFP4/FP8 weights x FP16 activations, FP32 accumulation",
            "l2": "inputs larger than L2: %d rotating weight copies, %.0f MB" %
                  (COPIES, COPIES * sum(weight_bytes(s) for s in si.MIXED_LAYER) / 1e6),
            "bytes_per_step": step_bytes(), "launch": "CUDA graph per step",
            "parallelism": "replicas" if world > 1 else "single GPU"}


def copy_for(step: int, pass_idx: int) -> int:
    return (2 * step + pass_idx) % COPIES


def launch_step(weights, xs, ys, ws, step: int):
    """Enqueue one step (both passes) on the current stream."""
    for pi, M in enumerate(PASSES):
        wc = weights[copy_for(step, pi)]
        for i in range(len(si.MIXED_LAYER)):
            launch_one(ys[M][i], xs[M][i], wc[i], ws)


def capture_step_graphs(weights, xs, ys, ws):
    """One CUDA graph per rotation phase (a step's launches are fixed by step % 3)."""
    import torch

    graphs = []
    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        launch_step(weights, xs, ys, ws, 0)  # warm the driver paths before capture
    torch.cuda.current_stream().wait_stream(stream)
    torch.cuda.synchronize()
    for phase in range(COPIES):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            launch_step(weights, xs, ys, ws, phase)
        graphs.append(g)
    return graphs


def clone_weight(w):
    import fp8_weight_only_w4a16_b200 as sk

    if isinstance(w, sk.PackedNVFP4):
        return sk.PackedNVFP4(w.data.clone(), w.global_scale, w.N, w.K)
    return sk.PackedFP8(w.codes.clone(), w.channel_scale, w.N, w.K)


def per_launch_us(weights, xs, ys, ws, launches: int = 30, replays: int = 3, trials: int = 10, passes=PASSES):
    """Device time of one launch of each GEMM of the step, [pass][gemm] in us:
    the median and the best of `trials` trials.

    Each GEMM is timed as a CUDA graph of `launches` back-to-back launches on one
    stream, rotating through enough copies of its weights to exceed 4x the L2
    cache (so no launch finds its weights in L2); a trial is `replays` replays
    of that graph between CUDA events on the launching stream, divided by the
    launches it ran.  No event sits between the launches (an event-record node
    in a graph costs several microseconds)."""
    import torch

    l2 = torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size
    out = np.zeros((len(passes), len(si.MIXED_LAYER)))
    best = np.zeros_like(out)
    stream = torch.cuda.Stream()
    for i, spec in enumerate(si.MIXED_LAYER):
        base = weights[0][i]
        n_copy = max(COPIES, int(np.ceil(4 * l2 / weight_bytes(spec))))
        copies = [weights[c][i] for c in range(COPIES)] + [clone_weight(base) for _ in range(n_copy - COPIES)]
        for pi, M in enumerate(passes):
            stream.wait_stream(torch.cuda.current_stream())
            with torch.cuda.stream(stream):
                launch_one(ys[M][i], xs[M][i], copies[0], ws)
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                for r in range(launches):
                    launch_one(ys[M][i], xs[M][i], copies[r % n_copy], ws)
            g.replay()
            g.replay()
            torch.cuda.synchronize()
            t = []
            for _ in range(trials):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record()
                for _ in range(replays):
                    g.replay()
                e1.record()
                torch.cuda.synchronize()
                t.append(1e3 * e0.elapsed_time(e1) / (replays * launches))
            out[pi, i] = float(np.median(t))
            best[pi, i] = float(np.min(t))
            del g
        del copies
    torch.cuda.empty_cache()
    return out, best


def m16_per_gemm(weights, ws, dur_us, peak):
    """Each GEMM of the step at M = 16 (two MMA token blocks), timed like the
    M = 1 and M = 8 launches, next to its M = 8 time."""
    import torch

    dev = ws.device
    xs = {16: [torch.from_numpy(si.activations(16, s.K, seed=0, cfg_id=si.MIXED_CFG_ID, tensor_id=200 + i)).to(dev)
               for i, s in enumerate(si.MIXED_LAYER)]}
    ys = {16: [torch.empty((16, s.N), dtype=torch.float32 if s.out == "f32" else torch.float16, device=dev)
               for s in si.MIXED_LAYER]}
    med, best = per_launch_us(weights, xs, ys, ws, passes=(16,))
    rows = []
    for i, spec in enumerate(si.MIXED_LAYER):
        b16, b8 = gemm_bytes(spec, 16), gemm_bytes(spec, 8)
        g16, g8 = b16 / med[0, i] / 1e3, b8 / float(dur_us[PASSES.index(8), i]) / 1e3
        rows.append({"gemm": spec.name, "fmt": spec.fmt, "us": round(float(med[0, i]), 3),
                     "us_best": round(float(best[0, i]), 3), "GB/s": round(g16, 1), "frac": round(g16 / peak, 4),
                     "GB/s_vs_M8": round(g16 / g8, 4)})
    return rows


def grouped_attention_us(weights, xs, ys, ws, peak, launches: int = 30, replays: int = 3, trials: int = 10):
    """The step's three 5120 x 5120 NVFP4 projections (q, kv, o: own x, own y)
    as ONE grouped launch, at M = 1 and 8: per-launch device time (median and
    best of `trials`), timed like the standalone GEMMs (graphs of back-to-back
    launches over weight copies > 4x L2)."""
    import torch

    import fp8_weight_only_w4a16_b200 as sk

    idx = [i for i, s in enumerate(si.MIXED_LAYER) if s.fmt == "nvfp4" and s.N == 5120 and s.K == 5120]
    l2 = torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size
    per_set = sum(weight_bytes(si.MIXED_LAYER[i]) for i in idx)
    n_set = max(COPIES, int(np.ceil(4 * l2 / per_set)))
    sets = [[weights[c][i] for i in idx] for c in range(COPIES)]
    sets += [[clone_weight(weights[0][i]) for i in idx] for _ in range(n_set - COPIES)]
    rows = []
    stream = torch.cuda.Stream()
    for M in PASSES:
        xg = [xs[M][i] for i in idx]
        yg = [ys[M][i] for i in idx]
        stream.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(stream):
            sk.gemm_grouped_into(yg, xg, sets[0], workspace=ws)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for r in range(launches):
                sk.gemm_grouped_into(yg, xg, sets[r % n_set], workspace=ws)
        g.replay()
        torch.cuda.synchronize()
        t = []
        for _ in range(trials):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            for _ in range(replays):
                g.replay()
            e1.record()
            torch.cuda.synchronize()
            t.append(1e3 * e0.elapsed_time(e1) / (replays * launches))
        del g
        b = sum(gemm_bytes(si.MIXED_LAYER[i], M) for i in idx)
        us = float(np.median(t))
        rows.append({"M": M, "us": round(us, 3), "us_best": round(float(np.min(t)), 3), "GB/s": round(b / us / 1e3, 1),
                     "frac": round(b / us / 1e3 / peak, 4)})
    del sets
    torch.cuda.empty_cache()
    return {"gemms": ["%s nvfp4 5120x5120" % si.MIXED_LAYER[i].name for i in idx], "passes": rows,
            "note": "one skinny_nvfp4_gemm_grouped launch of the three attention projections; the step itself "
                    "runs them as three launches"}


def _random_packed_copies(dev, N, K, gen):
    """Packed NVFP4 tiles drawn on the device (random E2M1 codes, UE4M3 block
    scales in [2^-4, 2^4]), as many copies as it takes to exceed 4x L2."""
    import torch

    import fp8_weight_only_w4a16_b200 as sk

    nbytes = sk.nvfp4_packed_bytes(N, K)
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    n_copy = max(2, int(np.ceil(4 * l2 / nbytes)))
    copies = []
    for _ in range(n_copy):
        t = torch.randint(0, 256, (nbytes // 36864, 36864), dtype=torch.uint8, device=dev, generator=gen)
        t[:, 32768:] = torch.randint(0x18, 0x59, (nbytes // 36864, 4096), dtype=torch.uint8, device=dev,
                                     generator=gen)
        copies.append(t.view(-1))
    return copies, nbytes


def _graph_us(one, n_copy, launches, replays, trials: int = 10):
    """Device time of one launch, median over `trials`: a CUDA graph of
    back-to-back launches rotating over the weight copies, CUDA events around
    each trial's replays."""
    import torch

    stream = torch.cuda.Stream()
    stream.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(stream):
        one(0)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for r in range(launches):
            one(r % n_copy)
    g.replay()
    torch.cuda.synchronize()
    t = []
    for _ in range(trials):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(replays):
            g.replay()
        e1.record()
        torch.cuda.synchronize()
        t.append(1e3 * e0.elapsed_time(e1) / (replays * launches))
    del g
    return float(np.median(t))


def fused_epilogues_us(dev, launches: int = 20, replays: int = 3):
    """Per-launch device time of the two fused epilogues next to the plain GEMM
    they replace, at M = 1 and 8:
      * the vocabulary projection 151936 x 5120 fused with the per-token argmax
        vs the same GEMM writing FP32 logits;
      * the gate+up projection 34816 x 5120 fused with SiLU*mul (17408 FP16
        outputs) vs the same GEMM writing its 34816 FP16 outputs;
      * the attention output projection 5120 x 5120 adding its result into
        the FP16 residual stream in place vs the same GEMM writing y."""
    import torch

    import fp8_weight_only_w4a16_b200 as sk
    from fp8_weight_only_w4a16_b200 import PackedGateUp, PackedNVFP4

    gen = torch.Generator(device=dev)
    gen.manual_seed(5)
    result = {}
    for name, N, K in (("lm_head_argmax", 151936, 5120), ("gate_up_silu_mul", 34816, 5120),
                       ("o_proj_residual_add", 5120, 5120)):
        copies, nbytes = _random_packed_copies(dev, N, K, gen)
        plain = [PackedNVFP4(c, 1.0, N, K) for c in copies]
        gu = [PackedGateUp(c, 1.0 / 448, N // 2, K) for c in copies]
        ws = sk.make_workspace(sk.FMT_NVFP4, 8, N, K, dev)
        rows = []
        for M in PASSES:
            x = torch.randn((M, K), generator=gen, device=dev).to(torch.float16)
            row = {"M": M}
            if name == "lm_head_argmax":
                y = torch.empty((M, N), dtype=torch.float32, device=dev)
                idx = torch.empty((M,), dtype=torch.int32, device=dev)
                val = torch.empty((M,), dtype=torch.float32, device=dev)
                kinds = {"fused_argmax": (lambda c: sk.gemm_argmax_into(idx, val, x, plain[c], ws), M * 8),
                         "gemm_fp32": (lambda c: sk.gemm_into(y, x, plain[c], workspace=ws), M * N * 4)}
            elif name == "gate_up_silu_mul":
                y = torch.empty((M, N), dtype=torch.float16, device=dev)
                h = torch.empty((M, N // 2), dtype=torch.float16, device=dev)
                kinds = {"fused_silu_mul": (lambda c: sk.gemm_silu_mul_into(h, x, gu[c], workspace=ws), M * N),
                         "gemm_fp16": (lambda c: sk.gemm_into(y, x, plain[c], workspace=ws), M * N * 2)}
            else:
                y = torch.zeros((M, N), dtype=torch.float16, device=dev)
                kinds = {"fused_residual_add": (lambda c: sk.gemm_add_into(y, x, plain[c], y, workspace=ws),
                                                2 * M * N * 2),
                         "gemm_fp16": (lambda c: sk.gemm_into(y, x, plain[c], workspace=ws), M * N * 2)}
            for kind, (one, out_bytes) in kinds.items():
                us = _graph_us(one, len(copies), launches, replays)
                alg = nbytes + 4 + M * K * 2 + out_bytes
                row[kind] = {"us": round(us, 3), "GB/s": round(alg / us / 1e3, 1)}
            rows.append(row)
        result[name] = {"gemm": "nvfp4 %dx%d" % (N, K), "passes": rows}
        del copies, plain, gu, ws
        torch.cuda.empty_cache()
    return result


READ_CEILING_BYTES = 4 << 30


def read_only_ceiling(dev, trials: int = 5):
    """The in-run read-only HBM ceiling: the library's streaming-read kernels
    (16-byte loads from every thread, and 36 KB bulk copies into a shared-memory
    ring) over a 4 GiB buffer, best of `trials` each, CUDA events on the
    launching stream.  The faster method is the ceiling."""
    import ctypes

    import torch

    import fp8_weight_only_w4a16_b200 as sk

    buf = torch.empty(READ_CEILING_BYTES, dtype=torch.uint8, device=dev)
    buf.random_(0, 256)   # the 16-byte loads could otherwise be fed by compressed zero pages
    sink = torch.zeros(4, dtype=torch.int32, device=dev)
    lib = sk.library()
    stream = torch.cuda.current_stream()
    out = {}
    for method, name, nbytes in ((0, "ldg", READ_CEILING_BYTES),
                                 (1, "bulk", READ_CEILING_BYTES // 36864 * 36864)):
        def run():
            st = lib.skinny_stream_read(ctypes.c_void_p(buf.data_ptr()), READ_CEILING_BYTES, method,
                                        ctypes.c_void_p(sink.data_ptr()), ctypes.c_void_p(stream.cuda_stream))
            if st != sk.OK:
                raise sk.SkinnyError(st, "skinny_stream_read")
        run()
        torch.cuda.synchronize()
        ts = []
        for _ in range(trials):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record()
            run()
            e1.record()
            torch.cuda.synchronize()
            ts.append(e0.elapsed_time(e1) * 1e-3)
        out[name] = {"GB/s": round(nbytes / min(ts) / 1e9, 1), "GB/s_median": round(nbytes / float(np.median(ts)) / 1e9, 1),
                     "bytes": nbytes}
    del buf
    torch.cuda.empty_cache()
    best = max(v["GB/s"] for v in out.values())
    return best, out


def launch_one(y, x, w, ws):
    import fp8_weight_only_w4a16_b200 as sk

    sk.gemm_into(y, x, w, workspace=ws)


def e2e_run(weights, xs, ys, ws, steps: int, warmup: int):
    """Same workload through the public API with host buffers.  Every step
    copies all its activations from pinned host memory to the device (one
    copy: they share one device buffer), runs the ten GEMMs (one CUDA graph),
    and reads all its outputs back to pinned host memory (one copy).  The
    activations and outputs are double-buffered on the device: step i's
    copy-in runs on one copy stream while step i-1's GEMMs run, and step i-1's
    read-back on another, ordered by events (a buffer is refilled only after
    the GEMMs two steps back have read it, and overwritten only after its
    read-back).  Every step's copies are inside the timed region."""
    import torch

    dev = xs["buffer"].device
    bufs = [(xs, ys), make_io_buffers(dev)]
    hx = xs["buffer"].cpu().pin_memory()
    hys = [torch.empty(ys["buffer"].shape, dtype=ys["buffer"].dtype).pin_memory() for _ in range(2)]
    h2d = xs["buffer"].numel()
    d2h = ys["buffer"].numel()

    graphs = {}
    compute = torch.cuda.Stream()
    compute.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(compute):
        for b, (bx, by) in enumerate(bufs):
            launch_step(weights, bx, by, ws, 0)
    torch.cuda.synchronize()
    for b, (bx, by) in enumerate(bufs):
        for phase in range(COPIES):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                launch_step(weights, bx, by, ws, phase)
            graphs[phase, b] = g
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()   # noqa: E731
    in_done = [ev(), ev()]
    gemm_done = [ev(), ev()]
    out_done = [ev(), ev()]
    for b in range(2):   # every buffer starts free
        gemm_done[b].record(compute)
        out_done[b].record(s_out)

    def one(i):
        b = i % 2
        x_buf, y_buf = bufs[b][0]["buffer"], bufs[b][1]["buffer"]
        s_in.wait_event(gemm_done[b])            # the GEMMs of step i-2 have read x_buf
        with torch.cuda.stream(s_in):
            x_buf.copy_(hx, non_blocking=True)
        in_done[b].record(s_in)
        compute.wait_event(in_done[b])
        compute.wait_event(out_done[b])          # step i-2's outputs have been read back
        with torch.cuda.stream(compute):
            graphs[i % COPIES, b].replay()
        gemm_done[b].record(compute)
        s_out.wait_event(gemm_done[b])
        with torch.cuda.stream(s_out):
            hys[b].copy_(y_buf, non_blocking=True)
        out_done[b].record(s_out)

    for i in range(warmup):
        one(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(compute)
    s_in.wait_stream(compute)
    for i in range(steps):
        one(warmup + i)
    compute.wait_stream(s_out)
    e1.record(compute)
    torch.cuda.synchronize()
    del graphs
    return e0.elapsed_time(e1), h2d, d2h


# ---------------------------------------------------------------------------
# The oracle on the host cores (CPU baseline and the reference arm)
# ---------------------------------------------------------------------------

def _oracle_inputs(frac: float):
    """Row samples of every GEMM of a step (both passes), as oracle inputs."""
    items = []
    for i, spec in enumerate(si.MIXED_LAYER):
        rows = max(1, int(round(spec.N * frac)))
        sub = si.GemmSpec(spec.name, spec.fmt, rows, spec.K, spec.scale_dist, spec.global_scale, spec.out)
        logical = si.weights_for(sub, seed=0, cfg_id=si.MIXED_CFG_ID, tensor_id=10 * i)
        for M in PASSES:
            x = si.activations(M, spec.K, seed=0, cfg_id=si.MIXED_CFG_ID, tensor_id=100 + i)
            items.append((sub, M, logical, x))
    return items


def _oracle_run(items, threads):
    import oracle

    t0 = time.perf_counter()
    for spec, M, logical, x in items:
        if spec.fmt == "nvfp4":
            oracle.nvfp4_gemm(x, logical[0], logical[1], spec.global_scale, threads=threads)
        else:
            oracle.fp8_gemm(x, logical[0], logical[1], threads=threads)
    return time.perf_counter() - t0


def _oracle_bytes(items) -> int:
    return sum(gemm_bytes(spec, M) for spec, M, _, _ in items)


def oracle_sample_frac(target_s: float, threads: int) -> float:
    """Row fraction whose oracle time is about target_s (two probes, so that the
    fixed per-call cost of the first does not skew the estimate)."""
    frac = 1.0 / 1024
    for _ in range(2):
        t = _oracle_run(_oracle_inputs(frac), threads)
        frac = float(min(1.0, max(1.0 / 4096, frac * target_s / max(t, 1e-3))))
        if t > 0.25 * target_s:
            break
    return frac


def _timed_oracle(target_s: float, threads: int):
    frac = oracle_sample_frac(target_s, threads)
    items = _oracle_inputs(frac)
    t, reps = 0.0, 0
    while t < 0.8 * target_s or reps == 0:   # the whole workload may take less than target_s
        t += _oracle_run(items, threads)
        reps += 1
    return reps * _oracle_bytes(items) / t / 1e9, frac, reps, t


def cpu_baseline(target_s: float = 12.0, single_core_s: float = 6.0):
    """The float64 oracle on every host core, and on one core."""
    import oracle

    threads = oracle.default_threads()
    value, frac, reps, t = _timed_oracle(target_s, threads)
    one, frac1, reps1, t1 = _timed_oracle(single_core_s, 1)
    return {"value": round(value, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": "float64 C oracle, %d threads, on the first %.3f%% of the rows of each of the 5 GEMMs of %s at "
                      "M=1 and M=8 (same byte formula), %d pass(es), %.1f s" % (threads, 100 * frac, WORKLOAD, reps, t),
            "single_core": {"value": round(one, 4), "unit": "GB/s", "cores": 1,
                            "sample": "the same oracle on 1 thread, first %.3f%% of the rows, %d pass(es), %.1f s"
                                      % (100 * frac1, reps1, t1)}}


def reference_arm(args):
    """The oracle as the reference arm: each step a bounded row sample of the workload."""
    import oracle

    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    threads = oracle.default_threads()
    # About 150 s of oracle time for the whole run, whatever K and W are.
    per_step_s = max(0.01, min(6.0, 150.0 / max(1, args.steps + args.warmup)))
    frac = oracle_sample_frac(per_step_s, threads)
    items = _oracle_inputs(frac)
    for _ in range(args.warmup):
        _oracle_run(items, threads)
    t = sum(_oracle_run(items, threads) for _ in range(args.steps))
    value = _oracle_bytes(items) * args.steps / t / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * t / args.steps, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": bench_config(args.gpus),
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": threads, "kind": "oracle",
                             "sample": "float64 C oracle on the first %.3f%% of the rows of each GEMM of %s "
                                       "at M=1 and M=8" % (100 * frac, WORKLOAD)},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def single_gemm(args):
    """Time one GEMM of the workload alone (direct launches, rotating weight
    copies): the small case that ncu captures are taken on."""
    import torch

    import fp8_weight_only_w4a16_b200 as sk

    name, M = args.single.split(":")
    M = int(M)
    idx = [s.name for s in si.MIXED_LAYER].index(name)
    spec = si.MIXED_LAYER[idx]
    torch.cuda.set_device(0)
    weights, xs, ys, ws = build_device_workload(torch.device("cuda", 0))
    if M not in xs:
        xs[M] = [torch.from_numpy(si.activations(M, s.K, seed=0, cfg_id=si.MIXED_CFG_ID, tensor_id=100 + i)).cuda()
                 for i, s in enumerate(si.MIXED_LAYER)]
        ys[M] = [torch.empty((M, s.N), dtype=torch.float16, device="cuda") for s in si.MIXED_LAYER]
    for i in range(args.warmup):
        sk.gemm_into(ys[M][idx], xs[M][idx], weights[i % COPIES][idx], workspace=ws)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for i in range(args.steps):
        sk.gemm_into(ys[M][idx], xs[M][idx], weights[i % COPIES][idx], workspace=ws)
    e1.record()
    torch.cuda.synchronize()
    us = 1e3 * e0.elapsed_time(e1) / args.steps
    b = gemm_bytes(spec, M)
    print(json.dumps({"single": args.single, "us_per_launch": round(us, 3), "GB/s": round(b / us / 1e3, 1),
                      "alg_bytes": b}), flush=True)
    return 0


# ---------------------------------------------------------------------------
# Main (our arm)
# ---------------------------------------------------------------------------

def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="skinny", choices=["skinny", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--single", default=None, help="NAME:M -- time one GEMM of the workload alone")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    if args.impl == "reference":
        return reference_arm(args)
    if args.single:
        return single_gemm(args)

    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit("--gpus %d but WORLD_SIZE=%d" % (args.gpus, world))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime

        dist.init_process_group("nccl", device_id=dev, timeout=datetime.timedelta(seconds=300))

    import fp8_weight_only_w4a16_b200 as sk

    peak, peak_src = load_peaks()
    weights, xs, ys, ws = build_device_workload(dev)
    graphs = capture_step_graphs(weights, xs, ys, ws)

    sampler = ClockSampler(local)
    # Per-launch device time of each GEMM (CUDA events around graphs of
    # back-to-back launches); this also brings the GPU to its loaded clocks.
    dur_us, best_us = per_launch_us(weights, xs, ys, ws)
    ro_peak, ro_methods = read_only_ceiling(dev)
    grouped = grouped_attention_us(weights, xs, ys, ws, peak)
    m16 = m16_per_gemm(weights, ws, dur_us, peak)
    fused = fused_epilogues_us(dev)

    for i in range(args.warmup):
        graphs[i % COPIES].replay()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.nvtx.range_push("timed_steps")   # lets a profiler list exactly the step's launches
    e0.record()
    for i in range(args.steps):
        graphs[i % COPIES].replay()
    e1.record()
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_pop()
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    # Ten more trials of the same K steps (not part of the value): their median
    # and best show how steady the timed region was.
    trial_ms = []
    for _ in range(10):
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record()
        for i in range(args.steps):
            graphs[i % COPIES].replay()
        t1.record()
        torch.cuda.synchronize()
        trial_ms.append(t0.elapsed_time(t1) / args.steps)
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    assert sk.device_error(clear=True) == 0, "a device-side wait gave up"

    e2e_ms, h2d, d2h = e2e_run(weights, xs, ys, ws, args.steps, args.warmup)
    e2e_ms = max_over_ranks(e2e_ms, world, dev)

    sb = step_bytes()
    value = whole_job_gbs(world, sb, args.steps, ms)
    e2e_value = whole_job_gbs(world, sb, args.steps, e2e_ms)

    # Roofline of the dominant kernel (the NVFP4 GEMM: 8 of 10 launches, most of the bytes).
    per = []
    nv_bytes = nv_us = 0.0
    nv_launches = 0
    for pi, M in enumerate(PASSES):
        for i, spec in enumerate(si.MIXED_LAYER):
            b = gemm_bytes(spec, M)
            d = float(dur_us[pi, i])
            per.append({"gemm": spec.name, "fmt": spec.fmt, "M": M, "N": spec.N, "K": spec.K,
                        "us": round(d, 3), "us_best": round(float(best_us[pi, i]), 3),
                        "GB/s": round(b / d / 1e3, 1), "frac": round(b / d / 1e3 / peak, 4)})
            if spec.fmt == "nvfp4":
                nv_bytes += b
                nv_us += d
                nv_launches += 1
    achieved = nv_bytes / nv_us / 1e3
    traffic = recorded_traffic(nv_bytes / nv_launches)

    line = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": bench_config(world),
        "frac_of_peak": round(value / world / peak, 4),
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(achieved / peak, 4), "traffic": traffic, "peak_source": peak_src,
                     "peak_read_only": ro_peak, "frac_read_only": round(achieved / ro_peak, 4),
                     "read_only_ceiling": dict(ro_methods, note="measured in this run: the library's read-only "
                                               "streaming kernels over 4 GiB, best of 5; the faster is peak_read_only"),
                     "kernel": "gemm_kernel<NVFP4>", "launches_in_step": nv_launches,
                     "method": "per-launch device time from CUDA events around graphs of 30 back-to-back launches "
                               "of each GEMM over rotating weight copies > 4x L2, measured in this process before "
                               "the timed region; achieved = algorithmic bytes / time summed over the step's NVFP4 "
                               "launches"},
        "sum_launch_us": round(float(dur_us.sum()), 2),
        "step_trials": {"ms_per_step_median": round(float(np.median(trial_ms)), 5),
                        "ms_per_step_best": round(float(np.min(trial_ms)), 5), "trials": len(trial_ms),
                        "note": "10 more runs of the same K steps after the timed region (not part of value)"},
        "per_gemm": per,
        "grouped_attention": grouped,
        "per_gemm_m16": m16,
        "fused_epilogues": dict(fused, note="next rows: the per-token argmax, the SiLU*mul activation and the "
                                            "residual add fused into the GEMM epilogue, each next to the plain "
                                            "GEMM it replaces; per-launch device time, not part of the step"),
        "e2e": {"value": round(e2e_value, 2), "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": len(PASSES) * len(si.MIXED_LAYER) * args.steps,
        "clocks": clocks,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline()
    del graphs
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
