"""Benchmark of the W4A16 linear layer: effective HBM GB/s and TFLOP/s against the roofline.

One step = the Llama-7B-shaped W4A16 layer set ((K, N) = (4096, 12288) fused QKV,
(4096, 4096) out-proj, (4096, 22016) gate+up, (11008, 4096) down; g = 128) at every batch
size M in {1, 2, 4, 8, 16, 32, 64, 128}: 32 calls of the layer. Inputs are seeded synthetic
data with the distributions of the layer configuration (fp16 N(0,1) activations, uniform
4-bit codes, fp16 scales 0.002 + 0.01|N(0,1)|). Prepacking happens once, outside timing.

Four prepacked copies of the layer set (404 MB of weights) rotate across the M values, so a
copy is re-read only after three other copies (303 MB) went through the 126 MB L2: every
weight byte of a call comes from HBM. The step is captured once in a CUDA graph and replayed.

Printed: one JSON line (rank 0). ``value`` = algorithmic bytes of all ranks' steps / the
slowest rank's device time (GB/s); algorithmic bytes of one call = K*N/2 (codes) +
2*(K/g)*N (scales) + 2*M*K (A) + 2*M*N (Y). ``--gpus N`` runs N independent replicas (the
layer does not shard across GPUs here), one process per GPU under torchrun.
``--impl reference`` times the CPU fp64 oracle on a bounded sample of the same workload.
``--case K,N,g,M`` replaces the layer set by one layer (profiling runs): a step is then one
call on each of enough rotated prepacked copies to exceed L2 three times over.
"""
from __future__ import annotations

import argparse
import datetime
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

import synth  # noqa: E402

LAYERS = [(4096, 12288), (4096, 4096), (4096, 22016), (11008, 4096)]
M_SWEEP = [1, 2, 4, 8, 16, 32, 64, 128]
G = 128
COPIES = 4
METRIC = "W4A16 GEMM TFLOP/s and effective HBM GB/s vs roofline fraction at M=1..128"
WORKLOAD = "llama7b_w4a16_layer_set_M1-128_g128"

# Fallback denominators (an earlier measurement on this machine) when MEASURED_PEAKS.json is absent.
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0

# DRAM traffic per launch of the dominant kernel (dram__bytes_read.sum + dram__bytes_write.sum
# from ncu captures of single launches on one layer of the set, scaled to this workload's launches
# by their algorithmic bytes), valid for the kernel sources whose hash is recorded with it and
# reported as null once they change.
TRAFFIC = {"kernel_sha": "7f2277a5710e86ea", "bytes_per_launch": 26125031, "algo_bytes_per_launch": 26291379,
           "how": "dram__bytes_read.sum + dram__bytes_write.sum of one launch of the dominant kernel on the "
                  "4096x22016 layer at M = 1 and M = 16 (1.0004 and 0.9869 of their algorithmic bytes), the mean "
                  "ratio times this workload's average algorithmic bytes per launch of that kernel"}


def kernel_sha() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "bit_weight_quantized_prepack_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        if f.endswith((".cu", ".cuh", ".h")):
            h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def algo_bytes(M, K, N, g=G):
    return K * N // 2 + 2 * (K // g) * N + 2 * M * K + 2 * M * N


def algo_flops(M, K, N):
    return 2 * M * N * K


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


def step_totals():
    b = sum(algo_bytes(M, K, N) for M in M_SWEEP for (K, N) in LAYERS)
    f = sum(algo_flops(M, K, N) for M in M_SWEEP for (K, N) in LAYERS)
    return b, f


def roofline_time(M, K, N, hbm_gbs, tflops, g=None):
    return max(algo_bytes(M, K, N, G if g is None else g) / (hbm_gbs * 1e9), algo_flops(M, K, N) / (tflops * 1e12))


def fp16_bound_time(M, K, N, hbm_gbs):
    """Time to move a dense fp16 weight, A and Y at the copy bandwidth: what the same layer with
    fp16 weights cannot beat. (time of this bound) / (measured time) is the speedup over it."""
    return (2 * K * N + 2 * M * K + 2 * M * N) / (hbm_gbs * 1e9)


def launch_times(torch, stream, fns, reps):
    """Per-launch device times (s) of isolated launches: fns are single calls, made round robin
    (so consecutive launches read different weight copies), each between two CUDA events on the
    launching stream. An isolated launch does not overlap its neighbours, unlike the step's
    back-to-back launches (which set up while the previous kernel finishes)."""
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(reps)]
    with torch.cuda.stream(stream):
        for fn in fns:
            fn()
        for i in range(reps):
            evs[i][0].record(stream)
            fns[i % len(fns)]()
            evs[i][1].record(stream)
    stream.synchronize()
    return [a.elapsed_time(b) / 1e3 for a, b in evs]


def pct_us(ts):
    """(p10, median, p90) of times in seconds, as microseconds."""
    return [round(float(np.percentile(ts, q)) * 1e6, 2) for q in (10, 50, 90)]


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu = gpu_id
        self.proc = None
        self.path = None
        self.t_start = self.t_stop = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu=timestamp,{self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def mark(self, which):
        setattr(self, "t_" + which, datetime.datetime.now())

    def stop(self):
        time.sleep(0.15)
        if self.proc:
            self.proc.terminate()
            self.proc.wait()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f")
            except ValueError:
                continue
            rows.append((ts, parts))
        os.unlink(self.path)
        inside = [r for r in rows if self.t_start and self.t_stop and self.t_start <= r[0] <= self.t_stop]
        used = inside if inside else rows
        if not used:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no nvidia-smi samples"], "samples": 0}
        sm = [float(r[1][2]) for r in used if r[1][2].replace(".", "").isdigit()]
        smax = [float(r[1][3]) for r in used if r[1][3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in used for i, v in enumerate(r[1][6:10]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(used), "samples_in_window": len(inside)}


# ------------------------------------------------------------------ multi-rank helpers
def max_over_ranks(x: float, device) -> float:
    """The largest x over all ranks (the slowest rank's time); x itself when not distributed."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, bytes_per_step: float, steps: int, seconds: float) -> float:
    """Whole-job GB/s: every rank runs the same step (replicas), timed by the slowest rank."""
    return world * bytes_per_step * steps / seconds / 1e9


# ------------------------------------------------------------------ breakdowns outside the timed region
COMPUTE_SWEEP = {"K": 8192, "N": 8192, "g": 128, "M": [256, 512, 1024, 4096]}
W4A8_LAYERS = [(4096, 11008), (11008, 4096)]
W4A8_M = [1, 16, 128, 1024]


def _graph_time(torch, stream, fn, reps):
    """Seconds per call of fn(r) for r in 0..reps-1, captured once in a CUDA graph and replayed."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(g, stream=stream):
            for r in range(reps):
                fn(r)
        g.replay()
        stream.synchronize()
        a0 = torch.cuda.Event(enable_timing=True)
        a1 = torch.cuda.Event(enable_timing=True)
        a0.record(stream)
        for _ in range(5):
            g.replay()
        a1.record(stream)
    stream.synchronize()
    t = a0.elapsed_time(a1) / 1e3 / (5 * reps)
    del g
    return t


LAYERS_70B = [(8192, 10240), (8192, 8192), (8192, 57344), (28672, 8192)]
M_70B = [1, 16, 64, 128]


def rows_70b(torch, wq, dev, stream, hbm_gbs, tflops):
    """The 70B-shaped W4A16 layers at M in {1, 16, 64, 128}, each with g = 128 and with one scale
    per column (g = K): per-launch p10 / median / p90 over rotated weight copies (more than 3x
    L2 per rotation), effective GB/s, roofline fraction and the speedup over the dense fp16
    weight-read bound, all from the median."""
    out = {}
    for K, N in LAYERS_70B:
        for g in (128, K):
            d = synth.w4a16_inputs(K, N, g, max(M_70B), seed=21)
            Q, s = torch.from_numpy(d["Q"]).to(dev), torch.from_numpy(d["s"]).to(dev)
            wbytes = K * N // 2 + 2 * (K // g) * N
            copies = int(min(12, max(2, -(-3 * 126_000_000 // wbytes))))
            Wps = [wq.wq_prepack(Q, s, g) for _ in range(copies)]
            A = torch.from_numpy(d["A"]).to(dev)
            for M in M_70B:
                Am = A[:M].contiguous()
                Y = torch.empty((M, N), dtype=torch.float16, device=dev)
                wq.wq_workspace_reserve(wq.wq_workspace_bytes(0, M, N, K), stream=stream)
                fns = [(lambda W: lambda: wq.wq_gemm_w4a16(Am, W, N, g, Y=Y, stream=stream))(W) for W in Wps]
                ts = launch_times(torch, stream, fns, max(12, 2 * copies))
                p10, med, p90 = pct_us(ts)
                t = med / 1e6
                out[f"{K}x{N}_g{'K' if g == K else g}_M{M}"] = {
                    "us_p10_med_p90": [p10, med, p90],
                    "gbs": round(algo_bytes(M, K, N, g) / t / 1e9, 1),
                    "tflops": round(algo_flops(M, K, N) / t / 1e12, 2),
                    "roofline_frac": round(roofline_time(M, K, N, hbm_gbs, tflops, g) / t, 3),
                    "speedup_vs_fp16_bound": round(fp16_bound_time(M, K, N, hbm_gbs) / t, 2)}
            del Wps, Q, s, A
    return out


SPARSE_LAYERS = LAYERS + [(8192, 57344)]
SPARSE_M = [1, 4, 16]


def sparse_algo_bytes(M, K, N, g=G):
    """Algorithmic bytes of one 2:4 sparse call: the kept codes (K/2 x N x 4 bits), their
    positions (K/4 groups x N x 4 bits), the scales, A and Y."""
    return K * N // 4 + K * N // 8 + 2 * (K // g) * N + 2 * M * K + 2 * M * N


def rows_sparse24(torch, wq, dev, stream, hbm_gbs):
    """2:4 sparse W4A16 (the Llama-7B layers and the 70B gate/up layer, g = 128, M in {1, 4, 16}):
    the same pruned weight through the dense and the sparse buffer, each call back to back in a
    CUDA graph over rotated copies (more than 3x L2 per rotation); per call: microseconds, GB/s
    of the sparse call's own algorithmic bytes, its roofline fraction, and the dense call's time
    over the sparse call's."""
    out = {}
    for K, N in SPARSE_LAYERS:
        d = synth.w4a16_sparse24_inputs(K, N, G, max(SPARSE_M), seed=31)
        Q, s = torch.from_numpy(d["Q"]).to(dev), torch.from_numpy(d["s"]).to(dev)
        copies = int(min(12, max(2, -(-3 * 126_000_000 // (K * N * 3 // 8)))))
        Wd = [wq.wq_prepack(Q, s, G) for _ in range(copies)]
        Ws = [wq.wq_prepack_sparse24(Q, s, G) for _ in range(copies)]
        A = torch.from_numpy(d["A"]).to(dev)
        for M in SPARSE_M:
            Am = A[:M].contiguous()
            Y = torch.empty((M, N), dtype=torch.float16, device=dev)
            wq.wq_workspace_reserve(wq.wq_workspace_bytes(0, M, N, K), stream=stream)
            td = _graph_time(torch, stream, lambda r: wq.wq_gemm_w4a16(Am, Wd[r % copies], N, G, Y=Y, stream=stream),
                             2 * copies)
            ts = _graph_time(torch, stream,
                             lambda r: wq.wq_gemm_w4a16_sparse24(Am, Ws[r % copies], N, G, Y=Y, stream=stream),
                             2 * copies)
            b = sparse_algo_bytes(M, K, N)
            out[f"{K}x{N}_M{M}"] = {"us": round(ts * 1e6, 2), "dense_us": round(td * 1e6, 2),
                                   "gbs": round(b / ts / 1e9, 1), "roofline_frac": round(b / (hbm_gbs * 1e9) / ts, 3),
                                   "speedup_vs_dense": round(td / ts, 3)}
        del Wd, Ws, Q, s, A
    return out


MIXED_FRAC4 = 0.15


def mixed_algo_bytes(M, K, N, n4, g=G):
    """Algorithmic bytes of one mixed 2/4-bit call: 2-bit and 4-bit code blocks (1024 or 2048
    bytes per 32 x 128 block), the scales, A and Y (the blob table is bookkeeping, not counted)."""
    blocks = (K // 32) * -(-N // 128)
    return (blocks - n4) * 1024 + n4 * 2048 + 2 * (K // g) * N + 2 * M * K + 2 * M * N


def rows_mixed(torch, wq, dev, stream, hbm_gbs):
    """Mixed 2/4-bit W4A16 (the Llama-7B layers and the 70B gate/up layer, g = 128, 15 % of the
    32 x 128 blocks at 4 bits, M in {1, 4, 16}): the same weight through the dense buffer and the
    mixed one, each call back to back in a CUDA graph over rotated copies; per call:
    microseconds, GB/s of the mixed call's own algorithmic bytes, its roofline fraction, and the
    dense call's time over the mixed call's."""
    out = {}
    for K, N in SPARSE_LAYERS:
        d = synth.w4a16_mixed_inputs(K, N, G, max(SPARSE_M), seed=37, frac4=MIXED_FRAC4)
        Q, s = torch.from_numpy(d["Q"]).to(dev), torch.from_numpy(d["s"]).to(dev)
        W = torch.from_numpy(d["widths"]).to(dev)
        n4 = int((d["widths"] == 4).sum())
        nb = wq.wq_prepacked_bytes_mixed(K, N, G, n4)
        copies = int(min(12, max(2, -(-3 * 126_000_000 // nb))))
        Wd = [wq.wq_prepack(Q, s, G) for _ in range(copies)]
        Wm = [wq.wq_prepack_mixed(Q, s, W, G) for _ in range(copies)]
        A = torch.from_numpy(d["A"]).to(dev)
        for M in SPARSE_M:
            Am = A[:M].contiguous()
            Y = torch.empty((M, N), dtype=torch.float16, device=dev)
            wq.wq_workspace_reserve(wq.wq_workspace_bytes(0, M, N, K), stream=stream)
            td = _graph_time(torch, stream, lambda r: wq.wq_gemm_w4a16(Am, Wd[r % copies], N, G, Y=Y, stream=stream),
                             2 * copies)
            tm = _graph_time(torch, stream,
                             lambda r: wq.wq_gemm_w4a16_mixed(Am, Wm[r % copies], N, G, Y=Y, stream=stream), 2 * copies)
            b = mixed_algo_bytes(M, K, N, n4)
            out[f"{K}x{N}_M{M}"] = {"us": round(tm * 1e6, 2), "dense_us": round(td * 1e6, 2),
                                   "gbs": round(b / tm / 1e9, 1), "roofline_frac": round(b / (hbm_gbs * 1e9) / tm, 3),
                                   "speedup_vs_dense": round(td / tm, 3), "bits_per_weight": round(8 * nb / (K * N), 2)}
        del Wd, Wm, Q, s, A
    return out


def extra_breakdowns(torch, wq, dev, stream, hbm_gbs, tflops):
    """The compute-bound W4A16 sweep (K = N = 8192) and the W4A8 layers, each timed alone."""
    out = {"compute_sweep": {}, "w4a8": {}}
    cs = COMPUTE_SWEEP
    K, N, g = cs["K"], cs["N"], cs["g"]
    d = synth.w4a16_inputs(K, N, g, max(cs["M"]), seed=11)
    Wp = wq.wq_prepack(torch.from_numpy(d["Q"]).to(dev), torch.from_numpy(d["s"]).to(dev), g)
    A = torch.from_numpy(d["A"]).to(dev)
    for M in cs["M"]:
        Am = A[:M].contiguous()
        Y = torch.empty((M, N), dtype=torch.float16, device=dev)
        wq.wq_workspace_reserve(wq.wq_workspace_bytes(0, M, N, K), stream=stream)
        t = _graph_time(torch, stream, lambda r: wq.wq_gemm_w4a16(Am, Wp, N, g, Y=Y, stream=stream), 4)
        f = 2 * M * N * K
        out["compute_sweep"][str(M)] = {"us": round(t * 1e6, 2), "tflops": round(f / t / 1e12, 1),
                                        "tensor_frac": round(f / t / 1e12 / tflops, 3)}
    del Wp, A
    int8_peak = 2 * tflops  # int8 dense peak: the measured bf16 peak times the nominal 2x ratio
    for K, N in W4A8_LAYERS:
        d = synth.w4a8_inputs(K, N, max(W4A8_M), seed=12)
        Q = torch.from_numpy(d["Q"]).to(dev)
        copies = max(2, -(-3 * 126_000_000 // (K * N // 2)))
        Wps = [wq.wq_prepack_w4a8(Q) for _ in range(copies)]
        sw = torch.from_numpy(d["sw"]).to(dev)
        A = torch.from_numpy(d["A"]).to(dev)
        sa = torch.from_numpy(d["sa"]).to(dev)
        for M in W4A8_M:
            Am, sam = A[:M].contiguous(), sa[:M].contiguous()
            Y = torch.empty((M, N), dtype=torch.float16, device=dev)
            wq.wq_workspace_reserve(wq.wq_workspace_bytes(1, M, N, K), stream=stream)
            t = _graph_time(torch, stream,
                            lambda r: wq.wq_gemm_w4a8(Am, sam, Wps[r % copies], sw, N, Y=Y, stream=stream), 2 * copies)
            b = K * N // 2 + 4 * N + M * K + 4 * M + 2 * M * N
            ops = 2 * M * N * K
            troof = max(b / (hbm_gbs * 1e9), ops / (int8_peak * 1e12))
            out["w4a8"][f"{K}x{N}_M{M}"] = {"us": round(t * 1e6, 2), "gbs": round(b / t / 1e9, 1),
                                           "tops": round(ops / t / 1e12, 1), "roofline_frac": round(troof / t, 3)}
        del Wps
    # the layer on fp16 activations (per-token quantisation to 8 bits, W4A8, or to 4 bits, W4A4, then
    # the int8 layer, one call) and the 8-bit quantisation kernel alone (HBM-bound: 2MK bytes read,
    # MK + 4M written)
    out["w4a8_fp16act"] = {}
    for K, N in W4A8_LAYERS:
        d = synth.w4a8_inputs(K, N, 1, seed=13)
        Q = torch.from_numpy(d["Q"]).to(dev)
        copies = max(2, -(-3 * 126_000_000 // (K * N // 2)))
        Wps = [wq.wq_prepack_w4a8(Q) for _ in range(copies)]
        sw = torch.from_numpy(d["sw"]).to(dev)
        for M in W4A8_M:
            A16 = torch.randn((M, K), generator=torch.Generator().manual_seed(M), dtype=torch.float32).half().to(dev)
            Y = torch.empty((M, N), dtype=torch.float16, device=dev)
            Aq = torch.empty((M, K), dtype=torch.int8, device=dev)
            sa = torch.empty((M,), dtype=torch.float32, device=dev)
            wq.wq_workspace_reserve(wq.wq_workspace_bytes(2, M, N, K), stream=stream)
            t = _graph_time(torch, stream,
                            lambda r: wq.wq_gemm_w4a8_fp16act(A16, Wps[r % copies], sw, N, Y=Y, stream=stream), 2 * copies)
            tq = _graph_time(torch, stream, lambda r: wq.wq_quantize_act(A16, Aq, sa, stream=stream), 8)
            bq = 3 * M * K + 4 * M
            t4 = _graph_time(torch, stream, lambda r: wq.wq_gemm_w4a8_fp16act(A16, Wps[r % copies], sw, N, Y=Y,
                                                                                stream=stream, act_bits=4), 2 * copies)
            out["w4a8_fp16act"][f"{K}x{N}_M{M}"] = {"us": round(t * 1e6, 2), "w4a4_us": round(t4 * 1e6, 2),
                                                   "quantize_us": round(tq * 1e6, 2),
                                                   "quantize_gbs": round(bq / tq / 1e9, 1)}
        del Wps
    out["peaks"] = {"tensor_tflops": tflops, "int8_tops": int8_peak,
                    "note": "int8 peak = measured bf16 peak x the nominal 2x ratio"}
    out["layers_70b"] = rows_70b(torch, wq, dev, stream, hbm_gbs, tflops)
    out["sparse24"] = rows_sparse24(torch, wq, dev, stream, hbm_gbs)
    out["mixed24"] = rows_mixed(torch, wq, dev, stream, hbm_gbs)
    return out


# ------------------------------------------------------------------ our implementation
def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    import bit_weight_quantized_prepack_b200 as wq

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180), device_id=dev)

    hbm_gbs, tflops, tflops_sus, peak_src = peaks()

    # inputs: one seeded draw per layer; A holds 128 rows, smaller M use the first rows
    layers = []
    for li, (K, N) in enumerate(LAYERS):
        d = synth.w4a16_inputs(K, N, G, max(M_SWEEP), seed=li)
        Q = torch.from_numpy(d["Q"]).to(dev)
        s = torch.from_numpy(d["s"]).to(dev)
        Wp0 = wq.wq_prepack(Q, s, G)
        copies = [Wp0] + [Wp0.clone() for _ in range(COPIES - 1)]
        A = torch.from_numpy(d["A"]).to(dev)
        layers.append({"K": K, "N": N, "Wp": copies, "A": {M: A[:M].contiguous() for M in M_SWEEP},
                       "Y": {M: torch.empty((M, N), dtype=torch.float16, device=dev) for M in M_SWEEP},
                       "A_host": {M: A[:M].cpu() for M in M_SWEEP}})
        del Q, s
    torch.cuda.synchronize()

    stream = torch.cuda.Stream(device=dev)
    ws = max(wq.wq_workspace_bytes(0, M, L["N"], L["K"]) for M in M_SWEEP for L in layers)
    wq.wq_workspace_reserve(ws, stream=stream)

    def step_calls(st):
        for mi, M in enumerate(M_SWEEP):
            c = mi % COPIES
            for L in layers:
                wq.wq_gemm_w4a16(L["A"][M], L["Wp"][c], L["N"], G, Y=L["Y"][M], stream=st)

    launches_per_step = len(M_SWEEP) * len(LAYERS)
    with torch.cuda.stream(stream):
        step_calls(stream)  # eager once (also checks the status path)
    stream.synchronize()
    if wq.wq_get_device_status(stream) != wq.WQ_OK:
        raise RuntimeError("device status not OK after the first step")
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(graph, stream=stream):
            step_calls(stream)
    stream.synchronize()

    for _ in range(args.warmup):
        with torch.cuda.stream(stream):
            graph.replay()
    stream.synchronize()

    props = torch.cuda.get_device_properties(dev)
    uuid = str(getattr(props, "uuid", "") or "")
    sampler = ClockSampler(("GPU-" + uuid) if uuid and not uuid.startswith("GPU-") else (uuid or str(local_rank)))
    sampler.start()
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    sampler.mark("start")
    with torch.cuda.stream(stream):
        ev0.record(stream)
        for _ in range(args.steps):
            graph.replay()
        ev1.record(stream)
    torch.cuda.synchronize()
    # a timed region shorter than the sampling period may hold no clock sample: the same step is
    # then replayed, untimed, until half a second has passed, and the samples of that whole window
    # are reported (the window is named in the record)
    window = "timed region"
    t_reg = (datetime.datetime.now() - sampler.t_start).total_seconds()
    if t_reg < 0.5:
        window = "timed region and untimed replays of the same step right after it (0.5 s in all)"
        with torch.cuda.stream(stream):
            while (datetime.datetime.now() - sampler.t_start).total_seconds() < 0.5:
                for _ in range(20):
                    graph.replay()
                stream.synchronize()
    sampler.mark("stop")
    if world > 1:
        dist.barrier()
    clocks = sampler.stop()
    clocks["window"] = window
    t_local = ev0.elapsed_time(ev1) / 1e3
    t = max_over_ranks(t_local, dev)
    if wq.wq_get_device_status(stream) != wq.WQ_OK:
        raise RuntimeError("device status not OK after the timed region")

    bytes_step, flops_step = step_totals()
    value = job_throughput(world, bytes_step, args.steps, t)
    ms_per_step = t / args.steps * 1e3

    # ---------------------------------------------------------- end to end through the public API
    # Every step copies all of its inputs (the 32 calls' A, one pinned host buffer) to the
    # device, makes the 32 public-API calls on views of that buffer, and copies all of their
    # results back to one pinned host buffer, all inside the timed region. Device buffers are
    # double-buffered and the copies run on their own streams, so that the next step's inputs
    # go in and the previous step's results come out while the kernels run (events order each
    # buffer's reuse).
    e2e_steps = max(1, min(args.steps, args.e2e_steps))
    calls = [(mi, M, li) for mi, M in enumerate(M_SWEEP) for li in range(len(layers))]
    a_off, y_off, ao, yo = [], [], 0, 0
    for mi, M, li in calls:
        a_off.append(ao)
        y_off.append(yo)
        ao += M * layers[li]["K"]
        yo += M * layers[li]["N"]
    h2d, d2h = 2 * ao, 2 * yo
    a_host = torch.empty(ao, dtype=torch.float16).pin_memory()
    for (mi, M, li), o in zip(calls, a_off):
        a_host[o:o + M * layers[li]["K"]].copy_(layers[li]["A_host"][M].reshape(-1))
    y_host = torch.empty(yo, dtype=torch.float16).pin_memory()
    a_dev = [torch.empty(ao, dtype=torch.float16, device=dev) for _ in range(2)]
    y_dev = [torch.empty(yo, dtype=torch.float16, device=dev) for _ in range(2)]
    s_in = torch.cuda.Stream(device=dev)
    s_out = torch.cuda.Stream(device=dev)
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_mm = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0.record(stream)
    s_in.wait_stream(stream)
    s_out.wait_stream(stream)
    for step in range(e2e_steps):
        b = step & 1
        with torch.cuda.stream(s_in):
            if step >= 2:
                s_in.wait_event(ev_mm[b])     # the kernels of step - 2 have read this buffer
            a_dev[b].copy_(a_host, non_blocking=True)
            ev_in[b].record(s_in)
        stream.wait_event(ev_in[b])
        if step >= 2:
            stream.wait_event(ev_out[b])      # step - 2's results have left this buffer
        for (mi, M, li), oa, oy in zip(calls, a_off, y_off):
            L = layers[li]
            A = a_dev[b][oa:oa + M * L["K"]].view(M, L["K"])
            Y = y_dev[b][oy:oy + M * L["N"]].view(M, L["N"])
            wq.wq_gemm_w4a16(A, L["Wp"][mi % COPIES], L["N"], G, Y=Y, stream=stream)
        ev_mm[b].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_mm[b])
            y_host.copy_(y_dev[b], non_blocking=True)
            ev_out[b].record(s_out)
    stream.wait_stream(s_in)
    stream.wait_stream(s_out)
    e1.record(stream)
    torch.cuda.synchronize()
    te = max_over_ranks(e0.elapsed_time(e1) / 1e3, dev)
    e2e_value = job_throughput(world, bytes_step, e2e_steps, te)

    # ---------------------------------------------------------- per-M breakdown (rank 0, outside timing)
    per_m = {}
    c1_row = {}  # the single 4096 x 4096 layer at M = 1, g = 128, timed alone
    if rank == 0 and not args.no_breakdown:
        for mi, M in enumerate(M_SWEEP):
            g2 = torch.cuda.CUDAGraph()
            reps = 8
            with torch.cuda.stream(stream):
                with torch.cuda.graph(g2, stream=stream):
                    for r in range(reps):
                        for L in layers:
                            wq.wq_gemm_w4a16(L["A"][M], L["Wp"][r % COPIES], L["N"], G, Y=L["Y"][M], stream=stream)
                g2.replay()
                stream.synchronize()
                a0 = torch.cuda.Event(enable_timing=True)
                a1 = torch.cuda.Event(enable_timing=True)
                a0.record(stream)
                for _ in range(10):
                    g2.replay()
                a1.record(stream)
            stream.synchronize()
            tm = a0.elapsed_time(a1) / 1e3 / (10 * reps)
            b = sum(algo_bytes(M, L["K"], L["N"]) for L in layers)
            f = sum(algo_flops(M, L["K"], L["N"]) for L in layers)
            troof = sum(roofline_time(M, L["K"], L["N"], hbm_gbs, tflops) for L in layers)
            t16 = sum(fp16_bound_time(M, L["K"], L["N"], hbm_gbs) for L in layers)
            per_m[str(M)] = {"us": round(tm * 1e6, 2), "gbs": round(b / tm / 1e9, 1),
                             "tflops": round(f / tm / 1e12, 2), "roofline_frac": round(troof / tm, 3),
                             "speedup_vs_fp16_bound": round(t16 / tm, 2), "launch_us_p10_med_p90": {}}
            del g2
            # per-launch distribution: each layer alone, one launch per graph replay
            for L in layers:
                fns = [(lambda W: lambda: wq.wq_gemm_w4a16(L["A"][M], W, L["N"], G, Y=L["Y"][M], stream=stream))(W)
                       for W in L["Wp"]]
                ts = launch_times(torch, stream, fns, 4 * COPIES)
                per_m[str(M)]["launch_us_p10_med_p90"][f"{L['K']}x{L['N']}"] = pct_us(ts)
                if (L["K"], L["N"]) == (4096, 4096) and M == 1:
                    t = float(np.median(ts))
                    c1_row.update({"us_p10_med_p90": pct_us(ts), "gbs": round(algo_bytes(1, 4096, 4096) / t / 1e9, 1),
                                   "roofline_frac": round(roofline_time(1, 4096, 4096, hbm_gbs, tflops) / t, 3),
                                   "speedup_vs_fp16_bound": round(fp16_bound_time(1, 4096, 4096, hbm_gbs) / t, 2)})

    # ---------------------------------------------------------- the dominant kernel's roofline
    # The calls whose plan is the register-operand kernel (576 threads: the small M of decoding)
    # take the largest share of the step's device time. They are captured in their own graph, in
    # the step's order and weight copies, and timed like the step (events on the launching stream
    # around whole replays).
    def family(M):
        pl = wq.wq_plan(0, M, LAYERS[0][1], LAYERS[0][0], G)
        if pl["threads"] == 576:
            return "wq_gemm_rf<fp16 groups> (register-operand tiles)"
        return f"wq_gemm_small<fp16 groups, {pl['tile_m']}-row tiles>" if pl["tile_m"] <= 32 else "wq_gemm_large<fp16 groups>"

    dom_ms = sorted({M for M in M_SWEEP if wq.wq_plan(0, M, LAYERS[0][1], LAYERS[0][0], G)["threads"] == 576})
    if not dom_ms:  # a single-layer case (--case) whose M runs another kernel: that kernel is the one timed
        dom_ms = sorted(set(M_SWEEP))
    dom_kernel = family(dom_ms[0])
    dom_calls = [(mi, M, L) for mi, M in enumerate(M_SWEEP) if M in dom_ms for L in layers]
    gd = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(gd, stream=stream):
            for mi, M, L in dom_calls:
                wq.wq_gemm_w4a16(L["A"][M], L["Wp"][mi % COPIES], L["N"], G, Y=L["Y"][M], stream=stream)
        for _ in range(3):
            gd.replay()
        d0 = torch.cuda.Event(enable_timing=True)
        d1 = torch.cuda.Event(enable_timing=True)
        d0.record(stream)
        dom_reps = max(5, min(args.steps, 200))
        for _ in range(dom_reps):
            gd.replay()
        d1.record(stream)
    stream.synchronize()
    t_dom = d0.elapsed_time(d1) / 1e3 / dom_reps / len(dom_calls)  # average launch duration
    b_dom = sum(algo_bytes(M, L["K"], L["N"]) for mi, M, L in dom_calls) / len(dom_calls)
    del gd

    extras = {}
    if rank == 0 and not args.no_breakdown and not args.case:
        extras = extra_breakdowns(torch, wq, dev, stream, hbm_gbs, tflops)

    troof_step = sum(roofline_time(M, K, N, hbm_gbs, tflops) for M in M_SWEEP for (K, N) in LAYERS)
    achieved = b_dom / t_dom / 1e9
    sha = kernel_sha()
    # the recorded figure belongs to the default workload (the layer set) and these kernel sources
    traffic = TRAFFIC["bytes_per_launch"] if TRAFFIC["kernel_sha"] == sha and not args.case else None

    out = {
        "metric": METRIC, "value": round(value, 1), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "fp16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "layers_KN": LAYERS, "M": M_SWEEP, "g": G,
                   "l2": f"inputs larger than L2: {COPIES} rotated prepacked copies of the layer set "
                         f"({COPIES * sum(K * N // 2 + 2 * (K // G) * N for K, N in LAYERS) / 1e6:.0f} MB)",
                   "parallelism": f"replicas{world}" if world > 1 else "single"},
        "tflops": round(world * flops_step * args.steps / t / 1e12, 2),
        "roofline_time_frac": round(troof_step / (t_local / args.steps), 3),
        "step_roofline": {"time_frac": round(troof_step / (t_local / args.steps), 3),
                          "note": "the step's headline fraction: the sum over its 32 calls of max(algorithmic "
                                  "bytes / measured copy bandwidth, flops / measured bf16 peak), over the step's "
                                  "device time (M = 64 and 128 are past the ridge, so a pure bandwidth fraction "
                                  "of the whole step would understate them)"},
        "roofline": {"bound": "hbm", "kernel": f"{dom_kernel}: the step's M = {', '.join(map(str, dom_ms))} calls",
                     "achieved": round(achieved, 1), "peak": hbm_gbs, "unit": "GB/s",
                     "frac": round(achieved / hbm_gbs, 3), "traffic": traffic,
                     "traffic_how": TRAFFIC["how"] if traffic is not None else None,
                     "traffic_algo_bytes": round(b_dom),
                     "launch_us": round(t_dom * 1e6, 2),
                     "peak_source": f"{peak_src} hbm_gbs (copy bandwidth), of measured",
                     "note": f"achieved = average algorithmic bytes per launch of the {len(dom_calls)} calls "
                             f"(weights + scales + A + Y) / their average launch duration, CUDA events over "
                             f"{dom_reps} replays of a graph holding just those calls in the step's order"},
        "c1_4096x4096_M1": c1_row,
        "e2e": {"value": round(e2e_value, 1), "unit": "GB/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps, "copies": "per step one pinned host-to-device copy of all inputs and one "
                                              "device-to-host copy of all results, on their own streams, "
                                              "double-buffered so that they overlap the kernels"},
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
        "per_m": per_m,
        **extras,
        "kernel_sha": sha,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(args.cpu_sample)
    del graph
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out), flush=True)


# ------------------------------------------------------------------ the oracle as the CPU baseline
def _cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


def _host_info():
    """CPU model and the BLAS threads numpy uses (what the oracle's matrix product runs on)."""
    model = None
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                model = line.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    threads = None
    try:
        from threadpoolctl import threadpool_info
        threads = max((i.get("num_threads") or 0) for i in threadpool_info() if i.get("user_api") == "blas") or None
    except Exception:
        pass
    return {"cpu_model": model, "blas_threads": threads}


def _oracle_pairs():
    return [(M, K, N, li) for M in M_SWEEP for li, (K, N) in enumerate(LAYERS)]


def cpu_baseline(n_pairs: int):
    """The oracle as it stands, on the host cores, over the first n (M, layer) pairs of the step."""
    import oracle
    pairs = _oracle_pairs()[:n_pairs]
    inputs = {li: synth.w4a16_inputs(K, N, G, max(M_SWEEP), seed=li) for li, (K, N) in enumerate(LAYERS)}
    t0 = time.perf_counter()
    b = 0
    for (M, K, N, li) in pairs:
        d = inputs[li]
        oracle.w4a16(d["A"][:M], d["Q"], d["s"], G)
        b += algo_bytes(M, K, N)
    dt = time.perf_counter() - t0
    return {"value": round(b / dt / 1e9, 4), "unit": "GB/s", "cores": _cores(), "kind": "oracle",
            "sample": f"{len(pairs)} of the step's 32 (M, layer) calls, fp64 dequantise + numpy BLAS matmul, "
                      f"{dt:.1f} s", **_host_info()}


def run_reference(args, rank, world):
    """--impl reference: the CPU oracle timed on this host, same metric and workload, rank 0 only.

    One step = the oracle on one (M, layer) call of the step, cycling through the 32 calls,
    restricted to a block of output columns sized so that the whole run stays near
    ``--reference-budget`` seconds whatever --steps is. The bytes counted are the algorithmic
    bytes of the columns computed.
    """
    if rank != 0:
        return
    import oracle
    pairs = _oracle_pairs()
    inputs = {li: synth.w4a16_inputs(K, N, G, max(M_SWEEP), seed=li) for li, (K, N) in enumerate(LAYERS)}
    # calibration (untimed): seconds per output column of each layer at M = 128
    per_col = {}
    for li, (K, N) in enumerate(LAYERS):
        d = inputs[li]
        c = min(N, 1024)
        t0 = time.perf_counter()
        oracle.w4a16(d["A"], d["Q"][:, :c], d["s"][:, :c], G)
        per_col[li] = (time.perf_counter() - t0) / c
    per_step = args.reference_budget / max(1, args.steps + args.warmup)

    def one(i):
        M, K, N, li = pairs[i % len(pairs)]
        d = inputs[li]
        cols = int(min(N, max(8, per_step / per_col[li]))) // 8 * 8
        n0 = (i * 4096) % (N - cols + 1)
        oracle.w4a16(d["A"][:M], d["Q"][:, n0:n0 + cols], d["s"][:, n0:n0 + cols], G)
        return algo_bytes(M, K, cols), cols

    for i in range(args.warmup):
        one(i)
    t0 = time.perf_counter()
    b = 0
    ncols = 0
    for i in range(args.steps):
        bi, ci = one(args.warmup + i)
        b += bi
        ncols += ci
    dt = time.perf_counter() - t0
    v = b / dt / 1e9
    sample = (f"{args.steps} steps, each the fp64 oracle on one (M, layer) call of the 32, "
              f"{ncols / args.steps:.0f} output columns on average, {dt:.1f} s")
    out = {"impl": "reference", "metric": METRIC, "value": round(v, 4), "unit": "GB/s", "n_gpus": world,
           "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 3),
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
           "config": {"workload": WORKLOAD, "layers_KN": LAYERS, "M": M_SWEEP, "g": G,
                      "step": "one (M, layer) call of the layer set on a block of output columns"},
           "cpu_baseline": {"value": round(v, 4), "unit": "GB/s", "cores": _cores(), "kind": "oracle",
                            "sample": sample, **_host_info()},
           "e2e": {"value": round(v, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--cpu-sample", type=int, default=32, help="(M, layer) calls the oracle baseline times")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-breakdown", action="store_true", help="skip the per-M breakdown (short profiler runs)")
    ap.add_argument("--reference-budget", type=float, default=90.0, help="seconds the reference arm aims for")
    ap.add_argument("--case", default=None, help="K,N,g,M: one layer instead of the layer set (profiling)")
    args = ap.parse_args(argv)
    if args.case:
        global LAYERS, M_SWEEP, G, COPIES, WORKLOAD
        K, N, g, M = (int(v) for v in args.case.split(","))
        LAYERS, G = [(K, N)], g
        COPIES = int(min(64, max(2, -(-3 * 126e6 // (K * N // 2 + 2 * (K // g) * N)))))
        M_SWEEP = [M] * COPIES
        WORKLOAD = f"single_layer_K{K}_N{N}_g{g}_M{M}_x{COPIES}_copies"
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        if world == 1 and args.gpus > 1:
            raise SystemExit("for --gpus N > 1 launch with torchrun --nproc-per-node N")
    if args.impl == "reference":
        return run_reference(args, rank, world)
    return run_ours(args, rank, world, local_rank)


if __name__ == "__main__":
    main()
