#!/usr/bin/env python
"""Benchmark: SmolVLA action-chunk generation on B200 through libsvla.

One step = one pass of the whole hot path over one batch: prefix prefill into
the per-layer K/V cache, then the 10-step Euler denoise of the 50 x 32 chunk.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Default workload: smolvla_b1 (B = 1, 177 prefix tokens, chunk 50, 10 steps),
on which the headline metric "ms per 50-action chunk (b=1)" is quoted; a
secondary line-item measures chunks/s at b = 32 (smolvla_b32). For N > 1 (one
process per GPU under torchrun) every rank runs its own replica of the same
workload (independent queries, no collective on the path): weak scaling.

Further objects of the line, each measured after the headline's timed region:
the per-step spread, the prefill / denoise breakdown, the prefix assembly, the
int8 (vlm-8bit) prefix at batch 1 and 32, the batch-8 / prefix-321 / chunk-100
step and the batch-256 denoise ("batched"), and the expert's training step.
The CPU leg times the oracle on the host's cores and on one core and reports
the headline chunk's difference from the oracle's.
    --no-secondary  skip batch 32 and the batched workloads
    --no-int8 / --no-train / --no-cpu   skip those blocks
    --train-only    time only the training step
    --batched-only  time only the batch-8 and batch-256 workloads
    --profile CASE  run a workload untimed for ncu (the commands in profiles/)

Prints ONE JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

METRIC = "ms per 50-action chunk (b=1)"
L2_BYTES = 126 * 1024 * 1024

# DRAM bytes (read + write) per launch of the dominant kernels, from the ncu
# captures summarised in profiles/ncu_traffic.json. Each entry records a hash
# of the CUDA sources it was taken on; when the sources have changed since,
# the figure no longer describes the kernel and is reported as None.
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "ncu_traffic.json")


def sources_sha16() -> str:
    """First 16 hex digits of the SHA-256 over the CUDA sources and the header."""
    import glob
    h = hashlib.sha256()
    files = sorted(glob.glob(os.path.join(ROOT, "vision_language_action_b200", "csrc", "*")))
    for f in files + [os.path.join(ROOT, "include", "svla.h")]:
        h.update(os.path.basename(f).encode())
        with open(f, "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str):
    """DRAM bytes per launch of `kernel` from its capture, or None (no capture,
    or the sources changed since it was taken)."""
    try:
        rec = json.load(open(TRAFFIC_FILE))["kernels"].get(kernel)
    except (OSError, ValueError, KeyError):
        return None
    if not rec or rec.get("sources_sha16") != sources_sha16():
        return None
    return float(rec["dram_bytes_per_launch"])


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return d["hbm_gbs"], d["bf16_tflops"], d.get("bf16_tflops_sustained", d["bf16_tflops"]), "measured"
    return 6650.0, 1590.0, 1400.0, "fallback"


# ---------------------------------------------------------------------------
# algorithmic work of one chunk
# ---------------------------------------------------------------------------
def gemm_list(s, B, L, H, n_steps):
    """Every GEMM launch of one chunk as (M, N, K, out_bytes_per_elem, rmw)."""
    hd = s.head_dim
    qp, kvp = s.p_heads * hd, s.p_kv_heads * hd
    qe, kve = s.e_heads * hd, s.e_kv_heads * hd
    Mp, Me = B * L, B * H
    g = []
    for l in range(s.p_layers):
        g.append((Mp, qp + 2 * kvp, s.p_width, 2, False))
        if l == s.p_layers - 1:
            break
        g += [(Mp, s.p_width, qp, 4, True), (Mp, 2 * s.p_ffn, s.p_width, 1, False),
              (Mp, s.p_width, s.p_ffn, 4, True)]
    for l in range(1, s.e_layers, 2):
        g += [(Mp, kve, kvp, 2, False)] * 2
    step = [(Me, s.e_width, s.e_width, 2, False), (Me, s.e_width, s.e_width, 4, False)]
    for l in range(s.e_layers):
        step.append((Me, qe + 2 * kve, s.e_width, 2, False) if l % 2 == 0 else (Me, qe, s.e_width, 2, False))
        step += [(Me, s.e_width, qe, 4, True), (Me, 2 * s.e_ffn, s.e_width, 1, False),
                 (Me, s.e_width, s.e_ffn, 4, True)]
    return g + step * n_steps


def gemm_bytes(M, N, K, ob, rmw):
    return 2 * (M * K + N * K) + M * N * ob * (2 if rmw else 1)


def chunk_work(s, B, L, H, n_steps):
    """(algorithmic HBM bytes, GEMM FLOPs, attention FLOPs) of one chunk."""
    flops = sum(2 * M * N * K for M, N, K, _, _ in gemm_list(s, B, L, H, n_steps))
    wbytes = sum(2 * int(np.prod(shp)) for _, shp in synth.manifest(s))
    hd = s.head_dim
    kvw = s.p_kv_heads * hd
    kv_bytes = 2 * s.p_layers * B * L * kvw * 2
    n_odd = s.e_layers // 2
    kvx_bytes = n_odd * 2 * B * L * s.e_kv_width * 2
    # weights once for prefill + once per denoise step (the expert's 196 MB do not fit in L2),
    # K/V written once, odd-layer cache read once by the hoist, projected K'/V' read every step
    pre_w = sum(2 * int(np.prod(shp)) for n, shp in synth.manifest(s) if n.startswith("p"))
    exp_w = wbytes - pre_w
    hbm = pre_w + kv_bytes + (kv_bytes // 2) + kvx_bytes + n_steps * (exp_w + kvx_bytes)
    att = 0
    for _ in range(s.p_layers - 1):
        att += 4 * B * s.p_heads * L * L * hd
    att_step = 0
    for l in range(s.e_layers):
        att_step += 4 * B * s.e_heads * H * (H if l % 2 == 0 else L) * hd
    att += n_steps * att_step
    return hbm, flops, att


def prefix_projection_bytes(s, bits):
    """Bytes of the prefix projections one prefill reads (the last layer stops
    after its QKV): bf16 weights, or int8 codes plus a bf16 (alpha, beta) pair
    per 64 weights (the vlm-8bit preset)."""
    D, hd = s.p_width, s.head_dim
    mats = [((s.p_heads + 2 * s.p_kv_heads) * hd, D), (D, s.p_heads * hd), (2 * s.p_ffn, D), (D, s.p_ffn)]
    tot = 0
    for l in range(s.p_layers):
        for i, (N, K) in enumerate(mats):
            if l == s.p_layers - 1 and i > 0:
                break
            tot += 2 * N * K if bits == 16 else N * K + N * ((K + 63) // 64) * 4
    return tot


def expert_projection_bytes(s, bits, cross=None):
    """Bytes of the expert layers' projections: bf16 weights, or int8 codes
    plus a bf16 (alpha, beta) pair per group of 64 inputs, the last group of a
    row holding the K mod 64 remaining inputs (the int8 expert). cross=None:
    all of them; True: only the odd layers' cross K / V projections (read once
    per denoise call, by the hoist); False: the others (read every step)."""
    tot = 0
    for name, shp in synth.manifest(s):
        layer, _, mat = name.partition(".")
        if not layer.startswith("e") or mat not in ("wq", "wk", "wv", "wo", "wg", "wu", "wd"):
            continue
        is_cross = int(layer[1:]) % 2 == 1 and mat in ("wk", "wv")
        if cross is not None and is_cross != cross:
            continue
        N, K = shp
        tot += 2 * N * K if bits == 16 else N * K + N * ((K + 63) // 64) * 4
    return tot


def train_flops(s, B, L, H):
    """Algorithmic FLOPs of one training step of the expert (svla_train_step):
    every forward GEMM, its weight gradient, and its input gradient except
    where the input is frozen (the prefix cache of the cross projections) or
    not needed (the time half of the time MLP's input); attention forward 2
    products per score block, backward 5 (scores again, dP, dQ, dK, dV)."""
    hd = s.head_dim
    M, Lb, E, F = B * H, B * L, s.e_width, s.e_ffn
    qw, kvw, pkvw = s.e_heads * hd, s.e_kv_heads * hd, s.p_kv_width
    g = 2 * M * 2 * E * E * 2 + 2 * M * E * E        # W_t1: forward + weight grad, input grad of the action half
    g += 2 * M * E * E * 3                            # W_t2
    att = 0
    for l in range(s.e_layers):
        if l % 2 == 0:
            g += 2 * M * E * (qw + 2 * kvw) * 3
            tk = H
        else:
            g += 2 * M * E * qw * 3 + 2 * (2 * Lb * pkvw * kvw) * 2
            tk = L
        g += 2 * M * qw * E * 3 + 2 * M * E * 2 * F * 3 + 2 * M * F * E * 3
        att += (2 + 5) * 2 * B * s.e_heads * H * tk * hd
    return g + att


def launches_per_chunk(s, n_steps, fused):
    """Kernels libsvla launches for one prefill + denoise (the CUDA graphs' kernel nodes)."""
    pre = 2 + s.p_layers + 4 * (s.p_layers - 1)   # positions, residual init, QKV per layer, attn/O/GU/D
    hoist = 2 * (s.e_layers // 2)
    if fused:
        return pre + hoist + 1                     # the whole Euler loop is one persistent kernel
    step = 1 + 2 + 5 * s.e_layers + 1              # step begin, time MLP, 5 per layer, step end
    return pre + hoist + n_steps * step


def denoise_bytes(s, B, L, H, n_steps):
    """Algorithmic HBM bytes of one svla_denoise call: the hoisted cross K/V
    projection (odd-layer cache read, W_k/W_v, K'/V' written) once, then per
    Euler step every expert weight the step multiplies by (streamed from HBM:
    196 MB do not stay in the 126 MB L2) and the projected K'/V' it reads."""
    man = dict(synth.manifest(s))
    nbytes = lambda n: 2 * int(np.prod(man[n]))  # noqa: E731
    kvw = s.p_kv_heads * s.head_dim
    n_odd = s.e_layers // 2
    kvx = n_odd * 2 * B * L * s.e_kv_width * 2
    hoist = n_odd * 2 * B * L * kvw * 2 + kvx
    step_w = 0
    for l in range(s.e_layers):
        names = ["in_norm", "wq", "wo", "post_norm", "wg", "wu", "wd"] + (["wk", "wv"] if l % 2 == 0 else [])
        hoist += 0 if l % 2 == 0 else nbytes(f"e{l}.wk") + nbytes(f"e{l}.wv")
        step_w += sum(nbytes(f"e{l}.{n}") for n in names)
    step_w += sum(nbytes(n) for n in ("final_norm", "w_in", "b_in", "w_t1", "b_t1", "w_t2", "b_t2", "w_out", "b_out"))
    return hoist + n_steps * (step_w + kvx)


# ---------------------------------------------------------------------------
# clocks sampled during the timed region
# ---------------------------------------------------------------------------
CLOCK_REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
                 ("sw_power_cap", 0x4))


def summarize_clocks(samples):
    """[(sm_mhz, max_sm_mhz, reasons_bitmask)] sampled during a timed region ->
    {"sm_mhz": median, "sm_max_mhz", "reasons": the clock-event reasons seen
    active among hw_slowdown, hw_thermal_slowdown, sw_thermal_slowdown,
    sw_power_cap, "samples"}; None without samples."""
    if not samples:
        return None
    reasons = sorted({name for _, _, m in samples for name, bit in CLOCK_REASONS if m & bit})
    return {"sm_mhz": statistics.median(s[0] for s in samples), "sm_max_mhz": max(s[1] for s in samples),
            "reasons": reasons, "samples": len(samples)}


class Clocks:
    """SM clocks and clock-event reasons of the bench's GPU, sampled during the
    timed region: NVML polled from a thread every 10 ms (the device found by the
    UUID torch reports, so a CUDA_VISIBLE_DEVICES remapping cannot point it at
    another GPU), else nvidia-smi every 50 ms. Read-only: no setting changes."""
    Q = ("uuid,clocks.sm,clocks.max.sm,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, cuda_dev):
        self.dev = cuda_dev
        self.samples = []
        self.thread = None
        self.stop_flag = False
        self.proc = None
        self.path = None
        self.uuid = None
        try:
            import torch
            u = str(torch.cuda.get_device_properties(cuda_dev).uuid)
            self.uuid = u if u.startswith("GPU-") else "GPU-" + u
        except Exception:
            self.uuid = None

    def _poll(self, nv, handle):
        while not self.stop_flag:
            try:
                sm = nv.nvmlDeviceGetClockInfo(handle, nv.NVML_CLOCK_SM)
                mx = nv.nvmlDeviceGetMaxClockInfo(handle, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(handle)
                self.samples.append((float(sm), float(mx), int(rs)))
            except Exception:
                return
            time.sleep(0.01)

    def start(self):
        self.samples = []
        self.stop_flag = False
        try:
            import threading
            import pynvml as nv
            nv.nvmlInit()
            handle = nv.nvmlDeviceGetHandleByUUID(self.uuid)
            self.thread = threading.Thread(target=self._poll, args=(nv, handle), daemon=True)
            self.thread.start()
            while not self.samples and self.thread.is_alive():  # sampling runs before the region starts
                time.sleep(0.001)
            return
        except Exception:
            self.thread = None
        try:
            import tempfile
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            target = self.uuid if self.uuid else str(self.dev)
            self.proc = subprocess.Popen(["nvidia-smi", "-i", target, f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "50"],
                                         stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            t0 = time.time()
            while os.path.getsize(self.path) == 0 and time.time() - t0 < 5:
                time.sleep(0.01)
        except Exception:
            self.proc = None

    def stop(self):
        if self.thread is not None:
            self.stop_flag = True
            self.thread.join(timeout=2)
            return summarize_clocks(self.samples)
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) >= 7 and f[1].replace(".", "").isdigit() and f[2].replace(".", "").isdigit():
                bits = sum(bit for (name, bit), v in zip(CLOCK_REASONS, f[3:7]) if v.lower() == "active")
                rows.append((float(f[1]), float(f[2]), bits))
        os.unlink(self.path)
        return summarize_clocks(rows)


# ---------------------------------------------------------------------------
# CPU oracle (baseline and reference arm)
# ---------------------------------------------------------------------------
def _blas_threads():
    try:
        from threadpoolctl import threadpool_info
        info = threadpool_info()
        return max((d.get("num_threads", 1) for d in info), default=1)
    except Exception:
        return os.cpu_count() or 1


def oracle_chunk_timer(wl_name):
    """Returns a callable running the oracle on one chunk of query 0 (ms)."""
    import oracle
    wl = synth.WORKLOADS[wl_name]
    s = wl.model
    W = oracle.load_weights(synth.gen_weights(s, wl.seed))
    inp = synth.gen_inputs(wl, B=1)
    emb = synth.bf16_bits_to_f32(inp["embeds"][0]).astype(np.float64)
    valid = inp["valid"][0]
    noise = inp["noise"][0].astype(np.float64)

    def run():
        t0 = time.perf_counter()
        run.chunk = oracle.sample(W, s, emb, valid, noise, wl.n_steps)[-1]
        return (time.perf_counter() - t0) * 1e3
    run.chunk = None
    return run


# Seeded query subsets of the batched workloads on which the oracle is timed
# (queries are independent, so the full batch's oracle time is extrapolated).
ORACLE_SUBSETS = {"smolvla_b32": 4, "long_prefix_b8": 2, "denoise_b256": 4}


def oracle_subset_time(wl_name, n_queries):
    """The oracle on the first n_queries queries of a batched workload (prefill,
    unless the K/V cache is given, and the Euler denoise): ms per chunk, and the
    full batch's time extrapolated from it."""
    import oracle
    wl = synth.WORKLOADS[wl_name]
    s = wl.model
    W = oracle.load_weights(synth.gen_weights(s, wl.seed))
    inp = synth.gen_inputs(wl, B=n_queries)
    per = []
    for b in range(n_queries):
        valid = inp["valid"][b]
        noise = inp["noise"][b].astype(np.float64)
        if wl.prefix_kind == "kv_given":
            K = synth.bf16_bits_to_f32(inp["k"][:, b]).astype(np.float64)
            V = synth.bf16_bits_to_f32(inp["v"][:, b]).astype(np.float64)
            t0 = time.perf_counter()
        else:
            emb = synth.bf16_bits_to_f32(inp["embeds"][b]).astype(np.float64)
            t0 = time.perf_counter()
            K, V = oracle.prefill(W, s, emb, valid)
        oracle.denoise(W, s, K, V, valid, noise, wl.n_steps)
        per.append((time.perf_counter() - t0) * 1e3)
    ms = float(np.mean(per))
    return {"queries_timed": n_queries, "batch": wl.B, "ms_per_chunk": round(ms, 1),
            "ms_full_batch_extrapolated": round(ms * wl.B, 1),
            "includes": "denoise from the given K/V cache" if wl.prefix_kind == "kv_given" else "prefill + denoise"}


def chunk_delta(gpu: np.ndarray, ref: np.ndarray, gate: float = 2e-2) -> dict:
    """|GPU chunk - oracle chunk| over [H, A]: median, p95 and max overall and per
    action dimension, beside the parity gate on the max."""
    d = np.abs(np.asarray(gpu, np.float64) - np.asarray(ref, np.float64))
    return {"median": float(np.median(d)), "p95": float(np.percentile(d, 95)), "max": float(d.max()),
            "per_dim_p95": [round(float(x), 7) for x in np.percentile(d, 95, axis=0)],
            "per_dim_max": [round(float(x), 7) for x in d.max(axis=0)],
            "gate_max": gate, "pass": bool(d.max() <= gate)}


def reference_arm(args, rank):
    """The oracle as it stands, timed on this machine's host cores (rank 0 only)."""
    if rank != 0:
        return
    wl = synth.WORKLOADS["smolvla_b1"]
    run = oracle_chunk_timer(wl.name)
    for _ in range(max(args.warmup, 0)):
        run()
    times = [run() for _ in range(args.steps)]
    ms = float(np.mean(times))
    cores = _blas_threads()
    sample = "one full chunk of smolvla_b1 per step (prefill + 10 Euler steps, query 0)"
    line = {"impl": "reference", "metric": METRIC, "value": ms, "unit": "ms", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": wl.name, "batch": 1, "prefix_len": wl.L, "chunk": wl.H,
                       "euler_steps": wl.n_steps, "parallelism": "host oracle"},
            "cpu_baseline": {"value": ms, "unit": "ms", "cores": cores, "kind": "oracle", "sample": sample},
            "e2e": {"value": ms, "unit": "ms", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# GPU arm
# ---------------------------------------------------------------------------
def gpu_setup(wl_name, dev, B=None, prefix_int8=False, hash_blob=False, expert_int8=False):
    import torch
    from vision_language_action_b200.runtime import SmolVLA
    wl = synth.WORKLOADS[wl_name]
    s = wl.model
    B = wl.B if B is None else B
    blob = synth.pack_blob(s, synth.gen_weights(s, wl.seed))
    m = SmolVLA(s, blob, max_batch=B, max_prefix=wl.L, max_chunk=wl.H, device=dev, prefix_int8=prefix_int8,
                expert_int8=expert_int8)
    m.blob_sha256 = hashlib.sha256(blob.tobytes()).hexdigest() if hash_blob else None
    del blob
    inp = synth.gen_inputs(wl, B=B)
    host = {
        "embeds": torch.from_numpy(inp["embeds"].view(np.int16)).view(torch.bfloat16).pin_memory(),
        "valid": torch.from_numpy(inp["valid"]).pin_memory(),
        "noise": torch.from_numpy(inp["noise"]).pin_memory(),
    }
    d = {k: v.to(f"cuda:{dev}") for k, v in host.items()}
    d["kv"] = m.new_kv_cache(B, wl.L)
    d["actions"] = torch.empty_like(d["noise"])
    return m, wl, host, d


def max_over_ranks(x: float, world: int, device: str) -> float:
    """The largest value of x over the ranks (the job's time is its slowest rank's)."""
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def ms_per_chunk(ms_total_max: float, steps: int, batch_per_rank: int, world: int) -> float:
    """Job-level metric: the timed region (max over ranks) over every chunk all ranks produced."""
    return ms_total_max / (steps * batch_per_rank * world)


def time_steps(fn, steps, warmup, barrier):
    import torch
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(steps):
        fn()
    e1.record()
    torch.cuda.synchronize()
    barrier()
    return e0.elapsed_time(e1)


def step_spread(fn, steps):
    """Per-step device times (an event after every step, after the timed region):
    median, p10 and p90 in ms."""
    import torch
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    torch.cuda.synchronize()
    ev[0].record()
    for i in range(steps):
        fn()
        ev[i + 1].record()
    torch.cuda.synchronize()
    t = np.array([ev[i].elapsed_time(ev[i + 1]) for i in range(steps)])
    return {"median": round(float(np.median(t)), 4), "p10": round(float(np.percentile(t, 10)), 4),
            "p90": round(float(np.percentile(t, 90)), 4), "steps": steps}


def gemm_roofline(s, B, L, H, n_steps, dev, hbm_peak):
    """Live CUDA-event timing of the GEMM kernel over one chunk's GEMM launches.

    The launches of the prefill (+ hoisted cross K/V projection) and of one
    denoise step are captured, with the same shapes and tile/split plans as the
    path and distinct weight buffers per launch (nothing is served from L2 that
    the path would not), into two CUDA graphs that are replayed back to back
    (PDL-chained like the path) and timed with events on the launch stream.
    achieved = algorithmic bytes of a chunk's GEMMs / their time per chunk."""
    import ctypes
    import torch
    from vision_language_action_b200 import _abi
    lib = _abi.load()
    pre = gemm_list(s, B, L, H, 0)
    step = gemm_list(s, B, L, H, 1)[len(pre):]

    def build(launches):
        acts, plans = {}, []
        for (M, N, K, ob, rmw) in launches:
            W = torch.randn(N, K, device=dev).to(torch.bfloat16)
            if (M, K) not in acts:
                acts[(M, K)] = torch.randn(M, K, device=dev).to(torch.bfloat16)
            C = torch.zeros(M, N, device=dev, dtype=torch.float32 if ob == 4 else torch.bfloat16)
            epi = _abi.EPI_ADD_F32 if rmw else (_abi.EPI_F32 if ob == 4 else _abi.EPI_BF16)
            plans.append((epi, acts[(M, K)], W, C, M, N, K))
        return plans

    P = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731

    def run(plans):
        st = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        for epi, A, W, C, M, N, K in plans:
            _abi.check(lib.svla_op_gemm(epi, P(A), K, P(W), K, M, N, K, P(C), N, None, 0, None, 0, None, st))

    def graph_time(plans, reps=10):
        cs = torch.cuda.Stream()
        with torch.cuda.stream(cs):
            run(plans)
            torch.cuda.synchronize()
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=cs):
                run(plans)
            g.replay()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(cs)
            for _ in range(reps):
                g.replay()
            e1.record(cs)
            torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    t_pre = graph_time(build(pre))
    t_step = graph_time(build(step))
    b_pre = sum(gemm_bytes(*x) for x in pre)
    b_step = sum(gemm_bytes(*x) for x in step)
    t_chunk = t_pre + n_steps * t_step
    bytes_chunk = b_pre + n_steps * b_step
    n_launch = len(pre) + n_steps * len(step)
    achieved = bytes_chunk / (t_chunk * 1e-3) / 1e9
    return {"bound": "hbm", "kernel": "gemm_tc_kernel", "achieved": round(achieved, 1), "peak": hbm_peak,
            "unit": "GB/s", "frac": round(achieved / hbm_peak, 4),
            "traffic": ncu_traffic("gemm_tc_kernel_b1"),
            "launches_per_chunk": n_launch, "avg_launch_us": round(1e3 * t_chunk / n_launch, 2),
            "algorithmic_bytes_per_launch": int(bytes_chunk / n_launch),
            "gemm_ms_per_chunk": round(float(t_chunk), 4)}


def int8_prefix(args, dev, barrier, hbm_peak, peak_kind):
    """The vlm-8bit preset (weight-only int8 prefix projections) at batch 1 and
    batch 32: prefill and chunk times on one handle, switched between its int8
    and dense prefix weights, and the int8 prefill's bytes against HBM."""
    out = {"preset": "vlm-8bit: prefix projections int8, affine groups of 64 (bf16 alpha, beta); expert bf16"}
    for name in ("smolvla_b1", "smolvla_b32"):
        m, wl, _, d = gpu_setup(name, dev, prefix_int8=True)
        s = wl.model
        steps = args.steps if wl.B == 1 else max(3, args.steps // 2)

        def pre():
            m.prefill(d["embeds"], d["valid"], d["kv"])

        def chunk():
            pre()
            m.denoise(d["kv"], d["valid"], d["noise"], wl.n_steps, actions=d["actions"])

        t8 = time_steps(pre, steps, args.warmup, barrier) / steps
        c8 = time_steps(chunk, steps, args.warmup, barrier) / steps
        m.set_prefix_weights(16)
        t16 = time_steps(pre, steps, args.warmup, barrier) / steps
        m.set_prefix_weights(8)
        if m.device_status() != 0:
            raise RuntimeError("device status after the int8 prefill timing")
        m.close()
        del d
        w8, w16 = prefix_projection_bytes(s, 8), prefix_projection_bytes(s, 16)
        pre_bytes = chunk_work(s, wl.B, wl.L, wl.H, 0)[0] - w16 + w8
        achieved = pre_bytes / (t8 * 1e-3) / 1e9
        if wl.B == 1:
            M, N, K = wl.L, 2 * s.p_ffn, s.p_width
            out["gemm_w8_gate_up_b1"] = {"kernel": "gemm_w8_kernel<64, SwiGLU, 4>", "M": M, "N": N, "K": K,
                                         "algorithmic_bytes_per_launch": int(N * K + N * ((K + 63) // 64) * 4 + 2 * M * K),
                                         "traffic": ncu_traffic("gemm_w8_kernel_gate_up_b1")}
        out[name] = {"prefill_ms": round(t8, 4), "prefill_ms_dense_same_handle": round(t16, 4),
                     "chunk_ms": round(c8 / wl.B, 4) if wl.B == 1 else None,
                     "chunks_per_s": round(wl.B / (c8 * 1e-3), 2) if wl.B > 1 else None,
                     "projection_bytes_int8": int(w8), "projection_bytes_bf16": int(w16),
                     "prefill_roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_peak,
                                          "unit": "GB/s", "frac": round(achieved / hbm_peak, 4),
                                          "algorithmic_bytes": int(pre_bytes), "peak_kind": peak_kind}}
    import torch
    torch.cuda.empty_cache()
    return out


def int8_expert(args, dev, barrier, hbm_peak, peak_kind):
    """The int8 expert (the vlm-8bit scheme on the expert's projections) at
    batch 1 (persistent kernel) and batch 32 (multi-kernel path): denoise and
    chunk times on one handle, switched between its int8 and dense expert
    weights, the denoise's bytes against HBM, and at batch 1 the chunk with
    both the prefix and the expert in int8."""
    out = {"preset": "expert int8: the expert layers' projections (cross K/V included) in int8, affine groups "
                     "of 64 (a 720-wide row's last group holds 16 inputs), bf16 (alpha, beta); prefix and heads bf16"}
    for name in ("smolvla_b1", "smolvla_b32"):
        m, wl, _, d = gpu_setup(name, dev, expert_int8=True)
        s = wl.model
        steps = args.steps if wl.B == 1 else max(3, args.steps // 2)

        def den():
            m.denoise(d["kv"], d["valid"], d["noise"], wl.n_steps, actions=d["actions"])

        def chunk():
            m.prefill(d["embeds"], d["valid"], d["kv"])
            den()

        chunk()
        t8 = time_steps(den, steps, args.warmup, barrier) / steps
        c8 = time_steps(chunk, steps, args.warmup, barrier) / steps
        m.set_expert_weights(16)
        t16 = time_steps(den, steps, args.warmup, barrier) / steps
        m.set_expert_weights(8)
        if m.device_status() != 0:
            raise RuntimeError("device status after the int8 expert timing")
        m.close()
        del d
        e8, e16 = expert_projection_bytes(s, 8, False), expert_projection_bytes(s, 16, False)
        x8, x16 = expert_projection_bytes(s, 8, True), expert_projection_bytes(s, 16, True)
        den_bytes8 = denoise_bytes(s, wl.B, wl.L, wl.H, wl.n_steps) - wl.n_steps * (e16 - e8) - (x16 - x8)
        achieved = den_bytes8 / (t8 * 1e-3) / 1e9
        row = {"denoise_ms": round(t8, 4), "denoise_ms_dense_same_handle": round(t16, 4),
               "chunk_ms": round(c8 / wl.B, 4) if wl.B == 1 else None,
               "chunks_per_s": round(wl.B / (c8 * 1e-3), 2) if wl.B > 1 else None,
               "projection_bytes_per_step_int8": int(e8), "projection_bytes_per_step_bf16": int(e16),
               "denoise_roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm_peak,
                                    "unit": "GB/s", "frac": round(achieved / hbm_peak, 4),
                                    "algorithmic_bytes": int(den_bytes8), "peak_kind": peak_kind}}
        if wl.B == 1:
            m, wl, _, d = gpu_setup(name, dev, prefix_int8=True, expert_int8=True)

            def chunk_all():
                m.prefill(d["embeds"], d["valid"], d["kv"])
                m.denoise(d["kv"], d["valid"], d["noise"], wl.n_steps, actions=d["actions"])

            chunk_all()
            ca = time_steps(chunk_all, steps, args.warmup, barrier) / steps
            if m.device_status() != 0:
                raise RuntimeError("device status after the int8 prefix + expert timing")
            m.close()
            del d
            row["chunk_ms_prefix_and_expert_int8"] = round(ca, 4)
        out[name] = row
    import torch
    torch.cuda.empty_cache()
    return out


def batched_configs(args, dev, barrier, hbm_peak, tf_peak, tf_sus, peak_kind):
    """The two batched workloads beside the headline and batch 32: batch 8 with
    prefix 321 and chunk 100 (prefill + denoise, tensor and HBM fractions), and
    the batch-256 denoise from a given K/V cache."""
    import torch
    from vision_language_action_b200.runtime import SmolVLA
    out = {}
    # batch 8, prefix 321, chunk 100
    m, wl, _, d = gpu_setup("long_prefix_b8", dev)
    s = wl.model
    steps = max(3, args.steps // 4)

    def pre():
        m.prefill(d["embeds"], d["valid"], d["kv"])

    def den():
        m.denoise(d["kv"], d["valid"], d["noise"], wl.n_steps, actions=d["actions"])

    def step():
        pre()
        den()

    ms_step = time_steps(step, steps, args.warmup, barrier) / steps
    ms_pre = time_steps(pre, steps, args.warmup, barrier) / steps
    ms_den = time_steps(den, steps, args.warmup, barrier) / steps
    if m.device_status() != 0:
        raise RuntimeError("device status after the batch-8 timing")
    m.close()
    del d
    hbm, g, att = chunk_work(s, wl.B, wl.L, wl.H, wl.n_steps)
    hbm0, g0, att0 = chunk_work(s, wl.B, wl.L, wl.H, 0)
    den_tf = ((g - g0) + (att - att0)) / (ms_den * 1e-3) / 1e12
    pre_tf = (g0 + att0) / (ms_pre * 1e-3) / 1e12
    out["long_prefix_b8"] = {
        "config": {"batch": wl.B, "prefix_len": wl.L, "chunk": wl.H, "euler_steps": wl.n_steps},
        "ms_per_step": round(ms_step, 4), "chunks_per_s": round(wl.B / (ms_step * 1e-3), 2),
        "prefill_ms": round(ms_pre, 4), "denoise_ms": round(ms_den, 4),
        "denoise_tensor": {"achieved": round(den_tf, 1), "peak": tf_sus, "unit": "TFLOP/s",
                           "frac": round(den_tf / tf_sus, 4), "peak_kind": f"{peak_kind} sustained bf16"},
        "prefill_tensor": {"achieved": round(pre_tf, 1), "peak": tf_peak, "unit": "TFLOP/s",
                           "frac": round(pre_tf / tf_peak, 4), "peak_kind": f"{peak_kind} bf16"},
        "step_hbm": {"achieved": round(hbm / (ms_step * 1e-3) / 1e9, 1), "peak": hbm_peak, "unit": "GB/s",
                     "frac": round(hbm / (ms_step * 1e-3) / 1e9 / hbm_peak, 4), "algorithmic_bytes": int(hbm)}}
    torch.cuda.empty_cache()
    # batch 256, denoise only from a given cache (tail pads)
    wl = synth.WORKLOADS["denoise_b256"]
    s = wl.model
    m = SmolVLA(s, synth.pack_blob(s, synth.gen_weights(s, wl.seed)), max_batch=wl.B, max_prefix=wl.L,
                max_chunk=wl.H, device=dev)
    inp = synth.gen_inputs(wl)
    dv = f"cuda:{dev}"
    kv = np.stack([inp["k"], inp["v"]]).reshape(2, s.p_layers, wl.B, wl.L, -1)
    kv = torch.from_numpy(kv.view(np.int16)).to(dv).view(torch.bfloat16)
    valid = torch.from_numpy(inp["valid"]).to(dv)
    noise = torch.from_numpy(inp["noise"]).to(dv)
    actions = torch.empty_like(noise)
    del inp
    steps5 = 3
    ms5 = time_steps(lambda: m.denoise(kv, valid, noise, wl.n_steps, actions=actions), steps5, args.warmup,
                     barrier) / steps5
    if m.device_status() != 0:
        raise RuntimeError("device status after the batch-256 timing")
    m.close()
    _, g, att = chunk_work(s, wl.B, wl.L, wl.H, wl.n_steps)
    _, g0, att0 = chunk_work(s, wl.B, wl.L, wl.H, 0)
    tf5 = ((g - g0) + (att - att0)) / (ms5 * 1e-3) / 1e12
    out["denoise_b256"] = {
        "config": {"batch": wl.B, "prefix_len": wl.L, "chunk": wl.H, "euler_steps": wl.n_steps,
                   "prefix": "given K/V cache, per-query tail pads"},
        "denoise_ms": round(ms5, 3), "chunks_per_s": round(wl.B / (ms5 * 1e-3), 1),
        "tensor": {"achieved": round(tf5, 1), "peak": tf_peak, "unit": "TFLOP/s", "frac": round(tf5 / tf_peak, 4),
                   "peak_kind": f"{peak_kind} bf16 burst"}}
    torch.cuda.empty_cache()
    return out


def train_block(args, dev, barrier, tf_peak, peak_kind):
    """The expert's training step (svla_train_step: loss and every gradient) on
    the SmolVLA shape with two queries, the shape its GPU parity test covers."""
    import torch
    from vision_language_action_b200.runtime import SmolVLA
    s = synth.SHAPES["smolvla"]
    B, L, H = 2, 177, 50
    d = f"cuda:{dev}"
    m = SmolVLA(s, synth.pack_blob(s, synth.gen_weights(s, 7, random_affine=True)), max_batch=B, max_prefix=L,
                max_chunk=H, device=dev, train=True)
    try:
        rng = np.random.default_rng(7)
        kv = torch.from_numpy(synth.f32_to_bf16_bits(rng.standard_normal((2, s.p_layers, B, L, s.p_kv_width))
                                                     .astype(np.float32)).view(np.int16)).to(d).view(torch.bfloat16)
        valid = torch.ones((B, L), dtype=torch.uint8, device=d)
        a = torch.from_numpy((0.5 * rng.standard_normal((B, H, s.action_dim))).astype(np.float32)).to(d)
        eps = torch.from_numpy(rng.standard_normal((B, H, s.action_dim)).astype(np.float32)).to(d)
        t = torch.from_numpy(rng.uniform(0.05, 0.95, B).astype(np.float32)).to(d)
        grads = torch.empty(int(m.lib.svla_train_grad_elems(m.h)), dtype=torch.float32, device=d)
        steps = max(3, args.steps // 4)
        ms = time_steps(lambda: m.train_step(kv, valid, a, eps, t, grads=grads), steps, args.warmup, barrier) / steps
        if m.device_status() != 0:
            raise RuntimeError("device status after the training step timing")
    finally:
        m.close()
    fl = train_flops(s, B, L, H)
    tf = fl / (ms * 1e-3) / 1e12
    return {"workload": "smolvla expert, 2 queries, prefix 177, chunk 50 (frozen prefix cache)",
            "ms_per_step": round(ms, 4), "steps": steps, "samples_per_s": round(B / (ms * 1e-3), 2),
            "algorithmic_flops": int(fl),
            "roofline": {"bound": "tensor", "achieved": round(tf, 2), "peak": tf_peak, "unit": "TFLOP/s",
                         "frac": round(tf / tf_peak, 5), "peak_kind": f"{peak_kind} bf16"}}


def ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist
    dev = local_rank
    torch.cuda.set_device(dev)
    barrier = (lambda: dist.barrier()) if world > 1 else (lambda: None)
    hbm_peak, tf_peak, tf_sus, peak_kind = _peaks()

    m, wl, host, d = gpu_setup("smolvla_b1", dev, hash_blob=True)
    s = wl.model

    def step():
        m.prefill(d["embeds"], d["valid"], d["kv"])
        m.denoise(d["kv"], d["valid"], d["noise"], wl.n_steps, actions=d["actions"])

    clocks = Clocks(dev)
    for _ in range(3):
        step()
    torch.cuda.synchronize()
    clocks.start()
    ms_total = time_steps(step, args.steps, args.warmup, barrier)
    clk = clocks.stop()
    st = m.device_status()
    if st != 0:
        raise RuntimeError(f"device status {st} after the timed region")
    ms_total = max_over_ranks(ms_total, world, f"cuda:{dev}")
    ms_step = ms_total / args.steps
    chunks_per_step = wl.B * world
    value = ms_per_chunk(ms_total, args.steps, wl.B, world)

    # end to end through the public API with host buffers: H2D inputs, both calls, D2H actions
    out_host = torch.empty_like(host["noise"]).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = out_host.numel() * out_host.element_size()

    def e2e_step():
        d["embeds"].copy_(host["embeds"], non_blocking=True)
        d["valid"].copy_(host["valid"], non_blocking=True)
        d["noise"].copy_(host["noise"], non_blocking=True)
        m.prefill(d["embeds"], d["valid"], d["kv"])
        m.denoise(d["kv"], d["valid"], d["noise"], wl.n_steps, actions=d["actions"])
        out_host.copy_(d["actions"], non_blocking=True)
        torch.cuda.current_stream().synchronize()

    ms_e2e = max_over_ranks(time_steps(e2e_step, args.steps, args.warmup, barrier), world, f"cuda:{dev}")
    try:  # per-step distribution, outside the timed region
        spread = step_spread(step, args.steps)
    except Exception as exc:
        spread = {"error": f"{type(exc).__name__}: {exc}"}

    # the two calls of a step timed on their own (same warm-up and step count)
    ms_pre = time_steps(lambda: m.prefill(d["embeds"], d["valid"], d["kv"]), args.steps, args.warmup, barrier)
    ms_den = time_steps(lambda: m.denoise(d["kv"], d["valid"], d["noise"], wl.n_steps, actions=d["actions"]),
                        args.steps, args.warmup, barrier)

    # prefix assembly upstream of the step (connector + state token, svla_assemble_prefix),
    # timed alone: the headline step starts from the assembled prefix embeddings
    asm = None
    ash = synth.ASSEMBLY_SHAPES["smolvla"]
    if wl.L == ash.n_img * ash.tokens_per_image + ash.text_len + 1:
        wbits = synth.gen_assembly_weights(ash, s.p_width, wl.seed)
        m.set_assembly(synth.pack_assembly_blob(ash, s.p_width, wbits), ash.vis_width, ash.grid, ash.shuffle,
                       ash.state_dim, ash.n_img)
        ai = synth.gen_assembly_inputs(ash, s.p_width, wl.B, wl.seed)
        av = torch.from_numpy(ai["vis"].view(np.int16)).to(f"cuda:{dev}").view(torch.bfloat16)
        at = torch.from_numpy(ai["text"].view(np.int16)).to(f"cuda:{dev}").view(torch.bfloat16)
        atv = torch.from_numpy(ai["text_valid"]).to(f"cuda:{dev}")
        ast = torch.from_numpy(ai["state"]).to(f"cuda:{dev}")
        ms_asm = time_steps(lambda: m.assemble_prefix(av, at, atv, ast), args.steps, args.warmup, barrier)
        conn_w = 2 * s.p_width * ash.conn_in
        asm_bytes = conn_w + 2 * 2 * wl.B * ash.n_img * ash.grid * ash.grid * ash.vis_width \
            + 2 * wl.B * wl.L * s.p_width
        asm = {"assemble_ms": round(ms_asm / args.steps, 4), "images": ash.n_img,
               "algorithmic_bytes": int(asm_bytes),
               "note": "pixel-shuffle gather + connector GEMM (12288 -> 960) + state token and layout, 3 kernels"}

    gpu_chunk = d["actions"][0].cpu().numpy()  # query 0 of the last timed step (same inputs every step)
    blob_sha = m.blob_sha256[:16]
    hbm_bytes, gflops, aflops = chunk_work(s, wl.B, wl.L, wl.H, wl.n_steps)
    chunk_s = value * 1e-3 * world  # per-rank chunk latency in s
    fused = m.fused_supported(wl.B, wl.H)
    graph_gemm = gemm_roofline(s, wl.B, wl.L, wl.H, wl.n_steps, f"cuda:{dev}", hbm_peak)
    if fused:
        # dominant kernel: the persistent denoise kernel, timed live as the denoise
        # call it makes up (the call's graph also holds the 16 hoisted K'/V'
        # projections, whose bytes are counted too)
        dbytes = denoise_bytes(s, wl.B, wl.L, wl.H, wl.n_steps)
        t_den = ms_den / args.steps * 1e-3
        achieved = dbytes / t_den / 1e9
        roof = {"bound": "hbm", "kernel": "denoise_fused_kernel", "achieved": round(achieved, 1), "peak": hbm_peak,
                "unit": "GB/s", "frac": round(achieved / hbm_peak, 4), "traffic": ncu_traffic("denoise_fused_kernel_b1"),
                "algorithmic_bytes_per_launch": int(dbytes), "launch_ms": round(t_den * 1e3, 4),
                "timed_as": "svla_denoise call (16 hoisted K'/V' projection GEMMs + denoise_fused_kernel), CUDA events",
                "peak_kind": f"{peak_kind} HBM copy"}
    else:
        roof = graph_gemm
    m.close()
    del d
    torch.cuda.empty_cache()

    q8 = None if args.no_int8 else int8_prefix(args, dev, barrier, hbm_peak, peak_kind)
    e8 = None if args.no_int8 else int8_expert(args, dev, barrier, hbm_peak, peak_kind)

    secondary = None
    if not args.no_secondary:
        m3, wl3, host3, d3 = gpu_setup("smolvla_b32", dev)

        def step3():
            m3.prefill(d3["embeds"], d3["valid"], d3["kv"])
            m3.denoise(d3["kv"], d3["valid"], d3["noise"], wl3.n_steps, actions=d3["actions"])

        def den3():
            m3.denoise(d3["kv"], d3["valid"], d3["noise"], wl3.n_steps, actions=d3["actions"])

        steps3 = max(3, args.steps // 2)
        ms3 = time_steps(step3, steps3, args.warmup, barrier) / steps3
        msd = time_steps(den3, steps3, args.warmup, barrier) / steps3
        _, g3, a3 = chunk_work(wl3.model, wl3.B, wl3.L, wl3.H, wl3.n_steps)
        _, g3p, a3p = chunk_work(wl3.model, wl3.B, wl3.L, wl3.H, 0)
        den_flops = (g3 - g3p) + (a3 - a3p)
        den_tf = den_flops / (msd * 1e-3) / 1e12
        secondary = {"metric": "chunks/s (b=32)", "value": round(wl3.B * world / (ms3 * 1e-3), 2),
                     "unit": "chunks/s", "ms_per_step": round(ms3, 4), "denoise_ms": round(msd, 4),
                     "denoise_roofline": {"bound": "tensor", "achieved": round(den_tf, 1), "peak": tf_sus,
                                          "unit": "TFLOP/s", "frac": round(den_tf / tf_sus, 4),
                                          "peak_kind": f"{peak_kind} sustained bf16"},
                     "config": {"workload": wl3.name, "batch": wl3.B, "prefix_len": wl3.L, "chunk": wl3.H,
                                "euler_steps": wl3.n_steps}}
        m3.close()

    batched = None
    if not args.no_secondary:
        try:
            batched = batched_configs(args, dev, barrier, hbm_peak, tf_peak, tf_sus, peak_kind)
        except Exception as exc:  # the headline line must not depend on this block
            batched = {"error": f"{type(exc).__name__}: {exc}"}

    train = None
    if not args.no_train:
        try:
            train = train_block(args, dev, barrier, tf_peak, peak_kind)
        except Exception as exc:  # the headline line must not depend on this block
            train = {"error": f"{type(exc).__name__}: {exc}"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        run = oracle_chunk_timer("smolvla_b1")
        run()
        times = [run() for _ in range(3)]
        cpu = {"value": round(float(np.mean(times)), 2), "unit": "ms", "cores": _blas_threads(), "kind": "oracle",
               "sample": "3 full chunks of smolvla_b1 (prefill + 10 Euler steps, query 0), float64 numpy"}
        try:  # the headline chunk against the oracle's, same weights, embeddings and noise
            cpu["delta_vs_gpu"] = chunk_delta(gpu_chunk, run.chunk)
        except Exception as exc:
            cpu["delta_vs_gpu"] = {"error": f"{type(exc).__name__}: {exc}"}
        try:  # the same oracle on one core
            from threadpoolctl import threadpool_limits
            with threadpool_limits(limits=1):
                cpu["one_core"] = {"value": round(run(), 2), "unit": "ms", "cores": 1, "sample": "1 chunk"}
        except Exception as exc:
            cpu["one_core"] = {"error": f"{type(exc).__name__}: {exc}"}
        subsets = {}
        if not args.no_secondary:
            for name, nq in ORACLE_SUBSETS.items():
                try:
                    subsets[name] = oracle_subset_time(name, nq)
                except Exception as exc:
                    subsets[name] = {"error": f"{type(exc).__name__}: {exc}"}
        cpu["batched_subsets"] = subsets
        # the schema of the result line keeps value / unit / cores / kind / sample
        # of cpu_baseline: the one-core time and the chunk delta are restated in
        # the sample text, and the whole record is repeated as cpu_oracle
        oc, dv = cpu.get("one_core", {}), cpu.get("delta_vs_gpu", {})
        cpu["sample"] += (f"; one core: {oc.get('value', 'n/a')} ms per chunk"
                          f"; GPU chunk vs oracle max |diff| {dv.get('max', float('nan')):.3g} (gate 2e-2)")

    if rank == 0:
        achieved_chunk = hbm_bytes / chunk_s / 1e9
        line = {
            "metric": METRIC, "value": round(value, 4), "unit": "ms", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": False,
            "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": wl.name, "batch": wl.B, "prefix_len": wl.L, "chunk": wl.H,
                       "euler_steps": wl.n_steps, "global_batch": wl.B * world,
                       "parallelism": f"replicas x{world}", "weights_sha256": blob_sha,
                       "l2_policy": "no flush: every step streams 514 MB of weights (> 126 MB L2)"},
            "roofline": roof,
            "chunk_roofline": {"bound": "hbm", "achieved": round(achieved_chunk, 1), "peak": hbm_peak,
                               "unit": "GB/s", "frac": round(achieved_chunk / hbm_peak, 4),
                               "algorithmic_bytes": int(hbm_bytes), "peak_kind": peak_kind},
            "cpu_baseline": cpu,
            "cpu_oracle": cpu,
            "e2e": {"value": round(ms_e2e / (args.steps * chunks_per_step), 4), "unit": "ms",
                    "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)},
            "step_spread_ms": spread,
            "breakdown": {"prefill_ms": round(ms_pre / args.steps, 4), "denoise_ms": round(ms_den / args.steps, 4),
                          "note": "each call timed alone on rank 0, same steps and warm-up"},
            "prefix_assembly": asm,
            "int8_prefix": q8,
            "int8_expert": e8,
            "train_step": train,
            "gpu_launches": launches_per_chunk(s, wl.n_steps, fused) * args.steps,
            "graph_gemm_roofline": graph_gemm if fused else None,
            "clocks": clk,
            "secondary": secondary,
            "batched": batched,
        }
        print(json.dumps(line), flush=True)


def profile_case(spec, dev, reps):
    """A workload run for a profiler to attach to (untimed): 'NAME' runs the
    prefill and the denoise of workload NAME `reps` times after one warm-up
    call; options ':graph' / ':fused' pick the denoise path, ':int8p' /
    ':int8e' the int8 prefix / expert; 'denoise_b256' runs the batch-256
    denoise from its given K/V cache; 'train' the expert's training step on
    the inputs train_block times."""
    import torch
    from vision_language_action_b200 import _abi
    from vision_language_action_b200.runtime import SmolVLA
    name, *opts = spec.split(":")
    if name == "train":
        s = synth.SHAPES["smolvla"]
        B, L, H = 2, 177, 50
        d = f"cuda:{dev}"
        m = SmolVLA(s, synth.pack_blob(s, synth.gen_weights(s, 7, random_affine=True)), max_batch=B, max_prefix=L,
                    max_chunk=H, device=dev, train=True)
        rng = np.random.default_rng(7)
        kv = torch.from_numpy(synth.f32_to_bf16_bits(rng.standard_normal((2, s.p_layers, B, L, s.p_kv_width))
                                                     .astype(np.float32)).view(np.int16)).to(d).view(torch.bfloat16)
        valid = torch.ones((B, L), dtype=torch.uint8, device=d)
        a = torch.from_numpy((0.5 * rng.standard_normal((B, H, s.action_dim))).astype(np.float32)).to(d)
        eps = torch.from_numpy(rng.standard_normal((B, H, s.action_dim)).astype(np.float32)).to(d)
        t = torch.from_numpy(rng.uniform(0.05, 0.95, B).astype(np.float32)).to(d)
        grads = torch.empty(int(m.lib.svla_train_grad_elems(m.h)), dtype=torch.float32, device=d)
        for _ in range(1 + reps):
            m.train_step(kv, valid, a, eps, t, grads=grads)
        torch.cuda.synchronize()
        st = m.device_status()
        m.close()
        print(json.dumps({"profile_case": spec, "calls": 1 + reps, "status": st}), flush=True)
        if st != 0:
            raise SystemExit(1)
        return
    if name == "denoise_b256":
        wl = synth.WORKLOADS[name]
        s = wl.model
        m = SmolVLA(s, synth.pack_blob(s, synth.gen_weights(s, wl.seed)), max_batch=wl.B, max_prefix=wl.L,
                    max_chunk=wl.H, device=dev)
        inp = synth.gen_inputs(wl)
        kv = np.stack([inp["k"], inp["v"]]).reshape(2, s.p_layers, wl.B, wl.L, -1)
        d = {"kv": torch.from_numpy(kv.view(np.int16)).to(f"cuda:{dev}").view(torch.bfloat16),
             "valid": torch.from_numpy(inp["valid"]).to(f"cuda:{dev}"),
             "noise": torch.from_numpy(inp["noise"]).to(f"cuda:{dev}")}
        d["actions"] = torch.empty_like(d["noise"])
        pre = None
    else:
        m, wl, _, d = gpu_setup(name, dev, prefix_int8="int8p" in opts, expert_int8="int8e" in opts)

        def pre():
            m.prefill(d["embeds"], d["valid"], d["kv"])
    path = {"graph": _abi.DENOISE_GRAPH, "fused": _abi.DENOISE_FUSED}
    for o in opts:
        if o in path:
            m.set_denoise_path(path[o])

    def call():
        if pre:
            pre()
        m.denoise(d["kv"], d["valid"], d["noise"], wl.n_steps, actions=d["actions"])

    for _ in range(1 + reps):
        call()
    torch.cuda.synchronize()
    st = m.device_status()
    m.close()
    print(json.dumps({"profile_case": spec, "calls": 1 + reps, "status": st}), flush=True)
    if st != 0:
        raise SystemExit(1)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-int8", action="store_true")
    ap.add_argument("--no-train", action="store_true")
    ap.add_argument("--train-only", action="store_true", help="time only the expert's training step")
    ap.add_argument("--batched-only", action="store_true", help="time only the batch-8 and batch-256 workloads")
    ap.add_argument("--profile", metavar="CASE", help="run CASE untimed for a profiler (see profile_case)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        reference_arm(args, rank)
        return
    if args.profile:
        import torch
        torch.cuda.set_device(local_rank)
        profile_case(args.profile, local_rank, max(1, args.steps))
        return
    if args.batched_only:
        import torch
        torch.cuda.set_device(local_rank)
        hbm_peak, tf_peak, tf_sus, peak_kind = _peaks()
        print(json.dumps({"batched": batched_configs(args, local_rank, lambda: None, hbm_peak, tf_peak, tf_sus,
                                                     peak_kind)}), flush=True)
        return
    if args.train_only:
        import torch
        torch.cuda.set_device(local_rank)
        _, tf_peak, _, peak_kind = _peaks()
        print(json.dumps({"train_step": train_block(args, local_rank, lambda: None, tf_peak, peak_kind)}), flush=True)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
