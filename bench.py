#!/usr/bin/env python
"""W4A16 g128 GEMM on B200: GB/s at M = 1 (decode) and TFLOP/s at M = 2048 (prefill).

One step of the headline workload is one decode GEMM (M = 1 token, 4-bit weights, groups of
128) on each of the three decoder shapes [N, K] = [4096, 4096], [11008, 4096], [4096, 11008],
with weights quantized by awq_quantize_pack on per-channel scales s = m^0.5 (m: lognormal
channel magnitudes with 1% outliers x20). Inputs are already resident in HBM. The weights
rotate through enough copies to exceed twice the L2, so every step streams from HBM; each
run of steps is captured in one CUDA graph. `value` is the algorithmic bytes of all ranks' steps
(codes + fp16 scales + uint8 zeros + X + Y) over the slowest rank's device time.

The line also carries: the prefill GEMMs at M = 2048 on [28672, 8192], [8192, 28672] and
[10240, 8192] (TFLOP/s, 2MNK per GEMM), the per-(shape, M) decode sweep, the dominant
kernel's roofline fraction, an end-to-end figure through the Python binding with host
buffers (copies inside the timed region), the CPU oracle on a bounded sample, and the SM
clocks sampled during the timed region.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import synth  # noqa: E402

METRIC = "W4A16 g128 GEMM: GB/s at M=1, TFLOP/s at M=2048; % of B200 roofline"
GROUP = 128


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum) come from the committed
# ncu summaries under profiles/: a summary states them on a line
#   bench-traffic: <kernel> <bytes per launch> <sha256 prefix of the kernel's source files>
# and the figure is used only while the sources still hash to that value (else null: the
# kernel changed since the counters were taken).
KERNEL_SOURCES = {
    "gemv_stream_decode_M1": ["gemv.cuh", "common.cuh"],
    "tc_gemm_prefill_28672x8192_M2048": ["gemm_tc.cuh", "common.cuh"],
}


def source_hash(kernel):
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "weight_only_int4_stats_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(kernel):
    """(bytes per launch, note) from the profile summaries, or (None, why not)."""
    want = source_hash(kernel)
    pdir = os.path.join(ROOT, "profiles")
    seen = False
    for name in sorted(os.listdir(pdir)) if os.path.isdir(pdir) else []:
        with open(os.path.join(pdir, name)) as f:
            for line in f:
                parts = line.strip().strip("`").split()
                if len(parts) == 4 and parts[0] == "bench-traffic:" and parts[1] == kernel:
                    seen = True
                    if parts[3] == want:
                        return float(parts[2]), f"profiles/{name}"
    return None, ("kernel changed since its ncu capture" if seen else "no ncu capture")


def search_executed_flops(M, N, K, n_alpha):
    """Tensor-core flops one awq_search_scale call executes, and its form. Direct (M < 2K):
    both fp16 parts of the error operand times X, 2 * n_alpha * 2 M N_pad K. Gram (M >= 2K):
    the tiles of G = X^T X on or above the diagonal over the token-padded X (about M_pad K^2),
    then three MMAs per k step (hi*hi, hi*lo, lo*hi) of the error operand against G,
    n_alpha * 3 * 2 N_pad K^2."""
    n_pad = -(-N // 128) * 128
    if M >= 2 * K:
        m_pad = -(-M // 128) * 128
        # G is built from its 128 x 256 tiles that reach the diagonal or above it
        tiles = sum(1 for r in range(K // 128) for c in range(-(-K // 256)) if r * 128 < (c + 1) * 256)
        return 2 * m_pad * 128 * 256 * tiles + n_alpha * 3 * 2 * n_pad * K * K, "gram"
    return 2 * n_alpha * 2 * M * n_pad * K, "direct"


def gemm_bytes(M, N, K, bits=4):
    return N * K * bits // 8 + N * (K // GROUP) * 3 + 2 * M * K + 2 * M * N


# ----------------------------------------------------------------------------- distributed

def dist_setup():
    """One process per GPU under torchrun (RANK / LOCAL_RANK / WORLD_SIZE / MASTER_*): NCCL
    on GPUs; gloo on a host without one (the replica bookkeeping is the same)."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                    device_id=torch.device("cuda", local))
        else:
            dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world):
    if world == 1:
        return x
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_rate(units_per_rank, seconds, world):
    """Whole-job rate: the units all ranks processed over the slowest rank's time (every
    rank runs the same fixed work). Returns (rate, slowest time)."""
    t_max = max_over_ranks(seconds, world)
    return units_per_rank * world / t_max, t_max


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = max(float(r[2]) for r in rows if r[2].replace(".", "").isdigit())
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        loaded = [v for v in sm if v > 0.5 * mx] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": reasons,
                "samples": len(rows)}


# ----------------------------------------------------------------------------- workloads

class DecodeShape:
    """One decode shape's rotating weight copies and its input/output buffers."""

    def __init__(self, awq, N, K, m_max, l2_bytes, device, bf16=False, bits=4):
        W, mag, X = synth.decode_layer(N, K, m_max)
        s = torch.from_numpy(np.power(mag.astype(np.float64), 0.5).astype(np.float32)).to(device)
        Wd = torch.from_numpy(W).to(device)
        self.bits = bits
        base = awq.awq_quantize_pack(Wd, s, bits)
        del Wd
        per_copy = sum(t.numel() * t.element_size() for t in base)
        self.copies = max(2, math.ceil(2 * l2_bytes / per_copy))
        self.w = [base] + [tuple(t.clone() for t in base) for _ in range(self.copies - 1)]
        self.N, self.K = N, K
        dt = torch.bfloat16 if bf16 else torch.float16
        self.X = torch.from_numpy(X).to(device).to(dt)
        self.Y = torch.empty(m_max, N, dtype=dt, device=device)
        self.Xh = torch.from_numpy(X).to(dt).pin_memory()
        self.Yh = torch.empty(m_max, N, dtype=dt).pin_memory()

    def call(self, awq, M, r, stream=None):
        # the packed weights are static (no kernel writes them between steps), which is the
        # AWQ_GEMM_WEIGHTS_READY contract: each GEMM may stream them while the previous runs
        qw, sc, z = self.w[r % self.copies]
        awq.awq_gemm_w4a16(self.X[:M], qw, sc, z, self.N, self.K, self.bits, out=self.Y[:M],
                           stream=stream, weights_ready=True)


def capture_run(fn_per_step, first, count, stream):
    """One CUDA graph holding `count` consecutive steps (step r uses rotation index r), so
    the kernels run back to back without a graph launch between them."""
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for r in range(first, first + count):
            fn_per_step(r)
    return g


def time_steps(fn_per_step, steps, warmup, stream, world):
    """Warm-up graph of `warmup` steps, then a graph of exactly `steps` steps timed with
    CUDA events on `stream`, with a barrier and a device synchronisation on both sides. The
    timed graph is also replayed once before the timed replay (its first replay uploads the
    graph to the device), so the untimed warm-up is `warmup + steps` steps."""
    gw = capture_run(fn_per_step, 0, warmup, stream)
    gt = capture_run(fn_per_step, warmup, steps, stream)
    with torch.cuda.stream(stream):
        gw.replay()
        gt.replay()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        gt.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    del gw, gt
    return e0.elapsed_time(e1) / 1e3   # seconds


def oracle_decode_jobs(shapes, rows=None):
    """The oracle's own packing of each decode shape's weight (rows: the first rows only)."""
    import oracle as O
    jobs = []
    for (N, K) in shapes:
        W, mag, X = synth.decode_layer(N, K, 1)
        s = np.power(mag.astype(np.float64), 0.5).astype(np.float32)
        Wr = W if rows is None else W[:rows]
        jobs.append((X[:1], *O.quantize_pack(Wr, s, 4, GROUP), K, 4, GROUP))
    return jobs


def cpu_oracle_sample(shapes, min_seconds=10.0, max_seconds=30.0):
    """The oracle (numpy, fp64) running the headline step -- the M = 1 decode GEMM over every
    row of each decode shape -- on every host core (one spawned process per core, each on a
    slice of the output rows), repeated for 10-30 s. Returns (GB/s of algorithmic bytes,
    seconds, cores, description)."""
    from oracle.parallel import OracleGemmPool, cpu_model
    jobs = oracle_decode_jobs(shapes)
    pool = OracleGemmPool(jobs)
    try:
        pool.run_once()   # warm-up
        total, passes = 0.0, 0
        while total < min_seconds and (passes == 0 or total + total / passes < max_seconds):
            total += pool.run_once()
            passes += 1
    finally:
        pool.close()
    step_bytes = sum(gemm_bytes(1, qw.shape[0], K) for _, qw, _, _, K, _, _ in jobs)
    desc = (f"oracle gemm_w4a16 (numpy fp64) at M=1 over all rows of {list(shapes)}, "
            f"{passes} passes, output rows split across {pool.cores} spawned processes "
            f"(1 BLAS thread each) on {cpu_model()}")
    return step_bytes * passes / total / 1e9, total, pool.cores, desc


# ----------------------------------------------------------------------------- other rows

def time_call(fn, reps, warm=1):
    """Median device time of `fn` over `reps` calls (CUDA events on the current stream)."""
    for _ in range(warm):
        fn()
    torch.cuda.synchronize()
    ts = []
    for _ in range(reps):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        fn()
        e1.record()
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1) / 1e3)
    return statistics.median(ts)


def decoder_layer_rows(awq, dev, pk):
    """The other hot-path rows on the 7B-shaped decoder layer and its 65536-token calibration
    batch: activation statistics, down_proj's calibration input computed as the gated MLP
    produces it (silu(X W_gate^T) * (X W_up^T) from the fp16 weights), the 20-point searches
    (q/k/v and gate/up jointly), packing, and the W4A16 GEMM of every linear over the
    calibration batch -- timed per stage and as one pipeline. Also quantize-and-pack on the
    largest prefill weight."""
    rows = {}
    acts = synth.decoder_layer_activations(names=("hidden", "o_in"))
    Ws = synth.decoder_layer_weights()
    alphas = torch.from_numpy(np.arange(20, dtype=np.float32) / np.float32(20)).to(dev)
    Xd = {k: torch.from_numpy(v).to(dev) for k, v in acts.items()}
    del acts
    Wd = {k: torch.from_numpy(v).to(dev) for k, v in Ws.items()}
    del Ws
    # down_proj's calibration input: the gated MLP's output on the hidden state
    Mtok = int(Xd["hidden"].shape[0])
    Xd["down_in"] = torch.empty(Mtok, Wd["gate_proj"].shape[0], dtype=torch.float16, device=dev)
    t = time_call(lambda: awq.awq_silu_mul_gemm(Xd["hidden"], Wd["gate_proj"], Wd["up_proj"],
                                                out=Xd["down_in"]), 3)
    fl = 4 * Mtok * Wd["gate_proj"].shape[0] * Wd["gate_proj"].shape[1]
    rows["gated_mlp_input"] = {"M": Mtok, "I": Wd["gate_proj"].shape[0],
                               "K": Wd["gate_proj"].shape[1], "ms": t * 1e3,
                               "TFLOP/s": fl / t / 1e12, "frac_tensor": fl / t / 1e12 / pk["bf16_tflops"]}

    # act_stats (HBM-bound: 2MK bytes)
    out = []
    for name in ("hidden", "down_in"):
        X = Xd[name]
        M, K = X.shape
        ws = torch.empty(max(awq.lib().awq_act_stats_workspace_size(M, K), 16), dtype=torch.uint8,
                         device=dev)
        sx = torch.empty(K, dtype=torch.float32, device=dev)
        t = time_call(lambda: awq.awq_act_stats(X, out=sx, workspace=ws), 5)
        gbs = 2 * M * K / t / 1e9
        out.append({"M": M, "K": K, "us": t * 1e6, "GB/s": gbs, "frac_hbm": gbs / pk["hbm_gbs"]})
    rows["act_stats"] = out

    # the joint gate/up search at full size (the largest of the layer's four searches)
    Wgu = torch.cat([Wd["gate_proj"], Wd["up_proj"]]).contiguous()
    X = Xd["hidden"]
    sx = awq.awq_act_stats(X)
    M, K = X.shape
    Ngu = Wgu.shape[0]
    ws = torch.empty(awq.lib().awq_search_scale_workspace_size(M, Ngu, K, 20), dtype=torch.uint8,
                     device=dev)
    t = time_call(lambda: awq.awq_search_scale(Wgu, X, sx, alphas, 4, workspace=ws), 2)
    flops = 20 * 2 * M * Ngu * K
    ex, form = search_executed_flops(M, Ngu, K, 20)
    rows["search_gate_up"] = {"M": M, "N": Ngu, "K": K, "grid": 20, "ms": t * 1e3,
                              "form": form,
                              "TFLOP/s (definition, 20*2MNK)": flops / t / 1e12,
                              "TFLOP/s (executed)": ex / t / 1e12,
                              "frac_tensor_executed": ex / t / 1e12 / pk["bf16_tflops"]}
    del ws, Wgu
    torch.cuda.empty_cache()

    # the whole layer as one pipeline: stats -> gated-MLP input of down_proj and its stats ->
    # 4 searches -> 7 packs -> 7 GEMMs over the batch (outputs and workspaces allocated before
    # the timed region)
    y_buf = torch.empty(Mtok * max(W.shape[0] for W in Wd.values()), dtype=torch.float16,
                        device=dev)
    g_ws = torch.empty(awq.lib().awq_gemm_workspace_size(Mtok, 1, max(W.shape[1] for W in
                                                                       Wd.values()), 4),
                       dtype=torch.uint8, device=dev)
    jobs = [("hidden", ["q_proj", "k_proj", "v_proj"]), ("hidden", ["gate_proj", "up_proj"]),
            ("o_in", ["o_proj"]), ("down_in", ["down_proj"])]
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
    chosen = {}
    search_flops = 0
    stacked = {tuple(names): (torch.cat([Wd[n] for n in names]).contiguous() if len(names) > 1
                              else Wd[names[0]]) for _, names in jobs}
    ws_bytes = max(awq.lib().awq_search_scale_workspace_size(Xd[x].shape[0], W.shape[0],
                                                            W.shape[1], 20)
                   for (x, names), W in zip(jobs, stacked.values()))
    search_ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    torch.cuda.synchronize()
    ev[0].record()
    awq.awq_silu_mul_gemm(Xd["hidden"], Wd["gate_proj"], Wd["up_proj"], out=Xd["down_in"])
    stats = {name: awq.awq_act_stats(Xd[name]) for name in ("hidden", "o_in", "down_in")}
    ev[1].record()
    for xname, names in jobs:
        W = stacked[tuple(names)]
        _, best, best_s, _, best_inv = awq.awq_search_scale(W, Xd[xname], stats[xname], alphas,
                                                            4, workspace=search_ws, inv=True)
        search_flops += search_executed_flops(Xd[xname].shape[0], W.shape[0], W.shape[1], 20)[0]
        for n in names:
            chosen[n] = (best, best_s, best_inv)
    ev[2].record()
    packed = {n: awq.awq_quantize_pack(Wd[n], chosen[n][1], 4) for n in Wd}
    ev[3].record()
    gemm_flops = 0
    xin = {"q_proj": "hidden", "k_proj": "hidden", "v_proj": "hidden", "gate_proj": "hidden",
           "up_proj": "hidden", "o_proj": "o_in", "down_proj": "down_in"}
    invs = {n: chosen[n][2] for n in packed}
    ev3b = torch.cuda.Event(enable_timing=True)
    ev3b.record()
    for n, (qw, sc, z) in packed.items():
        N, K = Wd[n].shape
        Y = y_buf[:Mtok * N].view(Mtok, N)
        awq.awq_gemm_w4a16(Xd[xin[n]], qw, sc, z, N, K, 4, inv_s=invs[n], out=Y, workspace=g_ws)
        gemm_flops += 2 * Mtok * N * K
    ev[4].record()
    torch.cuda.synchronize()
    st = [ev[i].elapsed_time(ev[i + 1]) / 1e3 for i in range(4)]
    st_gemm_only = ev3b.elapsed_time(ev[4]) / 1e3
    rows["decoder_layer_pipeline"] = {
        "tokens": int(Xd["hidden"].shape[0]), "seconds": sum(st),
        "stats_and_gated_input_s": st[0], "search_s": st[1], "pack_s": st[2], "gemm_s": st[3],
        "search_TFLOP/s (executed)": search_flops / st[1] / 1e12,
        "gemm_TFLOP/s": gemm_flops / st_gemm_only / 1e12,
        "alpha_index": {n: int(chosen[n][0].item()) for n in chosen},
    }
    del Xd, Wd, packed, stats, chosen, stacked, search_ws, y_buf, g_ws
    torch.cuda.empty_cache()

    # quantize-and-pack on the largest prefill weight (HBM-bound)
    N, K = synth.PREFILL_SHAPES[0]
    W, mag, _ = synth.prefill_layer(N, K, 1)
    Wt = torch.from_numpy(W).to(dev)
    del W
    s = torch.from_numpy(np.power(mag.astype(np.float64), 0.5).astype(np.float32)).to(dev)
    out = []
    for bits in (4, 3):
        t = time_call(lambda: awq.awq_quantize_pack(Wt, s, bits), 5)
        b = 2 * N * K + N * K * bits // 8 + 3 * N * (K // GROUP)
        out.append({"N": N, "K": K, "bits": bits, "us": t * 1e6, "GB/s": b / t / 1e9,
                    "frac_hbm": b / t / 1e9 / pk["hbm_gbs"]})
    rows["quantize_pack"] = out
    del Wt
    torch.cuda.empty_cache()
    return rows


def profile_rows(awq, dev):
    """Small cases of the other kernels for detailed profiling (a few GB on the device):
    act_stats on one 65536 x 4096 calibration input, quantize-and-pack of one
    [28672, 8192] weight, and the 20-point search of one [4096, 4096] linear over it."""
    X = torch.from_numpy(synth.decoder_layer_activations(names=("o_in",))["o_in"]).to(dev)
    sx = awq.awq_act_stats(X)
    N, K = synth.PREFILL_SHAPES[0]
    W, mag, _ = synth.prefill_layer(N, K, 1)
    Wt = torch.from_numpy(W).to(dev)
    del W
    s = torch.from_numpy(np.power(mag.astype(np.float64), 0.5).astype(np.float32)).to(dev)
    awq.awq_quantize_pack(Wt, s, 4)
    del Wt
    Wo = torch.from_numpy(synth.decoder_layer_weights()["o_proj"]).to(dev)
    alphas = torch.from_numpy(np.arange(20, dtype=np.float32) / np.float32(20)).to(dev)
    awq.awq_search_scale(Wo, X, sx, alphas, 4)
    torch.cuda.synchronize()


def segment_launches(records):
    """Splits the trace build's per-CTA records (in CTA start order) into launches. A
    launch's CTAs all start before the next launch's first CTA (which launches only after
    every CTA of this one has passed its dependency wait), and each blockIdx (word 6)
    appears once per launch, so a launch ends where a blockIdx repeats."""
    launches, cur, seen = [], [], set()
    for rec in records:
        b = int(rec[6])
        if b in seen:
            launches.append(np.array(cur))
            cur, seen = [], set()
        cur.append(rec)
        seen.add(b)
    if cur:
        launches.append(np.array(cur))
    return launches


def trace_decode(awq, dev, l2, stream, steps):
    """The headline step (M = 1 on the three decode shapes, weights-ready, one CUDA graph) on
    the trace build: the per-launch timeline of the streaming decode kernel from its CTAs'
    %globaltimer records. Steady-state medians per shape, in microseconds:
      span: from the previous launch's last CTA end to this launch's last CTA end;
      early_start: how long before the previous launch ended this launch's first CTA started;
      wait_release: from the previous launch's end to this launch's dependency wait returning
        (the producer's; mean over CTAs);
      x_staging: from that wait to X staged in shared memory (mean over CTAs; the consumers'
        own wait may return before the producer's);
      per_unit: interval between consecutive units (16 KB of codes) landing (mean over CTAs);
      units_max: the most units any CTA of the launch has;
      tail: from the mean CTA end to the last CTA end.
    %globaltimer ticks every 256 ns on this part; the means over CTAs and steps resolve below
    that."""
    from weight_only_int4_stats_b200 import build
    awq.use_library(build.build(trace=True))
    shapes = [DecodeShape(awq, N, K, 1, l2, dev) for (N, K) in synth.DECODE_SHAPES]
    for sh in shapes:
        sh.call(awq, 1, 0)
    torch.cuda.synchronize()
    g = capture_run(lambda r: [sh.call(awq, 1, r) for sh in shapes], 0, steps, stream)
    with torch.cuda.stream(stream):
        g.replay()            # the first replay uploads the graph
    torch.cuda.synchronize()
    awq.trace_reset()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        g.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    step_us = e0.elapsed_time(e1) * 1e3 / steps
    launches = segment_launches(awq.trace_read().astype(np.int64))
    per = {j: [] for j in range(len(shapes))}
    for li in range(len(shapes), len(launches)):
        L, prev = launches[li], launches[li - 1]
        j = li % len(shapes)
        prev_end = prev[:, 5].max()
        units = L[:, 1]
        gaps = []
        for rec, n in zip(L, units):
            k = int(min(n, 24))
            if k >= 2:   # first-to-last over k - 1 intervals
                gaps.append((rec[8 + k - 1] - rec[8]) / (k - 1))
        # %globaltimer ticks coarsely (256 ns here): means over the CTAs average the tick out
        per[j].append([L[:, 5].max() - prev_end, prev_end - L[:, 2].min(),
                       L[:, 3].mean() - prev_end, (L[:, 4] - L[:, 3]).mean(),
                       np.mean(gaps) if gaps else float("nan"), units.max(),
                       L[:, 5].max() - L[:, 5].mean()])
    keys = ["span", "early_start", "wait_release", "x_staging", "per_unit", "units_max", "tail"]
    out = []
    for j, sh in enumerate(shapes):
        m = np.median(np.array(per[j], dtype=np.float64), axis=0)
        row = {"N": sh.N, "K": sh.K}
        for k, v in zip(keys, m):
            row[k] = int(v) if k == "units_max" else round(float(v) / 1e3, 3)
        out.append(row)
    print(json.dumps({"metric": "decode timeline (trace build), M=1", "steps": steps,
                      "step_us": round(step_us, 2), "launches": len(launches),
                      "per_shape": out}), flush=True)


# ----------------------------------------------------------------------------- main arms

def run_reference(args, world, rank):
    """The CPU oracle timed as the reference arm (rank 0 only): each step is the headline
    step (the M = 1 decode GEMM on the three decode shapes) on every host core, on all rows
    when a pass takes under half a second, else on the first rows of each shape."""
    if rank != 0:
        return
    from oracle.parallel import OracleGemmPool, cpu_model
    shapes = synth.DECODE_SHAPES
    rows = None
    probe = OracleGemmPool(oracle_decode_jobs(shapes, rows=512))
    t512 = min(probe.run_once() for _ in range(3))
    probe.close()
    full = sum(n for n, _ in shapes)
    if t512 * full / (512 * len(shapes)) > 0.5:
        rows = max(64, int(512 * 0.5 / t512))
    jobs = oracle_decode_jobs(shapes, rows=rows)
    pool = OracleGemmPool(jobs)
    try:
        for _ in range(args.warmup):
            pool.run_once()
        dt = sum(pool.run_once() for _ in range(args.steps))
    finally:
        pool.close()
    step_bytes = sum(gemm_bytes(1, qw.shape[0], K) for _, qw, _, _, K, _, _ in jobs)
    v = step_bytes * args.steps / dt / 1e9
    sample = (f"each step: oracle gemm_w4a16 (numpy fp64) at M=1 on "
              f"{'all rows' if rows is None else f'the first {rows} rows'} of each decode shape "
              f"{shapes}, rows split across {pool.cores} spawned processes on {cpu_model()}")
    line = {
        "impl": "reference", "metric": METRIC, "value": v, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": "decode GEMM M=1 over [4096,4096], [11008,4096], [4096,11008] "
                               "(W4 g128), CPU oracle"},
        "cpu_baseline": {"value": v, "unit": "GB/s", "cores": pool.cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_b200(args, world, rank, local):
    import weight_only_int4_stats_b200 as awq
    dev = torch.device("cuda", torch.cuda.current_device())
    props = torch.cuda.get_device_properties(dev)
    l2 = getattr(props, "L2_cache_size", 126 * 1024 * 1024)
    pk = peaks()
    stream = torch.cuda.Stream()
    if args.only == "profile":
        profile_rows(awq, dev)
        return
    if args.only == "trace":
        trace_decode(awq, dev, l2, stream, args.steps)
        return
    if args.only == "rows":
        rows = decoder_layer_rows(awq, dev, pk)
        if rank == 0:
            print(json.dumps({"metric": METRIC, "rows": rows}), flush=True)
        return

    # ---- headline: decode GEMM at M = 1 over the three shapes
    shapes = [DecodeShape(awq, N, K, 16, l2, dev) for (N, K) in synth.DECODE_SHAPES]
    for sh in shapes:                     # first calls outside capture
        sh.call(awq, 1, 0)
    torch.cuda.synchronize()
    def step(r):
        for sh in shapes:
            sh.call(awq, 1, r)
    step_bytes = sum(gemm_bytes(1, sh.N, sh.K) for sh in shapes)

    clocks = ClockSampler(local)
    clocks.start()
    dt = time_steps(step, args.steps, args.warmup, stream, world)
    clk = clocks.stop()
    value, dt_max = job_rate(step_bytes * args.steps / 1e9, dt, world)
    per_gpu = step_bytes * args.steps / dt / 1e9
    launches = args.steps * len(shapes)

    # ---- decode sweep: each (shape, M) on its own
    sweep = []
    for sh in (shapes if args.only in ("all", "decode") else []):
        for M in synth.DECODE_M:
            t = time_steps(lambda r, sh=sh, M=M: sh.call(awq, M, r), 200, 10, stream, world)
            b = gemm_bytes(M, sh.N, sh.K)
            gbs = b * 200 / t / 1e9
            sweep.append({"N": sh.N, "K": sh.K, "M": M, "us": t / 200 * 1e6, "GB/s": gbs,
                          "TFLOP/s": 2 * M * sh.N * sh.K * 200 / t / 1e12,
                          "frac_hbm": gbs / pk["hbm_gbs"]})

    # ---- end to end through the binding with host buffers (no graph, copies timed)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e2e_steps = min(args.steps, 200)
    h2d = sum(2 * sh.K for sh in shapes)
    d2h = sum(2 * sh.N for sh in shapes)

    def e2e_step(r):
        for sh in shapes:
            sh.X[:1].copy_(sh.Xh[:1], non_blocking=True)
            sh.call(awq, 1, r)
            sh.Yh[:1].copy_(sh.Y[:1], non_blocking=True)
    with torch.cuda.stream(stream):
        for r in range(3):
            e2e_step(r)
        torch.cuda.synchronize()
        e0.record(stream)
        for r in range(e2e_steps):
            e2e_step(r)
        e1.record(stream)
    torch.cuda.synchronize()
    t_e2e = max_over_ranks(e0.elapsed_time(e1) / 1e3, world)
    e2e = {"value": step_bytes * e2e_steps * world / t_e2e / 1e9, "unit": "GB/s",
           "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
           "how": "python binding call per GEMM, pinned-host X copied in and Y copied out "
                  "every step on the same stream, no graph"}
    del shapes
    torch.cuda.empty_cache()

    # ---- batched decode / small prefill: M in 32..256 on the batched shapes (weights > L2 in
    #      rotation), GB/s and TFLOP/s per (shape, M)
    batched = []
    for (N, K) in (synth.BATCHED_SHAPES if args.only in ("all", "batched") else []):
        W, mag, X = synth.batched_layer(N, K)
        s_ = torch.from_numpy(np.power(mag.astype(np.float64), 0.5).astype(np.float32)).to(dev)
        Wt = torch.from_numpy(W).to(dev)
        base = awq.awq_quantize_pack(Wt, s_, 4)
        del Wt
        per = sum(t.numel() * t.element_size() for t in base)
        ncp = max(2, math.ceil(2 * l2 / per))
        cps = [base] + [tuple(t.clone() for t in base) for _ in range(ncp - 1)]
        Xt = torch.from_numpy(X).to(dev)
        Yt = torch.empty(X.shape[0], N, dtype=torch.float16, device=dev)
        for M in synth.BATCHED_M:
            f = (lambda r, M=M: awq.awq_gemm_w4a16(Xt[:M], *cps[r % ncp], N, K, 4, out=Yt[:M]))
            f(0)
            t = time_steps(f, 100, 5, stream, world)
            b = gemm_bytes(M, N, K)
            batched.append({"N": N, "K": K, "M": M, "us": t / 100 * 1e6,
                            "GB/s": b * 100 / t / 1e9, "TFLOP/s": 2 * M * N * K * 100 / t / 1e12,
                            "frac_hbm": b * 100 / t / 1e9 / pk["hbm_gbs"],
                            "frac_tensor": 2 * M * N * K * 100 / t / 1e12 / pk["bf16_tflops"]})
        del cps, base, Xt, Yt
        torch.cuda.empty_cache()

    # ---- prefill at M = 2048 (4-bit on the three shapes, then the 3-bit variant)
    prefill = []
    pf_cases = [(N, K, 4) for (N, K) in synth.PREFILL_SHAPES] + [(*synth.PREFILL_SHAPES[0], 3)]
    for (N, K, bits) in (pf_cases if args.only in ("all", "prefill") else []):
        m_list = synth.PREFILL_M if bits == 4 else [2048]
        W, mag, X = synth.prefill_layer(N, K, max(m_list))
        s = torch.from_numpy(np.power(mag.astype(np.float64), 0.5).astype(np.float32)).to(dev)
        Wd = torch.from_numpy(W).to(dev)
        del W
        packs = [awq.awq_quantize_pack(Wd, s, bits)]
        del Wd
        packs.append(tuple(t.clone() for t in packs[0]))   # two copies > L2 with X
        Xall = torch.from_numpy(X).to(dev)
        Yall = torch.empty(max(m_list), N, dtype=torch.float16, device=dev)
        for M in m_list:
            Xd, Yd = Xall[:M], Yall[:M]
            for p in packs:
                awq.awq_gemm_w4a16(Xd, *p, N, K, bits, out=Yd)
            torch.cuda.synchronize()
            iters = max(5, 20 * 2048 // M)
            t = time_steps(lambda r: awq.awq_gemm_w4a16(Xd, *packs[r % 2], N, K, bits, out=Yd),
                           iters, 3, stream, world)
            tfl = 2 * M * N * K * iters / t / 1e12
            prefill.append({"N": N, "K": K, "M": M, "bits": bits, "ms": t / iters * 1e3,
                            "TFLOP/s": tfl, "frac_tensor": tfl / pk["bf16_tflops"]})
        del packs, Xall, Yall
        torch.cuda.empty_cache()
    pf4 = [p for p in prefill if p["bits"] == 4 and p["M"] == 2048]
    pf_flops = sum(2 * 2048 * p["N"] * p["K"] for p in pf4)
    pf_time = sum(p["ms"] for p in pf4) / 1e3
    pf_value = pf_flops / pf_time / 1e12 if pf4 else None

    # ---- bf16 activations: the headline decode step and the M = 2048 prefill GEMM
    bf16 = {}
    if args.only in ("all", "bf16"):
        shapes_b = [DecodeShape(awq, N, K, 1, l2, dev, bf16=True) for (N, K) in synth.DECODE_SHAPES]
        for sh in shapes_b:
            sh.call(awq, 1, 0)
        t = time_steps(lambda r: [sh.call(awq, 1, r) for sh in shapes_b], 200, 10, stream, world)
        b = sum(gemm_bytes(1, sh.N, sh.K) for sh in shapes_b)
        bf16["decode_M1_step"] = {"us_per_step": t / 200 * 1e6, "GB/s": b * 200 / t / 1e9,
                                  "frac_hbm": b * 200 / t / 1e9 / pk["hbm_gbs"]}
        del shapes_b
        # 3-bit codes, fp16 activations: the same headline step
        shapes_3 = [DecodeShape(awq, N, K, 1, l2, dev, bits=3) for (N, K) in synth.DECODE_SHAPES]
        for sh in shapes_3:
            sh.call(awq, 1, 0)
        t = time_steps(lambda r: [sh.call(awq, 1, r) for sh in shapes_3], 200, 10, stream, world)
        b = sum(gemm_bytes(1, sh.N, sh.K, 3) for sh in shapes_3)
        bf16["decode_M1_step_3bit_fp16"] = {"us_per_step": t / 200 * 1e6,
                                            "GB/s": b * 200 / t / 1e9,
                                            "frac_hbm": b * 200 / t / 1e9 / pk["hbm_gbs"]}
        del shapes_3
        N, K = synth.PREFILL_SHAPES[0]
        W, mag, X = synth.prefill_layer(N, K, 2048)
        s_ = torch.from_numpy(np.power(mag.astype(np.float64), 0.5).astype(np.float32)).to(dev)
        Wt = torch.from_numpy(W).to(dev)
        del W
        packs = [awq.awq_quantize_pack(Wt, s_, 4)]
        del Wt
        packs.append(tuple(t_.clone() for t_ in packs[0]))
        Xb = torch.from_numpy(X).to(dev).to(torch.bfloat16)
        Yb = torch.empty(2048, N, dtype=torch.bfloat16, device=dev)
        t = time_steps(lambda r: awq.awq_gemm_w4a16(Xb, *packs[r % 2], N, K, 4, out=Yb), 20, 3,
                       stream, world)
        tfl = 2 * 2048 * N * K * 20 / t / 1e12
        bf16["prefill_M2048_28672x8192"] = {"ms": t / 20 * 1e3, "TFLOP/s": tfl,
                                            "frac_tensor": tfl / pk["bf16_tflops"]}
        del packs, Xb, Yb
        torch.cuda.empty_cache()

    rows = decoder_layer_rows(awq, dev, pk) if args.only == "all" else None

    if rank != 0:
        return
    cpu_gbs, cpu_t, cpu_cores, cpu_desc = (cpu_oracle_sample(synth.DECODE_SHAPES)
                                           if args.only == "all"
                                           else (None, None, None, "skipped (--only)"))
    dec_traffic, dec_traffic_src = profiled_traffic("gemv_stream_decode_M1")
    pf_traffic, pf_traffic_src = profiled_traffic("tc_gemm_prefill_28672x8192_M2048")
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt_max / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
        "data": "synthetic",
        "config": {
            "workload": "decode GEMM, M=1, W4 g128, [N,K] in [4096,4096], [11008,4096], "
                        "[4096,11008]; one GEMM per shape per step",
            "inputs": "weights rotate through copies totalling > 2x L2 (L2 not flushed)",
            "replay": "warm-up steps and the K timed steps each captured in one CUDA graph "
                      "(kernels back to back, programmatic dependent launch between them)",
            "flags": "AWQ_GEMM_WEIGHTS_READY (static weights: each GEMM streams its weights "
                     "while the previous GEMM runs; activations are read after it completes)",
            "parallelism": f"replicas x{world} (no data-path collective)",
        },
        "roofline": {"bound": "hbm", "achieved": per_gpu, "peak": pk["hbm_gbs"],
                     "unit": "GB/s", "frac": per_gpu / pk["hbm_gbs"],
                     "traffic": dec_traffic, "traffic_source": dec_traffic_src,
                     "algorithmic_bytes_per_launch": step_bytes / len(synth.DECODE_SHAPES),
                     "kernel": "gemv_stream_kernel<1, true, false, 4>", "peak_source": pk["source"],
                     "peak_kind": "measured copy bandwidth (burst)",
                     "frac_of_8TBps_nominal": per_gpu / 8000.0},
        "prefill": {"metric": "TFLOP/s at M=2048", "value": pf_value, "unit": "TFLOP/s",
                    "per_shape": prefill, "peak": pk["bf16_tflops"],
                    "peak_kind": "measured bf16 cuBLAS burst (fp16 has the same dense rate)",
                    "traffic_28672x8192": pf_traffic, "traffic_source": pf_traffic_src,
                    "frac": pf_value / pk["bf16_tflops"] if prefill else None,
                    "kernel": "tc_gemm_kernel"},
        "sweep": sweep,
        "batched": batched,
        "bf16_and_3bit": bf16,
        "rows": rows,
        "cpu_baseline": {"value": cpu_gbs, "unit": "GB/s", "cores": cpu_cores,
                         "kind": "oracle", "sample": cpu_desc, "seconds": cpu_t},
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clk,
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["b200", "reference"], default="b200")
    ap.add_argument("--only", choices=["all", "decode", "batched", "prefill", "bf16", "rows",
                                       "profile", "trace"],
                    default="all",
                    help="run one section only (used by the profiling commands)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world, rank, local = dist_setup()
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_b200(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
