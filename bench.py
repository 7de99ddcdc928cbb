#!/usr/bin/env python
"""Decode throughput of the int8 per-window recurrent state on B200.

Workload (default): Gated DeltaNet decode, batch 256 x 32 heads, d_k = d_v =
128, bf16 q/k/v/o, int8 state with per-row scales, window W = 16, r = 4
Compensator Tokens, smoothing on.  One STEP is one window: W decode launches
and the window commit through the C ABI, i.e. batch * W tokens.

Timing: W_warm untimed steps, then exactly K steps bracketed by a barrier and
torch.cuda.synchronize() on both sides, timed with CUDA events on the
launching stream, max over ranks.  Each step replays a CUDA graph of the
window's launches; event-record nodes inside the graph time every launch for
the roofline.  Each decode launch reads 160-300 MB (int8 state, records,
inputs), above the 126 MB L2, so every launch streams from HBM.

Other modes: --mode prefill | fp32step | init | ragged | mse (see --help);
--bits 6 | 4 | 16 runs any decode mode on the narrow-code or BF16 state variants.

Multi-GPU (torchrun): every rank decodes its own shard of sequences (batch
per rank fixed: weak scaling); no collective on the data path; the host
gathers the max elapsed time at the end.

--impl reference times the CPU oracle (plain C, FP64) on the host cores on a
bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import json
import math
import os
import re
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "decode tokens/s (state-update+output) and HBM GB/s as % of B200 peak"
FALLBACK_HBM_GBS = 6650.0
# FP32 FMA peak of one B200: 148 SMs x 128 FP32 lanes x 2 FLOP x 1.965 GHz
FP32_ALU_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


# --------------------------------------------------------------------------
# Algorithmic bytes (per (sequence, head) and launch)
# --------------------------------------------------------------------------

def snapshot_bytes(dk, dv, r, bits=8, svd=False):
    """Codes (one byte per code, half a byte at 4 bits, two bytes per BF16
    value at 16), row scales, smoothing factors and compensators of one head
    (row indices and k~_c rows; with the SVD rule also the u_c vectors)."""
    codes = dv * dk // 2 if bits == 4 else 2 * dv * dk if bits == 16 else dv * dk
    return codes + 4 * dv + 4 * dk + r * (4 + 4 * dk) + (4 * r * dv if svd else 0)


def record_bytes(dk, dv, gate):
    return 4 * ((dk if gate == "diag" else 1) + dk + dv)


def decode_launch_bytes(dk, dv, r, gate, e, t, bits=8, svd=False):
    """Bytes one decode launch at window position t must move per head:
    read the snapshot and the t-1 buffered records, read q, k, v, alpha,
    beta, write o and record t."""
    G = dk if gate == "diag" else 1
    rec = record_bytes(dk, dv, gate)
    return (snapshot_bytes(dk, dv, r, bits, svd) + (t - 1) * rec + e * (2 * dk + dv) + 4 * G + 4
            + e * dv + rec)


def commit_launch_bytes(dk, dv, r, gate, n, bits=8, svd=False):
    """Bytes the commit of a window of n records must move per head: read the
    snapshot and the n records, write the new snapshot."""
    return 2 * snapshot_bytes(dk, dv, r, bits, svd) + n * record_bytes(dk, dv, gate)


# --------------------------------------------------------------------------
# Helpers
# --------------------------------------------------------------------------

def _dist():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def aggregate(elapsed_ms: float, tokens_per_rank: int, world: int, group=None):
    """Max elapsed time over ranks and the whole-job token rate (host-side
    reduction of two scalars; no data-path collective)."""
    import torch
    import torch.distributed as dist
    if world > 1:
        dev = "cuda" if dist.get_backend(group) == "nccl" else "cpu"
        t = torch.tensor([elapsed_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
        elapsed_ms = float(t.item())
    return elapsed_ms, tokens_per_rank * world / (elapsed_ms / 1e3)


def shard(rank: int, world: int, batch_per_rank: int):
    """This rank's sequences: a contiguous block of the global batch
    (world * batch_per_rank sequences).  Each (sequence, head) state is
    independent, so ranks share nothing but the final timing reduction."""
    if not (0 <= rank < world) or batch_per_rank < 1:
        raise ValueError("bad shard")
    b0 = rank * batch_per_rank
    return range(b0, b0 + batch_per_rank)


def shard_tokens(wl, rank: int, world: int, t0: int, t1: int, device):
    """Inputs of tokens t0..t1-1 for this rank's shard, drawn by global
    sequence index (the counter-based generator is keyed by it): the N ranks
    together decode exactly the global batch one rank would."""
    from linear_attention_recurrent_int8_b200 import synth
    return synth.torch_tokens(wl.seed, list(shard(rank, world, wl.batch)), wl.heads, t0, t1,
                              wl.d_k, wl.d_v, wl.gate, wl.io, device)


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def measured_bf16_tflops(sustained: bool):
    """Dense BF16 tensor peak (TFLOP/s): the measured cuBLAS figure (burst, or
    sustained under the power cap), else the pool's earlier measurement."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        key = "bf16_tflops_sustained" if sustained else "bf16_tflops"
        if key in d:
            return float(d[key]), "measured"
    return (1400.0 if sustained else 1590.0), "fallback"


# the sources of each kernel's translation unit (the .cu and the headers it includes)
KERNEL_SOURCES = {
    "decode": ["lq_decode.cu", "lq_common.cuh", "lq_quant.cuh", "lq_tc.cuh", "lq_kernels.h"],
    "commit": ["lq_commit.cu", "lq_common.cuh", "lq_quant.cuh", "lq_tc.cuh", "lq_kernels.h"],
}


def source_digest(kernel: str) -> str:
    h = hashlib.sha1()
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, "linear_attention_recurrent_int8_b200", "csrc", name), "rb") as fh:
            h.update(name.encode())
            h.update(fh.read())
    return h.hexdigest()[:12]


def profiled_traffic(kernel_key: str, directory: str | None = None):
    """dram bytes per launch recorded by an ncu capture summary under
    profiles/, if it was taken on the current kernel sources."""
    digest = source_digest(kernel_key.split(":")[0])
    for f in glob.glob(os.path.join(directory or os.path.join(ROOT, "profiles"), "*.md")):
        text = open(f).read()
        m_key = re.search(r"^traffic_key:\s*(\S+)", text, re.M)
        m_src = re.search(r"^source_sha1:\s*(\S+)", text, re.M)
        m_val = re.search(r"^traffic_bytes_per_launch:\s*([0-9.eE+]+)", text, re.M)
        if m_key and m_src and m_val and m_key.group(1) == kernel_key and m_src.group(1) == digest:
            return float(m_val.group(1))
    return None


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled every 50 ms."""

    FIELDS = ["clocks.sm", "clocks.max.sm", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]

    def __init__(self, device_index: int):
        self.rows = []
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(device_index), "--query-gpu=" + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append((time.monotonic(), [x.strip() for x in line.split(",")]))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self, t0, t1, t_warm0):
        def pick(a, b):
            return [r for (t, r) in self.rows if a <= t <= b and len(r) == len(self.FIELDS)]
        rows = pick(t0, t1)
        window = "timed region"
        if len(rows) < 3:
            rows = pick(t_warm0, t1)
            window = "warm-up and timed region (timed region shorter than 3 samples)"
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm = sorted(float(r[0]) for r in rows if r[0].replace(".", "").isdigit())
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[3 + i].lower() == "active"})
        mx = rows[0][1]
        return {"sm_mhz": sm[len(sm) // 2] if sm else None,
                "sm_max_mhz": float(mx) if mx.replace(".", "").isdigit() else None,
                "reasons": reasons, "samples": len(rows), "window": window}


# --------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline and the reference arm)
# --------------------------------------------------------------------------

def oracle_window_rate(wl, n_seq: int, w_index: int = 0, bits: int = 8):
    """Times the CPU oracle on n_seq sequences x all heads for one window of
    decode plus its commit (codes of width `bits`).  Returns (tokens/s,
    seconds, threads)."""
    import numpy as np
    cores = len(os.sched_getaffinity(0))
    os.environ.setdefault("OMP_NUM_THREADS", str(cores))
    import oracle
    from linear_attention_recurrent_int8_b200 import synth
    bs = np.arange(n_seq)
    hs = np.arange(wl.heads)
    S0 = synth.initial_state(wl.seed, bs, hs, wl.d_k, wl.d_v, wl.outlier_rows, wl.outlier_cols,
                             wl.outlier_scale).reshape(n_seq * wl.heads, wl.d_v, wl.d_k)
    tok = synth.tokens(wl.seed, bs, hs, w_index * wl.window, (w_index + 1) * wl.window, wl.d_k,
                       wl.d_v, wl.gate, wl.io)

    def hm(x):
        x = np.asarray(x)
        B, T, H = x.shape[:3]
        return np.ascontiguousarray(np.swapaxes(x, 1, 2).reshape((B * H, T) + x.shape[3:]))

    inst = oracle.kda_instance if wl.gate == "diag" else oracle.gdn_instance
    d, kt, b = inst(hm(tok["alpha"]), hm(tok["beta"]), hm(tok["k"]))
    v, q = hm(tok["v"]), hm(tok["q"])
    snap = oracle.quantize(S0, wl.n_comp, wl.smoothing, bits)
    gdim = wl.d_k if wl.gate == "diag" else 1
    t0 = time.perf_counter()
    rec = oracle.empty_records(n_seq * wl.heads, wl.window, wl.d_k, wl.d_v, gdim)
    oracle.window(snap, rec, 0, d, kt, b, v, q)
    oracle.commit(snap, rec, wl.window, wl.n_comp, wl.smoothing, bits)
    dt = time.perf_counter() - t0
    return n_seq * wl.window / dt, dt, int(os.environ["OMP_NUM_THREADS"])


def calibrated_sample(wl, target_s: float, bits: int = 8):
    _, dt1, _ = oracle_window_rate(wl, 1, bits=bits)
    n = int(max(1, min(wl.batch, math.floor(target_s / max(dt1, 1e-6)))))
    return n


# --------------------------------------------------------------------------
# Arms
# --------------------------------------------------------------------------

def run_reference(args, wl):
    rank, world, _ = _dist()
    if rank != 0:
        return None
    n_seq = calibrated_sample(wl, args.ref_seconds, args.bits)
    for i in range(args.warmup):
        oracle_window_rate(wl, n_seq, i, args.bits)
    total_tok, total_s = 0, 0.0
    for i in range(args.steps):
        rate, dt, cores = oracle_window_rate(wl, n_seq, args.warmup + i, args.bits)
        total_tok += n_seq * wl.window
        total_s += dt
    value = total_tok / total_s
    sample = (f"{n_seq} of {wl.batch} sequences x {wl.heads} heads, one window of {wl.window} "
              f"decode tokens plus its commit per step")
    return {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total_s / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(wl, args),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def state_words(bits):
    return {8: "int8 codes", 6: "6-bit codes (one per byte)", 4: "4-bit codes (two per byte)",
            16: "bf16 residual"}[bits]


def profile_key(kernel, wl, args):
    """Key of the ncu summary under profiles/ that holds this kernel's DRAM
    traffic: the workload's name, plus every override of its window,
    compensators, smoothing or code width (no summary exists for those)."""
    base = synth_workload(wl.name)
    key = f"{kernel}:{wl.name}"
    if (wl.window, wl.n_comp, bool(wl.smoothing)) != (base.window, base.n_comp, bool(base.smoothing)) \
            or args.bits != 8:
        key += f"_W{wl.window}_r{wl.n_comp}_s{int(bool(wl.smoothing))}_b{args.bits}"
    if getattr(args, "comp_rule", "rows") == "svd":
        key += "_svd"
    return key


def decode_kernel_name(wl, args):
    """The decode kernel the library launches for this workload: the
    tensor-core matvec for d_k = d_v = 128 with one code per byte, else the
    dp4a / FP32 kernel."""
    return "decode_tc_kernel" if wl.d_k == 128 and wl.d_v == 128 and args.bits in (8, 6) else "decode_kernel"


def synth_workload(name):
    from linear_attention_recurrent_int8_b200 import synth
    return synth.WORKLOADS[name]


def workload_config(wl, args):
    return {
        "workload": (f"{wl.name}: {'KDA per-channel' if wl.gate == 'diag' else 'GDN scalar'}-gate "
                     f"{'' if wl.delta else 'b = 0 (no delta rule) '}decode, batch {wl.batch} x {wl.heads} heads, d_k={wl.d_k}, d_v={wl.d_v}, "
                     f"window W={wl.window}, r={wl.n_comp} compensators, {wl.io} q/k/v/o, "
                     f"{state_words(args.bits)} state with per-row scales"),
        "batch_per_gpu": wl.batch, "heads": wl.heads, "d_k": wl.d_k, "d_v": wl.d_v,
        "window": wl.window, "n_comp": wl.n_comp, "gate": wl.gate, "io": wl.io,
        "smoothing": bool(wl.smoothing), "bits": args.bits, "delta": wl.delta,
        "comp_rule": args.comp_rule,
        "state": f"{state_words(args.bits)} + fp32 row scales",
        "step": f"one window: {wl.window} decode launches and the window commit",
        "tokens_per_step_per_gpu": wl.batch * wl.window,
        "l2": l2_note(wl.batch * wl.heads * decode_launch_bytes(
            wl.d_k, wl.d_v, wl.n_comp, wl.gate, 2 if wl.io == "bf16" else 4, 1, args.bits)),
        "graph": not args.no_graph,
        "launch_timing": ("per-launch CUDA events only in the last `slots` windows of the timed "
                          "region (the roofline's launch durations); the other windows run "
                          "without event nodes"),
    }


L2_BYTES = 126e6  # B200 L2


def l2_note(launch_bytes):
    """How the timing treats L2: the workloads whose decode launches read more
    than the L2 holds stream from HBM every launch; smaller ones are reported
    as L2-resident (effective GB/s), not flushed."""
    mb = launch_bytes / 1e6
    if launch_bytes > L2_BYTES:
        return f"inputs larger than L2: each decode launch reads ~{mb:.0f} MB vs 126 MB L2"
    return (f"inputs smaller than L2 (~{mb:.0f} MB per decode launch vs 126 MB L2), not flushed: "
            f"L2-resident, effective GB/s")


def run_lq(args, wl):
    import numpy as np
    import torch

    import linear_attention_recurrent_int8_b200 as lq
    from linear_attention_recurrent_int8_b200 import synth

    rank, world, local = _dist()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    group = None
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=dev)

    lq.load_library()
    cfg = lq.Config(batch=wl.batch, heads=wl.heads, d_k=wl.d_k, d_v=wl.d_v, window=wl.window,
                    n_comp=wl.n_comp, gate=lq.LQ_GATE_DIAG if wl.gate == "diag" else lq.LQ_GATE_SCALAR,
                    io_dtype=lq.LQ_BF16 if wl.io == "bf16" else lq.LQ_F32,
                    smoothing=int(wl.smoothing), auto_commit=0, delta=wl.delta, bits=args.bits,
                    comp_rule=lq.LQ_COMP_SVD if args.comp_rule == "svd" else lq.LQ_COMP_ROWS)
    svd = args.comp_rule == "svd" and wl.n_comp > 0
    W = wl.window
    e = 2 if wl.io == "bf16" else 4
    st = lq.State(cfg, dev)
    # this rank's shard of sequences: global sequence index offset
    bs, hs = np.array(shard(rank, world, wl.batch)), np.arange(wl.heads)
    S0 = synth.torch_initial_state(wl.seed, bs, hs, wl.d_k, wl.d_v, wl.outlier_rows, wl.outlier_cols,
                                   wl.outlier_scale, dev)
    lq.lq_state_init(st, S0.reshape(wl.nh, wl.d_v, wl.d_k))
    del S0

    n_slots = max(1, min(args.slots, args.steps + args.warmup))
    slots = []
    for sidx in range(n_slots):
        tok = shard_tokens(wl, rank, world, sidx * W, (sidx + 1) * W, dev)
        per_t = []
        for t in range(W):
            per_t.append([tok[k][:, t:t + 1].contiguous() for k in ("q", "k", "v", "alpha", "beta")])
        o = torch.empty((wl.batch, 1, wl.heads, wl.d_v), dtype=cfg.io_torch_dtype, device=dev)
        slots.append((per_t, o))
    torch.cuda.synchronize()

    def run_window(slot, events=None):
        per_t, o = slot
        if events:
            events[0].record()
        for t in range(W):
            lq.lq_decode_window(st, *per_t[t], 1, o)
            if events:
                events[t + 1].record()
        lq.lq_window_commit(st)
        if events:
            events[W + 1].record()

    # one eager window (also sets kernel attributes before any capture)
    run_window(slots[0])
    torch.cuda.synchronize()

    # Each slot has a graph without event nodes and one with an event node
    # around every launch.  An event node adds about 5 us to a window (18 per
    # window), so the timed region replays the plain graphs except in its
    # last len(graphs) windows, whose per-launch events give the launch
    # durations of the roofline; one warm-up round replays the instrumented
    # graphs once before the timing.
    graphs = []
    if not args.no_graph:
        s = torch.cuda.Stream(device=dev)
        for slot in slots:
            g_plain = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g_plain, stream=s):
                run_window(slot)
            # external events become event-record nodes of the graph
            evs = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(W + 2)]
            g_inst = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g_inst, stream=s):
                run_window(slot, evs)
            graphs.append((g_plain, g_inst, evs))
        assert st.pos == 0
    else:
        for slot in slots:
            graphs.append((None, None, [torch.cuda.Event(enable_timing=True) for _ in range(W + 2)]))
    n_g = len(graphs)

    def step(i, timed=None):
        g_plain, g_inst, evs = graphs[i % n_g]
        inst = timed >= args.steps - n_g if timed is not None else n_g <= i < 2 * n_g
        if g_plain is not None:
            (g_inst if inst else g_plain).replay()
        else:
            run_window(slots[i % len(slots)], evs if inst else None)

    sampler = ClockSampler(local) if not args.no_clocks else None
    t_warm0 = time.monotonic()
    for i in range(args.warmup):
        step(i)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    cur = torch.cuda.current_stream(dev)
    t0 = time.monotonic()
    start.record(cur)
    for i in range(args.steps):
        step(args.warmup + i, i)
    end.record(cur)
    torch.cuda.synchronize()
    t1 = time.monotonic()
    if world > 1:
        dist.barrier()
    if sampler:
        sampler.stop()
    elapsed = start.elapsed_time(end)
    elapsed_max, value = aggregate(elapsed, wl.batch * W * args.steps, world, group)

    # per-launch times from the event nodes of the instrumented windows (the
    # last n_g of the timed region, one per slot)
    dec_ms, com_ms, dec_bytes = [], [], 0.0
    nh = wl.nh
    used = sorted({(args.warmup + j) % n_g for j in range(max(0, args.steps - n_g), args.steps)})
    for gi in used:
        evs = graphs[gi][2]
        for t in range(W):
            dec_ms.append(evs[t].elapsed_time(evs[t + 1]))
            dec_bytes += nh * decode_launch_bytes(wl.d_k, wl.d_v, wl.n_comp, wl.gate, e, t + 1, args.bits,
                                                  svd)
        com_ms.append(evs[W].elapsed_time(evs[W + 1]))
    peak, peak_kind = measured_peaks()
    dec_avg_ms = sum(dec_ms) / len(dec_ms)
    achieved = dec_bytes / len(dec_ms) / (dec_avg_ms / 1e3) / 1e9
    traffic = profiled_traffic(profile_key("decode", wl, args))
    roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
            "frac": achieved / peak, "traffic": traffic,
            "kernel": f"{decode_kernel_name(wl, args)} (window positions 1..W)",
            "bytes_per_launch": dec_bytes / len(dec_ms), "avg_launch_us": dec_avg_ms * 1e3,
            "peak_source": f"{peak_kind} hbm_gbs (copy)"}
    extra = {}
    # average duration of the launch at each window position (us), then the commit
    pos_us = []
    for t in range(W):
        vals = [graphs[gi][2][t].elapsed_time(graphs[gi][2][t + 1]) for gi in used]
        pos_us.append(round(1e3 * sum(vals) / len(vals), 1))
    extra["launch_us_by_position"] = pos_us
    c_avg = sum(com_ms) / len(com_ms)
    c_bytes = nh * commit_launch_bytes(wl.d_k, wl.d_v, wl.n_comp, wl.gate, W, args.bits, svd)
    extra["commit"] = {"kernel": "commit_kernel", "avg_launch_us": c_avg * 1e3,
                       "bytes_per_launch": c_bytes, "achieved_gbs": c_bytes / (c_avg / 1e3) / 1e9,
                       "frac": c_bytes / (c_avg / 1e3) / 1e9 / peak,
                       "traffic": profiled_traffic(profile_key("commit", wl, args))}
    step_bytes = c_bytes + nh * sum(decode_launch_bytes(wl.d_k, wl.d_v, wl.n_comp, wl.gate, e, t + 1,
                                                        args.bits) for t in range(W))
    extra["step_gbs"] = step_bytes / (elapsed / args.steps / 1e3) / 1e9

    # end to end through the C ABI from pinned host buffers
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, wl, st, cfg, dev, world, group)

    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": elapsed_max / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8+f32",
        "data": "synthetic", "config": workload_config(wl, args),
        "roofline": roof, "gpu_launches": (W + 1) * args.steps,
        "detail": extra,
    }
    line["config"]["parallelism"] = f"dp{world} (independent sequence shards, no collective)"
    if e2e:
        line["e2e"] = e2e
    if sampler:
        line["clocks"] = sampler.summary(t0, t1, t_warm0)
    if rank == 0 and world == 1 and not args.no_cpu:
        n_seq = calibrated_sample(wl, args.cpu_seconds, args.bits)
        rate, dt, cores = oracle_window_rate(wl, n_seq, bits=args.bits)
        line["cpu_baseline"] = {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                                "sample": f"{n_seq} of {wl.batch} sequences x {wl.heads} heads, one "
                                          f"window of {W} decode tokens plus its commit ({dt:.1f} s)"}
    if lq.lq_device_errors() != 0:
        line["device_errors"] = True
    if world > 1:
        import torch.distributed as dist
        del graphs
        dist.destroy_process_group()
    return line if rank == 0 else None


def run_e2e(args, wl, st, cfg, dev, world, group):
    import torch

    import linear_attention_recurrent_int8_b200 as lq
    from linear_attention_recurrent_int8_b200 import synth
    W = wl.window
    rank, world_, _ = _dist()
    tok = shard_tokens(wl, rank, world_, 0, W, dev)
    # host layout [W][B, 1, H, ...]: each token's inputs are contiguous
    keys = ("q", "k", "v", "alpha", "beta")
    per_tok = {k: tok[k].transpose(0, 1).unsqueeze(2).contiguous() for k in keys}  # [W][B, 1, H, ...]
    # one pinned host buffer [W][bytes]: each token's q, k, v, alpha, beta
    # back to back (16-byte aligned segments), so that a chunk of tokens
    # moves with one copy; the device buffers are the same layout and the
    # tensors handed to the library are views into them
    seg, off = {}, 0
    for k in keys:
        nb = per_tok[k][0].numel() * per_tok[k].element_size()
        seg[k] = (off, nb)
        off += (nb + 15) // 16 * 16
    tok_bytes = off
    host = torch.empty((W, tok_bytes), dtype=torch.uint8, pin_memory=True)
    for k in keys:
        o0, nb = seg[k]
        host[:, o0:o0 + nb].copy_(per_tok[k].reshape(W, -1).cpu().view(torch.uint8))
    shapes = {k: (per_tok[k].dtype, tuple(per_tok[k].shape[1:])) for k in keys}
    dpack = [torch.empty((W, tok_bytes), dtype=torch.uint8, device=dev) for _ in range(2)]

    def views(buf, t):
        out = []
        for k in keys:
            o0, nb = seg[k]
            dt, shp = shapes[k]
            out.append(buf[t, o0:o0 + nb].view(dt).view(shp))
        return out

    dviews = [[views(dpack[j], t) for t in range(W)] for j in range(2)]
    # two device input sets (alternate windows) and two output sets, so that
    # window n + 1's uploads and window n's downloads overlap window n's
    # decode; tokens move in chunks of CH (one upload and one download each)
    CH = 4 if W % 4 == 0 else 1
    o_dev = [torch.empty((W, wl.batch, 1, wl.heads, wl.d_v), dtype=cfg.io_torch_dtype, device=dev)
             for _ in range(2)]
    o_host = torch.empty(o_dev[0].shape, dtype=o_dev[0].dtype, pin_memory=True)
    h2d = host.numel()  # the five input tensors of every token (plus alignment padding)
    d2h = o_host.numel() * o_host.element_size()
    comp = torch.cuda.current_stream(dev)
    up, down = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()
    # the last use of each input / output set by the compute stream
    set_free = [ev(), ev()]
    out_free = [ev(), ev()]
    for e in set_free + out_free:
        e.record(comp)
    step_no = [0]

    def one():
        n_ = step_no[0]
        step_no[0] += 1
        j = n_ % 2
        up.wait_event(set_free[j])
        ready = []
        for c0 in range(0, W, CH):
            with torch.cuda.stream(up):
                dpack[j][c0:c0 + CH].copy_(host[c0:c0 + CH], non_blocking=True)
                e = ev()
                e.record(up)
            ready.append(e)
        comp.wait_event(out_free[j])
        for c0 in range(0, W, CH):
            comp.wait_event(ready[c0 // CH])
            for t in range(c0, c0 + CH):
                lq.lq_decode_window(st, *dviews[j][t], 1, o_dev[j][t])
            done = ev()
            done.record(comp)
            down.wait_event(done)
            with torch.cuda.stream(down):
                o_host[c0:c0 + CH].copy_(o_dev[j][c0:c0 + CH], non_blocking=True)
        lq.lq_window_commit(st)
        set_free[j] = ev()
        set_free[j].record(comp)
        out_free[j] = ev()
        out_free[j].record(down)

    for _ in range(3):
        one()
    torch.cuda.synchronize()
    n = max(1, min(args.steps, args.e2e_steps))
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(comp)
    up.wait_event(a)
    down.wait_event(a)
    for _ in range(n):
        one()
    # the timed region ends when the last download has landed
    last = ev()
    last.record(down)
    comp.wait_event(last)
    b.record(comp)
    torch.cuda.synchronize()
    ms, rate = aggregate(a.elapsed_time(b), wl.batch * W * n, world, group)
    return {"value": rate, "unit": "tokens/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "steps": n, "copies": "chunks of 4 tokens on an upload and a download stream, overlapping the decode"}


DEFAULT_WORKLOAD = "gdn_256x32_d128_bf16"

# Secondary workloads of the default run: (name, mode, workload, steps, warmup,
# the equivalent command's flags).
SECONDARY = (
    ("kda_128x32_d128_bf16", "decode", "kda_128x32_d128_bf16", 40, 20,
     "--workload kda_128x32_d128_bf16 --steps 40 --warmup 20"),
    ("prefill_2x32_T65536", "prefill", DEFAULT_WORKLOAD, 3, 3, "--mode prefill --steps 3 --warmup 3"),
    ("ragged_gdn_256x32_d128_bf16", "ragged", DEFAULT_WORKLOAD, 20, 5, "--mode ragged --steps 20 --warmup 5"),
)


def run_secondary(args):
    """The default decode run also times, after the headline's timed region,
    short runs of the secondary workloads (KDA decode, the 65,536-token
    prefill, per-sequence window positions), each exactly as its own mode
    would (no CPU baseline, no e2e, no clock sampling), so that one run
    records them; a failure is reported in its entry, not raised."""
    import copy

    from linear_attention_recurrent_int8_b200 import synth
    out = {}
    for name, mode, workload, steps, warmup, flags in SECONDARY:
        a = copy.copy(args)
        a.mode, a.workload, a.steps, a.warmup = mode, workload, steps, warmup
        a.no_cpu = a.no_e2e = a.no_clocks = a.no_secondary = True
        try:
            wl = synth.WORKLOADS[workload]
            if mode == "prefill":
                l = run_prefill(a)
            elif mode == "ragged":
                l = run_ragged(a, wl)
            else:
                l = run_lq(a, wl)
            e = {k: l[k] for k in ("metric", "value", "unit", "ms_per_step", "steps", "warmup")}
            e["command"] = f"python bench.py {flags} --no-cpu --no-e2e --no-clocks"
            if "roofline" in l:
                e["roofline"] = {k: l["roofline"][k] for k in ("bound", "achieved", "peak", "unit", "frac",
                                                               "traffic", "avg_launch_us") if k in l["roofline"]}
            if "commit" in l.get("detail", {}):
                e["commit_avg_launch_us"] = l["detail"]["commit"]["avg_launch_us"]
            out[name] = e
        except Exception as exc:  # recorded, so that the headline line still prints
            out[name] = {"error": f"{type(exc).__name__}: {exc}"[:300]}
    return out


def run_prefill(args):
    """Prefill throughput: batch 2 x 32 heads, T tokens, bf16, a snapshot every
    1024 tokens (prompt tokens/s)."""
    import numpy as np
    import torch

    import linear_attention_recurrent_int8_b200 as lq
    from linear_attention_recurrent_int8_b200 import synth
    P = synth.PREFILL_WORKLOAD
    B, H, dk, dv, every, r = P["batch"], P["heads"], P["d_k"], P["d_v"], P["snapshot_every"], P["n_comp"]
    T = args.prefill_tokens or P["T"]
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    cfg = lq.Config(batch=B, heads=H, d_k=dk, d_v=dv, window=P["window"], n_comp=r,
                    gate=lq.LQ_GATE_SCALAR, io_dtype=lq.LQ_BF16, smoothing=1, auto_commit=1)
    st = lq.State(cfg, dev)
    lq.lq_state_init(st, None)
    q = torch.empty((B, T, H, dk), dtype=torch.bfloat16, device=dev)
    k, v = torch.empty_like(q), torch.empty((B, T, H, dv), dtype=torch.bfloat16, device=dev)
    alpha = torch.empty((B, T, H), dtype=torch.float32, device=dev)
    beta = torch.empty_like(alpha)
    for t0 in range(0, T, 4096):
        t1 = min(T, t0 + 4096)
        tok = synth.torch_tokens(P["seed"], B, H, t0, t1, dk, dv, "scalar", "bf16", dev)
        q[:, t0:t1], k[:, t0:t1], v[:, t0:t1] = tok["q"], tok["k"], tok["v"]
        alpha[:, t0:t1], beta[:, t0:t1] = tok["alpha"], tok["beta"]
    S = torch.zeros((B * H, dv, dk), dtype=torch.float32, device=dev)
    o = torch.empty((B, T, H, dv), dtype=torch.bfloat16, device=dev)
    snaps = [lq.Snapshot(cfg, dev) for _ in range(T // every)]

    ws = torch.empty(max(1, lq.lq_prefill_workspace_bytes(cfg)), dtype=torch.uint8, device=dev)

    def one():
        S.zero_()
        lq.lq_prefill_chunk(st, S, q, k, v, alpha, beta, T, every, snaps, o, workspace=ws)

    for _ in range(args.warmup):
        one()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.steps):
        one()
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / args.steps
    nbytes = B * T * H * (2 * (2 * dk + dv) + 8 + 2 * dv)
    # the chunked algorithm's products per 64-token chunk and head (C = 64):
    # [Q; K] K^T 2*2C*C*dk, X = [Q; K] S^T 2*2C*dk*dv, [PT; T] R 2*2C*C*dv,
    # K^T U^ 2*dk*C*dv; the tensor pipe runs each S / R / U product on three
    # BF16 parts (six for [PT; T] R), counted separately as executed work
    C = 64
    chunks = B * H * (T // C)
    f_alg = 2 * 2 * C * C * dk + 2 * 2 * C * dk * dv + 2 * 2 * C * C * dv + 2 * dk * C * dv
    f_exec = 2 * 2 * C * C * dk + 3 * 2 * 2 * C * dk * dv + 6 * 2 * 2 * C * C * dv + 3 * 2 * dk * C * dv
    tflops = chunks * f_alg / (ms / 1e3) / 1e12
    peak_t, peak_kind = measured_bf16_tflops(sustained=False)
    line = {"metric": "prefill tokens/s (state update + output, snapshots every 1024 tokens)",
            "value": B * T / (ms / 1e3), "unit": "tokens/s", "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": f"gdn prefill batch {B} x {H} heads, d={dk}, T={T}, bf16, "
                                   f"snapshot every {every} (r={r})"},
            # the chunked prefill on the tensor core: the whole call (chunk
            # preparation, the chunk scan, snapshot quantization) against the
            # dense BF16 peak, algorithmic FLOPs of the chunked algorithm
            "roofline": {"bound": "tensor", "achieved": tflops, "peak": peak_t, "unit": "TFLOP/s",
                         "frac": tflops / peak_t, "traffic": None, "peak_kind": peak_kind,
                         "kernel": "chunk_prep_kernel + chunk_scan_kernel + quantize_kernel (whole call)"},
            "detail": {"io_gbs": nbytes / (ms / 1e3) / 1e9, "snapshots": T // every,
                       "executed_tensor_tflops": chunks * f_exec / (ms / 1e3) / 1e12,
                       "us_per_chunk_per_head_chain": ms * 1e3 / (T // C),
                       "fp32_recurrence_equiv_tflops": B * T * H * 3 * 2 * dk * dv / (ms / 1e3) / 1e12}}
    if not args.no_cpu:
        rate, dt, cores, sample = oracle_prefill_rate(P, args.cpu_seconds)
        line["cpu_baseline"] = {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                                "sample": sample}
    return line


def oracle_prefill_rate(P, target_s: float):
    """The CPU oracle's prefill (FP64 recurrence, snapshots every 1024 tokens)
    on a bounded sample of heads and tokens; tokens/s counts sequence tokens
    (all heads of a sequence), scaled from the sampled heads."""
    import numpy as np
    cores = len(os.sched_getaffinity(0))
    os.environ.setdefault("OMP_NUM_THREADS", str(cores))
    import oracle
    from linear_attention_recurrent_int8_b200 import synth
    dk, dv, H, every, r = P["d_k"], P["d_v"], P["heads"], P["snapshot_every"], P["n_comp"]

    def run(nh, T):
        tok = synth.tokens(P["seed"], [0], list(range(nh)), 0, T, dk, dv, "scalar", "bf16")
        hm = lambda x: np.ascontiguousarray(np.swapaxes(np.asarray(x), 1, 2).reshape(
            (nh, T) + np.asarray(x).shape[3:]))
        d, kt, b = oracle.gdn_instance(hm(tok["alpha"]), hm(tok["beta"]), hm(tok["k"]))
        t0 = time.perf_counter()
        oracle.prefill(np.zeros((nh, dv, dk)), d, kt, b, hm(tok["v"]), hm(tok["q"]), every, r)
        return time.perf_counter() - t0

    dt1 = run(H, every)
    T = every * int(max(1, min(P["T"] // every, round(target_s / max(dt1, 1e-6)))))
    dt = run(H, T)
    return T / dt, dt, cores, f"one sequence (all {H} heads) x {T} tokens ({dt:.1f} s)"


def run_ragged(args, wl):
    """Continuous batching: every sequence decodes one token per step at its
    own window position (positions spread evenly over 0..W-1, so 1/W of the
    sequences commit at each step) through lq_decode_ragged."""
    import torch

    import linear_attention_recurrent_int8_b200 as lq
    from linear_attention_recurrent_int8_b200 import synth
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    W = wl.window
    cfg = lq.Config(batch=wl.batch, heads=wl.heads, d_k=wl.d_k, d_v=wl.d_v, window=W, n_comp=wl.n_comp,
                    gate=lq.LQ_GATE_DIAG if wl.gate == "diag" else lq.LQ_GATE_SCALAR,
                    io_dtype=lq.LQ_BF16 if wl.io == "bf16" else lq.LQ_F32, smoothing=int(wl.smoothing),
                    bits=args.bits, comp_rule=lq.LQ_COMP_SVD if args.comp_rule == "svd" else lq.LQ_COMP_ROWS)
    st = lq.State(cfg, dev)
    S0 = synth.torch_initial_state(wl.seed, range(wl.batch), range(wl.heads), wl.d_k, wl.d_v,
                                   wl.outlier_rows, wl.outlier_cols, wl.outlier_scale, dev)
    lq.lq_state_init(st, S0.reshape(wl.nh, wl.d_v, wl.d_k))
    del S0
    # staggered positions: the records below each position are those of a
    # synthetic earlier stretch of the sequence (any finite values do)
    seq_pos = (torch.arange(wl.batch, device=dev, dtype=torch.int32) % W).contiguous()
    st.buf_u.normal_(0.0, 0.1)
    st.buf_k.normal_(0.0, 0.05)
    st.buf_gate.copy_(-0.1 * torch.arange(1, W + 1, device=dev, dtype=torch.float32).reshape(
        (1, W) + (1,) * (st.buf_gate.dim() - 2)).expand_as(st.buf_gate))
    slots = []
    for sidx in range(4):
        tok = synth.torch_tokens(wl.seed, wl.batch, wl.heads, sidx, sidx + 1, wl.d_k, wl.d_v, wl.gate,
                                 wl.io, dev)
        slots.append([tok[k].contiguous() for k in ("q", "k", "v", "alpha", "beta")])
    o = torch.empty((wl.batch, 1, wl.heads, wl.d_v), dtype=cfg.io_torch_dtype, device=dev)
    lq.lq_decode_ragged(st, seq_pos, *slots[0], o)  # sets kernel attributes before capture
    torch.cuda.synchronize()
    # one graph per input slot (the positions live on the device, so replays advance them)
    graphs = []
    cs = torch.cuda.Stream(device=dev)
    for sl in slots:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cs):
            lq.lq_decode_ragged(st, seq_pos, *sl, o)
        graphs.append(g)
    for i in range(args.warmup):
        graphs[i % 4].replay()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    steps = args.steps * W
    a.record()
    for i in range(steps):
        graphs[i % 4].replay()
    b.record()
    torch.cuda.synchronize()
    assert lq.lq_device_errors() == 0
    ms = a.elapsed_time(b) / steps
    return {"metric": "decode tokens/s, per-sequence window positions", "value": wl.batch / (ms / 1e3),
            "unit": "tokens/s", "n_gpus": 1, "steps": steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int8+f32",
            "data": "synthetic", "config": dict(workload_config(wl, args),
                                                step="one token per sequence (decode, commit of the "
                                                     "sequences whose window filled, position update)")}


def run_init(args, wl):
    """State initialisation (I1): quantize an FP32 state of every (sequence,
    head) into the int8 snapshot (compensators, smoothing, codes)."""
    import torch

    import linear_attention_recurrent_int8_b200 as lq
    from linear_attention_recurrent_int8_b200 import synth
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    cfg = lq.Config(batch=wl.batch, heads=wl.heads, d_k=wl.d_k, d_v=wl.d_v, window=wl.window,
                    n_comp=wl.n_comp, gate=lq.LQ_GATE_DIAG if wl.gate == "diag" else lq.LQ_GATE_SCALAR,
                    io_dtype=lq.LQ_BF16 if wl.io == "bf16" else lq.LQ_F32,
                    smoothing=int(wl.smoothing), bits=args.bits)
    st = lq.State(cfg, dev)
    S0 = synth.torch_initial_state(wl.seed, range(wl.batch), range(wl.heads), wl.d_k, wl.d_v,
                                   wl.outlier_rows, wl.outlier_cols, wl.outlier_scale, dev)
    S0 = S0.reshape(wl.nh, wl.d_v, wl.d_k).contiguous()
    for _ in range(args.warmup):
        lq.lq_state_init(st, S0)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.steps):
        lq.lq_state_init(st, S0)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / args.steps
    nbytes = wl.nh * (4 * wl.d_v * wl.d_k + snapshot_bytes(wl.d_k, wl.d_v, wl.n_comp, args.bits))
    peak, kind = measured_peaks()
    gbs = nbytes / (ms / 1e3) / 1e9
    return {"metric": "state init: heads quantized per second", "value": wl.nh / (ms / 1e3),
            "unit": "heads/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "data": "synthetic", "config": workload_config(wl, args),
            "roofline": {"bound": "hbm", "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
                         "traffic": None, "kernel": "quantize_kernel",
                         "bytes_per_launch": nbytes, "peak_source": f"{kind} hbm_gbs (copy)"}}


def run_fp32step(args, wl):
    """FP32 per-step comparator: the whole FP32 state read and written every
    token (one launch per token, all heads)."""
    import torch

    import linear_attention_recurrent_int8_b200 as lq
    from linear_attention_recurrent_int8_b200 import synth
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    cfg = lq.Config(batch=wl.batch, heads=wl.heads, d_k=wl.d_k, d_v=wl.d_v,
                    gate=lq.LQ_GATE_DIAG if wl.gate == "diag" else lq.LQ_GATE_SCALAR,
                    io_dtype=lq.LQ_BF16 if wl.io == "bf16" else lq.LQ_F32)
    S = torch.randn((wl.nh, wl.d_v, wl.d_k), dtype=torch.float32, device=dev)
    toks = []
    for t in range(8):
        tok = synth.torch_tokens(wl.seed, wl.batch, wl.heads, t, t + 1, wl.d_k, wl.d_v, wl.gate,
                                 wl.io, dev)
        toks.append([tok[k2] for k2 in ("q", "k", "v", "alpha", "beta")])
    o = torch.empty((wl.batch, 1, wl.heads, wl.d_v), dtype=cfg.io_torch_dtype, device=dev)
    for i in range(args.warmup):
        lq.lq_fp32_step(cfg, S, *toks[i % 8], 1, o)
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for i in range(args.steps):
        lq.lq_fp32_step(cfg, S, *toks[i % 8], 1, o)
    b.record()
    torch.cuda.synchronize()
    ms = a.elapsed_time(b) / args.steps
    e = 2 if wl.io == "bf16" else 4
    nbytes = wl.nh * (8 * wl.d_v * wl.d_k + e * (2 * wl.d_k + 2 * wl.d_v) + 8)
    peak, kind = measured_peaks()
    return {"metric": "FP32 per-step comparator: decode tokens/s", "value": wl.batch / (ms / 1e3),
            "unit": "tokens/s", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "f32", "data": "synthetic", "config": workload_config(wl, args),
            "roofline": {"bound": "hbm", "achieved": nbytes / (ms / 1e3) / 1e9, "peak": peak,
                         "unit": "GB/s", "frac": nbytes / (ms / 1e3) / 1e9 / peak, "traffic": None}}


def run_mse(args, wl):
    """State MSE against the unquantized FP32 state (the FP32 per-step chain),
    per-window (W, r, smoothing as configured) versus per-token (W = 1,
    r = 0), over the same inputs, for a subset of sequences."""
    import dataclasses

    import torch

    import linear_attention_recurrent_int8_b200 as lq
    from linear_attention_recurrent_int8_b200 import synth
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    wl = dataclasses.replace(wl, batch=min(wl.batch, args.mse_batch))
    steps = args.mse_steps
    S0 = synth.torch_initial_state(wl.seed, range(wl.batch), range(wl.heads), wl.d_k, wl.d_v,
                                   wl.outlier_rows, wl.outlier_cols, wl.outlier_scale, dev)
    S0 = S0.reshape(wl.nh, wl.d_v, wl.d_k).contiguous()
    sm0 = int(wl.smoothing)
    variants = {"per_window": (wl.window, wl.n_comp, sm0, 8),
                "per_window_svd": (wl.window, wl.n_comp, sm0, 8, lq.LQ_COMP_SVD),
                "per_token": (1, 0, sm0, 8), "per_token_plain": (1, 0, 0, 8),
                "per_window_6bit": (wl.window, wl.n_comp, sm0, 6), "per_token_6bit": (1, 0, sm0, 6),
                "per_window_4bit": (wl.window, wl.n_comp, sm0, 4), "per_token_4bit": (1, 0, sm0, 4),
                "per_window_bf16": (wl.window, 0, 0, 16), "per_token_bf16": (1, 0, 0, 16)}
    states, cfgs = {}, {}
    for name, (W, r, sm, bits, *rule) in variants.items():
        cfg = lq.Config(batch=wl.batch, heads=wl.heads, d_k=wl.d_k, d_v=wl.d_v, window=W, n_comp=r,
                        gate=lq.LQ_GATE_DIAG if wl.gate == "diag" else lq.LQ_GATE_SCALAR,
                        io_dtype=lq.LQ_BF16 if wl.io == "bf16" else lq.LQ_F32, smoothing=sm,
                        auto_commit=1, bits=bits, comp_rule=rule[0] if rule else lq.LQ_COMP_ROWS)
        st = lq.State(cfg, dev)
        lq.lq_state_init(st, S0)
        states[name], cfgs[name] = st, cfg
    S = S0.clone()
    fcfg = cfgs["per_window"]
    o = torch.empty((wl.batch, 1, wl.heads, wl.d_v), dtype=fcfg.io_torch_dtype, device=dev)

    def codes_float(st):
        c = st.snap.t["codes"]
        if st.cfg.bits != 4:
            return c.float()
        # two per byte: in each 8-channel group, byte b holds channel b (low
        # nibble) and channel 4 + b (high nibble), two's complement
        p = c.to(torch.int16).reshape(c.shape[0], c.shape[1], -1, 4)
        nib = torch.stack([p & 0xF, (p >> 4) & 0xF], dim=-2)
        nib = torch.where(nib >= 8, nib - 16, nib)
        return nib.reshape(c.shape[0], c.shape[1], -1).float()

    def dequant(st):
        t = st.snap.t
        Sh = (t["row_scale"][:, :, None] * codes_float(st) * t["col_smooth"][:, None, :])
        if "comp_u" in t:  # SVD rule: rank-one compensators
            Sh += torch.einsum("hcv,hck->hvk", t["comp_u"], t["comp_val"])
        elif t["comp_row"].numel():
            Sh.scatter_add_(1, t["comp_row"].long()[:, :, None].expand(-1, -1, wl.d_k), t["comp_val"])
        return Sh

    curve = {n: [] for n in variants}
    W = wl.window
    for t in range(steps):
        tok = synth.torch_tokens(wl.seed, wl.batch, wl.heads, t, t + 1, wl.d_k, wl.d_v, wl.gate, wl.io,
                                 dev)
        args_t = [tok[k2] for k2 in ("q", "k", "v", "alpha", "beta")]
        lq.lq_fp32_step(fcfg, S, *args_t, 1, o)
        for name, st in states.items():
            lq.lq_decode_window(st, *args_t, 1, o)
        if (t + 1) % W == 0:
            ref_ms = float((S * S).mean())
            for name, st in states.items():
                curve[name].append(float(((dequant(st) - S) ** 2).mean()) / ref_ms)
    out = {n: {"final_rel_mse": c[-1], "mean_rel_mse": sum(c) / len(c)} for n, c in curve.items()}
    return {"report": "state MSE relative to the mean square of the FP32 state, at window ends",
            "workload": wl.name, "batch": wl.batch, "heads": wl.heads, "steps": steps,
            "window": W, "n_comp": wl.n_comp, "results": out,
            "variants": {n: {"window": v[0], "n_comp": v[1], "smoothing": bool(v[2]), "bits": v[3],
                             "comp_rule": "svd" if v[4:] == (lq.LQ_COMP_SVD,) else "rows"}
                         for n, v in variants.items()}}


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["lq", "reference"], default="lq")
    ap.add_argument("--mode", choices=["decode", "prefill", "fp32step", "mse", "init", "ragged"],
                    default="decode",
                    help="decode (default, the headline) or a comparator / report")
    ap.add_argument("--prefill-tokens", type=int, default=0)
    ap.add_argument("--mse-batch", type=int, default=16)
    ap.add_argument("--mse-steps", type=int, default=1024)
    ap.add_argument("--workload", default="gdn_256x32_d128_bf16")
    ap.add_argument("--window", type=int, default=None, help="override W (comparators / sweep)")
    ap.add_argument("--n-comp", type=int, default=None, help="override r")
    ap.add_argument("--no-smoothing", action="store_true")
    ap.add_argument("--delta", type=int, choices=[0, 1], default=None,
                    help="0: the b = 0 rows of equation 1 (linear attention / Mamba2 / GLA)")
    ap.add_argument("--comp-rule", choices=["rows", "svd"], default="rows",
                    help="compensator rule: top-r rows (default) or top-r singular triplets")
    ap.add_argument("--bits", type=int, choices=[8, 6, 4, 16], default=8,
                    help="code width of the state (8; 6 and 4 are the narrow variants; 16 = BF16)")
    ap.add_argument("--slots", type=int, default=8, help="distinct input windows (graphs)")
    ap.add_argument("--no-graph", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--no-clocks", action="store_true")
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--ref-seconds", type=float, default=5.0)
    ap.add_argument("--no-secondary", action="store_true",
                    help="skip the secondary workloads that the default decode run also times")
    args = ap.parse_args(argv)
    args.warmup = max(3, args.warmup)

    import dataclasses
    from linear_attention_recurrent_int8_b200 import synth
    wl = synth.WORKLOADS[args.workload]
    over = {}
    if args.window is not None:
        over["window"] = args.window
    if args.n_comp is not None:
        over["n_comp"] = args.n_comp
    if args.no_smoothing:
        over["smoothing"] = False
    if args.delta is not None:
        over["delta"] = args.delta
    if over:
        wl = dataclasses.replace(wl, **over)

    if args.impl == "reference":
        line = run_reference(args, wl)
    elif args.mode == "prefill":
        line = run_prefill(args)
    elif args.mode == "fp32step":
        line = run_fp32step(args, wl)
    elif args.mode == "mse":
        line = run_mse(args, wl)
    elif args.mode == "init":
        line = run_init(args, wl)
    elif args.mode == "ragged":
        line = run_ragged(args, wl)
    else:
        line = run_lq(args, wl)
        if line is not None and not over and _dist()[1] == 1 and not args.no_secondary and \
                args.workload == DEFAULT_WORKLOAD and args.bits == 8 and args.comp_rule == "rows":
            line["detail"]["secondary"] = run_secondary(args)
    if line is not None:
        print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
