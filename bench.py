"""Benchmark of the KDA hot path on B200: prefill tokens/s and decode-step HBM GB/s.

One timed "step" is one chunkwise prefill of the single-sequence workload
(B=1, H=32, T=8192, d_k=d_v=128, bf16 q/k/v, fp32 gates and state; inputs
~404 MB > L2, so no flush is needed). Further lines on the same JSON record:
  * varlen_16 (16 packed sequences, lengths U[512, 8192]), prefill_1m
    (T = 1,048,576) and tiny_f32 (H=2, T=256, d=64, fp32; L2 flushed before
    each timed call), each with tokens/s and its HBM roofline;
  * gdn (one gate per token and head), output_gate (RMSNorm + sigmoid gate
    fused), short_conv (the convolution before the recurrence), backward;
  * decode: 256 sequences x 32 heads, 512 MiB fp32 state in place (> L2),
    1000 consecutive steps on 1000 pregenerated inputs, as plain launches and
    replayed from a CUDA graph; decode_conv: the same with the convolution
    fused into the loads.
Everything runs in libkda's CUDA kernels; inputs are seeded synthetic tensors
(``kda_inputs``).

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kda|reference]
Multi-GPU: launched with torchrun, one rank per GPU; every rank runs its own
independent batch (weak scaling, no data-path collective).

``--impl reference`` times the fp64 CPU oracle (the only other implementation
of this path; it is test infrastructure) on the host cores, on a bounded
sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import kda_inputs as KI  # noqa: E402

METRIC = "KDA prefill tokens/s at H=32,d=128; decode-step HBM GB/s vs B200 peak"
PREFILL = "prefill_8k"
T8K, H, D = 8192, 32, 128
DEC_N = 256
BACKWARD_LAUNCHES = 7  # bw_offsets, bw_prep, bw_fwd, bw_bwd, bw_rowstate, bw_grads, bw_norm
# Algorithmic HBM bytes (inputs read once, outputs written once):
#   prefill per token (all 32 heads): q,k,v bf16 3*32*128*2 + log_alpha 32*128*4 + beta 32*4
#   + o 32*128*2 = 49,280 B; plus S0 read and S_T written (2 MiB each at H=32).
PREFILL_BYTES_PER_TOKEN = 3 * H * D * 2 + H * D * 4 + H * 4 + H * D * 2
PREFILL_STATE_BYTES = 2 * H * D * D * 4
# the Gated DeltaNet form: one fp32 gate per (token, head) instead of d_k
GDN_BYTES_PER_TOKEN = 3 * H * D * 2 + H * 4 + H * 4 + H * D * 2
# decode per step: state read + write, q,k,v bf16, log_alpha fp32, beta fp32, o bf16
DECODE_BYTES = DEC_N * H * (2 * D * D * 4 + 3 * D * 2 + D * 4 + 4 + D * 2)
CONV_W = 4  # short-convolution window of the conv lines (the pages leave it open)
# backward of prefill_8k: q, k, v, do (bf16), log_alpha, beta read; dq, dk, dv, dlog_alpha,
# dbeta (fp32) written; S0 and dS_T read, dS0 written
BACKWARD_BYTES = T8K * H * (4 * D * 2 + D * 4 + 4 + 4 * D * 4 + 4) + 3 * H * D * D * 4
# one short convolution over a [T8K, H*D] bf16 projection: x read, y written, taps,
# the state read and written
CONV_BYTES = 2 * T8K * H * D * 2 + H * D * CONV_W * 4 + 2 * (CONV_W - 1) * H * D * 2
# decode with the convolution fused into the q, k, v loads: + three states read and written, taps
DECODE_CONV_BYTES = DECODE_BYTES + 3 * (2 * DEC_N * (CONV_W - 1) * H * D * 2 + H * D * CONV_W * 4)


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def bf16_peak():
    """Dense bf16 tensor peak in TFLOP/s: the measured burst figure, else the fallback."""
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return 1590.0, "fallback"


# Prefill FLOPs per token at H heads: the pages' count (6 d^2 + 3 C d + C^2 per head-token)
# and this path's own count (6 d^2 + 10 C d per head-token: every Gram, solve-application
# and scan product at 2 flop per multiply-add).
FLOPS_PAGES_PER_TOKEN = H * (6 * D * D + 3 * 64 * D + 64 * 64)
FLOPS_OWN_PER_TOKEN = H * (6 * D * D + 10 * 64 * D)


class Clocks:
    """Sample SM clocks and throttle reasons while the timed region runs."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.Q,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        self.out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        rows = []
        for line in (self.out or "").splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                rows.append((float(f[1]), float(f[2]), f[5:9]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for _, _, r in rows for i, x in enumerate(r) if x == "Active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() and args.impl == "kda" else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x, world, device):
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# -------------------------------------------------------------- oracle ----

def oracle_sample(seconds_target=10.0, device="cpu"):
    """Time the fp64 oracle on a bounded sample of the prefill workload (some heads,
    all 8192 tokens). Returns (tokens/s at H=32, cores, description)."""
    import oracle
    cores = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else os.cpu_count()
    heads = max(1, min(H, cores))
    inp = KI.prefill_workload(PREFILL, "cpu", heads=heads)
    f = lambda x: x.to(torch.float64).numpy()
    args = [f(inp[n]) for n in ("q", "k", "v", "log_alpha", "beta")]
    S0 = f(inp["S0"])
    reps, elapsed = 0, 0.0
    while reps == 0 or (elapsed < seconds_target and reps < 50):
        t0 = time.perf_counter()
        oracle.recurrent(*args, S0, threads=cores)
        elapsed += time.perf_counter() - t0
        reps += 1
    tok = reps * T8K * heads / H  # tokens-equivalent of a 32-head token
    desc = "%d of %d heads x %d tokens, %d repetitions, fp64 recurrence, %d threads" % (
        heads, H, T8K, reps, cores)
    return tok / elapsed, cores, desc


def run_reference(args, world, rank):
    """Each step is one bounded oracle sample (``cores`` heads x 8192 tokens)."""
    if rank != 0:
        return
    for _ in range(args.warmup):
        oracle_sample(seconds_target=0.0)
    rates = []
    for _ in range(args.steps):
        r, cores, desc = oracle_sample(seconds_target=0.0)
        rates.append(r)
    v = len(rates) / sum(1.0 / r for r in rates)  # total tokens / total time
    desc = "%d steps, each: %s" % (args.steps, desc)
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": "tokens/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * T8K / v, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "prefill_8k: B=1 H=32 T=8192 d_k=d_v=128 (oracle sample)"},
            "cpu_baseline": {"value": v, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- kda ----

PREFILL_SOURCES = ["gated_delta_rule_125_b200/csrc/kda_prefill_tc.cu", "gated_delta_rule_125_b200/csrc/kda_tc.cuh",
                   "gated_delta_rule_125_b200/csrc/kda_internal.cuh"]
DECODE_SOURCES = ["gated_delta_rule_125_b200/csrc/kda_decode.cu", "gated_delta_rule_125_b200/csrc/kda_internal.cuh"]


def profiled_traffic(profile, sources):
    """DRAM bytes (read + write) per launch from a committed ncu summary under
    profiles/, or None when the summary is missing or the kernel's sources have
    changed since it was taken (the summary records their sha256)."""
    root = os.path.dirname(os.path.abspath(__file__))
    try:
        txt = open(os.path.join(root, "profiles", profile)).read()
        blob = b"".join(open(os.path.join(root, f), "rb").read() for f in sources)
    except OSError:
        return None
    m = re.search(r"traffic_bytes_per_launch:\s*(\d+)", txt)
    h = re.search(r"source_sha256:\s*([0-9a-f]{64})", txt)
    if not m or not h or hashlib.sha256(blob).hexdigest() != h.group(1):
        return None
    return int(m.group(1))


def timed(fn, steps, warmup, world, dev, stream):
    """CUDA-event time per call of ``fn`` over ``steps`` calls after ``warmup`` untimed ones,
    bracketed by a barrier and a device synchronisation. Returns (this rank's ms, max over ranks)."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    barrier(world)
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    for _ in range(steps):
        fn()
    ev1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ms = ev0.elapsed_time(ev1) / steps
    return ms, max_over_ranks(ms, world, dev)


def timed_flushed(fn, steps, warmup, world, dev, stream):
    """As ``timed`` for inputs that fit in L2: each call is timed alone, after a write of a
    buffer larger than L2 (the flush is outside the events). Returns (ms, max over ranks)."""
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    barrier(world)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for e0, e1 in evs:
        flush.fill_(1)
        e0.record(stream)
        fn()
        e1.record(stream)
    torch.cuda.synchronize()
    barrier(world)
    ms = sum(e0.elapsed_time(e1) for e0, e1 in evs) / steps
    del flush
    return ms, max_over_ranks(ms, world, dev)


def prefill_bytes(tokens, n_seqs, heads, d, io_bytes, gate_per_channel=True, reads_s0=True):
    """Algorithmic HBM bytes of one prefill: q, k, v read and o written in the io dtype,
    log_alpha and beta read (fp32), S_T written and S0 read (when given), fp32."""
    per_token = heads * (3 * d * io_bytes + (d if gate_per_channel else 1) * 4 + 4 + d * io_bytes)
    state = n_seqs * heads * d * d * 4
    return tokens * per_token + state * (2 if reads_s0 else 1)


def prefill_entry(tokens, ms_local, ms_max, world, nbytes, hbm, peak_src, workload, kernel,
                  traffic=None, flops=True, extra=None):
    """One prefill line: tokens/s over all ranks, the HBM roofline of one pass and the flop view."""
    achieved = nbytes / (ms_local * 1e-3) / 1e9
    e = {"value": world * tokens / (ms_max * 1e-3), "unit": "tokens/s", "ms_per_step": ms_max,
         "workload": workload,
         "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                      "frac": achieved / hbm, "traffic": traffic, "kernel": kernel,
                      "algorithmic_bytes": nbytes, "peak_source": peak_src}}
    if flops:
        pk, pk_src = bf16_peak()
        tp = FLOPS_PAGES_PER_TOKEN * tokens / (ms_local * 1e-3) / 1e12
        to = FLOPS_OWN_PER_TOKEN * tokens / (ms_local * 1e-3) / 1e12
        e["tensor"] = {"tflops_pages_count": tp, "tflops_own_count": to, "peak_tflops": pk,
                       "peak_source": pk_src, "frac_pages_count": tp / pk, "frac_own_count": to / pk}
    if extra:
        e.update(extra)
    return e


def run_kda(args, world, rank, local):
    import gated_delta_rule_125_b200 as kda
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream(dev)
    hbm, peak_src = peaks()
    launches = 0  # this library's kernel launches inside timed regions

    # ---- prefill workload, resident in HBM
    inp = KI.prefill_workload(PREFILL, dev, seed=rank)
    q, k, v, la, beta, S0, cu = (inp[n] for n in ("q", "k", "v", "log_alpha", "beta", "S0", "cu_seqlens"))
    o = torch.empty_like(v)
    S_T = torch.empty_like(S0)
    wsb = kda.kda_prefill_workspace_size(1, T8K, T8K, H, D, D, torch.bfloat16)
    ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
    launches_prefill = kda.kda_prefill_launches(1, T8K, T8K, H, D, D, torch.bfloat16, wsb)

    def prefill():
        kda.kda_prefill(q, k, v, la, beta, S0, cu, max_seqlen=T8K, o=o, S_T=S_T, workspace=ws)

    with Clocks(local) as clk:
        ms, ms_max = timed(prefill, args.steps, args.warmup, world, dev, stream)
    launches += args.steps * launches_prefill
    tokens_per_s = world * T8K / (ms_max * 1e-3)
    bytes_pass = T8K * PREFILL_BYTES_PER_TOKEN + PREFILL_STATE_BYTES
    achieved = bytes_pass / (ms * 1e-3) / 1e9

    # ---- the Gated DeltaNet form of the same workload: one gate per (token, head)
    gdn = KI.prefill_workload("gdn_8k", dev, seed=rank)

    def prefill_gdn():
        kda.kda_prefill(gdn["q"], gdn["k"], gdn["v"], gdn["log_alpha"], gdn["beta"], gdn["S0"], cu,
                        max_seqlen=T8K, o=o, S_T=S_T, workspace=ws)

    gdn_ms, gdn_ms_max = timed(prefill_gdn, args.steps, args.warmup, world, dev, stream)
    launches += args.steps * launches_prefill
    gdn_bytes = T8K * GDN_BYTES_PER_TOKEN + PREFILL_STATE_BYTES
    del gdn

    # ---- the same workload with the layer's output step fused (RMSNorm + sigmoid gate)
    g_gen = torch.Generator(device=dev)
    g_gen.manual_seed(1000 + rank)
    og = (torch.randn((T8K, H, D), generator=g_gen, device=dev).to(torch.bfloat16),
          1.0 + 0.1 * torch.randn((D,), generator=g_gen, device=dev), 1e-6)

    def prefill_gated():
        kda.kda_prefill(q, k, v, la, beta, S0, cu, max_seqlen=T8K, o=o, S_T=S_T, workspace=ws,
                        out_gate=og)

    og_ms, og_ms_max = timed(prefill_gated, args.steps, args.warmup, world, dev, stream)
    launches += args.steps * launches_prefill
    og_bytes = T8K * (PREFILL_BYTES_PER_TOKEN + H * D * 2) + PREFILL_STATE_BYTES
    del og

    # ---- the layer's step before the recurrence: short convolution + Swish on the
    #      q, k, v projections (W = 4, states written for a following decode), alone
    #      and followed by the prefill
    conv_in = [KI.conv_inputs(T8K, H * D, CONV_W, 1, torch.bfloat16, dev, seed=rank, tensor=i) for i in range(3)]
    conv_out = [torch.empty_like(c[0]) for c in conv_in]
    conv_st = [torch.empty_like(c[2]) for c in conv_in]
    conv_launches = kda.load_library().kda_short_conv_launches(CONV_W, 1, T8K)

    def convs():
        for (x, w, st), y, so in zip(conv_in, conv_out, conv_st):
            kda.kda_short_conv_swish(x, w, state_in=st, state_out=so, y=y)

    def conv_prefill():
        convs()
        kda.kda_prefill(conv_out[0].view(T8K, H, D), conv_out[1].view(T8K, H, D), conv_out[2].view(T8K, H, D),
                        la, beta, S0, cu, max_seqlen=T8K, o=o, S_T=S_T, workspace=ws)

    # the same, with the convolution inside the prefill's loads (kda_prefill_conv)
    fused_conv = tuple((w, st, so) for (x, w, st), so in zip(conv_in, conv_st))

    def prefill_conv():
        kda.kda_prefill(conv_in[0][0].view(T8K, H, D), conv_in[1][0].view(T8K, H, D), conv_in[2][0].view(T8K, H, D),
                        la, beta, S0, cu, max_seqlen=T8K, o=o, S_T=S_T, workspace=ws, conv=fused_conv)

    # Three short convolutions (two launches each, ~30 us of GPU time): the host issues them
    # more slowly than the GPU runs them, so the convolution line replays them from a CUDA
    # graph (captured once).
    conv_graph = None
    try:
        side = torch.cuda.Stream(dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            convs()
        torch.cuda.current_stream(dev).wait_stream(side)
        torch.cuda.synchronize()
        conv_graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(conv_graph):
            convs()
        torch.cuda.synchronize()
    except RuntimeError:
        conv_graph = None
    conv_ms = {}
    for name, fn in (("conv", conv_graph.replay if conv_graph is not None else convs), ("conv_prefill", conv_prefill),
                     ("prefill_conv", prefill_conv)):
        conv_ms[name] = timed(fn, args.steps, args.warmup, world, dev, stream)
    launches += args.steps * (3 * conv_launches) + args.steps * (3 * conv_launches + launches_prefill)
    launches += args.steps * (launches_prefill + 3)  # the fused form: prefill launches + three conv-state kernels
    conv_gbs = 3 * CONV_BYTES / (conv_ms["conv"][0] * 1e-3) / 1e9
    conv_graph_used = conv_graph is not None
    del conv_graph, conv_in, conv_out, conv_st

    # ---- end to end through the C ABI: pinned host inputs -> device -> host
    h_in = {n: inp[n].cpu().pin_memory() for n in ("q", "k", "v", "log_alpha", "beta", "S0")}
    h_o = torch.empty(o.shape, dtype=o.dtype).pin_memory()
    h_S = torch.empty(S_T.shape, dtype=S_T.dtype).pin_memory()
    d_in = {n: torch.empty_like(inp[n]) for n in h_in}
    h2d = sum(t.numel() * t.element_size() for t in h_in.values())
    d2h = h_o.numel() * h_o.element_size() + h_S.numel() * h_S.element_size()

    def e2e_step():
        for n in h_in:
            d_in[n].copy_(h_in[n], non_blocking=True)
        kda.kda_prefill(d_in["q"], d_in["k"], d_in["v"], d_in["log_alpha"], d_in["beta"],
                        d_in["S0"], cu, max_seqlen=T8K, o=o, S_T=S_T, workspace=ws)
        h_o.copy_(o, non_blocking=True)
        h_S.copy_(S_T, non_blocking=True)

    _, e2e_ms = timed(e2e_step, args.steps, args.warmup, world, dev, stream)
    launches += args.steps * launches_prefill
    del d_in, h_in, inp, q, k, v, la, beta, S0, o, S_T

    # ---- the other prefill workloads: packed variable length, 1M tokens, tiny fp32
    others = {}
    for name, steps in (("varlen_16", args.steps), ("prefill_1m", 3), ("tiny_f32", args.steps)):
        w = KI.WORKLOADS[name]
        lens = KI.workload_lengths(name, 0)  # the same sizes on every rank, own data
        wi = KI.prefill_workload(name, dev, seed=rank, lengths=lens)
        Tn, Nn, dn = sum(lens), len(lens), w["d"]
        dt = KI.torch_dtype(w["dtype"])
        s0 = wi["S0"] if w["s0_std"] else None  # S0 = 0: not passed (nothing to read)
        wo = torch.empty_like(wi["v"])
        wS = torch.empty((Nn, w["H"], dn, dn), dtype=torch.float32, device=dev)
        nb = kda.kda_prefill_workspace_size(Nn, Tn, max(lens), w["H"], dn, dn, dt)
        wws = torch.empty(nb, dtype=torch.uint8, device=dev)
        wl = kda.kda_prefill_launches(Nn, Tn, max(lens), w["H"], dn, dn, dt, nb)

        def fn(wi=wi, s0=s0, wo=wo, wS=wS, wws=wws, lens=lens):
            kda.kda_prefill(wi["q"], wi["k"], wi["v"], wi["log_alpha"], wi["beta"], s0, wi["cu_seqlens"],
                            max_seqlen=max(lens), o=wo, S_T=wS, workspace=wws)

        io = 2 if dt == torch.bfloat16 else 4
        nbytes = prefill_bytes(Tn, Nn, w["H"], dn, io, reads_s0=s0 is not None)
        in_l2 = nbytes < (64 << 20)
        t_local, t_max = (timed_flushed if in_l2 else timed)(fn, steps, args.warmup, world, dev, stream)
        launches += steps * wl
        others[name] = prefill_entry(
            Tn, t_local, t_max, world, nbytes, hbm, peak_src,
            "%s: %d sequence(s), %d tokens, H=%d, d_k=d_v=%d, %s q/k/v, fp32 gates/state, chunk 64%s" % (
                name, Nn, Tn, w["H"], dn, w["dtype"], ", S0=0" if s0 is None else ""),
            "kda_prefill (%s path, %d launches)" % ("tensor-core" if wl == 2 else "fp32 CUDA-core", wl),
            flops=(dt == torch.bfloat16),
            extra={"steps": steps, "l2": ("%d KB of inputs: L2 flushed before each timed call" % (nbytes >> 10))
                   if in_l2 else "inputs %.1f GB > L2 (no flush)" % (nbytes / 1e9)})
        del wi, wo, wS, wws, fn

    # ---- decode: 256 x 32 heads, state 512 MiB in place, 1000 consecutive steps on
    #      1000 pregenerated inputs; plain launches and the 1000 launches replayed from a
    #      CUDA graph
    dsteps = args.decode_steps
    dec = KI.decode_workload(DEC_N, H, D, dsteps, torch.bfloat16, dev, seed=rank)
    S = dec["S0"].clone()
    od = torch.empty((dsteps, DEC_N, H, D), dtype=torch.bfloat16, device=dev)

    def decode_all(conv=None):
        for t in range(dsteps):
            kda.kda_decode_step(dec["q"][t], dec["k"][t], dec["v"][t], dec["log_alpha"][t],
                                dec["beta"][t], S, o=od[t], conv=conv)

    dec_ms, dec_ms_max = timed(decode_all, 1, 1, world, dev, stream)
    launches += dsteps
    dec_us, dec_us_max = 1e3 * dec_ms / dsteps, 1e3 * dec_ms_max / dsteps
    dec_gbs = DECODE_BYTES / (dec_us * 1e-6) / 1e9
    dec_graph = {}
    try:
        side = torch.cuda.Stream(dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        with torch.cuda.stream(side):
            decode_all()
        torch.cuda.current_stream(dev).wait_stream(side)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            decode_all()
        gms, gms_max = timed(g.replay, 1, 1, world, dev, stream)
        launches += dsteps
        dec_graph = {"us_per_step": 1e3 * gms_max / dsteps,
                     "value": DECODE_BYTES / (1e-3 * gms_max / dsteps) / 1e9,
                     "frac": DECODE_BYTES / (1e-3 * gms / dsteps) / 1e9 / hbm}
        del g
    except RuntimeError as exc:
        dec_graph = {"error": str(exc)[:200]}

    # ---- decode with the short convolution fused into the q, k, v loads (states in place)
    dconv = []
    for i in range(3):
        _, w_, st_ = KI.conv_inputs(1, H * D, CONV_W, DEC_N, torch.bfloat16, dev, seed=rank, tensor=i)
        dconv.append((w_, st_, st_))
    dc_ms, dc_ms_max = timed(lambda: decode_all(tuple(dconv)), 1, 1, world, dev, stream)
    launches += dsteps
    dconv_us, dconv_us_max = 1e3 * dc_ms / dsteps, 1e3 * dc_ms_max / dsteps
    dconv_gbs = DECODE_CONV_BYTES / (dconv_us * 1e-6) / 1e9
    del dec, dconv, od, S

    # ---- backward of the prefill (training): gradients of prefill_8k given dL/do, dL/dS_T
    #      (an error of this line is reported in it, not fatal to the others)
    bw = {}
    bw_steps = 3
    try:
        inp = KI.prefill_workload(PREFILL, dev, seed=rank)
        g_bw = torch.Generator(device=dev)
        g_bw.manual_seed(2000 + rank)
        d_o = torch.randn((T8K, H, D), generator=g_bw, device=dev).to(torch.bfloat16)
        d_ST = torch.randn((1, H, D, D), generator=g_bw, device=dev)
        bw_wsb = kda.load_library().kda_backward_workspace_size(1, T8K, T8K, H, D, D, 1, 64, 0)
        bw_ws = torch.empty(bw_wsb, dtype=torch.uint8, device=dev)

        def backward():
            kda.kda_backward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], d_o, d_ST,
                             inp["S0"], inp["cu_seqlens"], max_seqlen=T8K, workspace=bw_ws)

        bw_ms, bw["ms"] = timed(backward, bw_steps, args.warmup, world, dev, stream)
        launches += bw_steps * BACKWARD_LAUNCHES
        bw["gbs"] = BACKWARD_BYTES / (bw_ms * 1e-3) / 1e9
        del bw_ws, d_o, d_ST, inp
    except RuntimeError as exc:  # KDAError included
        bw = {"error": str(exc)[:200]}

    line = {
        "metric": METRIC, "value": tokens_per_s, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": "prefill_8k: B=1 H=32 T=8192 d_k=d_v=128 bf16 q/k/v, fp32 "
                               "gates/state, chunk 64, S0~N(0,0.01^2), per rank",
                   "global_batch": world, "seq_len": T8K,
                   "l2": "inputs 404 MB > 126 MB L2 (no flush)",
                   "parallelism": "independent batch per GPU" if world > 1 else "1 GPU"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                     "frac": achieved / hbm,
                     "traffic": profiled_traffic("fused_kernel_prefill_8k.md", PREFILL_SOURCES),
                     "kernel": "kda_prefill = plan_kernel + persistent fused_kernel (timed together)",
                     "algorithmic_bytes": bytes_pass, "peak_source": peak_src},
        "tensor": {"bound_note": "HBM binds (intensity below the ridge); reported for the flop view",
                   "tflops_pages_count": FLOPS_PAGES_PER_TOKEN * T8K / (ms * 1e-3) / 1e12,
                   "tflops_own_count": FLOPS_OWN_PER_TOKEN * T8K / (ms * 1e-3) / 1e12,
                   "peak_tflops": bf16_peak()[0], "peak_source": bf16_peak()[1],
                   "frac_pages_count": FLOPS_PAGES_PER_TOKEN * T8K / (ms * 1e-3) / 1e12 / bf16_peak()[0],
                   "frac_own_count": FLOPS_OWN_PER_TOKEN * T8K / (ms * 1e-3) / 1e12 / bf16_peak()[0]},
        "e2e": {"value": world * T8K / (e2e_ms * 1e-3), "unit": "tokens/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
        "gpu_launches": launches,
        "clocks": clk.summary(),
        "varlen_16": others["varlen_16"],
        "prefill_1m": others["prefill_1m"],
        "tiny_f32": others["tiny_f32"],
        "gdn": prefill_entry(T8K, gdn_ms, gdn_ms_max, world, gdn_bytes, hbm, peak_src,
                             "gdn_8k: prefill_8k with one forget gate per (token, head) "
                             "(log_alpha [T][H], the Gated DeltaNet form)",
                             "kda_prefill with KDA_FLAG_SCALAR_GATE (timed like the main line)", flops=False),
        "output_gate": prefill_entry(T8K, og_ms, og_ms_max, world, og_bytes, hbm, peak_src,
                                     "prefill_8k with the output step fused: RMSNorm over d_v and "
                                     "a sigmoid gate [T][H][d_v] bf16 (page section 6.3)",
                                     "kda_prefill_ex with a kda_output_gate", flops=False),
        "decode": {"value": DECODE_BYTES / (dec_us_max * 1e-6) / 1e9, "unit": "GB/s",
                   "us_per_step": dec_us_max, "steps": dsteps,
                   "workload": "decode_256: 256 seqs x 32 heads, d=128, bf16 q/k/v, fp32 state "
                               "512 MiB in place (> L2); %d consecutive steps on %d pregenerated "
                               "inputs" % (dsteps, dsteps),
                   "roofline": {"bound": "hbm", "achieved": dec_gbs, "peak": hbm, "unit": "GB/s",
                                "frac": dec_gbs / hbm,
                                "traffic": profiled_traffic("decode_kernel_decode_256.md", DECODE_SOURCES),
                                "kernel": "decode_kernel<128,128,bf16>",
                                "algorithmic_bytes": DECODE_BYTES, "peak_source": peak_src},
                   "cuda_graph": dec_graph},
        "short_conv": {"value": world * T8K / (conv_ms["conv"][1] * 1e-3), "unit": "tokens/s",
                       "ms_per_step": conv_ms["conv"][1], "cuda_graph": conv_graph_used,
                       "workload": "short convolution (W=%d) + Swish of the q, k, v projections of prefill_8k "
                                   "([8192, 32*128] bf16 each, states written; page section 6.1)" % CONV_W,
                       "conv_then_prefill": {"value": world * T8K / (conv_ms["conv_prefill"][1] * 1e-3),
                                             "unit": "tokens/s", "ms_per_step": conv_ms["conv_prefill"][1]},
                       "prefill_conv": {"value": world * T8K / (conv_ms["prefill_conv"][1] * 1e-3),
                                        "unit": "tokens/s", "ms_per_step": conv_ms["prefill_conv"][1],
                                        "kernel": "kda_prefill_conv: the convolution of q, k in the prep engines' "
                                                  "loads and of v on the scan CTAs, then the three conv states"},
                       "roofline": {"bound": "hbm", "achieved": conv_gbs, "peak": hbm, "unit": "GB/s",
                                    "frac": conv_gbs / hbm, "traffic": None,
                                    "kernel": "conv_kernel<4,bf16> + conv_state_kernel (x3)",
                                    "algorithmic_bytes": 3 * CONV_BYTES, "peak_source": peak_src}},
        "backward": ({"value": world * T8K / (bw["ms"] * 1e-3), "unit": "tokens/s", "ms_per_step": bw["ms"],
                      "steps": bw_steps,
                      "workload": "gradients of prefill_8k w.r.t. q, k, v, log_alpha, beta, S0 given dL/do "
                                  "(bf16) and dL/dS_T (fp32); fp32 CUDA-core kernels",
                      "roofline": {"bound": "hbm", "achieved": bw["gbs"], "peak": hbm, "unit": "GB/s",
                                   "frac": bw["gbs"] / hbm, "traffic": None,
                                   "kernel": "bw_offsets + bw_prep + bw_fwd + bw_bwd + bw_rowstate + bw_grads + bw_norm",
                                   "algorithmic_bytes": BACKWARD_BYTES, "peak_source": peak_src}}
                     if "ms" in bw else bw),
        "decode_conv": {"value": DECODE_CONV_BYTES / (dconv_us_max * 1e-6) / 1e9, "unit": "GB/s",
                        "us_per_step": dconv_us_max, "steps": dsteps,
                        "workload": "decode_256 with the short convolution (W=%d) + Swish fused into the q, k, v "
                                    "loads, bf16 states [256, %d, 4096] x3 in place" % (CONV_W, CONV_W - 1),
                        "roofline": {"bound": "hbm", "achieved": dconv_gbs, "peak": hbm, "unit": "GB/s",
                                     "frac": dconv_gbs / hbm, "traffic": None,
                                     "kernel": "decode_kernel<128,128,bf16> with the convolution",
                                     "algorithmic_bytes": DECODE_CONV_BYTES, "peak_source": peak_src}},
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v_cpu, cores, desc = oracle_sample(seconds_target=args.cpu_seconds)
        line["cpu_baseline"] = {"value": v_cpu, "unit": "tokens/s", "cores": cores,
                                "kind": "oracle", "sample": desc}
    if rank == 0:
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["kda", "reference"], default="kda")
    ap.add_argument("--decode-steps", type=int, default=1000)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_kda(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
