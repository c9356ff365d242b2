"""Run one named KDA workload through the public API a few times, for profilers.

``python -m gated_delta_rule_125_b200.run_workload NAME [--calls N]`` builds the
seeded synthetic inputs of NAME (``kda_inputs``) on ``cuda:0`` and calls the
matching entry point N times (default 3), then synchronises. It times nothing
and checks nothing: it is the command an ncu capture wraps, so that one kernel
of one workload can be captured at a size that fits the profiler (a few GB).

Names: the prefill workloads of ``kda_inputs.WORKLOADS`` (``tiny_f32``,
``prefill_8k``, ``varlen_16``, ``gdn_8k``); ``decode_256`` (256 sequences x 32
heads, one step per call), ``decode_256_conv`` (the same with the short
convolution fused into the loads), ``short_conv_8k`` (the convolution of one
[8192, 32 * 128] projection), ``backward_1k`` (the backward of one 1024-token
sequence, 32 heads), ``prefill_8k_conv`` (prefill_8k from raw projections with the
width-4 short convolution of q, k, v inside the prefill), ``prefill_8k_gate`` (prefill_8k
with the fused output step).
"""
from __future__ import annotations

import argparse
import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import gated_delta_rule_125_b200 as kda  # noqa: E402
import kda_inputs as KI  # noqa: E402


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("name")
    ap.add_argument("--calls", type=int, default=3)
    args = ap.parse_args()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    n = args.name
    if n in KI.WORKLOADS and "lengths" in KI.WORKLOADS[n]:
        inp = KI.prefill_workload(n, dev)
        L = max(inp["lengths"])
        for _ in range(args.calls):
            kda.kda_prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["S0"],
                            inp["cu_seqlens"], max_seqlen=L)
    elif n in ("prefill_8k_conv", "prefill_8k_gate"):
        inp = KI.prefill_workload("prefill_8k", dev)
        T, H, D = inp["v"].shape
        kw = {}
        if n.endswith("_conv"):
            conv, raw = [], []
            for i in range(3):
                x, w, st = KI.conv_inputs(T, H * D, 4, 1, torch.bfloat16, dev, tensor=i)
                raw.append(x.view(T, H, D))
                conv.append((w, st, torch.empty_like(st)))
            inp["q"], inp["k"], inp["v"] = raw
            kw["conv"] = tuple(conv)
        else:
            g = torch.Generator(device=dev)
            g.manual_seed(1000)
            kw["out_gate"] = (torch.randn((T, H, D), generator=g, device=dev).to(torch.bfloat16),
                              1.0 + 0.1 * torch.randn((D,), generator=g, device=dev), 1e-6)
        for _ in range(args.calls):
            kda.kda_prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp["S0"],
                            inp["cu_seqlens"], max_seqlen=T, **kw)
    elif n in ("decode_256", "decode_256_conv"):
        steps, H, D, N = args.calls, 32, 128, 256
        d = KI.decode_workload(N, H, D, steps, torch.bfloat16, dev)
        S = d["S0"].clone()
        conv = None
        if n.endswith("_conv"):
            conv = []
            for i in range(3):
                _, w, st = KI.conv_inputs(1, H * D, 4, N, torch.bfloat16, dev, tensor=i)
                conv.append((w, st, st))
            conv = tuple(conv)
        for t in range(steps):
            kda.kda_decode_step(d["q"][t], d["k"][t], d["v"][t], d["log_alpha"][t], d["beta"][t], S, conv=conv)
    elif n == "short_conv_8k":
        x, w, st = KI.conv_inputs(8192, 32 * 128, 4, 1, torch.bfloat16, dev)
        so = torch.empty_like(st)
        for _ in range(args.calls):
            kda.kda_short_conv_swish(x, w, state_in=st, state_out=so)
    elif n == "backward_1k":
        inp = KI.prefill_workload("prefill_8k", dev, lengths=[1024])
        g = torch.Generator(device=dev)
        g.manual_seed(5)
        do = torch.randn(inp["v"].shape, generator=g, device=dev).to(torch.bfloat16)
        dST = torch.randn(inp["S0"].shape, generator=g, device=dev)
        for _ in range(args.calls):
            kda.kda_backward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], do, dST, inp["S0"],
                             inp["cu_seqlens"], max_seqlen=1024)
    else:
        raise SystemExit("unknown workload %r" % n)
    torch.cuda.synchronize()
    code = kda.kda_device_error(reset=True)
    print("%s: %d calls, device error word %d" % (n, args.calls, code))


if __name__ == "__main__":
    main()
