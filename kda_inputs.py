"""Seeded synthetic inputs for KDA workloads.

This module only draws random tensors with the shapes and value distributions
of the KDA workloads; it holds none of the operator's arithmetic. Both the
CUDA path and the fp64 oracle consume what it produces (the oracle gets the
exact stored bits copied to the host).

Recipe (every tensor seeded from ``(seed, tensor id, block)``; torch's
generator on the target device):

* q, k: N(0, 1) in fp32, scaled per (token, head) to unit L2 norm, then
  stored in the workload dtype (bf16 or fp32);
* v: N(0, 1) stored in the workload dtype;
* beta: sigmoid(N(0, 1)), fp32;
* log_alpha: -softplus(N(mu, 1)) per key channel, fp32 (mu = -3, or -4 for
  the long-memory 1M-token workload);
* S0: N(0, s0_std^2) fp32, or zeros;
* short-convolution inputs (the layer's q, k, v projections before the
  convolution): raw projections N(0, 1) in the workload dtype, taps
  N(0, 1/W) fp32 per channel, initial convolution states N(0, 1) in the
  workload dtype.
"""
from __future__ import annotations

import torch
import torch.nn.functional as F

_BLOCK = 1 << 16  # tokens drawn per generator call (bounds fp32 temporaries)

_IDS = {"q": 1, "k": 2, "v": 3, "beta": 4, "log_alpha": 5, "S0": 6, "len": 7, "log_alpha_scalar": 8,
        "conv_x": 9, "conv_w": 10, "conv_state": 11}


def _gen(device, seed, name, block=0):
    g = torch.Generator(device=device)
    g.manual_seed((int(seed) * 1_000_003 + _IDS[name] * 10_007 + block) & 0x7FFF_FFFF_FFFF_FFFF)
    return g


def _normal(shape, device, seed, name, block=0):
    return torch.randn(shape, generator=_gen(device, seed, name, block), device=device,
                       dtype=torch.float32)


def _unit_rows(x):
    # Data recipe: rows of N(0,1) scaled to unit length before storage.
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-30)


def varlen_lengths(n, lo, hi, seed):
    """``n`` sequence lengths drawn uniformly from [lo, hi] (inclusive)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed) * 7919 + _IDS["len"])
    return torch.randint(lo, hi + 1, (n,), generator=g).tolist()


def cu_from_lengths(lengths, device="cpu"):
    cu = [0]
    for n in lengths:
        cu.append(cu[-1] + int(n))
    return torch.tensor(cu, dtype=torch.int32, device=device)


def token_inputs(T, H, dk, dv, dtype=torch.bfloat16, device="cpu", seed=0, mu=-3.0):
    """q, k, v [T,H,d] (``dtype``), log_alpha [T,H,dk] fp32, beta [T,H] fp32."""
    q = torch.empty((T, H, dk), dtype=dtype, device=device)
    k = torch.empty((T, H, dk), dtype=dtype, device=device)
    v = torch.empty((T, H, dv), dtype=dtype, device=device)
    la = torch.empty((T, H, dk), dtype=torch.float32, device=device)
    beta = torch.empty((T, H), dtype=torch.float32, device=device)
    for b, t0 in enumerate(range(0, T, _BLOCK)):
        n = min(_BLOCK, T - t0)
        q[t0:t0 + n] = _unit_rows(_normal((n, H, dk), device, seed, "q", b)).to(dtype)
        k[t0:t0 + n] = _unit_rows(_normal((n, H, dk), device, seed, "k", b)).to(dtype)
        v[t0:t0 + n] = _normal((n, H, dv), device, seed, "v", b).to(dtype)
        la[t0:t0 + n] = -F.softplus(_normal((n, H, dk), device, seed, "log_alpha", b) + mu)
        beta[t0:t0 + n] = torch.sigmoid(_normal((n, H), device, seed, "beta", b))
    return q, k, v, la, beta


def scalar_gates(T, H, device="cpu", seed=0, mu=-3.0):
    """log_alpha [T,H] fp32 = -softplus(N(mu, 1)): one forget gate per (token, head),
    the Gated DeltaNet form; same distribution as the per-channel gates."""
    la = torch.empty((T, H), dtype=torch.float32, device=device)
    for b, t0 in enumerate(range(0, T, _BLOCK)):
        n = min(_BLOCK, T - t0)
        la[t0:t0 + n] = -F.softplus(_normal((n, H), device, seed, "log_alpha_scalar", b) + mu)
    return la


def initial_state(N, H, dk, dv, std, device="cpu", seed=0):
    """S0 [N,H,dk,dv] fp32 drawn N(0, std^2); zeros when ``std`` is 0 or None."""
    if not std:
        return torch.zeros((N, H, dk, dv), dtype=torch.float32, device=device)
    return _normal((N, H, dk, dv), device, seed, "S0") * float(std)


# Named workloads (sizes and distributions of the KDA benchmarks).
WORKLOADS = {
    "tiny_f32": dict(lengths=[256], H=2, d=64, dtype="f32", mu=-3.0, s0_std=0.0),
    "prefill_8k": dict(lengths=[8192], H=32, d=128, dtype="bf16", mu=-3.0, s0_std=0.01),
    "varlen_16": dict(lengths=("uniform", 16, 512, 8192), H=32, d=128, dtype="bf16", mu=-3.0,
                      s0_std=0.0),
    "prefill_1m": dict(lengths=[1 << 20], H=32, d=128, dtype="bf16", mu=-4.0, s0_std=0.0),
    "decode_256": dict(N=256, H=32, d=128, dtype="bf16", mu=-3.0, s0_std=0.01, steps=1000),
    # Gated DeltaNet form of prefill_8k: one gate per (token, head)
    "gdn_8k": dict(lengths=[8192], H=32, d=128, dtype="bf16", mu=-3.0, s0_std=0.01, scalar_gate=True),
}


def workload_lengths(name, seed=0):
    spec = WORKLOADS[name]["lengths"]
    if isinstance(spec, tuple):
        _, n, lo, hi = spec
        return varlen_lengths(n, lo, hi, seed)
    return list(spec)


def torch_dtype(tag):
    return {"f32": torch.float32, "bf16": torch.bfloat16}[tag]


def prefill_workload(name, device="cpu", seed=0, lengths=None, heads=None):
    """Inputs of a named prefill workload (``lengths``/``heads`` override its sizes)."""
    w = WORKLOADS[name]
    lengths = workload_lengths(name, seed) if lengths is None else list(lengths)
    H = w["H"] if heads is None else heads
    T = sum(lengths)
    q, k, v, la, beta = token_inputs(T, H, w["d"], w["d"], torch_dtype(w["dtype"]), device,
                                     seed, w["mu"])
    if w.get("scalar_gate"):
        la = scalar_gates(T, H, device, seed, w["mu"])
    S0 = initial_state(len(lengths), H, w["d"], w["d"], w["s0_std"], device, seed)
    return dict(q=q, k=k, v=v, log_alpha=la, beta=beta, S0=S0,
                cu_seqlens=cu_from_lengths(lengths, device), lengths=lengths)


def decode_workload(N, H, d, steps, dtype=torch.bfloat16, device="cpu", seed=0, mu=-3.0,
                    s0_std=0.01):
    """Per-step decode inputs ``[steps, N, H, d]`` and the initial state ``[N,H,d,d]``."""
    q, k, v, la, beta = token_inputs(steps * N, H, d, d, dtype, device, seed, mu)
    shp = (steps, N, H)
    return dict(q=q.view(*shp, d), k=k.view(*shp, d), v=v.view(*shp, d),
                log_alpha=la.view(*shp, d), beta=beta.view(*shp),
                S0=initial_state(N, H, d, d, s0_std, device, seed))


def conv_inputs(T, C, W, N=1, dtype=torch.bfloat16, device="cpu", seed=0, tensor=0, with_state=True):
    """Short-convolution inputs for one projection: x [T, C] N(0,1) in ``dtype``,
    taps [C, W] N(0, 1/W) fp32 and an initial state [N, W-1, C] N(0,1) in ``dtype``
    (None without state). ``tensor`` separates the q / k / v draws."""
    x = _normal((T, C), device, seed * 3 + tensor, "conv_x").to(dtype)
    w = _normal((C, W), device, seed * 3 + tensor, "conv_w") / float(W) ** 0.5
    st = None
    if with_state:
        st = _normal((N, W - 1, C), device, seed * 3 + tensor, "conv_state").to(dtype)
    return x, w, st
