"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Tolerances (bf16 q/k/v: max|o - o_ref| <= 2e-2 and relative Frobenius error of
the final state <= 1e-2; fp32: both <= 1e-4) are the gate of the workloads.
The oracle always runs on the exact bits the GPU consumed, copied to the host.
Full-size workloads are checked on sampled (sequence, head) units over their
whole length -- units are independent, so a sample is an exact check of its
members.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_125_b200 as kda
import kda_inputs as KI
import oracle
from bf16_round import bf16_neighbours

pytestmark = pytest.mark.gpu

TOL = {torch.bfloat16: (2e-2, 1e-2), torch.float32: (1e-4, 1e-4)}
DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    kda.load_library()


def host(x):
    return x.detach().to("cpu", torch.float64).numpy()


def rel_fro(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def ref_prefill(inp, heads=None, seqs=None, S0=True):
    """Oracle on the given (sub)set of heads/sequences. Returns o_ref, S_ref and the index."""
    cu = inp["cu_seqlens"].cpu().numpy().astype(np.int64)
    N = len(cu) - 1
    seqs = list(range(N)) if seqs is None else list(seqs)
    H = inp["q"].shape[1]
    heads = list(range(H)) if heads is None else list(heads)
    tok = np.concatenate([np.arange(cu[s], cu[s + 1]) for s in seqs]) if seqs else np.zeros(0, int)
    sub_cu = np.cumsum([0] + [cu[s + 1] - cu[s] for s in seqs])
    hi = torch.tensor(heads)
    ti = torch.from_numpy(tok)
    pick = lambda x: host(x.index_select(0, ti.to(x.device)).index_select(1, hi.to(x.device)))
    S0v = None
    if S0 and inp.get("S0") is not None:
        S0v = host(inp["S0"][torch.tensor(seqs).to(DEV)][:, hi.to(DEV)])
    o_ref, S_ref = oracle.recurrent(pick(inp["q"]), pick(inp["k"]), pick(inp["v"]),
                                    pick(inp["log_alpha"]), pick(inp["beta"]), S0v, sub_cu)
    return o_ref, S_ref, ti, hi, seqs


def check(o, S_T, inp, dtype, heads=None, seqs=None, label=""):
    o_ref, S_ref, ti, hi, seqs = ref_prefill(inp, heads, seqs)
    og = host(o.index_select(0, ti.to(o.device)).index_select(1, hi.to(o.device)))
    Sg = host(S_T[torch.tensor(seqs).to(DEV)][:, hi.to(DEV)])
    atol, stol = TOL[dtype]
    err = float(np.abs(og - o_ref).max()) if og.size else 0.0
    sf = rel_fro(Sg, S_ref)
    assert np.isfinite(og).all() and np.isfinite(Sg).all(), label
    assert err <= atol, "%s: max|o-o_ref| = %.3e > %.1e" % (label, err, atol)
    assert sf <= stol, "%s: relFro(S_T) = %.3e > %.1e" % (label, sf, stol)
    return err, sf


def make(lengths, H, dk, dv, dtype, seed=0, mu=-3.0, s0=0.1):
    T = sum(lengths)
    q, k, v, la, beta = KI.token_inputs(T, H, dk, dv, dtype, DEV, seed, mu)
    S0 = KI.initial_state(len(lengths), H, dk, dv, s0, DEV, seed)
    return dict(q=q, k=k, v=v, log_alpha=la, beta=beta, S0=S0,
                cu_seqlens=KI.cu_from_lengths(lengths, DEV), lengths=list(lengths))


def run(inp, **kw):
    o = torch.full(inp["v"].shape, float("nan"), dtype=inp["v"].dtype, device=DEV)
    N = len(inp["lengths"])
    S_T = torch.full((N,) + tuple(inp["S0"].shape[1:]), float("nan"), device=DEV)
    kda.kda_prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], inp.get("S0"),
                    inp["cu_seqlens"], max_seqlen=max(inp["lengths"] + [0]), o=o, S_T=S_T, **kw)
    torch.cuda.synchronize()
    return o, S_T


# ------------------------------------------------------------ prefill ----

def test_tiny_f32_workload():
    """B=1, H=2, T=256, d=64, fp32 throughout, S0 = 0 (tolerance 1e-4)."""
    inp = KI.prefill_workload("tiny_f32", DEV)
    o, S_T = run(inp)
    check(o, S_T, inp, torch.float32, label="tiny_f32")


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("dk,dv", [(64, 64), (128, 128), (64, 128), (128, 64)])
@pytest.mark.parametrize("T", [1, 63, 64, 65, 130])
def test_small_shapes(T, dk, dv, dtype):
    inp = make([T], 3, dk, dv, dtype, seed=T + dk + dv)
    o, S_T = run(inp)
    check(o, S_T, inp, dtype, label="T=%d dk=%d dv=%d %s" % (T, dk, dv, dtype))


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_varlen_with_empty_sequences(dtype):
    lengths = [0, 5, 64, 1, 200, 0, 129]
    inp = make(lengths, 4, 128, 128, dtype, seed=3)
    o, S_T = run(inp)
    check(o, S_T, inp, dtype, label="varlen")
    # empty sequences return their entry state
    assert torch.equal(S_T[0], inp["S0"][0]) and torch.equal(S_T[5], inp["S0"][5])


def test_varlen_equals_separate_calls():
    lengths = [70, 1, 191, 64]
    inp = make(lengths, 2, 128, 128, torch.bfloat16, seed=4)
    o, S_T = run(inp)
    cu = [0]
    for n in lengths:
        cu.append(cu[-1] + n)
    for s, n in enumerate(lengths):
        a, b = cu[s], cu[s + 1]
        # fresh copies: every pointer handed to the library must be 16-byte aligned
        one = dict(q=inp["q"][a:b].clone(), k=inp["k"][a:b].clone(), v=inp["v"][a:b].clone(),
                   log_alpha=inp["log_alpha"][a:b].clone(), beta=inp["beta"][a:b].clone(),
                   S0=inp["S0"][s:s + 1].clone(), cu_seqlens=KI.cu_from_lengths([n], DEV),
                   lengths=[n])
        o1, S1 = run(one)
        assert torch.equal(o1, o[a:b]) and torch.equal(S1[0], S_T[s])


@pytest.mark.parametrize("t0", [1, 37, 64, 100])
def test_split_prefill_continuity(t0):
    """prefill(x[0:T]) == prefill(x[t0:T], S0 = prefill(x[0:t0]).S_T): state across chunk edges."""
    T = 200
    inp = make([T], 2, 128, 128, torch.float32, seed=5)
    o, S_T = run(inp)
    sl = lambda a, b, S0: dict(q=inp["q"][a:b].clone(), k=inp["k"][a:b].clone(),
                               v=inp["v"][a:b].clone(), log_alpha=inp["log_alpha"][a:b].clone(),
                               beta=inp["beta"][a:b].clone(), S0=S0,
                               cu_seqlens=KI.cu_from_lengths([b - a], DEV), lengths=[b - a])
    oa, Sa = run(sl(0, t0, inp["S0"]))
    ob, Sb = run(sl(t0, T, Sa))
    torch.testing.assert_close(torch.cat([oa, ob]), o, atol=2e-5, rtol=0)
    torch.testing.assert_close(Sb, S_T, atol=2e-5, rtol=0)


def test_multi_wave_matches_single_wave():
    lengths = [300, 40, 513]
    inp = make(lengths, 3, 64, 64, torch.bfloat16, seed=6)
    o1, S1 = run(inp)
    L = max(lengths)
    mn = kda.kda_prefill_workspace_min(3, sum(lengths), L, 3, 64, 64, torch.bfloat16)
    ws = torch.empty(mn + 4096, dtype=torch.uint8, device=DEV)
    o2, S2 = run(inp, workspace=ws)
    assert torch.equal(o1, o2) and torch.equal(S1, S2)
    check(o2, S2, inp, torch.bfloat16, label="multi-wave")


def test_tensor_core_ring_sizes_and_many_units():
    """bf16, d = 128 with more (sequence, head) units than scan streams (72 over
    32: streams of 2 or 3 units of different lengths) and empty, one-token and
    ragged sequences. The smallest workspace (fewest ring slots per stream)
    gives bit-identical results to the recommended one; both match the oracle."""
    lengths = [0, 130, 1, 64, 700, 0, 65, 257]
    H = 9
    inp = make(lengths, H, 128, 128, torch.bfloat16, seed=21)
    o1, S1 = run(inp)
    mn = kda.kda_prefill_workspace_min(len(lengths), sum(lengths), max(lengths), H, 128, 128,
                                       torch.bfloat16)
    ws = torch.empty(mn, dtype=torch.uint8, device=DEV)
    o2, S2 = run(inp, workspace=ws)
    assert torch.equal(o1, o2) and torch.equal(S1, S2)
    check(o1, S1, inp, torch.bfloat16, label="tc streams")
    assert torch.equal(S1[0], inp["S0"][0]) and torch.equal(S1[5], inp["S0"][5])
    assert kda.kda_device_error() == 0


def test_strong_decay():
    inp = make([150], 2, 128, 128, torch.float32, seed=7)
    inp["log_alpha"] = inp["log_alpha"] * 400.0  # ~ -20 per token: exp(+G) would overflow
    o, S_T = run(inp)
    check(o, S_T, inp, torch.float32, label="strong decay")


@pytest.mark.parametrize("scale", [400.0, 30.0])
def test_strong_decay_tensor_core_path(scale):
    """bf16, d = 128: chunks whose decay range is too large for the factorised
    Gram go through the exact fallback (every chunk at scale 400, some at 30)."""
    inp = make([300, 64, 130], 4, 128, 128, torch.bfloat16, seed=13)
    inp["log_alpha"] = inp["log_alpha"] * scale
    o, S_T = run(inp)
    check(o, S_T, inp, torch.bfloat16, label="strong decay bf16 x%g" % scale)
    assert kda.kda_device_error() == 0


def test_tensor_core_matches_exact_path():
    """The tcgen05 path and the fp32 CUDA-core path agree within the bf16 tolerance."""
    inp = make([513, 77], 4, 128, 128, torch.bfloat16, seed=14)
    o1, S1 = run(inp)
    o2, S2 = run(inp, exact=True)
    assert float((o1.float() - o2.float()).abs().max()) <= 2e-2
    assert float((S1 - S2).norm() / S2.norm()) <= 1e-2
    check(o1, S1, inp, torch.bfloat16, label="tc")
    check(o2, S2, inp, torch.bfloat16, label="exact")


def test_no_device_error_after_runs():
    inp = make([1000], 8, 128, 128, torch.bfloat16, seed=15)
    run(inp)
    assert kda.kda_device_error() == 0


def test_no_l2norm_flag():
    inp = make([100], 2, 64, 64, torch.float32, seed=8)
    o1, S1 = run(inp)
    o2, S2 = run(inp, l2norm=False)  # inputs are already unit-norm
    torch.testing.assert_close(o2, o1, atol=1e-5, rtol=0)
    torch.testing.assert_close(S2, S1, atol=1e-5, rtol=0)


def test_deterministic():
    inp = make([257, 31], 4, 128, 128, torch.bfloat16, seed=9)
    o1, S1 = run(inp)
    o2, S2 = run(inp)
    assert torch.equal(o1, o2) and torch.equal(S1, S2)


def test_state_aliasing_in_place():
    """S_T may alias S0."""
    inp = make([150, 20], 2, 128, 128, torch.float32, seed=10)
    o_ref, S_ref = run(inp)
    S = inp["S0"].clone()
    kda.kda_prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], S,
                    inp["cu_seqlens"], max_seqlen=150, S_T=S)
    torch.cuda.synchronize()
    assert torch.equal(S, S_ref)


# ------------------------------------------------------------- decode ----

@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("dk,dv", [(128, 128), (64, 64), (64, 128), (128, 64)])
def test_decode_steps(dk, dv, dtype):
    N, H, steps = 5, 3, 4
    w = KI.decode_workload(N, H, dk, steps, dtype, DEV, seed=11, s0_std=0.1) if dk == dv else None
    if w is None:
        q, k, v, la, beta = KI.token_inputs(steps * N, H, dk, dv, dtype, DEV, 11, -3.0)
        w = dict(q=q.view(steps, N, H, dk), k=k.view(steps, N, H, dk), v=v.view(steps, N, H, dv),
                 log_alpha=la.view(steps, N, H, dk), beta=beta.view(steps, N, H),
                 S0=KI.initial_state(N, H, dk, dv, 0.1, DEV, 11))
    S = w["S0"].clone()
    S_ref = host(S)
    atol, stol = TOL[dtype]
    for t in range(steps):
        o = kda.kda_decode_step(w["q"][t], w["k"][t], w["v"][t], w["log_alpha"][t], w["beta"][t], S)
        torch.cuda.synchronize()
        o_ref, S_ref = oracle.decode_step(host(w["q"][t]), host(w["k"][t]), host(w["v"][t]),
                                          host(w["log_alpha"][t]), host(w["beta"][t]), S_ref)
        assert float(np.abs(host(o) - o_ref).max()) <= atol
        assert rel_fro(host(S), S_ref) <= stol


def test_prefill_then_decode_equals_longer_prefill():
    """Prefill of T-3 tokens then 3 decode steps == prefill of all T (one state layout)."""
    T, H = 131, 4
    inp = make([T], H, 128, 128, torch.float32, seed=12)
    o_all, S_all = run(inp)
    m = T - 3
    part = dict(q=inp["q"][:m], k=inp["k"][:m], v=inp["v"][:m], log_alpha=inp["log_alpha"][:m],
                beta=inp["beta"][:m], S0=inp["S0"], cu_seqlens=KI.cu_from_lengths([m], DEV),
                lengths=[m])  # prefixes keep the base pointers aligned
    _, S = run(part)
    for t in range(m, T):
        o = kda.kda_decode_step(inp["q"][t:t + 1].clone(), inp["k"][t:t + 1].clone(),
                                inp["v"][t:t + 1].clone(), inp["log_alpha"][t:t + 1].clone(),
                                inp["beta"][t:t + 1].clone(), S)
        torch.testing.assert_close(o[0], o_all[t], atol=2e-5, rtol=0)
    torch.testing.assert_close(S, S_all, atol=2e-5, rtol=0)


# ------------------------------------------------ full-size workloads ----

def test_workload_prefill_8k():
    """B=1, H=32, T=8192, d=128, bf16; every output of heads {0, 17, 31} vs the oracle."""
    inp = KI.prefill_workload("prefill_8k", DEV)
    o, S_T = run(inp)
    check(o, S_T, inp, torch.bfloat16, heads=[0, 17, 31], label="prefill_8k")


def test_workload_varlen_16():
    """16 packed sequences, lengths U[512, 8192]; sampled (sequence, head) units."""
    inp = KI.prefill_workload("varlen_16", DEV)
    o, S_T = run(inp)
    longest = int(np.argmax(inp["lengths"]))
    check(o, S_T, inp, torch.bfloat16, heads=[3, 30], seqs=[0, longest, 15], label="varlen_16")


def test_workload_prefill_1m():
    """B=1, H=32, T=1,048,576 (long memory); heads {0, 21} over all 1M tokens."""
    inp = KI.prefill_workload("prefill_1m", DEV)
    o, S_T = run(inp)
    check(o, S_T, inp, torch.bfloat16, heads=[0, 21], label="prefill_1m")


def test_workload_decode_256():
    """256 sequences x 32 heads, 1000 in-place steps; sequences {0, 101, 255} vs the oracle."""
    N, H, d, steps = 256, 32, 128, 1000
    w = KI.decode_workload(N, H, d, steps, torch.bfloat16, DEV, seed=0, s0_std=0.01)
    S = w["S0"].clone()
    seqs = [0, 101, 255]
    S_ref = host(S[seqs])
    o_all = torch.empty((steps, N, H, d), dtype=torch.bfloat16, device=DEV)
    for t in range(steps):
        kda.kda_decode_step(w["q"][t], w["k"][t], w["v"][t], w["log_alpha"][t], w["beta"][t], S,
                            o=o_all[t])
    torch.cuda.synchronize()
    worst = 0.0
    for t in range(steps):
        o_ref, S_ref = oracle.decode_step(host(w["q"][t][seqs]), host(w["k"][t][seqs]),
                                          host(w["v"][t][seqs]), host(w["log_alpha"][t][seqs]),
                                          host(w["beta"][t][seqs]), S_ref)
        worst = max(worst, float(np.abs(host(o_all[t][seqs]) - o_ref).max()))
    assert worst <= 2e-2
    assert rel_fro(host(S[seqs]), S_ref) <= 1e-2


# ------------------------------------------------- scalar gate (GDN) ----
# KDA_FLAG_SCALAR_GATE: log_alpha [T,H], one gate per (token, head), the Gated
# DeltaNet form of page "[Kimi-2] Kimi Linear" §3. The oracle is the KDA
# recurrence with that gate broadcast over d_k (the reduction the oracle pin
# `pin_gdn_special_case` checks against the explicit GDN matrices).

def _with_scalar_gate(inp, seed):
    T, H = inp["beta"].shape
    g = KI.scalar_gates(T, H, DEV, seed)
    dk = inp["q"].shape[-1]
    gdn = dict(inp, log_alpha=g)
    expanded = dict(inp, log_alpha=g[:, :, None].expand(T, H, dk).contiguous())
    return gdn, expanded


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64), (torch.bfloat16, 64)])
def test_scalar_gate_prefill(dtype, d):
    """Both prefill paths: the scalar-gate call equals the per-channel call with the
    gate broadcast (bit for bit), and both match the oracle; varlen with empty and
    ragged sequences."""
    inp = make([0, 130, 1, 257, 64], 3, d, d, dtype, seed=31)
    gdn, expanded = _with_scalar_gate(inp, 31)
    o1, S1 = run(gdn)
    o2, S2 = run(expanded)
    assert torch.equal(o1, o2) and torch.equal(S1, S2)
    check(o1, S1, expanded, dtype, label="scalar gate %s d=%d" % (dtype, d))


def test_scalar_gate_strong_decay_tensor_core_path():
    """Scalar gates large enough that every chunk takes the element-wise Gram."""
    inp = make([300, 64, 130], 4, 128, 128, torch.bfloat16, seed=33)
    gdn, expanded = _with_scalar_gate(inp, 33)
    gdn["log_alpha"] = gdn["log_alpha"] * 400.0
    expanded["log_alpha"] = expanded["log_alpha"] * 400.0
    o, S_T = run(gdn)
    check(o, S_T, expanded, torch.bfloat16, label="scalar gate strong decay")
    assert kda.kda_device_error() == 0


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_scalar_gate_decode(dtype):
    N, H, d, steps = 5, 3, 128, 4
    w = KI.decode_workload(N, H, d, steps, dtype, DEV, seed=35, s0_std=0.1)
    g = KI.scalar_gates(steps * N, H, DEV, 35).view(steps, N, H)
    S = w["S0"].clone()
    S_ref = host(S)
    atol, stol = TOL[dtype]
    for t in range(steps):
        o = kda.kda_decode_step(w["q"][t], w["k"][t], w["v"][t], g[t], w["beta"][t], S)
        torch.cuda.synchronize()
        la = host(g[t])[:, :, None].repeat(d, axis=2)
        o_ref, S_ref = oracle.decode_step(host(w["q"][t]), host(w["k"][t]), host(w["v"][t]), la,
                                          host(w["beta"][t]), S_ref)
        assert float(np.abs(host(o) - o_ref).max()) <= atol
        assert rel_fro(host(S), S_ref) <= stol


def test_workload_gdn_8k():
    """The Gated DeltaNet form of prefill_8k; every output of heads {3, 30} vs the oracle."""
    inp = KI.prefill_workload("gdn_8k", DEV)
    o, S_T = run(inp)
    T, H = inp["beta"].shape
    expanded = dict(inp, log_alpha=inp["log_alpha"][:, :, None].expand(T, H, 128).contiguous())
    check(o, S_T, expanded, torch.bfloat16, heads=[3, 30], label="gdn_8k")


# ------------------------------------------- fused output step (§6.3) ----
# kda_prefill_ex / kda_decode_step_ex with a kda_output_gate: o <- RMSNorm(o)
# * weight * sigmoid(gate) per (token, head). The oracle is its recurrence
# followed by oracle.output_gate (pinned in test_oracle_pins). RMSNorm rescales
# every row to unit mean square, so gated outputs are compared relative to
# their largest magnitude with the workload's tolerance for o.

def _gate_inputs(T, H, dv, dtype, seed):
    g = torch.Generator(device=DEV)
    g.manual_seed(1000 + seed)
    gate = torch.randn((T, H, dv), generator=g, device=DEV).to(dtype)
    w = 1.0 + 0.1 * torch.randn((dv,), generator=g, device=DEV)
    return gate, w, 1e-6


def _check_gated(o, inp, gate, w, eps, dtype, heads=None, label=""):
    o_ref, _, ti, hi, _ = ref_prefill(inp, heads)
    pick = lambda x: host(x.index_select(0, ti.to(x.device)).index_select(1, hi.to(x.device)))
    y_ref = oracle.output_gate(o_ref, pick(gate), host(w), eps)
    y = pick(o)
    atol = TOL[dtype][0] * max(1.0, float(np.abs(y_ref).max()))
    err = float(np.abs(y - y_ref).max())
    assert np.isfinite(y).all() and err <= atol, "%s: max|y-y_ref| = %.3e > %.3e" % (label, err, atol)


@pytest.mark.parametrize("dtype,d", [(torch.bfloat16, 128), (torch.float32, 64), (torch.float32, 128)])
def test_output_gate_prefill(dtype, d):
    inp = make([0, 130, 1, 257, 64], 3, d, d, dtype, seed=41)
    T = sum(inp["lengths"])
    gate, w, eps = _gate_inputs(T, 3, d, dtype, 41)
    o0, S0_ = run(inp)
    o1, S1 = run(inp, out_gate=(gate, w, eps))
    assert torch.equal(S0_, S1)  # the output step leaves the state alone
    _check_gated(o1, inp, gate, w, eps, dtype, label="gated %s d=%d" % (dtype, d))


def test_output_gate_many_units_small_ring():
    """Tensor-core path, 72 units over 32 streams and the smallest ring: the two scan
    CTAs of a stream exchange their halves' sums of squares chunk after chunk."""
    lengths = [0, 130, 1, 64, 700, 0, 65, 257]
    H = 9
    inp = make(lengths, H, 128, 128, torch.bfloat16, seed=43)
    gate, w, eps = _gate_inputs(sum(lengths), H, 128, torch.bfloat16, 43)
    mn = kda.kda_prefill_workspace_min(len(lengths), sum(lengths), max(lengths), H, 128, 128,
                                       torch.bfloat16)
    ws = torch.empty(mn, dtype=torch.uint8, device=DEV)
    o1, _ = run(inp, out_gate=(gate, w, eps), workspace=ws)
    o2, _ = run(inp, out_gate=(gate, w, eps))
    assert torch.equal(o1, o2)
    _check_gated(o1, inp, gate, w, eps, torch.bfloat16, label="gated streams")
    assert kda.kda_device_error() == 0


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_output_gate_decode(dtype):
    N, H, d, steps = 5, 3, 128, 3
    w_ = KI.decode_workload(N, H, d, steps, dtype, DEV, seed=45, s0_std=0.1)
    gate, w, eps = _gate_inputs(steps * N, H, d, dtype, 45)
    gate = gate.view(steps, N, H, d)
    S = w_["S0"].clone()
    S_ref = host(S)
    atol0 = TOL[dtype][0]
    for t in range(steps):
        o = kda.kda_decode_step(w_["q"][t], w_["k"][t], w_["v"][t], w_["log_alpha"][t], w_["beta"][t], S,
                                out_gate=(gate[t].contiguous(), w, eps))
        torch.cuda.synchronize()
        o_ref, S_ref = oracle.decode_step(host(w_["q"][t]), host(w_["k"][t]), host(w_["v"][t]),
                                          host(w_["log_alpha"][t]), host(w_["beta"][t]), S_ref)
        y_ref = oracle.output_gate(o_ref, host(gate[t]), host(w), eps)
        assert float(np.abs(host(o) - y_ref).max()) <= atol0 * max(1.0, float(np.abs(y_ref).max()))
        assert rel_fro(host(S), S_ref) <= TOL[dtype][1]


def test_output_gate_workload_prefill_8k():
    """prefill_8k with the fused output step; heads {5, 26} checked over all 8192 tokens."""
    inp = KI.prefill_workload("prefill_8k", DEV)
    gate, w, eps = _gate_inputs(8192, 32, 128, torch.bfloat16, 47)
    o, _ = run(inp, out_gate=(gate, w, eps))
    _check_gated(o, inp, gate, w, eps, torch.bfloat16, heads=[5, 26], label="gated prefill_8k")


# ------------------------------------- short convolution + Swish (§6.1) ----
# The convolution's output is one fp32 dot product of W taps then Swish, stored in
# the io dtype. The fp32 value z lies within CONV_FP32 = (relative, absolute) of
# the fp64 reference (absolute: the dot product's cancellation near zero). For
# bf16 the check separates that error from the rounding: rounding to nearest
# (ties to even) is monotone, so every output must lie between the roundings of
# y_ref - delta and y_ref + delta, delta = 4e-6 |y_ref| + 1e-6; the test reports
# how many outputs are not the rounding of y_ref itself. fp32 outputs: within
# 1e-5 relative + 1e-6 (fast exponential). States are raw input copies: bit-exact.
CONV_FP32 = (4e-6, 1e-6)


def _conv_ref(x, w, cu=None, st=None):
    return oracle.short_conv_swish(host(x).reshape(x.shape[0], -1), host(w),
                                   None if cu is None else cu.cpu().numpy(), None if st is None else host(st))


def _conv_close(y, y_ref, dtype, label):
    got = host(y).reshape(y_ref.shape)
    assert np.isfinite(got).all(), label
    if dtype != torch.bfloat16:
        err = np.abs(got - y_ref)
        assert np.all(err <= 1e-5 * np.abs(y_ref) + 1e-6), "%s: worst excess %.3e" % (
            label, float((err - 1e-5 * np.abs(y_ref) - 1e-6).max()))
        return 0
    delta = CONV_FP32[0] * np.abs(y_ref) + CONV_FP32[1]
    lo, hi = bf16_neighbours(y_ref - delta)[0], bf16_neighbours(y_ref + delta)[0]
    ok = (got >= lo) & (got <= hi)
    assert ok.all(), "%s: %d outputs are not a bf16 rounding of a value within the fp32 error (worst |y - y_ref| = %.3e)" % (
        label, int((~ok).sum()), float(np.abs(got - y_ref)[~ok].max()))
    return int((got != bf16_neighbours(y_ref)[0]).sum())  # not the rounding of y_ref itself


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("W", [1, 2, 3, 4, 8])
def test_short_conv_varlen(W, dtype):
    """Empty, one-token and ragged sequences (tiles of 32 tokens cross their boundaries)."""
    lengths = [37, 0, 1, 200, 5, 64, 3]
    T, N, C = sum(lengths), len(lengths), 96
    x, w, st = KI.conv_inputs(T, C, W, N, dtype, DEV, seed=W)
    cu = KI.cu_from_lengths(lengths, DEV)
    st_out = torch.full_like(st, float("nan"))
    y = kda.kda_short_conv_swish(x, w, cu, state_in=st, state_out=st_out)
    torch.cuda.synchronize()
    y_ref, st_ref = _conv_ref(x, w, cu, st)
    _conv_close(y, y_ref, dtype, "W=%d" % W)
    np.testing.assert_array_equal(host(st_out), st_ref)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
def test_short_conv_zero_state_and_aliased_state(dtype):
    T, C, W = 150, 64, 4
    x, w, st = KI.conv_inputs(T, C, W, 1, dtype, DEV, seed=21)
    y0 = kda.kda_short_conv_swish(x, w)  # one sequence, no state: zero history
    y_ref, st_ref0 = _conv_ref(x, w)
    _conv_close(y0, y_ref, dtype, "zero state")
    st_keep = st.clone()
    y1 = kda.kda_short_conv_swish(x, w, state_in=st, state_out=st)  # state updated in place
    torch.cuda.synchronize()
    y_ref1, st_ref1 = _conv_ref(x, w, None, st_keep)
    _conv_close(y1, y_ref1, dtype, "aliased state")
    np.testing.assert_array_equal(host(st), st_ref1)


def test_short_conv_rejects_bad_arguments():
    x, w, _ = KI.conv_inputs(16, 64, 4, 1, torch.bfloat16, DEV, seed=22, with_state=False)
    with pytest.raises(kda.KDAError):
        kda.kda_short_conv_swish(x, torch.zeros((64, 9), device=DEV))  # width 9 > KDA_MAX_CONV_WIDTH
    with pytest.raises(kda.KDAError):
        kda.kda_short_conv_swish(x, w, y=x)  # y overlaps x
    wl = KI.decode_workload(2, 1, 128, 1, torch.bfloat16, DEV, seed=22, s0_std=0.1)
    w5 = torch.zeros((128, 5), device=DEV)  # the fused decode step takes windows up to 4
    with pytest.raises(kda.KDAError):
        kda.kda_decode_step(wl["q"][0], wl["k"][0], wl["v"][0], wl["log_alpha"][0], wl["beta"][0],
                            wl["S0"].clone(), conv=((w5, None, None), None, None))
    lib = kda.load_library()
    assert lib.kda_short_conv_launches(4, 1, 16) == 2 and lib.kda_short_conv_launches(1, 1, 16) == 1
    assert lib.kda_short_conv_launches(4, 0, 0) == 0 and lib.kda_short_conv_launches(0, 0, 16) == -1


def test_short_conv_workload_prefill_8k():
    """The q projection of prefill_8k (T=8192, C=32*128), W=4: every output vs the oracle."""
    x, w, st = KI.conv_inputs(8192, 4096, 4, 1, torch.bfloat16, DEV, seed=23)
    st_out = torch.empty_like(st)
    y = kda.kda_short_conv_swish(x, w, state_in=st, state_out=st_out)
    torch.cuda.synchronize()
    y_ref, st_ref = _conv_ref(x, w, None, st)
    _conv_close(y, y_ref, torch.bfloat16, "prefill_8k q")
    np.testing.assert_array_equal(host(st_out), st_ref)


def test_short_conv_then_prefill():
    """q, k, v through the convolution, then the prefill (the oracle on the same bits)."""
    lengths, H, d, W = [100, 64, 1], 2, 128, 4
    T, N = sum(lengths), len(lengths)
    cu = KI.cu_from_lengths(lengths, DEV)
    outs = []
    for i in range(3):
        x, w, st = KI.conv_inputs(T, H * d, W, N, torch.bfloat16, DEV, seed=24, tensor=i)
        outs.append(kda.kda_short_conv_swish(x, w, cu, state_in=st).view(T, H, d))
    inp = make(lengths, H, d, d, torch.bfloat16, seed=24)
    inp.update(q=outs[0], k=outs[1], v=outs[2])
    o, S_T = run(inp)
    check(o, S_T, inp, torch.bfloat16, label="conv then prefill")


@pytest.mark.parametrize("dtype,d,with_v", [(torch.bfloat16, 128, True), (torch.float32, 64, True),
                                            (torch.bfloat16, 128, False)])
def test_decode_conv_steps(dtype, d, with_v):
    """Decode steps with the convolution fused into the q, k (, v) loads; states in place."""
    N, H, W, steps = 4, 3, 4, 4
    wl = KI.decode_workload(N, H, d, steps, dtype, DEV, seed=25, s0_std=0.1)
    convs, refs = [], []
    for i in range(3):
        x, w, st = KI.conv_inputs(steps * N, H * d, W, N, dtype, DEV, seed=25, tensor=i)
        raw = x.view(steps, N, H, d)
        convs.append((w, st, st, raw))
        refs.append(host(st))
    if not with_v:
        convs[2] = (None, None, None, wl["v"])
    S = wl["S0"].clone()
    S_ref = host(S)
    atol, stol = TOL[dtype]
    for t in range(steps):
        cq, ck, cv = [None if c[0] is None else (c[0], c[1], c[2]) for c in convs]
        o = kda.kda_decode_step(convs[0][3][t], convs[1][3][t], convs[2][3][t], wl["log_alpha"][t],
                                wl["beta"][t], S, conv=(cq, ck, cv))
        torch.cuda.synchronize()
        xs = []
        for i in range(3):
            if convs[i][0] is None:
                xs.append(host(wl["v"][t]))
                continue
            y, refs[i] = oracle.short_conv_step(host(convs[i][3][t]).reshape(N, H * d), host(convs[i][0]), refs[i])
            xs.append(y.reshape(N, H, d))
        o_ref, S_ref = oracle.decode_step(xs[0], xs[1], xs[2], host(wl["log_alpha"][t]), host(wl["beta"][t]), S_ref)
        assert float(np.abs(host(o) - o_ref).max()) <= atol, "step %d" % t
        assert rel_fro(host(S), S_ref) <= stol, "step %d" % t
        for i in range(3):
            if convs[i][0] is not None:
                np.testing.assert_array_equal(host(convs[i][1]), refs[i])


@pytest.mark.parametrize("W,which,dk", [(2, (False, True, True), 128), (3, (True, False, False), 128),
                                        (4, (True, True, True), 64)])
def test_decode_conv_windows_separate_states(W, which, dk):
    """Decode with the convolution on a subset of q, k, v, windows 2..4 and d_k 64 or 128
    (d_v = 128: the state split over a two-CTA cluster), reading the conv states from one
    buffer and writing them to another (the input states stay untouched)."""
    N, H, dv, steps = 5, 3, 128, 3
    g = torch.Generator(device=DEV)
    g.manual_seed(31)
    dims = (dk, dk, dv)
    raw = [torch.randn(steps, N, H, dims[i], generator=g, device=DEV).to(torch.bfloat16) for i in range(3)]
    la = -torch.nn.functional.softplus(torch.randn(steps, N, H, dk, generator=g, device=DEV) - 3.0)
    beta = torch.sigmoid(torch.randn(steps, N, H, generator=g, device=DEV))
    S = 0.1 * torch.randn(N, H, dk, dv, generator=g, device=DEV)
    S_ref = host(S)
    w = [torch.randn(H * dims[i], W, generator=g, device=DEV) / W ** 0.5 for i in range(3)]
    st = [torch.randn(N, W - 1, H * dims[i], generator=g, device=DEV).to(torch.bfloat16) for i in range(3)]
    refs = [host(x) for x in st]
    for t in range(steps):
        outs = [torch.empty_like(x) for x in st]
        cv = tuple((w[i], st[i], outs[i]) if which[i] else None for i in range(3))
        keep = [x.clone() for x in st]
        o = kda.kda_decode_step(raw[0][t], raw[1][t], raw[2][t], la[t], beta[t], S, conv=cv)
        torch.cuda.synchronize()
        xs = []
        for i in range(3):
            if not which[i]:
                xs.append(host(raw[i][t]))
                continue
            y, refs[i] = oracle.short_conv_step(host(raw[i][t]).reshape(N, H * dims[i]), host(w[i]), refs[i])
            xs.append(y.reshape(N, H, dims[i]))
        o_ref, S_ref = oracle.decode_step(xs[0], xs[1], xs[2], host(la[t]), host(beta[t]), S_ref)
        assert float(np.abs(host(o) - o_ref).max()) <= 2e-2, "step %d" % t
        assert rel_fro(host(S), S_ref) <= 1e-2, "step %d" % t
        for i in range(3):
            assert torch.equal(st[i], keep[i]), "input conv state %d written" % i
            if which[i]:
                np.testing.assert_array_equal(host(outs[i]), refs[i])
                st[i] = outs[i]


def test_decode_conv_continues_prefill_conv():
    """fp32: conv + prefill over T-3 tokens, then 3 decode steps with the fused convolution
    continuing from the prefill's conv states == conv + prefill over all T tokens."""
    T, H, d, W = 67, 2, 128, 4
    m = T - 3
    raw, ws = [], []
    for i in range(3):
        x, w, _ = KI.conv_inputs(T, H * d, W, 1, torch.float32, DEV, seed=26, tensor=i, with_state=False)
        raw.append(x)
        ws.append(w)
    inp = make([T], H, d, d, torch.float32, seed=26)
    full = [kda.kda_short_conv_swish(raw[i], ws[i]).view(T, H, d) for i in range(3)]
    inp_all = dict(inp, q=full[0], k=full[1], v=full[2])
    o_all, S_all = run(inp_all)
    states, part = [], []
    for i in range(3):
        st = torch.empty((1, W - 1, H * d), device=DEV)
        part.append(kda.kda_short_conv_swish(raw[i][:m].contiguous(), ws[i], state_out=st).view(m, H, d))
        states.append(st)
    inp_m = dict(q=part[0], k=part[1], v=part[2], log_alpha=inp["log_alpha"][:m], beta=inp["beta"][:m],
                 S0=inp["S0"], cu_seqlens=KI.cu_from_lengths([m], DEV), lengths=[m])
    _, S = run(inp_m)
    for t in range(m, T):
        xs = [raw[i][t:t + 1].view(1, H, d).clone() for i in range(3)]
        cv = [(ws[i], states[i], states[i]) for i in range(3)]
        o = kda.kda_decode_step(xs[0], xs[1], xs[2], inp["log_alpha"][t:t + 1].clone(),
                                inp["beta"][t:t + 1].clone(), S, conv=tuple(cv))
        torch.testing.assert_close(o[0], o_all[t], atol=2e-5, rtol=0)
    torch.testing.assert_close(S, S_all, atol=2e-5, rtol=0)


# ------------------------------- short convolution fused into the prefill ----

def _conv_case(lengths, H, W, which, seed, with_state=True):
    """Raw q, k, v projections with conv taps and initial states for the inputs in `which`."""
    inp = make(lengths, H, 128, 128, torch.bfloat16, seed=seed)
    N = len(lengths)
    convs = []
    for i, name in enumerate(("q", "k", "v")):
        if not which[i]:
            convs.append(None)
            continue
        x, w, st = KI.conv_inputs(sum(lengths), H * 128, W, N, torch.bfloat16, DEV, seed=seed, tensor=i,
                                  with_state=with_state)
        inp[name] = x.view(-1, H, 128)
        convs.append((w, st))
    return inp, convs


def _two_step(inp, convs, out_gate=None):
    """kda_short_conv_swish on each convolved input, then kda_prefill_ex; the states written."""
    x = dict(inp)
    states = []
    for i, name in enumerate(("q", "k", "v")):
        if convs[i] is None:
            states.append(None)
            continue
        w, st = convs[i]
        so = torch.empty((len(inp["lengths"]), w.shape[1] - 1, w.shape[0]), dtype=torch.bfloat16, device=DEV)
        y = kda.kda_short_conv_swish(inp[name].reshape(-1, w.shape[0]), w, inp["cu_seqlens"], state_in=st,
                                     state_out=so)
        x[name] = y.view(inp[name].shape)
        states.append(so)
    o, S_T = run(x, out_gate=out_gate)
    return o, S_T, states, x


def _fused(inp, convs, out_gate=None, in_place=False):
    states, conv = [], []
    for c in convs:
        if c is None:
            states.append(None)
            conv.append(None)
            continue
        w, st = c
        if in_place:
            so = st.clone() if st is not None else torch.zeros((len(inp["lengths"]), w.shape[1] - 1, w.shape[0]),
                                                               dtype=torch.bfloat16, device=DEV)
            conv.append((w, so if st is not None else None, so))
        else:
            so = torch.empty((len(inp["lengths"]), w.shape[1] - 1, w.shape[0]), dtype=torch.bfloat16, device=DEV)
            conv.append((w, st, so))
        states.append(so)
    o, S_T = run(inp, conv=tuple(conv), out_gate=out_gate)
    return o, S_T, states


@pytest.mark.parametrize("lengths,H,W,which", [
    ([300], 4, 4, (True, True, True)),
    ([1, 2, 3, 64, 65, 130, 0, 200], 3, 4, (True, True, True)),
    ([129, 70], 2, 3, (True, False, True)),
    ([64, 5, 190], 2, 2, (False, True, False)),
    ([2048, 700], 4, 1, (True, True, True)),
])
def test_prefill_conv_equals_conv_then_prefill(lengths, H, W, which):
    """kda_prefill_conv (convolution inside the prefill's loads) gives o, S_T and the conv
    states bit for bit equal to kda_short_conv_swish on each input followed by kda_prefill."""
    inp, convs = _conv_case(lengths, H, W, which, seed=40 + W)
    o2, S2, st2, _ = _two_step(inp, convs)
    o1, S1, st1 = _fused(inp, convs)
    assert torch.equal(o1, o2)
    assert torch.equal(S1, S2)
    for a, b in zip(st1, st2):
        if a is not None and W > 1:
            assert torch.equal(a, b)
    assert kda.kda_device_error(reset=True) == 0


def test_prefill_conv_in_place_states_and_no_initial_state():
    """States updated in place (state_in == state_out), and no initial state (zeros)."""
    lengths, H, W = [77, 2, 260], 2, 4
    inp, convs = _conv_case(lengths, H, W, (True, True, True), seed=47)
    o2, S2, st2, _ = _two_step(inp, convs)
    o1, S1, st1 = _fused(inp, convs, in_place=True)
    assert torch.equal(o1, o2) and torch.equal(S1, S2)
    for a, b in zip(st1, st2):
        assert torch.equal(a, b)
    inp0, convs0 = _conv_case(lengths, H, W, (True, True, True), seed=48, with_state=False)
    o2, S2, _, _ = _two_step(inp0, convs0)
    o1, S1, _ = _fused(inp0, convs0)
    assert torch.equal(o1, o2) and torch.equal(S1, S2)


def test_prefill_conv_matches_oracle():
    """Against the oracle: short_conv_swish on each raw input (fp64), then the recurrence."""
    lengths, H, W = [190, 3, 64], 2, 4
    inp, convs = _conv_case(lengths, H, W, (True, True, True), seed=49)
    o, S_T, _ = _fused(inp, convs)
    cu = inp["cu_seqlens"].cpu().numpy().astype(np.int64)
    ref = dict(inp)
    for i, name in enumerate(("q", "k", "v")):
        w, st = convs[i]
        y, _ = oracle.short_conv_swish(host(inp[name]).reshape(-1, H * 128), host(w), cu, host(st))
        ref[name] = torch.from_numpy(y.reshape(-1, H, 128)).to(DEV)
    ref["q"], ref["k"], ref["v"] = (ref[n].to(torch.float64) for n in ("q", "k", "v"))
    check(o, S_T, ref, torch.bfloat16, label="conv in the prefill vs oracle")


def test_prefill_conv_with_output_step():
    """The fused convolution and the fused output step together."""
    lengths, H, W = [150, 40], 3, 4
    inp, convs = _conv_case(lengths, H, W, (True, True, True), seed=50)
    g = torch.Generator(device=DEV)
    g.manual_seed(51)
    og = (torch.randn((sum(lengths), H, 128), generator=g, device=DEV).to(torch.bfloat16),
          1.0 + 0.1 * torch.randn((128,), generator=g, device=DEV), 1e-6)
    o2, S2, _, _ = _two_step(inp, convs, out_gate=og)
    o1, S1, _ = _fused(inp, convs, out_gate=og)
    assert torch.equal(o1, o2) and torch.equal(S1, S2)


def test_prefill_conv_unsupported():
    """fp32 inputs (the CUDA-core path) and windows above 4 are refused, not approximated."""
    inp = make([70], 2, 128, 128, torch.float32, seed=52)
    w = torch.randn(256, 4, device=DEV)
    with pytest.raises(kda.KDAError) as e:
        run(inp, conv=((w, None, None), None, None))
    assert e.value.status == kda.KDA_ERR_UNSUPPORTED
    inp = make([70], 2, 128, 128, torch.bfloat16, seed=52)
    w5 = torch.randn(256, 5, device=DEV)
    with pytest.raises(kda.KDAError) as e:
        run(inp, conv=((w5, None, None), None, None))
    assert e.value.status == kda.KDA_ERR_UNSUPPORTED


# ------------------------------------------------ backward (training) ----
# The CUDA backward (fp32 CUDA cores) against the fp64 oracle's token backward on
# the same input bits: gradients agree to fp32 accumulation error, checked as
# max|g - g_ref| <= 1e-3 * max(1, max|g_ref|) per gradient tensor.

def _bw_inputs(lengths, H, d, dtype, seed):
    inp = make(lengths, H, d, d, dtype, seed=seed)
    T, N = sum(lengths), len(lengths)
    gen = torch.Generator(device=DEV)
    gen.manual_seed(9000 + seed)
    do = torch.randn((T, H, d), generator=gen, device=DEV).to(dtype)
    dST = torch.randn((N, H, d, d), generator=gen, device=DEV)
    return inp, do, dST


def _bw_check(got, inp, do, dST, l2norm=True, label=""):
    assert kda.kda_device_error(reset=True) == 0, label  # no chunk flagged, no wait ran out
    ref = oracle.backward(host(inp["q"]), host(inp["k"]), host(inp["v"]), host(inp["log_alpha"]),
                          host(inp["beta"]), host(do), None if dST is None else host(dST), host(inp["S0"]),
                          inp["cu_seqlens"].cpu().numpy(), l2norm=l2norm)
    for name, g, w in zip(["dq", "dk", "dv", "dlog_alpha", "dbeta", "dS0"], got, ref):
        if g is None:
            continue
        gh = host(g)
        assert np.isfinite(gh).all(), (label, name)
        err = float(np.abs(gh - w).max()) if w.size else 0.0
        assert err <= 1e-3 * max(1.0, float(np.abs(w).max()) if w.size else 0.0), "%s %s: %.3e" % (label, name, err)


@pytest.mark.parametrize("dtype,d", [(torch.float32, 64), (torch.bfloat16, 128), (torch.float32, 128)])
def test_backward_matches_oracle(dtype, d):
    """Partial chunks, an empty and a one-token sequence, S0 and dS_T given."""
    inp, do, dST = _bw_inputs([70, 0, 130, 1], 2, d, dtype, seed=51)
    got = kda.kda_backward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], do, dST, inp["S0"],
                           inp["cu_seqlens"], max_seqlen=130)
    torch.cuda.synchronize()
    _bw_check(got, inp, do, dST, label="backward %s d=%d" % (dtype, d))


def test_backward_no_l2norm_no_state_gradient():
    inp, do, _ = _bw_inputs([100, 37], 1, 64, torch.float32, seed=52)
    got = kda.kda_backward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], do, None, inp["S0"],
                           inp["cu_seqlens"], max_seqlen=100, l2norm=False)
    torch.cuda.synchronize()
    _bw_check(got, inp, do, None, l2norm=False, label="no l2norm")


@pytest.mark.parametrize("dtype,d", [(torch.float32, 64), (torch.bfloat16, 128)])
def test_backward_scalar_gate(dtype, d):
    """One gate per (token, head) (the Gated DeltaNet form): log_alpha [T][H], its gradient
    [T][H], against the oracle's backward with the same per-head gates; varlen with an empty
    and a one-token sequence."""
    inp, do, dST = _bw_inputs([90, 0, 1, 140], 2, d, dtype, seed=53)
    inp["log_alpha"] = inp["log_alpha"][..., 0].contiguous()
    got = kda.kda_backward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], do, dST, inp["S0"],
                           inp["cu_seqlens"], max_seqlen=140)
    torch.cuda.synchronize()
    assert got[3].shape == inp["log_alpha"].shape
    _bw_check(got, inp, do, dST, label="backward scalar gate %s d=%d" % (dtype, d))


def test_backward_flags_strong_decay():
    """A chunk whose decay range exceeds 60 nats (log_alpha about -1.5 per token, 64 rows)
    is not computed by the factorised backward: it sets device error code 2."""
    inp, do, dST = _bw_inputs([100], 1, 64, torch.float32, seed=54)
    inp["log_alpha"] = torch.full_like(inp["log_alpha"], -1.5)
    assert kda.kda_device_error(reset=True) == 0
    kda.kda_backward(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"], do, dST, inp["S0"],
                     inp["cu_seqlens"], max_seqlen=100)
    torch.cuda.synchronize()
    assert kda.kda_device_error(reset=True) == 2
    assert kda.kda_device_error(reset=True) == 0
