"""Pins for the fp64 oracle against what the pages and the mathematics fix.

Each check here computes its expected value by a route other than the
oracle's own three-step update: the worked decay example printed on a page,
closed forms, the gradient-step definition of the delta rule (via autograd),
explicit transition matrices (product / DPLR / GDN / DeltaNet forms), the
read-back property of the delta rule, and the chunkwise form against the
token recurrence. ``test_pins_catch_planted_mistakes`` plants plausible
mistakes in a copy of the oracle's C source and checks that the pins fail.
"""
import os
import shutil
import subprocess

import numpy as np
import pytest
import torch

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))


def rnd(seed, T, H, dk, dv, unit=True, mu=-1.0, N=1):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((T, H, dk))
    k = rng.standard_normal((T, H, dk))
    if unit:
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((T, H, dv))
    la = -np.log1p(np.exp(rng.standard_normal((T, H, dk)) + mu))
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((T, H))))
    S0 = 0.3 * rng.standard_normal((N, H, dk, dv))
    return q, k, v, la, beta, S0


# ---------------------------------------------------------------- pins ----

def pin_worked_decay_example(orc):
    """Page "Kimi Linear — 逐通道的遺忘", section "KDA：把衰減拆到每個通道": (8,6) -> (4,3) / (8,0.6)."""
    rows = []
    with open(os.path.join(HERE, "golden", "channel_decay_example.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                rows.append([np.array(p.split(), dtype=float) for p in line.split("|")])
    assert len(rows) == 2
    for s_before, alpha, s_after in rows:
        S0 = s_before.reshape(1, 1, 2, 1)
        for ch in range(2):
            q = np.zeros((1, 1, 2)); q[0, 0, ch] = 1.0
            k = np.array([[[1.0, 0.0]]])
            v = np.array([[[5.0]]])
            la = np.log(alpha).reshape(1, 1, 2)
            beta = np.zeros((1, 1))  # decay step only: no correction/write
            o, ST = orc.recurrent(q, k, v, la, beta, S0)
            np.testing.assert_allclose(ST.reshape(2), s_after, rtol=0, atol=1e-14)
            np.testing.assert_allclose(o[0, 0, 0], s_after[ch], rtol=0, atol=1e-14)


def pin_pure_decay_closed_form(orc):
    """beta = 0 leaves only per-channel decay: S_T = Diag(exp(sum log alpha)) S0."""
    q, k, v, la, beta, S0 = rnd(1, 9, 2, 5, 3)
    beta[:] = 0.0
    o, ST = orc.recurrent(q, k, v, la, beta, S0)
    G = np.cumsum(la, axis=0)  # [T,H,dk]
    for h in range(2):
        np.testing.assert_allclose(ST[0, h], np.exp(G[-1, h])[:, None] * S0[0, h], rtol=1e-13, atol=1e-15)
        for t in range(9):
            St = np.exp(G[t, h])[:, None] * S0[0, h]
            np.testing.assert_allclose(o[t, h], St.T @ q[t, h], rtol=1e-12, atol=1e-14)


def pin_delta_readback(orc):
    """beta = 1 and a unit key: the updated state reads back exactly v_t at k_t,
    whatever the decay (page "[Kimi-2] Kimi Linear" §2: error ~ 0 once written)."""
    q, k, v, la, beta, S0 = rnd(2, 12, 2, 6, 4)
    beta[:] = 1.0
    q = k.copy()
    o, _ = orc.recurrent(q, k, v, la, beta, S0)
    np.testing.assert_allclose(o, v, rtol=0, atol=1e-12)


def pin_overwrite(orc):
    """Two writes to the same key with beta = 1, alpha = 1: only the last value is read."""
    rng = np.random.default_rng(3)
    kk = rng.standard_normal(5); kk /= np.linalg.norm(kk)
    k = np.stack([kk, kk, kk])[:, None, :]
    v = rng.standard_normal((3, 1, 4))
    la = np.zeros((3, 1, 5))
    beta = np.array([[1.0], [1.0], [0.0]])
    o, _ = orc.recurrent(k.copy(), k, v, la, beta, 0.5 * rng.standard_normal((1, 1, 5, 4)))
    np.testing.assert_allclose(o[2, 0], v[1, 0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(o[1, 0], v[1, 0], rtol=0, atol=1e-12)


def pin_gradient_step(orc):
    """Page "[Kimi-2] Kimi Linear" §2-§3: the update is one gradient step of size beta_t on
    1/2 ||S~^T k_t - v_t||^2 taken at the decayed state S~ = Diag(alpha_t) S_{t-1}.
    The gradient comes from torch autograd, not from a closed form."""
    T, dk, dv = 10, 5, 4
    q, k, v, la, beta, S0 = rnd(4, T, 1, dk, dv)
    o, ST = orc.recurrent(q, k, v, la, beta, S0)
    S = torch.tensor(S0[0, 0])
    for t in range(T):
        St = (torch.exp(torch.tensor(la[t, 0]))[:, None] * S).detach().requires_grad_(True)
        kt, vt = torch.tensor(k[t, 0]), torch.tensor(v[t, 0])
        loss = 0.5 * ((St.T @ kt - vt) ** 2).sum()
        (g,) = torch.autograd.grad(loss, St)
        S = (St - float(beta[t, 0]) * g).detach()
        np.testing.assert_allclose(o[t, 0], (S.T @ torch.tensor(q[t, 0])).numpy(), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(ST[0, 0], S.numpy(), rtol=1e-12, atol=1e-13)


def _A(la_t, k_t, b_t):
    return (np.eye(len(k_t)) - b_t * np.outer(k_t, k_t)) @ np.diag(np.exp(la_t))


def pin_unrolled_product_form(orc):
    """Page "[Kimi-2] Kimi Linear" §8: o_t = sum_i [q_t^T (prod_{j=i+1..t} A_j) k_i] v_i,
    read with the write strength beta_i restored and the S0 term added."""
    T, dk, dv = 7, 4, 3
    q, k, v, la, beta, S0 = rnd(5, T, 1, dk, dv)
    o, ST = orc.recurrent(q, k, v, la, beta, S0)
    A = [_A(la[j, 0], k[j, 0], beta[j, 0]) for j in range(T)]

    def prod(i, t):  # A_t A_{t-1} ... A_{i}  (i > t -> identity)
        M = np.eye(dk)
        for j in range(i, t + 1):
            M = A[j] @ M
        return M

    for t in range(T):
        St = prod(0, t) @ S0[0, 0]
        for i in range(t + 1):
            St = St + beta[i, 0] * np.outer(prod(i + 1, t) @ k[i, 0], v[i, 0])
        np.testing.assert_allclose(o[t, 0], St.T @ q[t, 0], rtol=1e-12, atol=1e-13)
        if t == T - 1:
            np.testing.assert_allclose(ST[0, 0], St, rtol=1e-12, atol=1e-13)


def pin_dplr_form(orc):
    """Page "[Kimi-2] Kimi Linear" §4: A_t = D_t - a_t b_t^T with D = Diag(alpha), a = beta k,
    b = alpha * k (both sides tied to the same key)."""
    T, dk, dv = 8, 5, 3
    q, k, v, la, beta, S0 = rnd(6, T, 1, dk, dv)
    o, ST = orc.recurrent(q, k, v, la, beta, S0)
    S = S0[0, 0].copy()
    for t in range(T):
        al = np.exp(la[t, 0])
        A = np.diag(al) - np.outer(beta[t, 0] * k[t, 0], al * k[t, 0])
        S = A @ S + beta[t, 0] * np.outer(k[t, 0], v[t, 0])
        np.testing.assert_allclose(o[t, 0], S.T @ q[t, 0], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(ST[0, 0], S, rtol=1e-12, atol=1e-13)


def pin_gdn_special_case(orc):
    """Channel-constant alpha reduces KDA to Gated DeltaNet, page "[Kimi-2] Kimi Linear" §3:
    S_t = alpha_t (I - beta_t k k^T) S_{t-1} + beta_t k v^T."""
    T, dk, dv = 9, 4, 6
    q, k, v, la, beta, S0 = rnd(7, T, 1, dk, dv)
    la[:] = la[:, :, :1]
    o, ST = orc.recurrent(q, k, v, la, beta, S0)
    S = S0[0, 0].copy()
    for t in range(T):
        a = np.exp(la[t, 0, 0])
        S = a * (np.eye(dk) - beta[t, 0] * np.outer(k[t, 0], k[t, 0])) @ S + beta[t, 0] * np.outer(k[t, 0], v[t, 0])
        np.testing.assert_allclose(o[t, 0], S.T @ q[t, 0], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(ST[0, 0], S, rtol=1e-12, atol=1e-13)


def pin_deltanet_special_case(orc):
    """alpha = 1 reduces KDA to DeltaNet, page "[Kimi-2] Kimi Linear" §2:
    S_t = S_{t-1} + beta_t k_t (v_t - S_{t-1}^T k_t)^T."""
    T, dk, dv = 9, 6, 5
    q, k, v, la, beta, S0 = rnd(8, T, 1, dk, dv)
    la[:] = 0.0
    o, ST = orc.recurrent(q, k, v, la, beta, S0)
    S = S0[0, 0].copy()
    for t in range(T):
        S = S + beta[t, 0] * np.outer(k[t, 0], v[t, 0] - S.T @ k[t, 0])
        np.testing.assert_allclose(o[t, 0], S.T @ q[t, 0], rtol=1e-12, atol=1e-13)


def pin_l2norm(orc):
    """Page "[Kimi-2] Kimi Linear" §6.2: q, k are L2-normalised, so scaling them changes nothing."""
    q, k, v, la, beta, S0 = rnd(9, 11, 2, 5, 3)
    o1, S1 = orc.recurrent(q, k, v, la, beta, S0)
    sc = np.random.default_rng(10).uniform(0.1, 7.0, size=(11, 2, 1))
    o2, S2 = orc.recurrent(q * sc, k * sc[::-1], v, la, beta, S0)
    np.testing.assert_allclose(o2, o1, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(S2, S1, rtol=1e-12, atol=1e-13)
    o3, S3 = orc.recurrent(q, k, v, la, beta, S0, l2norm=False)
    np.testing.assert_allclose(o3, o1, rtol=1e-12, atol=1e-13)


def pin_decode_step(orc):
    """Page "[Kimi-2] Kimi Linear" §5: a decode step is one token of the same recurrence."""
    N, H, dk, dv = 3, 2, 5, 4
    q, k, v, la, beta, S0 = rnd(11, N, H, dk, dv, N=N)
    o, S1 = orc.decode_step(q, k, v, la, beta, S0)
    for s in range(N):
        o_r, S_r = orc.recurrent(q[s:s + 1], k[s:s + 1], v[s:s + 1], la[s:s + 1], beta[s:s + 1], S0[s:s + 1])
        np.testing.assert_allclose(o[s], o_r[0], rtol=1e-14, atol=1e-15)
        np.testing.assert_allclose(S1[s], S_r[0], rtol=1e-14, atol=1e-15)


def pin_chunkwise_equals_recurrent(orc):
    """Page "[Kimi-2] Kimi Linear" §5: the chunkwise form reaches the recurrence's result."""
    lengths = [1, 63, 64, 65, 150]
    cu = np.cumsum([0] + lengths)
    q, k, v, la, beta, S0 = rnd(12, int(cu[-1]), 2, 8, 6, N=len(lengths))
    o_r, S_r = orc.recurrent(q, k, v, la, beta, S0, cu)
    for C in (1, 3, 16, 64):
        o_c, S_c = orc.chunkwise(q, k, v, la, beta, S0, cu, chunk=C)
        np.testing.assert_allclose(o_c, o_r, rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(S_c, S_r, rtol=1e-11, atol=1e-12)


ALL_PINS = [pin_worked_decay_example, pin_pure_decay_closed_form, pin_delta_readback,
            pin_overwrite, pin_gradient_step, pin_unrolled_product_form, pin_dplr_form,
            pin_gdn_special_case, pin_deltanet_special_case, pin_l2norm, pin_decode_step,
            pin_chunkwise_equals_recurrent]


@pytest.mark.parametrize("pin", ALL_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin(oracle)


# ------------------------------------------------------ structural tests ----

def test_varlen_packing_equals_separate_calls():
    lengths = [5, 1, 17, 64, 70]
    cu = np.cumsum([0] + lengths)
    q, k, v, la, beta, S0 = rnd(13, int(cu[-1]), 3, 6, 7, N=len(lengths))
    for fn in (oracle.recurrent, lambda *a, **kw: oracle.chunkwise(*a, chunk=16, **kw)):
        o, ST = fn(q, k, v, la, beta, S0, cu)
        for s in range(len(lengths)):
            a, b = cu[s], cu[s + 1]
            o1, S1 = oracle.recurrent(q[a:b], k[a:b], v[a:b], la[a:b], beta[a:b], S0[s:s + 1])
            np.testing.assert_allclose(o[a:b], o1, rtol=1e-11, atol=1e-12)
            np.testing.assert_allclose(ST[s], S1[0], rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("t0", [1, 37, 64, 100])
def test_split_continuity(t0):
    """prefill(x[0:T]) == prefill(x[t0:T], S0 = prefill(x[0:t0]).S_T) (chunk-boundary state)."""
    T = 160
    q, k, v, la, beta, S0 = rnd(14, T, 2, 8, 8)
    o, ST = oracle.chunkwise(q, k, v, la, beta, S0, chunk=64)
    oa, Sa = oracle.chunkwise(q[:t0], k[:t0], v[:t0], la[:t0], beta[:t0], S0, chunk=64)
    ob, Sb = oracle.chunkwise(q[t0:], k[t0:], v[t0:], la[t0:], beta[t0:], Sa, chunk=64)
    np.testing.assert_allclose(np.concatenate([oa, ob]), o, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(Sb, ST, rtol=1e-11, atol=1e-12)


def test_strong_decay_chunkwise_finite():
    """log alpha far below what exp(+-G) factorisations survive: chunkwise stays exact."""
    q, k, v, la, beta, S0 = rnd(15, 130, 1, 8, 4)
    la[:] = -np.abs(la) * 40.0
    o_r, S_r = oracle.recurrent(q, k, v, la, beta, S0)
    o_c, S_c = oracle.chunkwise(q, k, v, la, beta, S0, chunk=64)
    assert np.isfinite(o_c).all()
    np.testing.assert_allclose(o_c, o_r, rtol=1e-11, atol=1e-12)


def test_state_norm_bounded():
    """Invariant: with unit k, beta in [0,1] and alpha in (0,1] the transition is a
    contraction (||A_t||_2 <= 1), so ||S_t||_F <= ||S0||_F + sum_t beta_t ||v_t||."""
    q, k, v, la, beta, S0 = rnd(16, 200, 1, 6, 5, mu=-4.0)
    o, ST = oracle.recurrent(q, k, v, la, beta, S0)
    bound = np.linalg.norm(S0) + np.sum(beta[:, 0] * np.linalg.norm(v[:, 0], axis=-1))
    assert np.linalg.norm(ST) <= bound
    for t in range(20):
        A = _A(la[t, 0], k[t, 0], beta[t, 0])
        assert np.linalg.norm(A, 2) <= 1.0 + 1e-12


def test_threads_do_not_change_results():
    lengths = [40, 90]
    cu = np.cumsum([0] + lengths)
    q, k, v, la, beta, S0 = rnd(17, int(cu[-1]), 4, 8, 8, N=2)
    o1, S1 = oracle.recurrent(q, k, v, la, beta, S0, cu, threads=1)
    o2, S2 = oracle.recurrent(q, k, v, la, beta, S0, cu, threads=5)
    assert np.array_equal(o1, o2) and np.array_equal(S1, S2)


# ---------------------------------------------- planted-mistake check ----

class _Orc:
    """The oracle's Python wrapper bound to another build of its C source."""

    def __init__(self, lib):
        self.lib = lib

    def _call(self, fn, *a, **kw):
        saved = oracle._lib
        oracle._lib = self.lib
        try:
            return fn(*a, **kw)
        finally:
            oracle._lib = saved

    def recurrent(self, *a, **kw):
        return self._call(oracle.recurrent, *a, **kw)

    def chunkwise(self, *a, **kw):
        return self._call(oracle.chunkwise, *a, **kw)

    def decode_step(self, *a, **kw):
        return self._call(oracle.decode_step, *a, **kw)


_O_BLOCK = """    /* o_t = S_t^T q_t. */
    for (int j = 0; j < dv; ++j) o[j] = 0.0;
    for (int i = 0; i < dk; ++i) {
        const double *row = S + (size_t)i * dv;
        for (int j = 0; j < dv; ++j) o[j] += row[j] * qn[i];
    }
"""
_DECAY_MARK = "    /* S~ = Diag(alpha_t) S_{t-1}"

MUTANTS = {
    "sign_of_correction": [("y[j] = beta * (v[j] - y[j]);", "y[j] = beta * (v[j] + y[j]);")],
    "dropped_beta": [("y[j] = beta * (v[j] - y[j]);", "y[j] = (v[j] - y[j]);")],
    "gate_not_exponentiated": [("double a = exp(la[i]);", "double a = 1.0 + la[i];")],
    "gate_index_dropped": [("double a = exp(la[i]);", "double a = exp(la[0]);")],
    "write_along_query": [("row[j] += kn[i] * y[j];", "row[j] += qn[i] * y[j];")],
    "read_before_update": [(_O_BLOCK, ""), (_DECAY_MARK, _O_BLOCK + _DECAY_MARK)],
    "no_l2norm": [("    if (!on) {\n        memcpy", "    if (1) {\n        memcpy")],
    "chunk_solve_without_beta": [("for (int c = 0; c < wx; ++c) xr[c] *= b;", "")],
    "chunk_exponent_sign": [("double e = exp(G[(size_t)r * dk + c] - G[(size_t)i * dk + c]);",
                             "double e = exp(G[(size_t)i * dk + c] - G[(size_t)r * dk + c]);")],
    "chunk_P_without_diagonal": [("P[(size_t)r * C + i] = (i <= r) ? p : 0.0;",
                                  "P[(size_t)r * C + i] = (i < r) ? p : 0.0;")],
    "chunk_state_not_decayed": [("double acc = exp(gl[c]) * S[(size_t)c * dv + j];",
                                 "double acc = S[(size_t)c * dv + j];")],
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistakes(name, tmp_path):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    src = open(os.path.join(os.path.dirname(oracle.__file__), "kda_oracle.c")).read()
    for old, new in MUTANTS[name]:
        assert src.count(old) == 1, (name, old)
        src = src.replace(old, new)
    c = tmp_path / "mutant.c"
    c.write_text(src)
    so = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-pthread", "-o",
                           str(so), str(c), "-lm"])
    orc = _Orc(oracle.load_library(str(so)))
    failed = []
    for pin in ALL_PINS:
        try:
            pin(orc)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, "planted mistake %r passed every pin" % name


# ------------------------------------------------ output gate (§6.3) ----
# oracle.output_gate: head-wise RMSNorm of o_t, then a sigmoid gate ("[Kimi-2]
# Kimi Linear" §6 and §6.3). Pinned to hand arithmetic and to properties the
# definition fixes; each planted mistake below must fail at least one pin.

def og_pin_worked_example(f):
    # o = (3, 4): mean square 12.5; w = (2, 1); g = (0, ln 3): sigmoid = (1/2, 3/4).
    # y = (3 * 2 * 1/2, 4 * 1 * 3/4) / sqrt(12.5) = (3, 3) / sqrt(12.5).
    y = f(np.array([[3.0, 4.0]]), np.array([[0.0, np.log(3.0)]]), np.array([2.0, 1.0]), 0.0)
    np.testing.assert_allclose(y, [[3.0 / np.sqrt(12.5), 3.0 / np.sqrt(12.5)]], rtol=1e-14)


def og_pin_unit_rms(f):
    # w = 1 and a saturated gate leave the RMSNorm, whose mean square is 1 (eps = 0).
    o = np.random.default_rng(1).normal(size=(5, 3, 16)) * 7.0
    y = f(o, np.full_like(o, 60.0), np.ones(16), 0.0)
    np.testing.assert_allclose(np.mean(y * y, axis=-1), 1.0, rtol=1e-12)


def og_pin_scale_invariance(f):
    rng = np.random.default_rng(2)
    o, g, w = rng.normal(size=(4, 2, 8)), rng.normal(size=(4, 2, 8)), rng.normal(size=8)
    np.testing.assert_allclose(f(3.5 * o, g, w, 0.0), f(o, g, w, 0.0), rtol=1e-12)


def og_pin_heads_independent(f):
    # head-wise: a head's output does not depend on the other heads' values
    rng = np.random.default_rng(3)
    o, g, w = rng.normal(size=(4, 2, 8)), rng.normal(size=(4, 2, 8)), rng.normal(size=8)
    o2 = o.copy()
    o2[:, 1] *= 100.0
    np.testing.assert_allclose(f(o2, g, w, 1e-6)[:, 0], f(o, g, w, 1e-6)[:, 0], rtol=1e-14)


def og_pin_zero_row(f):
    # eps keeps an all-zero row finite (and zero)
    y = f(np.zeros((2, 8)), np.zeros((2, 8)), np.ones(8), 1e-6)
    assert np.all(y == 0.0)


OG_PINS = [og_pin_worked_example, og_pin_unit_rms, og_pin_scale_invariance,
           og_pin_heads_independent, og_pin_zero_row]


@pytest.mark.parametrize("pin", OG_PINS, ids=lambda p: p.__name__)
def test_output_gate_pin(pin):
    pin(oracle.output_gate)


def _og_mutant(kind):
    def f(o, g, w, eps):
        o, g, w = (np.asarray(x, dtype=np.float64) for x in (o, g, w))
        ms = np.mean(o * o, axis=-1, keepdims=True)
        if kind == "sum_not_mean":
            ms = np.sum(o * o, axis=-1, keepdims=True)
        if kind == "across_heads":
            ms = np.mean(o * o, axis=(-2, -1), keepdims=True) if o.ndim > 2 else ms
        if kind == "no_eps":
            eps = 0.0
        gate = np.tanh(g) if kind == "tanh_gate" else 1.0 / (1.0 + np.exp(-g))
        if kind == "no_weight":
            w = np.ones_like(w)
        with np.errstate(invalid="ignore", divide="ignore"):
            return o / np.sqrt(ms + eps) * w * gate
    return f


@pytest.mark.parametrize("kind", ["sum_not_mean", "across_heads", "no_eps", "tanh_gate", "no_weight"])
def test_output_gate_pins_catch_planted_mistakes(kind):
    f = _og_mutant(kind)
    failed = 0
    for pin in OG_PINS:
        try:
            pin(f)
        except AssertionError:
            failed += 1
    assert failed > 0, kind


# ------------------------------------------ short conv + Swish (§6.1) ----
# oracle.short_conv_swish / short_conv_step: a causal short convolution over the
# token axis, then Swish ("[Kimi-2] Kimi Linear" §6 and §6.1; "Kimi Delta
# Attention：把遗忘门做到每个通道", the pre-processing of q, k). Pinned to a library
# convolution, closed forms and the properties "causal" and "per sequence" fix;
# each planted mistake below must fail at least one pin.

def _silu_ref(z):
    from scipy.special import expit
    return z * expit(z)


def sc_pin_numpy_convolve(f):
    # one sequence from zero history: per channel, the pre-activation is the
    # library's full convolution with the taps reversed, cut to the first T outputs
    rng = np.random.default_rng(11)
    x, w = rng.normal(size=(23, 5)), rng.normal(size=(5, 4))
    y, _ = f(x, w)
    for c in range(5):
        z = np.convolve(x[:, c], w[c, ::-1])[:23]
        np.testing.assert_allclose(y[:, c], _silu_ref(z), rtol=1e-12, atol=1e-14)


def sc_pin_impulse(f):
    # a unit impulse at t0 gives silu(w[c, W-1-j]) at t0 + j (j < W), zero elsewhere
    W, t0 = 4, 5
    w = np.array([[0.5, -1.0, 2.0, 3.0], [1.5, 0.25, -0.75, 1.0]])
    x = np.zeros((12, 2))
    x[t0] = 1.0
    y, _ = f(x, w)
    want = np.zeros((12, 2))
    for j in range(W):
        want[t0 + j] = _silu_ref(w[:, W - 1 - j])
    np.testing.assert_allclose(y, want, rtol=1e-14, atol=0.0)


def sc_pin_swish_values(f):
    # W = 1, w = 1: y = silu(x); silu(0) = 0, silu(1) = 1/(1+e^-1), silu(-1) = -1/(1+e)
    y, st = f(np.array([[0.0], [1.0], [-1.0]]), np.ones((1, 1)))
    np.testing.assert_allclose(y[:, 0], [0.0, 1.0 / (1.0 + np.exp(-1.0)), -1.0 / (1.0 + np.e)], rtol=1e-15)
    assert st.shape == (1, 0, 1)


def sc_pin_sequences_independent(f):
    # varlen: equal to each sequence run alone (nothing crosses a boundary)
    rng = np.random.default_rng(12)
    lens = [3, 1, 9, 2]
    cu = np.concatenate([[0], np.cumsum(lens)])
    x, w = rng.normal(size=(cu[-1], 3)), rng.normal(size=(3, 3))
    s0 = rng.normal(size=(4, 2, 3))
    y, st = f(x, w, cu, s0)
    for s in range(4):
        ys, sts = f(x[cu[s]:cu[s + 1]], w, None, s0[s:s + 1])
        np.testing.assert_allclose(y[cu[s]:cu[s + 1]], ys, rtol=1e-14, atol=0.0)
        np.testing.assert_allclose(st[s], sts[0], rtol=0, atol=0)


def sc_pin_continuation(f):
    # a sequence split anywhere, the second part started from the first part's
    # final state, gives the same outputs and final state (also splits shorter than W-1)
    rng = np.random.default_rng(13)
    x, w = rng.normal(size=(17, 4)), rng.normal(size=(4, 4))
    y, st = f(x, w)
    for t1 in (1, 2, 7):
        y1, st1 = f(x[:t1], w)
        y2, st2 = f(x[t1:], w, None, st1)
        np.testing.assert_allclose(np.concatenate([y1, y2]), y, rtol=1e-14, atol=0.0)
        np.testing.assert_allclose(st2, st, rtol=0, atol=0)


def sc_pin_state_holds_last_inputs(f):
    # the final state is the last W-1 raw inputs, oldest first
    x = np.arange(10, dtype=np.float64).reshape(5, 2)
    _, st = f(x, np.ones((2, 3)))
    np.testing.assert_array_equal(st[0], x[3:5])


SC_PINS = [sc_pin_numpy_convolve, sc_pin_impulse, sc_pin_swish_values, sc_pin_sequences_independent,
           sc_pin_continuation, sc_pin_state_holds_last_inputs]


@pytest.mark.parametrize("pin", SC_PINS, ids=lambda p: p.__name__)
def test_short_conv_pin(pin):
    pin(oracle.short_conv_swish)


def test_short_conv_decode_steps_match_prefill():
    # T single-token steps on a carried state equal the sequence form
    rng = np.random.default_rng(14)
    x, w, s0 = rng.normal(size=(3, 11, 6)), rng.normal(size=(6, 4)), rng.normal(size=(3, 3, 6))
    cu = np.arange(0, 34, 11)
    y, st = oracle.short_conv_swish(x.reshape(33, 6), w, cu, s0)
    state = s0.copy()
    for t in range(11):
        yt, state = oracle.short_conv_step(x[:, t], w, state)
        np.testing.assert_allclose(yt, y.reshape(3, 11, 6)[:, t], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(state, st, rtol=0, atol=0)


def _sc_mutant(kind):
    def f(x, w, cu_seqlens=None, state0=None):
        x, w = np.asarray(x, dtype=np.float64), np.asarray(w, dtype=np.float64)
        T, C = x.shape
        W = w.shape[1]
        cu = np.array([0, T]) if cu_seqlens is None else np.asarray(cu_seqlens)
        if kind == "leaks_across_sequences":
            cu = np.array([0, T])
        N = len(cu) - 1
        y, st = np.zeros((T, C)), np.zeros((N, W - 1, C))
        for s in range(N):
            bos, eos = int(cu[s]), int(cu[s + 1])
            hist = np.zeros((W - 1, C))
            if state0 is not None and kind != "ignores_state":
                hist = np.asarray(state0[s], dtype=np.float64)
            xs = np.concatenate([hist, x[bos:eos]])
            L = eos - bos
            for t in range(L):
                taps = w[:, ::-1] if kind == "taps_reversed" else w
                z = sum(taps[:, j] * xs[t + j] for j in range(W))
                if kind == "off_by_one":
                    z = sum(taps[:, j] * xs[t + j - 1] for j in range(W)) if t > 0 else z
                y[bos + t] = z if kind == "no_swish" else z / (1.0 + np.exp(-z))
            st[s] = xs[L:L + W - 1] if kind != "state_newest_first" else xs[L:L + W - 1][::-1]
        if kind == "leaks_across_sequences" and cu_seqlens is not None:
            st = np.repeat(st, len(cu_seqlens) - 1, axis=0)
        return y, st
    return f


@pytest.mark.parametrize("kind", ["taps_reversed", "no_swish", "off_by_one", "ignores_state",
                                  "leaks_across_sequences", "state_newest_first"])
def test_short_conv_pins_catch_planted_mistakes(kind):
    f = _sc_mutant(kind)
    failed = 0
    for pin in SC_PINS:
        try:
            pin(f)
        except (AssertionError, ValueError, IndexError):
            failed += 1
    assert failed > 0, kind


# ------------------------------------------- backward (training, §5) ----
# oracle.backward: gradients of L = <do, o> + <dS_T, S_T> through the recurrence,
# derived by hand (the pages give no backward). Pinned to central finite
# differences of oracle.recurrent (itself pinned above) and to torch autograd of
# a separately written forward; each planted mistake below must fail the
# finite-difference pin.

def _bw_case(seed, scalar_gate=False):
    rng = np.random.default_rng(seed)
    T, H, dk, dv = 7, 2, 3, 2
    cu = np.array([0, 4, 4, 7])  # an empty sequence in the middle
    q, k = rng.normal(size=(T, H, dk)), rng.normal(size=(T, H, dk))
    v = rng.normal(size=(T, H, dv))
    la = -np.abs(rng.normal(size=(T, H) if scalar_gate else (T, H, dk))) * 0.4
    b = 1.0 / (1.0 + np.exp(-rng.normal(size=(T, H))))
    S0 = rng.normal(size=(3, H, dk, dv))
    Wo, WS = rng.normal(size=(T, H, dv)), rng.normal(size=(3, H, dk, dv))
    return dict(q=q, k=k, v=v, la=la, b=b, S0=S0, cu=cu, Wo=Wo, WS=WS)


def _bw_fd(c, l2norm=True):
    """Central finite differences of L through oracle.recurrent, for every input."""
    names = ["q", "k", "v", "la", "b", "S0"]

    def loss(vals):
        la = vals["la"]
        if la.ndim == 2:  # one gate per (token, head): the same gate on every key channel
            la = np.repeat(la[..., None], c["q"].shape[2], axis=-1)
        o, ST = oracle.recurrent(vals["q"], vals["k"], vals["v"], la, vals["b"], vals["S0"],
                                 c["cu"], l2norm=l2norm, threads=1)
        return float((o * c["Wo"]).sum() + (ST * c["WS"]).sum())

    out = []
    h = 1e-6
    for n in names:
        x = c[n]
        g = np.zeros_like(x)
        for idx in np.ndindex(x.shape):
            vals = {m: c[m] for m in names}
            xp, xm = x.copy(), x.copy()
            xp[idx] += h
            xm[idx] -= h
            vals[n] = xp
            lp = loss(vals)
            vals[n] = xm
            g[idx] = (lp - loss(vals)) / (2 * h)
        out.append(g)
    return out


def _bw_run(f, c, l2norm=True):
    return f(c["q"], c["k"], c["v"], c["la"], c["b"], c["Wo"], c["WS"], c["S0"], c["cu"], l2norm=l2norm)


@pytest.mark.parametrize("scalar_gate,l2norm", [(False, True), (True, True), (False, False)])
def test_backward_matches_finite_differences(scalar_gate, l2norm):
    c = _bw_case(31 + scalar_gate, scalar_gate)
    fd = _bw_fd(c, l2norm)
    for name, g, want in zip(["q", "k", "v", "log_alpha", "beta", "S0"], _bw_run(oracle.backward, c, l2norm), fd):
        np.testing.assert_allclose(g, want, rtol=0, atol=2e-7 * max(1.0, np.abs(want).max()), err_msg=name)


def test_backward_matches_torch_autograd():
    c = _bw_case(35)
    t = {n: torch.tensor(c[n], dtype=torch.float64, requires_grad=True) for n in ["q", "k", "v", "la", "b", "S0"]}
    loss = torch.zeros((), dtype=torch.float64)
    for s in range(len(c["cu"]) - 1):
        for h in range(c["q"].shape[1]):
            S = t["S0"][s, h]
            for i in range(int(c["cu"][s]), int(c["cu"][s + 1])):
                qh = t["q"][i, h] / t["q"][i, h].norm()
                kh = t["k"][i, h] / t["k"][i, h].norm()
                Sd = torch.exp(t["la"][i, h])[:, None] * S
                u = t["b"][i, h] * (t["v"][i, h] - Sd.T @ kh)
                S = Sd + torch.outer(kh, u)
                loss = loss + (S.T @ qh) @ torch.tensor(c["Wo"][i, h])
            loss = loss + (S * torch.tensor(c["WS"][s, h])).sum()
    loss.backward()
    for name, g in zip(["q", "k", "v", "la", "b", "S0"], _bw_run(oracle.backward, c)):
        np.testing.assert_allclose(g, t[name].grad.numpy(), rtol=1e-11, atol=1e-12, err_msg=name)


def test_backward_beta_zero_closed_form():
    # beta = 0: no write, so dL/dv = 0 and, without a normalisation, dL/dq_t = S_t do_t
    # with S_t = Diag(exp(sum of log_alpha)) S0 (the pure decay closed form)
    c = _bw_case(36)
    c["b"] = np.zeros_like(c["b"])
    gq, gk, gv, gla, gb, gS0 = _bw_run(oracle.backward, c, l2norm=False)
    assert np.all(gv == 0.0)
    s, h, t = 2, 1, 5  # token 5 of sequence 2 (tokens 4..6)
    St = np.exp(c["la"][4:t + 1, h].sum(axis=0))[:, None] * c["S0"][s, h]
    np.testing.assert_allclose(gq[t, h], St @ c["Wo"][t, h], rtol=1e-13)


_BW_MUTANTS = {
    "decay_not_propagated": ("G = a[:, None] * dSt", "G = dSt"),
    "write_sign": ("dSt = G - b[t, h] * np.outer(kh[t, h], du)", "dSt = G + b[t, h] * np.outer(kh[t, h], du)"),
    "dk_read_term_dropped": ("dkh[t, h] = G @ u - b[t, h] * (St @ du)", "dkh[t, h] = G @ u"),
    "gate_uses_new_state": ("g = a * np.sum(dSt * Sp, axis=1)", "g = a * np.sum(dSt * Sn, axis=1)"),
    "dbeta_wrong_factor": ("gb[t, h] = du @ r", "gb[t, h] = du @ u"),
    "readout_before_update": ("dqh[t, h] = Sn @ do[t, h]", "dqh[t, h] = Sp @ do[t, h]"),
    "no_norm_backward": ("gq, gk = _l2_back(q, dqh, eps), _l2_back(k, dkh, eps)", "gq, gk = dqh / nq, dkh / nk"),
}


@pytest.mark.parametrize("name", sorted(_BW_MUTANTS))
def test_backward_pins_catch_planted_mistakes(name):
    import inspect
    import textwrap
    src = textwrap.dedent(inspect.getsource(oracle.backward))
    old, new = _BW_MUTANTS[name]
    assert src.count(old) == 1, name
    ns = dict(vars(oracle))
    exec(compile(src.replace(old, new), "<mutant>", "exec"), ns)
    c = _bw_case(37)
    fd = _bw_fd(c)
    bad = False
    for g, want in zip(_bw_run(ns["backward"], c), fd):
        if not np.allclose(g, want, rtol=0, atol=2e-7 * max(1.0, np.abs(want).max())):
            bad = True
    assert bad, "planted mistake %r passed the finite-difference pin" % name


@pytest.mark.parametrize("chunk", [1, 16, 64])
def test_chunkwise_backward_equals_token_backward(chunk):
    # the chunked algebra (partial last chunks, an empty sequence) gives the token
    # form's gradients to rounding
    rng = np.random.default_rng(38)
    T, H, dk, dv = 150, 2, 8, 6
    cu = np.array([0, 70, 70, 150])
    q, k = rng.normal(size=(T, H, dk)), rng.normal(size=(T, H, dk))
    v = rng.normal(size=(T, H, dv))
    la = -np.log1p(np.exp(rng.normal(-3.0, 1.0, size=(T, H, dk))))
    b = 1.0 / (1.0 + np.exp(-rng.normal(size=(T, H))))
    S0, dST = rng.normal(size=(3, H, dk, dv)), rng.normal(size=(3, H, dk, dv))
    do = rng.normal(size=(T, H, dv))
    want = oracle.backward(q, k, v, la, b, do, dST, S0, cu)
    got = oracle.chunkwise_backward(q, k, v, la, b, do, dST, S0, cu, chunk=chunk)
    for name, g, w in zip(["q", "k", "v", "log_alpha", "beta", "S0"], got, want):
        np.testing.assert_allclose(g, w, rtol=0, atol=1e-12 * max(1.0, np.abs(w).max()), err_msg=name)


# ------------------------------------------------ segments of a sequence ----
# Each token's update is affine in the state ([P1] §3), so a segment of a sequence maps its entry
# state to its exit state by S_out = M S_in + B; oracle.segmented forms every segment's map from a
# zero state, composes them in order and replays each segment from its true entry state.

def _seg_case(seed, scalar_gate=False):
    rng = np.random.default_rng(seed)
    T, H, dk, dv = 150, 2, 6, 5
    cu = np.array([0, 70, 70, 150])
    q, k = rng.normal(size=(T, H, dk)), rng.normal(size=(T, H, dk))
    v = rng.normal(size=(T, H, dv))
    la = -np.log1p(np.exp(rng.normal(-3.0, 1.0, size=(T, H) if scalar_gate else (T, H, dk))))
    b = 1.0 / (1.0 + np.exp(-rng.normal(size=(T, H))))
    S0 = rng.normal(size=(3, H, dk, dv))
    return q, k, v, la, b, S0, cu


@pytest.mark.parametrize("cuts", [(), (37,), (1, 2, 3), (37, 38, 65, 79), (64,), (500,)])
@pytest.mark.parametrize("scalar_gate", [False, True])
def test_segmented_equals_recurrent(cuts, scalar_gate):
    """Cuts anywhere (on and off 64-token chunk edges, one-token segments, past the end),
    varlen with an empty sequence, per-channel and per-head gates."""
    q, k, v, la, b, S0, cu = _seg_case(61 + len(cuts), scalar_gate)
    la_full = la[..., None] * np.ones(q.shape[2]) if scalar_gate else la  # a per-head gate, broadcast
    o_ref, S_ref = oracle.recurrent(q, k, v, la_full, b, S0, cu)
    o, S = oracle.segmented(q, k, v, la, b, S0, cu, cuts=cuts)
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-12 * max(1.0, np.abs(o_ref).max()))
    np.testing.assert_allclose(S, S_ref, rtol=0, atol=1e-12 * max(1.0, np.abs(S_ref).max()))


def test_segment_map_closed_forms():
    rng = np.random.default_rng(62)
    dk, dv = 5, 4
    k, v = rng.normal(size=(1, dk)), rng.normal(size=(1, dv))
    la, b = -rng.uniform(0.0, 1.0, size=(1, dk)), np.array([0.7])
    M, B = oracle.segment_map(k, v, la, b)
    kh = k[0] / np.linalg.norm(k[0])
    np.testing.assert_allclose(M, (np.eye(dk) - 0.7 * np.outer(kh, kh)) @ np.diag(np.exp(la[0])), atol=1e-14)
    np.testing.assert_allclose(B, 0.7 * np.outer(kh, v[0]), atol=1e-14)
    # beta = 0: a pure decay, M = Diag(exp(sum log_alpha)), B = 0
    k, v = rng.normal(size=(9, dk)), rng.normal(size=(9, dv))
    la = -rng.uniform(0.0, 0.5, size=(9, dk))
    M, B = oracle.segment_map(k, v, la, np.zeros(9))
    np.testing.assert_allclose(M, np.diag(np.exp(la.sum(0))), atol=1e-14)
    assert np.abs(B).max() == 0


@pytest.mark.parametrize("mistake", ["map order", "drop B", "compose order"])
def test_segment_pins_catch_planted_mistakes(mistake):
    """A map multiplied in the wrong order, a dropped B, or segments composed in the wrong
    order each break the equality with the recurrence."""
    q, k, v, la, b, S0, cu = _seg_case(63)
    _, S_ref = oracle.recurrent(q, k, v, la, b, S0, cu)
    s, h = 0, 1
    bos, eos = int(cu[s]), int(cu[s + 1])
    edges = [bos, bos + 23, bos + 51, eos]
    kh = k[:, h] / np.linalg.norm(k[:, h], axis=-1, keepdims=True)
    maps = []
    for e0, e1 in zip(edges[:-1], edges[1:]):
        if mistake == "map order":  # M = M A instead of A M
            M, B = np.eye(k.shape[2]), np.zeros((k.shape[2], v.shape[2]))
            for t in range(e0, e1):
                A = (np.eye(k.shape[2]) - b[t, h] * np.outer(kh[t], kh[t])) * np.exp(la[t, h])[None, :]
                M, B = M @ A, A @ B + b[t, h] * np.outer(kh[t], v[t, h])
            maps.append((M, B))
        else:
            maps.append(oracle.segment_map(k[e0:e1, h], v[e0:e1, h], la[e0:e1, h], b[e0:e1, h]))
    if mistake == "compose order":
        maps = maps[::-1]
    S = S0[s, h].copy()
    for M, B in maps:
        S = M @ S + (0.0 if mistake == "drop B" else B)
    assert np.abs(S - S_ref[s, h]).max() > 1e-6


def test_chunk_map_from_the_chunkwise_quantities():
    """The map of one 64-token chunk from the chunkwise quantities a kernel forms
    (G = cumsum log_alpha, g its last row, Kg = K e^G, Kn = K e^-G, Kd = K e^(g-G),
    A = strict_lower(Kg Kn^T), T = (I + Diag(beta) A)^-1 Diag(beta), W = T Kg):
    S' = (Diag(e^g) - Kd^T W) S + Kd^T T V, equal to the token-by-token map."""
    rng = np.random.default_rng(64)
    C, dk, dv = 64, 8, 5
    k, v = rng.normal(size=(C, dk)), rng.normal(size=(C, dv))
    la = -np.log1p(np.exp(rng.normal(-3.0, 1.0, size=(C, dk))))
    b = 1.0 / (1.0 + np.exp(-rng.normal(size=C)))
    M_ref, B_ref = oracle.segment_map(k, v, la, b)
    kh = k / np.linalg.norm(k, axis=1, keepdims=True)
    G = np.cumsum(la, axis=0)
    g = G[-1]
    Kg, Kn, Kd = kh * np.exp(G), kh * np.exp(-G), kh * np.exp(g - G)
    A = np.tril(Kg @ Kn.T, -1)
    T = np.linalg.solve(np.eye(C) + b[:, None] * A, np.diag(b))
    W = T @ Kg
    np.testing.assert_allclose(np.diag(np.exp(g)) - Kd.T @ W, M_ref, atol=1e-12)
    np.testing.assert_allclose(Kd.T @ (T @ v), B_ref, atol=1e-12)
