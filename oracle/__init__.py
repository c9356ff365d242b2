"""fp64 CPU oracle for Kimi Delta Attention (KDA) -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline /
reference leg may import this package. The CUDA library never does, and the
two share no code: this side is plain C (``kda_oracle.c``, compiled with gcc)
plus the numpy marshalling below.

Functions and the passages they follow (pages cited by title and section):

* :func:`recurrent` -- the KDA recurrence token by token, "[Kimi-2] Kimi
  Linear：用 KDA 重写长上下文注意力" §3 (boxed update, three-step form) with the
  §1 readout ``o_t = S_t^T q_t`` and §6.2 L2 normalisation of q, k.
* :func:`chunkwise` -- the same outputs through the chunkwise form of §5 (UT
  transform inside a chunk, state passed between chunks), derived in the C
  source's comment.
* :func:`decode_step` -- one token of the recurrence on a resident state,
  §5 ("S_(t-1) + current token -> S_t + output").
* :func:`output_gate` -- the layer's output step after the recurrence, §6 and
  §6.3 (and "Kimi Linear — 逐通道的遺忘", 其他零件): head-wise RMSNorm of o_t,
  then a product with a sigmoid gate computed from the input.
* :func:`backward` -- gradients of the recurrence's outputs (o and the final
  state) with respect to every input, derived here by reverse-mode
  differentiation of the §3 three-step form token by token (the pages mention
  training but give no backward); pinned to central finite differences of
  :func:`recurrent` and to torch autograd.
* :func:`chunkwise_backward` -- the same gradients through the chunkwise form
  of §5 (a second CPU form: the algebra a chunked GPU backward implements),
  pinned to :func:`backward`.
* :func:`segment_map` / :func:`segmented` -- the recurrence by segments of a
  sequence: each token's update is affine in the state (§3), so a segment maps
  its entry state to its exit state by ``S_out = M S_in + B`` (M the product of
  the tokens' ``(I - beta k k^T) Diag(alpha)``, B the exit state from zero);
  the maps of all segments are independent, composed in order, and each
  segment's outputs then follow from its true entry state (the one-exchange
  form of splitting a long sequence); pinned to :func:`recurrent`.
* :func:`short_conv_swish` / :func:`short_conv_step` -- the layer's step before
  the recurrence, §6 and §6.1 (and "Kimi Delta Attention：把遗忘门做到每个通道",
  进状态之前 q/k 还要过一道预处理): a causal short convolution over the token
  axis, then Swish, on the q, k, v projections (the L2 norm of q, k follows, in
  the recurrence's functions above).

Arrays are ``numpy`` (any real dtype; converted to fp64). Layouts::

    q, k, log_alpha [T, H, dk]   v [T, H, dv]   beta [T, H]
    S0, S_T         [N, H, dk, dv]              cu_seqlens [N+1]
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB = os.path.join(_HERE, "libkda_oracle.so")
_lib = None

_D = ctypes.POINTER(ctypes.c_double)
_I64 = ctypes.POINTER(ctypes.c_int64)


def build(force: bool = False) -> str:
    """Compile ``kda_oracle.c`` into ``libkda_oracle.so`` with gcc (plain -O2)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp.%d" % os.getpid()
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared", "-pthread",
             "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def load_library(path: str | None = None):
    """Load the oracle library (building it first if needed)."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    if _lib is None:
        _lib = _bind(ctypes.CDLL(build()))
    return _lib


def _bind(lib):
    i, d = ctypes.c_int, ctypes.c_double
    lib.kda_oracle_recurrent.argtypes = [_D, _D, _D, _D, _D, _D, _I64, i, i, i, i, i, d, _D, _D, i]
    lib.kda_oracle_chunkwise.argtypes = [_D, _D, _D, _D, _D, _D, _I64, i, i, i, i, i, d, i, _D, _D, i]
    lib.kda_oracle_decode_step.argtypes = [_D, _D, _D, _D, _D, _D, i, i, i, i, i, d, _D]
    for f in (lib.kda_oracle_recurrent, lib.kda_oracle_chunkwise, lib.kda_oracle_decode_step):
        f.restype = ctypes.c_int
    return lib


def _f64(x):
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _p(x):
    return None if x is None else x.ctypes.data_as(_D)


def _prep(q, k, v, log_alpha, beta, S0, cu_seqlens):
    q, k, v, la, b = (_f64(x) for x in (q, k, v, log_alpha, beta))
    T, H, dk = q.shape
    dv = v.shape[2]
    if k.shape != (T, H, dk) or la.shape != (T, H, dk) or v.shape[:2] != (T, H) or b.shape != (T, H):
        raise ValueError("inconsistent shapes")
    cu = np.array([0, T] if cu_seqlens is None else np.asarray(cu_seqlens), dtype=np.int64)
    N = len(cu) - 1
    if cu[-1] != T:
        raise ValueError("cu_seqlens[-1] must equal T")
    if S0 is not None:
        S0 = _f64(S0)
        if S0.shape != (N, H, dk, dv):
            raise ValueError("S0 shape")
    return q, k, v, la, b, S0, cu, T, H, dk, dv, N


def _threads(threads):
    return threads if threads else (os.cpu_count() or 1)


def recurrent(q, k, v, log_alpha, beta, S0=None, cu_seqlens=None, l2norm=True, eps=1e-6,
              threads=None):
    """Token-by-token KDA recurrence in fp64. Returns ``(o [T,H,dv], S_T [N,H,dk,dv])``."""
    q, k, v, la, b, S0, cu, T, H, dk, dv, N = _prep(q, k, v, log_alpha, beta, S0, cu_seqlens)
    o = np.zeros((T, H, dv))
    ST = np.zeros((N, H, dk, dv))
    rc = load_library().kda_oracle_recurrent(
        _p(q), _p(k), _p(v), _p(la), _p(b), _p(S0), cu.ctypes.data_as(_I64), N, H, dk, dv,
        int(bool(l2norm)), float(eps), _p(o), _p(ST), _threads(threads))
    if rc:
        raise RuntimeError("kda_oracle_recurrent failed (%d)" % rc)
    return o, ST


def chunkwise(q, k, v, log_alpha, beta, S0=None, cu_seqlens=None, chunk=64, l2norm=True,
              eps=1e-6, threads=None):
    """Chunkwise (UT-transform) KDA in fp64. Returns ``(o, S_T)`` like :func:`recurrent`."""
    q, k, v, la, b, S0, cu, T, H, dk, dv, N = _prep(q, k, v, log_alpha, beta, S0, cu_seqlens)
    o = np.zeros((T, H, dv))
    ST = np.zeros((N, H, dk, dv))
    rc = load_library().kda_oracle_chunkwise(
        _p(q), _p(k), _p(v), _p(la), _p(b), _p(S0), cu.ctypes.data_as(_I64), N, H, dk, dv,
        int(bool(l2norm)), float(eps), int(chunk), _p(o), _p(ST), _threads(threads))
    if rc:
        raise RuntimeError("kda_oracle_chunkwise failed (%d)" % rc)
    return o, ST


def decode_step(q, k, v, log_alpha, beta, S, l2norm=True, eps=1e-6):
    """One decode step for N sequences: inputs ``[N,H,d]``, state ``[N,H,dk,dv]``.

    Returns ``(o [N,H,dv], S_new [N,H,dk,dv])``; the input ``S`` is not modified.
    """
    q, k, v, la = (_f64(x) for x in (q, k, v, log_alpha))
    b = _f64(beta)
    N, H, dk = q.shape
    dv = v.shape[2]
    Snew = np.array(S, dtype=np.float64, copy=True, order="C")
    if Snew.shape != (N, H, dk, dv) or b.shape != (N, H):
        raise ValueError("inconsistent shapes")
    o = np.zeros((N, H, dv))
    rc = load_library().kda_oracle_decode_step(
        _p(q), _p(k), _p(v), _p(la), _p(b), _p(Snew), N, H, dk, dv, int(bool(l2norm)),
        float(eps), _p(o))
    if rc:
        raise RuntimeError("kda_oracle_decode_step failed (%d)" % rc)
    return o, Snew


def output_gate(o, g, w, eps=1e-6):
    """Head-wise RMSNorm and sigmoid output gate, per (token, head) over the d_v
    channels: ``y = o / sqrt(mean(o^2) + eps) * w * sigmoid(g)``.

    o, g ``[..., dv]`` (g is the gate's pre-activation), w ``[dv]`` (one weight
    vector shared by the heads). The pages give no epsilon and do not say
    whether the weight is per head; this reads both as the plainest choice
    (a caller-chosen epsilon, one weight vector of d_v). fp64 numpy.
    """
    o = np.asarray(o, dtype=np.float64)
    g = np.asarray(g, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    rms = np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + eps)
    return o / rms * w / (1.0 + np.exp(-g))


def _unit_rows(x, eps):
    """x / max(||x||, eps) over the last axis (the L2 normalisation of §6.2)."""
    n = np.sqrt((x * x).sum(axis=-1, keepdims=True))
    return x / np.maximum(n, eps)


def segment_map(k, v, log_alpha, beta, l2norm=True, eps=1e-6):
    """Affine map of one (sequence, head) segment of n tokens: ``S_out = M S_in + B``.

    Each token's update ``S <- (I - beta k k^T) Diag(alpha) S + beta k v^T`` (§3) is
    affine in S, so the segment composes to M = A_n ... A_1 with
    ``A_t = (I - beta_t k_t k_t^T) Diag(alpha_t)`` and B = the exit state from S_in = 0.
    k [n, dk], v [n, dv], log_alpha [n, dk] (or [n]: one gate per token), beta [n].
    Returns ``(M [dk, dk], B [dk, dv])``; fp64, a loop over the tokens.
    """
    k, v, la, b = (np.asarray(x, dtype=np.float64) for x in (k, v, log_alpha, beta))
    n, dk = k.shape
    if l2norm:
        k = _unit_rows(k, eps)
    M, B = np.eye(dk), np.zeros((dk, v.shape[1]))
    for t in range(n):
        a = np.exp(la[t]) * np.ones(dk)
        A = (np.eye(dk) - b[t] * np.outer(k[t], k[t])) * a[None, :]
        M = A @ M
        B = A @ B + b[t] * np.outer(k[t], v[t])
    return M, B


def segmented(q, k, v, log_alpha, beta, S0=None, cu_seqlens=None, cuts=(), l2norm=True, eps=1e-6):
    """:func:`recurrent` computed by segments. Every sequence is cut at the offsets
    ``cuts`` (token positions within the sequence; those outside (0, len) are ignored);
    each segment's map (:func:`segment_map`) is formed from a zero state, independently
    of the others; the maps are composed in order from S0 (``S_in`` of a segment is
    ``M S_in + B`` of the one before); then each segment runs its tokens from its true
    entry state for the outputs ``o_t = S_t^T q_t``. Returns ``(o [T, H, dv],
    S_T [N, H, dk, dv])`` like :func:`recurrent`.
    """
    q, k, v, la, b = (np.asarray(x, dtype=np.float64) for x in (q, k, v, log_alpha, beta))
    T, H, dk = q.shape
    dv = v.shape[2]
    cu = np.array([0, T]) if cu_seqlens is None else np.asarray(cu_seqlens, dtype=np.int64)
    N = len(cu) - 1
    S0 = np.zeros((N, H, dk, dv)) if S0 is None else np.asarray(S0, dtype=np.float64)
    if l2norm:
        q, k = _unit_rows(q, eps), _unit_rows(k, eps)
    o, S_T = np.zeros((T, H, dv)), np.zeros((N, H, dk, dv))
    for s in range(N):
        bos, eos = int(cu[s]), int(cu[s + 1])
        edges = [bos] + sorted(bos + int(c) for c in set(cuts) if 0 < int(c) < eos - bos) + [eos]
        for h in range(H):
            gate = la[:, h] if la.ndim == 3 else la[:, h, None] * np.ones((1, dk))
            maps = [segment_map(k[e0:e1, h], v[e0:e1, h], gate[e0:e1], b[e0:e1, h], l2norm=False)
                    for e0, e1 in zip(edges[:-1], edges[1:])]
            S = S0[s, h].copy()
            for (e0, e1), (M, B) in zip(zip(edges[:-1], edges[1:]), maps):
                St = S.copy()  # the segment's true entry state
                for t in range(e0, e1):
                    a = np.exp(gate[t])
                    St = (np.eye(dk) - b[t, h] * np.outer(k[t, h], k[t, h])) @ (a[:, None] * St) \
                        + b[t, h] * np.outer(k[t, h], v[t, h])
                    o[t, h] = St.T @ q[t, h]
                S = M @ S + B  # the composed map; equals St
            S_T[s, h] = S
    return o, S_T


def _silu(x):
    return x / (1.0 + np.exp(-x))


def short_conv_swish(x, w, cu_seqlens=None, state0=None):
    """Causal depthwise short convolution over each sequence's tokens, then Swish.

    x ``[T, C]`` (C channels, e.g. H * d of a q, k or v projection), w ``[C, W]``:
    the pre-activation of token t, channel c is ``sum_j w[c, j] * x[t - W + 1 + j, c]``
    (``w[c, W-1]`` weighs the current token), positions before a sequence's start
    read its initial state ``state0[s]`` ``[W-1, C]`` (oldest first) or zero, and the
    output is ``z * sigmoid(z)``. The pages give neither the window nor a bias; the
    window is the caller's and there is no bias (the plainest reading of "a short
    causal convolution"). Returns ``(y [T, C], state_T [N, W-1, C])``, state_T
    holding each sequence's last W-1 inputs (oldest first, reaching into state0 when
    the sequence is shorter). fp64 numpy, a loop over the sequences.
    """
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    T, C = x.shape
    W = w.shape[1]
    cu = np.array([0, T]) if cu_seqlens is None else np.asarray(cu_seqlens, dtype=np.int64)
    N = len(cu) - 1
    y = np.zeros((T, C))
    state_T = np.zeros((N, W - 1, C))
    for s in range(N):
        bos, eos = int(cu[s]), int(cu[s + 1])
        hist = np.zeros((W - 1, C)) if state0 is None else np.asarray(state0[s], dtype=np.float64)
        xs = np.concatenate([hist, x[bos:eos]], axis=0)  # [W-1+L, C]
        L = eos - bos
        for t in range(L):
            z = np.zeros(C)
            for j in range(W):
                z += w[:, j] * xs[t + j]
            y[bos + t] = _silu(z)
        state_T[s] = xs[L:L + W - 1]
    return y, state_T


def short_conv_step(x, w, state):
    """One decode token of :func:`short_conv_swish` for N sequences: x ``[N, C]``,
    state ``[N, W-1, C]`` (the previous W-1 inputs, oldest first). Returns
    ``(y [N, C], new_state [N, W-1, C])``."""
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    state = np.asarray(state, dtype=np.float64)
    window = np.concatenate([state, x[:, None, :]], axis=1)  # [N, W, C], newest last
    z = np.einsum("cj,njc->nc", w, window)
    return _silu(z), window[:, 1:, :].copy()


def _l2_back(x, dxh, eps):
    """Gradient through xh = x / max(||x||, eps), per row of x [..., d]."""
    n = np.linalg.norm(x, axis=-1, keepdims=True)
    big = n > eps
    xh = x / np.where(big, n, 1.0)
    proj = np.sum(xh * dxh, axis=-1, keepdims=True)
    return np.where(big, (dxh - xh * proj) / np.where(big, n, 1.0), dxh / eps)


def backward(q, k, v, log_alpha, beta, do, dS_T=None, S0=None, cu_seqlens=None, l2norm=True,
             eps=1e-6):
    """Gradients of a loss L through the recurrence of :func:`recurrent`, given
    ``do = dL/do [T,H,dv]`` and ``dS_T = dL/dS_T [N,H,dk,dv]`` (None: zero).

    Per token, with q, k normalised (q^, k^) and a = exp(log_alpha_t):
    forward ``S~ = Diag(a) S_{t-1}``, ``u = beta (v - S~^T k^)``, ``S_t = S~ + k^ u^T``,
    ``o_t = S_t^T q^``; backward, from t = T down to 1 with G = dL/dS_t:
    ``G += q^ do_t^T``, ``dq^ = S_t do_t``, ``du = G^T k^``, ``dk^ = G u - beta S~ du``,
    ``dv = beta du``, ``dbeta = du . (v - S~^T k^)``, ``dS~ = G - beta k^ du^T``,
    ``dlog_alpha = a * rowsum(dS~ * S_{t-1})``, ``G <- Diag(a) dS~`` (dL/dS_{t-1});
    then through the normalisation. log_alpha [T,H] (one gate per head) gets the
    sum over the key channels. Returns ``(dq, dk, dv, dlog_alpha, dbeta, dS0)``.
    fp64 numpy, loops over sequences, heads and tokens (small cases).
    """
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    la = np.asarray(log_alpha, dtype=np.float64)
    b = np.asarray(beta, dtype=np.float64)
    do = np.asarray(do, dtype=np.float64)
    T, H, dk = q.shape
    dv = v.shape[2]
    scalar = la.ndim == 2
    cu = np.array([0, T]) if cu_seqlens is None else np.asarray(cu_seqlens, dtype=np.int64)
    N = len(cu) - 1
    S0 = np.zeros((N, H, dk, dv)) if S0 is None else np.asarray(S0, dtype=np.float64)
    dST = np.zeros((N, H, dk, dv)) if dS_T is None else np.asarray(dS_T, dtype=np.float64)
    if l2norm:
        nq = np.maximum(np.linalg.norm(q, axis=-1, keepdims=True), eps)
        nk = np.maximum(np.linalg.norm(k, axis=-1, keepdims=True), eps)
        qh, kh = q / nq, k / nk
    else:
        qh, kh = q, k
    dqh, dkh = np.zeros_like(q), np.zeros_like(k)
    gv, gla, gb = np.zeros_like(v), np.zeros_like(la), np.zeros_like(b)
    dS0 = np.zeros((N, H, dk, dv))
    for s in range(N):
        bos, eos = int(cu[s]), int(cu[s + 1])
        for h in range(H):
            alpha = lambda t: np.exp(np.full(dk, la[t, h]) if scalar else la[t, h])
            states = [S0[s, h].copy()]  # S_{t-1} of every token, then the last S_t
            for t in range(bos, eos):
                St = alpha(t)[:, None] * states[-1]
                u = b[t, h] * (v[t, h] - St.T @ kh[t, h])
                states.append(St + np.outer(kh[t, h], u))
            G = dST[s, h].copy()
            for i in range(eos - bos - 1, -1, -1):
                t = bos + i
                a = alpha(t)
                Sp, Sn = states[i], states[i + 1]
                St = a[:, None] * Sp
                r = v[t, h] - St.T @ kh[t, h]
                u = b[t, h] * r
                G += np.outer(qh[t, h], do[t, h])
                dqh[t, h] = Sn @ do[t, h]
                du = G.T @ kh[t, h]
                dkh[t, h] = G @ u - b[t, h] * (St @ du)
                gv[t, h] = b[t, h] * du
                gb[t, h] = du @ r
                dSt = G - b[t, h] * np.outer(kh[t, h], du)
                g = a * np.sum(dSt * Sp, axis=1)
                if scalar:
                    gla[t, h] = g.sum()
                else:
                    gla[t, h] = g
                G = a[:, None] * dSt
            dS0[s, h] = G
    if l2norm:
        gq, gk = _l2_back(q, dqh, eps), _l2_back(k, dkh, eps)
    else:
        gq, gk = dqh, dkh
    return gq, gk, gv, gla, gb, dS0


def chunkwise_backward(q, k, v, log_alpha, beta, do, dS_T=None, S0=None, cu_seqlens=None, chunk=64,
                       l2norm=True, eps=1e-6):
    """:func:`backward` through the chunkwise form. Per chunk (rows r, entry state S,
    G the inclusive cumsum of log_alpha, g its last row; Qg = Q e^G, Kg = K e^G,
    Kn = K e^-G, Kd = K e^(g-G); A = strict_lower(Kg Kn^T), P = lower(Qg Kn^T);
    X = (I + Diag(beta) A)^-1, T = X Diag(beta), W = T Kg, U = T V - W S;
    O = Qg S + P U, S' = Diag(e^g) S + Kd^T U), the reverse sweep over chunks,
    given dO and dS':

        dS  = Diag(e^g) dS' + Qg^T dO - W^T dU,   dU = Kd dS' + P^T dO
        dKd = U dS'^T,  dP = lower(dO U^T),  dQg = dO S^T,  dW = -dU S^T
        dT  = dU V^T + dW Kg^T,  dV = T^T dU,  dKg = T^T dW
        dX  = dT Diag(beta),  dM = -X^T dX X^T,  dA = strict_lower(Diag(beta) dM)
        dbeta_i = sum_r dT_ri X_ri + sum_i' dM_ii' A_ii'
        A, P: dKg += dA Kn,  dKn = dA^T Kg + dP^T Qg,  dQg += dP Kn
        exponents: dG = dQg Qg + dKg Kg - dKn Kn - dKd Kd (element-wise),
                   dg = colsum(dKd Kd) + e^g rowsum(dS' S)
        dlog_alpha_r = sum_{r' >= r} dG_r' + dg

    then through the normalisation of q, k. Entry states come from a forward pass
    over the chunks. Returns what :func:`backward` returns (KDA gates only).
    """
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    la = np.asarray(log_alpha, dtype=np.float64)
    b = np.asarray(beta, dtype=np.float64)
    do = np.asarray(do, dtype=np.float64)
    T, H, dk = q.shape
    dv = v.shape[2]
    cu = np.array([0, T]) if cu_seqlens is None else np.asarray(cu_seqlens, dtype=np.int64)
    N = len(cu) - 1
    S0 = np.zeros((N, H, dk, dv)) if S0 is None else np.asarray(S0, dtype=np.float64)
    dST = np.zeros((N, H, dk, dv)) if dS_T is None else np.asarray(dS_T, dtype=np.float64)
    if l2norm:
        nq = np.maximum(np.linalg.norm(q, axis=-1, keepdims=True), eps)
        nk = np.maximum(np.linalg.norm(k, axis=-1, keepdims=True), eps)
        qh, kh = q / nq, k / nk
    else:
        qh, kh = q, k
    dqh, dkh = np.zeros_like(q), np.zeros_like(k)
    gv, gla, gb = np.zeros_like(v), np.zeros_like(la), np.zeros_like(b)
    dS0 = np.zeros((N, H, dk, dv))

    def chunk_terms(rows, h):
        Q, K, V = qh[rows, h], kh[rows, h], v[rows, h]
        G = np.cumsum(la[rows, h], axis=0)
        g = G[-1]
        Qg, Kg, Kn, Kd = Q * np.exp(G), K * np.exp(G), K * np.exp(-G), K * np.exp(g - G)
        n = len(rows)
        A = np.tril(Kg @ Kn.T, -1)
        P = np.tril(Qg @ Kn.T)
        bt = b[rows, h]
        X = np.linalg.inv(np.eye(n) + bt[:, None] * A)
        Tm = X * bt[None, :]
        return dict(V=V, G=G, g=g, Qg=Qg, Kg=Kg, Kn=Kn, Kd=Kd, A=A, P=P, bt=bt, X=X, T=Tm, W=Tm @ Kg)

    for s in range(N):
        bos, eos = int(cu[s]), int(cu[s + 1])
        starts = list(range(bos, eos, chunk))
        for h in range(H):
            entry = [S0[s, h].copy()]
            for c0 in starts:
                rows = np.arange(c0, min(c0 + chunk, eos))
                m = chunk_terms(rows, h)
                S = entry[-1]
                U = m["T"] @ m["V"] - m["W"] @ S
                entry.append(np.exp(m["g"])[:, None] * S + m["Kd"].T @ U)
            dSn = dST[s, h].copy()  # dL/dS' of the current chunk
            for ci in range(len(starts) - 1, -1, -1):
                c0 = starts[ci]
                rows = np.arange(c0, min(c0 + chunk, eos))
                m = chunk_terms(rows, h)
                S = entry[ci]
                U = m["T"] @ m["V"] - m["W"] @ S
                dO = do[rows, h]
                eg = np.exp(m["g"])
                dU = m["Kd"] @ dSn + m["P"].T @ dO
                dKd = U @ dSn.T
                dP = np.tril(dO @ U.T)
                dQg = dO @ S.T
                dW = -dU @ S.T
                dS = eg[:, None] * dSn + m["Qg"].T @ dO - m["W"].T @ dU
                dT = np.tril(dU @ m["V"].T + dW @ m["Kg"].T)
                gv[rows, h] = m["T"].T @ dU
                dKg = m["T"].T @ dW
                dX = dT * m["bt"][None, :]
                dM = -m["X"].T @ dX @ m["X"].T
                dA = np.tril(m["bt"][:, None] * dM, -1)
                gb[rows, h] = np.sum(dT * m["X"], axis=0) + np.sum(dM * m["A"], axis=1)
                dKg = dKg + dA @ m["Kn"]
                dKn = dA.T @ m["Kg"] + dP.T @ m["Qg"]
                dQg = dQg + dP @ m["Kn"]
                dG = dQg * m["Qg"] + dKg * m["Kg"] - dKn * m["Kn"] - dKd * m["Kd"]
                dg = np.sum(dKd * m["Kd"], axis=0) + eg * np.sum(dSn * S, axis=1)
                gla[rows, h] = np.cumsum(dG[::-1], axis=0)[::-1] + dg[None, :]
                dqh[rows, h] = dQg * np.exp(m["G"])
                dkh[rows, h] = dKg * np.exp(m["G"]) + dKn * np.exp(-m["G"]) + dKd * np.exp(m["g"] - m["G"])
                dSn = dS
            dS0[s, h] = dSn
    if l2norm:
        gq, gk = _l2_back(q, dqh, eps), _l2_back(k, dkh, eps)
    else:
        gq, gk = dqh, dkh
    return gq, gk, gv, gla, gb, dS0
