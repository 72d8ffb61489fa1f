"""KDA oracle: slow, obviously correct CPU references (fp64).

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  It shares no code with
the CUDA library and never imports it.

Three independent formulations of the same operator:

* :func:`prefill` / :func:`decode` -- the token-by-token recurrence in plain C
  (``kda_oracle.c``), fp64, OpenMP over (sequence, head).  This is the
  definition every GPU result is compared with.
* :func:`brute_force` -- tiny inputs only: every step's transition
  (I - beta k k^T) Diag(alpha) is built as an explicit d_k x d_k matrix and
  applied with a matrix product, exactly the update written in the operator's
  definition ("Kimi Linear's 75% KV cache cut ...", theclarity.today, third
  paragraph; the delta rule of "Kimi Linear wlasnie pokonal pelna uwage ...",
  remio.ai, section "Jak Kimi Linear wykorzystuje inteligentniejsza pamiec
  rekurencyjna").
* :func:`chunked` -- the chunkwise (blockwise) algorithm with the WY/UT
  representation: a chunk's rank-1 updates become one unit-lower-triangular
  solve and dense matrix products ("Kimi Linear's 75% KV cache cut ...",
  fourth paragraph; blockwise training with a diagonal-plus-low-rank
  transition, remio.ai, same section).  The chunk algebra (derived from the
  recurrence) is, per chunk with incoming state S0 and g = per-channel
  inclusive cumulative sum of log_alpha inside the chunk:
      A[r,i] = beta_r sum_c k[r,c] k[i,c] exp(g[r,c]-g[i,c])   (i < r)
      M[r,i] =        sum_c q[r,c] k[i,c] exp(g[r,c]-g[i,c])   (i <= r)
      (I + A) U = Diag(beta) (V - (K*exp(g)) S0)
      O   = (Q*exp(g)) S0 + M U
      S_C = Diag(exp(g_last)) S0 + (K*exp(g_last - g))^T U
  It uses numpy's dense solve as a library step and no blocking beyond the
  chunk itself.

Masked (pad) positions: the state is not touched and the output is 0
("Transformers Community Reports Kimi Linear Cache Bug", ainews: pads must
neither decay nor write the recurrent state).

Head-wise gates: a log_alpha of shape [rows, H] is one decay per token and head,
the gating of Gated DeltaNet that KDA refines per channel ("Kimi Linear's 75% KV
cache cut ...", third paragraph; remio.ai, same section).  Diag(alpha) is then
alpha times the identity, i.e. the per-channel operator with that value in every
channel, which is how :func:`head_gate_channels` writes it out.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB = os.path.join(_HERE, "libkda_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle with gcc (-O2, OpenMP, IEEE arithmetic)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        f32p = np.ctypeslib.ndpointer(np.float32, flags="C_CONTIGUOUS")
        f64p = np.ctypeslib.ndpointer(np.float64, flags="C_CONTIGUOUS")
        i32p = np.ctypeslib.ndpointer(np.int32, flags="C_CONTIGUOUS")
        vp = ctypes.c_void_p
        lib.kda_oracle_prefill.argtypes = [ctypes.c_int, i32p, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_int, f32p, f32p, f32p, f32p, f32p, vp, vp,
                                           f64p, vp, ctypes.c_int]
        lib.kda_oracle_prefill.restype = ctypes.c_int
        lib.kda_oracle_decode.argtypes = [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          f32p, f32p, f32p, f32p, f32p, vp, f64p, f64p,
                                          ctypes.c_int]
        lib.kda_oracle_decode.restype = ctypes.c_int
        lib.kda_oracle_max_threads.restype = ctypes.c_int
        _lib = lib
    return _lib


def max_threads() -> int:
    return int(_load().kda_oracle_max_threads())


def _f32(x):
    return np.ascontiguousarray(x, dtype=np.float32)


def _ptr(x):
    return None if x is None else x.ctypes.data_as(ctypes.c_void_p)


def head_gate_channels(log_alpha, dk: int):
    """A head-wise gate [rows, H] as the per-channel gate [rows, H, dk] with the same
    value in every channel; a per-channel gate is returned unchanged."""
    la = np.asarray(log_alpha)
    if la.ndim == 2:
        return np.repeat(la[:, :, None], dk, axis=2)
    return la


def prefill(q, k, v, log_alpha, beta, cu_seqlens, pad_mask=None, init_state=None,
            nthreads: int = 0):
    """Token-by-token fp64 prefill.  Returns (o [N,H,dv] f64, final_state [B,H,dk,dv] f64).
    log_alpha is [N,H,dk] (per channel) or [N,H] (one gate per token and head)."""
    lib = _load()
    log_alpha = head_gate_channels(log_alpha, np.shape(q)[2])
    q, k, v, la, be = _f32(q), _f32(k), _f32(v), _f32(log_alpha), _f32(beta)
    cu = np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    N, H, dk = q.shape
    dv = v.shape[2]
    B = len(cu) - 1
    assert int(cu[-1]) == N
    mask = None if pad_mask is None else np.ascontiguousarray(pad_mask, dtype=np.uint8)
    s0 = None if init_state is None else _f32(init_state)
    o = np.zeros((N, H, dv), dtype=np.float64)
    fs = np.zeros((B, H, dk, dv), dtype=np.float64)
    rc = lib.kda_oracle_prefill(B, cu, H, dk, dv, q, k, v, la, be, _ptr(mask), _ptr(s0), o,
                                _ptr(fs), int(nthreads))
    if rc != 0:
        raise ValueError("kda_oracle_prefill: invalid arguments")
    return o, fs


def decode(q, k, v, log_alpha, beta, state, mask=None, nthreads: int = 0):
    """One fp64 decode step.  ``state`` [B,H,dk,dv] float64 is updated in place; returns o.
    log_alpha is [B,H,dk] or [B,H] (one gate per row and head)."""
    lib = _load()
    log_alpha = head_gate_channels(log_alpha, np.shape(q)[2])
    q, k, v, la, be = _f32(q), _f32(k), _f32(v), _f32(log_alpha), _f32(beta)
    B, H, dk = q.shape
    dv = v.shape[2]
    assert state.dtype == np.float64 and state.flags["C_CONTIGUOUS"]
    m = None if mask is None else np.ascontiguousarray(mask, dtype=np.uint8)
    o = np.zeros((B, H, dv), dtype=np.float64)
    rc = lib.kda_oracle_decode(B, H, dk, dv, q, k, v, la, be, _ptr(m), state, o, int(nthreads))
    if rc != 0:
        raise ValueError("kda_oracle_decode: invalid arguments")
    return o


# ----------------------------------------------------------------------------
# Pure numpy formulations (small inputs)
# ----------------------------------------------------------------------------
def brute_force(q, k, v, log_alpha, beta, S0=None, pad_mask=None):
    """One head, one sequence: q,k,log_alpha [T,dk], v [T,dv], beta [T].

    Each step applies the explicit transition matrix
    P_t = (I - beta_t k_t k_t^T) Diag(alpha_t) and adds beta_t k_t v_t^T.
    Returns (o [T,dv], S [dk,dv]) in fp64.
    """
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    la = np.asarray(log_alpha, dtype=np.float64)
    beta = np.asarray(beta, dtype=np.float64)
    T, dk = k.shape
    dv = v.shape[1]
    S = np.zeros((dk, dv)) if S0 is None else np.array(S0, dtype=np.float64)
    o = np.zeros((T, dv))
    eye = np.eye(dk)
    for t in range(T):
        if pad_mask is not None and pad_mask[t] == 0:
            continue
        P = (eye - beta[t] * np.outer(k[t], k[t])) @ np.diag(np.exp(la[t]))
        S = P @ S + beta[t] * np.outer(k[t], v[t])
        o[t] = S.T @ q[t]
    return o, S


def chunked(q, k, v, log_alpha, beta, chunk: int, S0=None, pad_mask=None):
    """One head, one sequence, chunkwise WY/UT form in fp64 (see module docstring).

    Pad positions become identity steps (log_alpha = 0, beta = 0, q = k = v = 0)
    and their output is 0.
    """
    q, k, v = (np.array(x, dtype=np.float64) for x in (q, k, v))
    la = np.array(log_alpha, dtype=np.float64)
    beta = np.array(beta, dtype=np.float64)
    T, dk = k.shape
    dv = v.shape[1]
    if pad_mask is not None:
        pad = np.asarray(pad_mask) == 0
        q[pad] = 0.0
        k[pad] = 0.0
        v[pad] = 0.0
        la[pad] = 0.0
        beta[pad] = 0.0
    S = np.zeros((dk, dv)) if S0 is None else np.array(S0, dtype=np.float64)
    o = np.zeros((T, dv))
    for c0 in range(0, T, chunk):
        Q, K, V = q[c0:c0 + chunk], k[c0:c0 + chunk], v[c0:c0 + chunk]
        b = beta[c0:c0 + chunk]
        g = np.cumsum(la[c0:c0 + chunk], axis=0)
        C = K.shape[0]
        r_idx, i_idx = np.meshgrid(np.arange(C), np.arange(C), indexing="ij")
        lower = i_idx <= r_idx
        # exp(g[r]-g[i]) only where i <= r (elsewhere it is never used)
        diff = np.where(lower[:, :, None], g[:, None, :] - g[None, :, :], -np.inf)
        D = np.exp(diff)
        A = b[:, None] * np.einsum("rc,ic,ric->ri", K, K, D) * (i_idx < r_idx)
        M = np.einsum("rc,ic,ric->ri", Q, K, D) * lower
        Gam = np.exp(g)
        rhs_v = b[:, None] * V
        rhs_k = b[:, None] * (K * Gam)
        L = np.eye(C) + A
        Uv = np.linalg.solve(L, rhs_v)
        W = np.linalg.solve(L, rhs_k)
        U = Uv - W @ S
        o[c0:c0 + C] = (Q * Gam) @ S + M @ U
        S = Gam[-1][:, None] * S + (K * np.exp(g[-1] - g)).T @ U
    if pad_mask is not None:
        o[np.asarray(pad_mask) == 0] = 0.0
    return o, S


def prefix_audit(run, T: int, perturb, tol: float = 0.0):
    """Prefix-invariance audit ("The Mask Is Not the Model", dev.to, audit procedure).

    ``run(x)`` returns per-position outputs [T, ...] for an input variant x in
    {0, 1}; variant 1 differs from variant 0 only at position T-1 (the caller's
    ``perturb`` builds it).  Returns (leak, onset, delta): delta[t] is the max-abs
    difference at position t < T-1, leak is True if any delta exceeds ``tol`` and
    onset is the first such position (None if clean).
    """
    h0 = np.asarray(run(0))
    h1 = np.asarray(run(perturb))
    d = np.abs(h0[: T - 1].astype(np.float64) - h1[: T - 1].astype(np.float64))
    d = d.reshape(T - 1, -1).max(axis=1)
    bad = np.nonzero(d > tol)[0]
    return (len(bad) > 0, (int(bad[0]) if len(bad) else None), d)


# ----------------------------------------------------------------------------
# Short causal convolution (the layer's convolution window, padding-correct)
# ----------------------------------------------------------------------------
def short_conv(x, weight, bias, cu_seqlens, pad_mask=None, state_in=None):
    """Depthwise causal convolution over each sequence's VALID positions, written as
    the sliding window it is: the window holds the W-1 previous valid inputs (the
    incoming state before the sequence's first ones); at a valid position the output
    is bias + sum_i weight[:, i] * u_i over the window followed by x_t, and x_t then
    enters the window; a pad position outputs 0 and leaves the window alone
    ("Transformers Community Reports Kimi Linear Cache Bug", ainews: padded entries
    must not enter the convolution window nor advance the convolution state).
    x [N, D]; weight [D, W]; bias [D] or None; state_in [B, W-1, D] or None.
    Returns (y [N, D] float64, state_out [B, W-1, D] float64)."""
    x = np.asarray(x, dtype=np.float64)
    w = np.asarray(weight, dtype=np.float64)
    N, D = x.shape
    W = w.shape[1]
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    B = len(cu) - 1
    b0 = np.zeros(D) if bias is None else np.asarray(bias, dtype=np.float64)
    y = np.zeros((N, D))
    s_out = np.zeros((B, W - 1, D))
    for b in range(B):
        window = [np.zeros(D) if state_in is None else np.asarray(state_in[b, j], dtype=np.float64)
                  for j in range(W - 1)]
        for t in range(int(cu[b]), int(cu[b + 1])):
            if pad_mask is not None and pad_mask[t] == 0:
                continue
            u = window + [x[t]]
            y[t] = b0 + sum(w[:, i] * u[i] for i in range(W))
            window = u[1:]
        for j in range(W - 1):
            s_out[b, j] = window[j]
    return y, s_out


def short_conv_at(x, weight, bias, cu_seqlens, positions, pad_mask=None, state_in=None):
    """Outputs of short_conv at the given packed positions only (for full-size checks):
    each one from its own window, found by walking back over the pad mask.
    Returns y [len(positions), D] float64."""
    w = np.asarray(weight, dtype=np.float64)
    D, W = w.shape
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    b0 = np.zeros(D) if bias is None else np.asarray(bias, dtype=np.float64)
    out = np.zeros((len(positions), D))
    for n, t in enumerate(positions):
        t = int(t)
        if pad_mask is not None and pad_mask[t] == 0:
            continue
        b = int(np.searchsorted(cu, t, side="right")) - 1
        prev = []                      # newest first
        s = t - 1
        while s >= cu[b] and len(prev) < W - 1:
            if pad_mask is None or pad_mask[s] != 0:
                prev.append(np.asarray(x[s], dtype=np.float64))
            s -= 1
        j = W - 2                      # newest state row first
        while len(prev) < W - 1:
            prev.append(np.zeros(D) if state_in is None else np.asarray(state_in[b, j], np.float64))
            j -= 1
        u = prev[::-1] + [np.asarray(x[t], dtype=np.float64)]
        out[n] = b0 + sum(w[:, i] * u[i] for i in range(W))
    return out


# ----------------------------------------------------------------------------
# Backward pass (reverse-mode derivative of the recurrence, token by token)
# ----------------------------------------------------------------------------
def prefill_backward(q, k, v, log_alpha, beta, cu_seqlens, do, dS_final=None, pad_mask=None,
                     init_state=None):
    """Gradients of the prefill's outputs (o and the final state) with respect to every
    input, for upstream gradients ``do`` [N,H,dv] and ``dS_final`` [B,H,dk,dv] (None = 0).
    The forward step is taken apart into its four operations -- decay S' = Diag(a) S,
    read p = S'^T k, correction u = beta (v - p), write S = S' + k u^T, output o = S^T q --
    and each one's adjoint is applied in reverse order (chain rule), in fp64, with the
    states recomputed forward.  Pads are identity steps: zero gradients there, the state
    gradient passes through.  Returns a dict with dq, dk, dv, dlog_alpha (the gate's
    layout), dbeta and dS0."""
    head_gate = np.asarray(log_alpha).ndim == 2
    dkk = np.shape(q)[2]
    la_full = np.asarray(head_gate_channels(log_alpha, dkk), dtype=np.float64)
    q, k, v = (np.asarray(x, dtype=np.float64) for x in (q, k, v))
    be = np.asarray(beta, dtype=np.float64)
    do = np.asarray(do, dtype=np.float64)
    N, H, dk = q.shape
    dv = v.shape[2]
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    B = len(cu) - 1
    g = {name: np.zeros_like(x) for name, x in (("dq", q), ("dk", k), ("dv", v))}
    g["dlog_alpha"] = np.zeros((N, H, dk))
    g["dbeta"] = np.zeros((N, H))
    g["dS0"] = np.zeros((B, H, dk, dv))
    for b in range(B):
        for h in range(H):
            S = np.zeros((dk, dv)) if init_state is None else np.asarray(init_state[b, h], np.float64)
            states = []                      # S_{t-1} before each position
            for t in range(int(cu[b]), int(cu[b + 1])):
                states.append(S.copy())
                if pad_mask is not None and pad_mask[t] == 0:
                    continue
                a = np.exp(la_full[t, h])
                Sp = a[:, None] * S
                p = Sp.T @ k[t, h]
                u = be[t, h] * (v[t, h] - p)
                S = Sp + np.outer(k[t, h], u)
            G = np.zeros((dk, dv)) if dS_final is None else np.asarray(dS_final[b, h], np.float64).copy()
            for idx in range(int(cu[b + 1]) - 1, int(cu[b]) - 1, -1):
                if pad_mask is not None and pad_mask[idx] == 0:
                    continue
                Sprev = states[idx - int(cu[b])]
                a = np.exp(la_full[idx, h])
                kt, qt, vt, bt, dot = k[idx, h], q[idx, h], v[idx, h], be[idx, h], do[idx, h]
                Sp = a[:, None] * Sprev
                p = Sp.T @ kt
                u = bt * (v[idx, h] - p)
                St = Sp + np.outer(kt, u)
                # o = S_t^T q
                g["dq"][idx, h] = St @ dot
                G = G + np.outer(qt, dot)
                # S_t = S' + k u^T
                dk_ = G @ u
                du = G.T @ kt
                Gp = G.copy()
                # u = beta (v - p)
                g["dv"][idx, h] = bt * du
                g["dbeta"][idx, h] = du @ (vt - p)
                dp = -bt * du
                # p = S'^T k
                Gp += np.outer(kt, dp)
                dk_ += Sp @ dp
                g["dk"][idx, h] = dk_
                # S' = Diag(a) S_{t-1}, a = exp(log_alpha)
                g["dlog_alpha"][idx, h] = (Gp * Sp).sum(axis=1)
                G = a[:, None] * Gp
            g["dS0"][b, h] = G
    if head_gate:
        g["dlog_alpha"] = g["dlog_alpha"].sum(axis=2)
    return g
