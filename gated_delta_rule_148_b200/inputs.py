"""Seeded synthetic inputs for the KDA operator.

This module only draws random numbers and lays them out; it holds none of the
operator's arithmetic.  The CUDA tests, the benchmark and the CPU oracle all
take their inputs from here, so both sides see the same values.

Distributions (the workloads in the model description the kernels target):
  q, k ~ N(0, 1), then L2-normalised per (token, head) in fp32;
  v ~ N(0, 1);
  beta = sigmoid(N(0, 1)) per (token, head), fp32;
  log_alpha = -softplus(N(-2, 1)) per (token, head, key channel), fp32;
  head-wise gates (one per token and head): -softplus(N(-2, 1)) per (token, head);
  initial state (where one is used) ~ N(0, 0.1) (standard deviation 0.1), fp32.
q, k and v are rounded to bf16 (round to nearest even) for bf16 workloads; the
arrays returned here always hold float32 values, which represent bf16 values
exactly, so the CPU side can read them without a conversion step.

Random streams: numpy PCG64.  Each tensor has its own stream id (q, k, v,
log_alpha, beta, state, structure), and its flattened elements are drawn in
blocks of 2**22, block i from SeedSequence([seed, stream, sub, i]); so the
values do not depend on how many threads fill the blocks, and generating one
tensor never shifts another.
"""
from __future__ import annotations

import dataclasses
import os
from concurrent.futures import ThreadPoolExecutor
from typing import Dict, List, Optional, Sequence

import numpy as np

SEED_BASE = 1480

_STREAMS = ("q", "k", "v", "log_alpha", "beta", "state", "structure", "decode_mask",
            "log_alpha_head", "conv_x", "conv_weight", "grad_o")


@dataclasses.dataclass(frozen=True)
class Workload:
    """A named workload: shapes, dtype and chunk size of one KDA call."""
    name: str
    seed: int
    H: int
    dk: int
    dv: int
    dtype: str               # "bf16" or "f32" for q, k, v and o
    chunk: int
    lengths: Optional[Sequence[int]] = None   # prefill: per-sequence lengths
    init_state: bool = False
    pads: bool = False       # prefill: 0-64 zero-valued pads left or right per sequence
    decode_rows: int = 0     # decode: rows per step
    decode_steps: int = 0
    decode_masked: int = 0   # decode: masked rows per step


def tiny_f32() -> Workload:
    """B=1, H=2, T=128, d=64, chunk 16, fp32 throughout, zero initial state."""
    return Workload("tiny_f32_T128_H2_d64", SEED_BASE + 0, 2, 64, 64, "f32", 16, lengths=(128,))


def prefill(T: int = 4096, H: int = 32, d: int = 128, seed: int = SEED_BASE + 1) -> Workload:
    """One sequence of T tokens, H heads, d_k = d_v = d, bf16 q/k/v, chunk 64, zero state."""
    return Workload(f"prefill_T{T}_H{H}_d{d}_bf16", seed, H, d, d, "bf16", 64, lengths=(T,))


def varlen_cached(H: int = 32, d: int = 128, n_seqs: int = 8, lo: int = 1024, hi: int = 16384,
                  seed: int = SEED_BASE + 2) -> Workload:
    """Packed batch with lengths uniform in [lo, hi], nonzero initial states and edge pads."""
    rng = _child(seed, "structure")
    lengths = tuple(int(x) for x in rng.integers(lo, hi + 1, size=n_seqs))
    return Workload(f"varlen_{n_seqs}seqs_H{H}_d{d}_bf16", seed, H, d, d, "bf16", 64,
                    lengths=lengths, init_state=True, pads=True)


def long_prefill(T: int = 131072) -> Workload:
    """B=1, H=32, T tokens (131072 headline; 16384 and 65536 for scaling), d=128, bf16."""
    return prefill(T=T, H=32, d=128, seed=SEED_BASE + 3)


def batched_decode(rows: int = 256, H: int = 32, d: int = 128, steps: int = 1000,
                   masked: int = 26) -> Workload:
    """256 rows x 32 heads, fp32 state ~ N(0, 0.1), bf16 q/k/v, 26 rows masked per step."""
    return Workload(f"decode_{rows}rows_H{H}_d{d}_bf16", SEED_BASE + 4, H, d, d, "bf16", 0,
                    init_state=True, decode_rows=rows, decode_steps=steps, decode_masked=masked)


# ----------------------------------------------------------------------------
def _child(seed: int, stream: str, sub: int = 0) -> np.random.Generator:
    ss = np.random.SeedSequence([seed, _STREAMS.index(stream), sub])
    return np.random.Generator(np.random.PCG64(ss))


_BLOCK = 1 << 22
_WORKERS = max(1, min(16, os.cpu_count() or 1))


def _blocks(n: int):
    return [(i, i * _BLOCK, min(n, (i + 1) * _BLOCK)) for i in range((n + _BLOCK - 1) // _BLOCK)]


def _par(fn, items):
    if len(items) <= 1:
        return [fn(it) for it in items]
    with ThreadPoolExecutor(_WORKERS) as ex:
        return list(ex.map(fn, items))


def _rows_map(fn, x: np.ndarray) -> np.ndarray:
    """Apply ``fn`` to blocks of leading rows of x in parallel (fn is row-local)."""
    lead = x.shape[0]
    per = max(1, _BLOCK // max(1, x[0].size))
    spans = [(a, min(lead, a + per)) for a in range(0, lead, per)]

    def one(sp):
        x[sp[0]:sp[1]] = fn(x[sp[0]:sp[1]])
    _par(one, spans)
    return x


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32.

    Finite inputs only (the uint32 sum cannot overflow below the NaN range)."""
    x = np.ascontiguousarray(x, dtype=np.float32)

    def rnd(blk):
        u = blk.view(np.uint32)
        u = (u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) & np.uint32(0xFFFF0000)
        return u.view(np.float32)
    return _rows_map(rnd, x.copy()) if x.ndim else rnd(x.reshape(1)).reshape(())


def _normal(seed: int, stream: str, shape, scale: float = 1.0, loc: float = 0.0) -> np.ndarray:
    n = int(np.prod(shape))
    out = np.empty(n, dtype=np.float32)
    sid = _STREAMS.index(stream)

    def fill(blk):
        i, a, b = blk
        g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, sid, 0, i])))
        g.standard_normal(out=out[a:b], dtype=np.float32)
        if scale != 1.0:
            out[a:b] *= np.float32(scale)
        if loc != 0.0:
            out[a:b] += np.float32(loc)
    _par(fill, _blocks(n))
    return out.reshape(shape)


def _unit_rows(x: np.ndarray) -> np.ndarray:
    def f(blk):
        n = np.sqrt(np.sum(blk * blk, axis=-1, keepdims=True, dtype=np.float32), dtype=np.float32)
        return (blk / np.maximum(n, np.float32(1e-30))).astype(np.float32)
    return _rows_map(f, x)


def _softplus(x: np.ndarray) -> np.ndarray:
    return _rows_map(lambda b: np.logaddexp(np.float32(0.0), b).astype(np.float32), x)


def _sigmoid(x: np.ndarray) -> np.ndarray:
    return _rows_map(lambda b: (1.0 / (1.0 + np.exp(-b))).astype(np.float32), x)


def token_tensors(seed: int, N: int, H: int, dk: int, dv: int, dtype: str) -> Dict[str, np.ndarray]:
    """q, k [N,H,dk], v [N,H,dv], log_alpha [N,H,dk], beta [N,H] (float32 arrays)."""
    q = _unit_rows(_normal(seed, "q", (N, H, dk)))
    k = _unit_rows(_normal(seed, "k", (N, H, dk)))
    v = _normal(seed, "v", (N, H, dv))
    if dtype == "bf16":
        q, k, v = round_bf16(q), round_bf16(k), round_bf16(v)
    log_alpha = _softplus(_normal(seed, "log_alpha", (N, H, dk), loc=-2.0))
    np.negative(log_alpha, out=log_alpha)
    beta = _sigmoid(_normal(seed, "beta", (N, H)))
    return dict(q=q, k=k, v=v, log_alpha=log_alpha, beta=beta)


def head_gates(seed: int, rows: int, H: int) -> np.ndarray:
    """log_alpha [rows, H] fp32 for one gate per token (or decode row) and head."""
    la = _softplus(_normal(seed, "log_alpha_head", (rows, H), loc=-2.0))
    np.negative(la, out=la)
    return la


def conv_inputs(seed: int, lengths: Sequence[int], D: int, W: int, dtype: str = "bf16",
                pad_frac: float = 0.0, state: bool = True) -> Dict[str, np.ndarray]:
    """Inputs of one short-convolution call: x [N, D] ~ N(0, 1) (bf16-rounded for bf16),
    weight [D, W] ~ N(0, 1/W), bias [D] ~ N(0, 0.1), cu_seqlens, pad_mask (each position
    a pad with probability pad_frac, or None), state [B, W-1, D] ~ N(0, 1) or None."""
    cu = np.zeros(len(lengths) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(lengths)
    N, B = int(cu[-1]), len(lengths)
    x = _normal(seed, "conv_x", (N, D))
    if dtype == "bf16" and N > 0:
        x = round_bf16(x)
    wb = _normal(seed, "conv_weight", (D * W + D,))
    out = dict(x=x, weight=(wb[:D * W].reshape(D, W) / np.sqrt(W)).astype(np.float32),
               bias=(0.1 * wb[D * W:]).astype(np.float32), cu_seqlens=cu, pad_mask=None,
               state=_normal(seed, "state", (B, W - 1, D)) if state else None)
    if pad_frac > 0:
        rng = _child(seed, "structure", 2)
        out["pad_mask"] = (rng.uniform(size=N) >= pad_frac).astype(np.uint8)
    return out


def grad_outputs(seed: int, N: int, H: int, dv: int) -> np.ndarray:
    """Upstream gradient of o for a backward pass: [N, H, dv] ~ N(0, 1), fp32."""
    return _normal(seed, "grad_o", (N, H, dv))


def prefill_inputs(w: Workload) -> Dict[str, np.ndarray]:
    """All inputs of one prefill call for workload ``w``.

    Returns q, k, v, log_alpha, beta, cu_seqlens (int32 [B+1]), pad_mask (uint8 [N]
    or None), init_state (float32 [B,H,dk,dv] or None) and, when pads are used,
    ``valid_lengths`` and ``pad_sides`` (the unpadded lengths and where the pads sit).
    Pads carry q = k = v = 0 but keep random nonzero gates, so an implementation
    that lets pads decay or write the state shows it.
    """
    assert w.lengths is not None
    valid = [int(x) for x in w.lengths]
    B = len(valid)
    pad_n = [0] * B
    pad_left = [False] * B
    if w.pads:
        rng = _child(w.seed, "structure", 1)
        pad_n = [int(x) for x in rng.integers(0, 65, size=B)]
        pad_left = [bool(x) for x in rng.integers(0, 2, size=B)]
    lengths = [valid[b] + pad_n[b] for b in range(B)]
    cu = np.zeros(B + 1, dtype=np.int32)
    cu[1:] = np.cumsum(lengths)
    N = int(cu[-1])
    out = token_tensors(w.seed, N, w.H, w.dk, w.dv, w.dtype)
    out["cu_seqlens"] = cu
    out["pad_mask"] = None
    if w.pads:
        mask = np.ones(N, dtype=np.uint8)
        for b in range(B):
            if pad_n[b] == 0:
                continue
            s = int(cu[b]) if pad_left[b] else int(cu[b + 1]) - pad_n[b]
            mask[s:s + pad_n[b]] = 0
        for key in ("q", "k", "v"):
            out[key][mask == 0] = 0.0
        out["pad_mask"] = mask
        out["valid_lengths"] = np.asarray(valid, dtype=np.int64)
        out["pad_sides"] = np.asarray([1 if p else 0 for p in pad_left], dtype=np.int8)
    out["init_state"] = None
    if w.init_state:
        out["init_state"] = _normal(w.seed, "state", (B, w.H, w.dk, w.dv), scale=0.1)
    return out


def unpad(inputs: Dict[str, np.ndarray]) -> Dict[str, np.ndarray]:
    """The same batch with every pad position removed (the unpadded baseline)."""
    mask = inputs["pad_mask"]
    if mask is None:
        return dict(inputs)
    keep = mask.astype(bool)
    cu = inputs["cu_seqlens"]
    new_len = [int(keep[cu[b]:cu[b + 1]].sum()) for b in range(len(cu) - 1)]
    ncu = np.zeros(len(cu), dtype=np.int32)
    ncu[1:] = np.cumsum(new_len)
    out = {key: (val[keep] if key in ("q", "k", "v", "log_alpha", "beta") else val)
           for key, val in inputs.items()}
    out["cu_seqlens"] = ncu
    out["pad_mask"] = None
    return out


def decode_state(w: Workload) -> np.ndarray:
    """Initial decode state [rows, H, dk, dv] float32 ~ N(0, 0.1)."""
    return _normal(w.seed, "state", (w.decode_rows, w.H, w.dk, w.dv), scale=0.1)


def decode_pool(w: Workload, pool: int = 16) -> List[Dict[str, np.ndarray]]:
    """``pool`` distinct token batches for decode; step s uses batch s % pool."""
    out = []
    for i in range(pool):
        t = token_tensors(w.seed * 1000 + i, w.decode_rows, w.H, w.dk, w.dv, w.dtype)
        out.append(t)
    return out


def decode_mask(w: Workload, step: int) -> np.ndarray:
    """uint8 [rows]: exactly ``decode_masked`` rows are 0, chosen by a seeded permutation."""
    rng = _child(w.seed, "decode_mask", step)
    m = np.ones(w.decode_rows, dtype=np.uint8)
    m[rng.permutation(w.decode_rows)[: w.decode_masked]] = 0
    return m


def random_case(seed: int, lengths: Sequence[int], H: int, dk: int, dv: int, dtype: str = "f32",
                init_state: bool = False) -> Dict[str, np.ndarray]:
    """A small ad-hoc case with the standard distributions (for tests)."""
    cu = np.zeros(len(lengths) + 1, dtype=np.int32)
    cu[1:] = np.cumsum(lengths)
    out = token_tensors(seed, int(cu[-1]), H, dk, dv, dtype)
    out["cu_seqlens"] = cu
    out["pad_mask"] = None
    out["init_state"] = (_normal(seed, "state", (len(lengths), H, dk, dv), scale=0.1)
                         if init_state else None)
    return out
