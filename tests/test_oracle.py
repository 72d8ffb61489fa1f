"""Pins for the CPU oracle: closed forms, hand cases, brute force, invariants.

None of these compares the oracle with itself: every expected value comes from
the mathematics of the operator (special cases with a closed form, an explicit
matrix-product formulation, the chunkwise WY/UT algebra, invariants) or from
hand-derived fixtures in tests/golden/.
"""
import json
import os

import numpy as np
import pytest

from oracle import kda_oracle as orc
from gated_delta_rule_148_b200 import inputs as gen

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_cases.json")


def _one(seed, T, dk, dv, la_scale=1.0):
    """Single-sequence single-head inputs with the standard distributions."""
    c = gen.random_case(seed, [T], 1, dk, dv, "f32")
    return (c["q"][:, 0], c["k"][:, 0], c["v"][:, 0], c["log_alpha"][:, 0] * la_scale,
            c["beta"][:, 0])


def _run1(q, k, v, la, beta, S0=None, mask=None):
    """C oracle on one head / one sequence."""
    T = q.shape[0]
    o, fs = orc.prefill(q[:, None], k[:, None], v[:, None], la[:, None], beta[:, None],
                        np.array([0, T], np.int32), pad_mask=mask,
                        init_state=None if S0 is None else S0[None, None])
    return o[:, 0], fs[0, 0]


# ---------------------------------------------------------------- hand cases
@pytest.mark.parametrize("case", json.load(open(GOLDEN))["cases"], ids=lambda c: c["name"])
def test_hand_cases(case):
    q, k, v = (np.array(case[x], np.float32) for x in ("q", "k", "v"))
    la = np.log(np.array(case["alpha"], np.float64)).astype(np.float32)
    beta = np.array(case["beta"], np.float32)
    S0 = np.array(case["S0"], np.float32)
    o, S = _run1(q, k, v, la, beta, S0)
    np.testing.assert_allclose(o, case["o"], rtol=0, atol=1e-6)
    np.testing.assert_allclose(S, case["S_final"], rtol=0, atol=1e-6)
    o2, S2 = orc.brute_force(q, k, v, la, beta, S0)
    np.testing.assert_allclose(o2, case["o"], rtol=0, atol=1e-6)
    o3, S3 = orc.chunked(q, k, v, la, beta, 2, S0)
    np.testing.assert_allclose(o3, case["o"], rtol=0, atol=1e-6)
    np.testing.assert_allclose(S3, case["S_final"], rtol=0, atol=1e-6)


# ---------------------------------------------------------------- closed forms
def test_beta_zero_is_pure_per_channel_decay():
    """beta = 0: S_T = Diag(exp(sum log_alpha)) S0 and o_t = (Diag(exp(cumsum)) S0)^T q_t."""
    T, dk, dv = 37, 12, 9
    q, k, v, la, _ = _one(1, T, dk, dv)
    S0 = np.random.default_rng(2).normal(0, 1, (dk, dv)).astype(np.float32)
    o, S = _run1(q, k, v, la, np.zeros(T, np.float32), S0)
    G = np.cumsum(la.astype(np.float64), axis=0)
    np.testing.assert_allclose(S, np.exp(G[-1])[:, None] * S0, rtol=1e-12, atol=1e-14)
    o_ref = np.stack([(np.exp(G[t])[:, None] * S0).T @ q[t] for t in range(T)])
    np.testing.assert_allclose(o, o_ref, rtol=1e-12, atol=1e-14)


def test_unit_gate_zero_beta_keeps_state():
    """alpha = 1, beta = 0: the state never changes and o_t = S0^T q_t."""
    T, dk, dv = 20, 8, 16
    q, k, v, _, _ = _one(3, T, dk, dv)
    S0 = np.random.default_rng(4).normal(0, 1, (dk, dv)).astype(np.float32)
    o, S = _run1(q, k, v, np.zeros((T, dk), np.float32), np.zeros(T, np.float32), S0)
    np.testing.assert_array_equal(S, S0.astype(np.float64))
    np.testing.assert_allclose(o, q.astype(np.float64) @ S0.astype(np.float64), rtol=1e-13)


@pytest.mark.parametrize("dk,dv,T", [(16, 16, 16), (16, 8, 11), (8, 24, 8)])
def test_orthonormal_keys_exact_retrieval(dk, dv, T):
    """alpha = 1, beta = 1, orthonormal keys, S0 = 0: S_T^T k_j = v_j for every j."""
    rng = np.random.default_rng(5)
    Qm, _ = np.linalg.qr(rng.normal(size=(dk, dk)))
    k = Qm[:T].astype(np.float32)            # rows orthonormal (to fp32 rounding)
    v = rng.normal(size=(T, dv)).astype(np.float32)
    q = rng.normal(size=(T, dk)).astype(np.float32)
    _, S = _run1(q, k, v, np.zeros((T, dk), np.float32), np.ones(T, np.float32))
    kd = k.astype(np.float64)
    # the keys are orthonormal to ~1e-7 after fp32 rounding: exactness holds to that level
    np.testing.assert_allclose(kd @ S, v, rtol=0, atol=1e-5)
    # with keys re-orthonormalised in fp64 the retrieval is exact to rounding
    kk, _ = np.linalg.qr(kd.T)
    kk = kk.T[:T]
    o, S2 = orc.brute_force(q, kk, v, np.zeros((T, dk)), np.ones(T))
    np.testing.assert_allclose(kk @ S2, v, rtol=0, atol=1e-12)


def test_delta_rule_overwrite():
    """alpha = 1, beta = 1, one unit key written twice: reading it returns the second value."""
    dk, dv = 6, 5
    rng = np.random.default_rng(6)
    key = rng.normal(size=dk)
    key = (key / np.linalg.norm(key)).astype(np.float32)
    v1 = rng.normal(size=dv).astype(np.float32)
    v2 = rng.normal(size=dv).astype(np.float32)
    k = np.stack([key, key])
    q = np.stack([key, key])
    o, S = _run1(q, k, np.stack([v1, v2]), np.zeros((2, dk), np.float32), np.ones(2, np.float32))
    nk = float(key.astype(np.float64) @ key.astype(np.float64))   # 1 up to fp32 rounding
    np.testing.assert_allclose(o[0], v1 * nk, rtol=1e-6)
    np.testing.assert_allclose(o[1], v2 * nk, rtol=1e-6)
    np.testing.assert_allclose(S.T @ key, v2 * nk, rtol=1e-6)


# ---------------------------------------------------------------- brute force
@pytest.mark.parametrize("seed", range(6))
def test_brute_force_tiny(seed):
    """Explicit d_k x d_k transition products vs the C oracle on tiny inputs."""
    rng = np.random.default_rng(100 + seed)
    T = int(rng.integers(1, 9))
    dk, dv = int(rng.integers(1, 5)), int(rng.integers(1, 5))
    q, k, v = (rng.normal(size=(T, d)).astype(np.float32) for d in (dk, dk, dv))
    la = -np.abs(rng.normal(size=(T, dk))).astype(np.float32)
    beta = rng.uniform(-0.5, 1.5, size=T).astype(np.float32)
    S0 = rng.normal(size=(dk, dv)).astype(np.float32)
    mask = (rng.uniform(size=T) > 0.3).astype(np.uint8)
    o, S = _run1(q, k, v, la, beta, S0, mask)
    o2, S2 = orc.brute_force(q, k, v, la, beta, S0, mask)
    np.testing.assert_allclose(o, o2, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(S, S2, rtol=1e-12, atol=1e-12)
    assert np.all(o[mask == 0] == 0.0)


# ---------------------------------------------------------------- chunkwise algebra
@pytest.mark.parametrize("chunk", [1, 2, 16, 64])
@pytest.mark.parametrize("T,dk,dv", [(77, 16, 16), (150, 8, 24), (64, 24, 8)])
def test_chunked_ut_equals_recurrence(chunk, T, dk, dv):
    q, k, v, la, beta = _one(7, T, dk, dv)
    S0 = np.random.default_rng(8).normal(0, 0.1, (dk, dv)).astype(np.float32)
    o, S = _run1(q, k, v, la, beta, S0)
    o2, S2 = orc.chunked(q, k, v, la, beta, chunk, S0)
    np.testing.assert_allclose(o2, o, rtol=0, atol=1e-10 * max(1.0, np.abs(o).max()))
    np.testing.assert_allclose(S2, S, rtol=0, atol=1e-10 * max(1.0, np.abs(S).max()))


def test_chunked_handles_pads_as_identity_steps():
    T, dk, dv = 90, 8, 8
    q, k, v, la, beta = _one(9, T, dk, dv)
    mask = np.ones(T, np.uint8)
    mask[[0, 1, 40, 41, 42, 89]] = 0
    S0 = np.random.default_rng(10).normal(0, 0.1, (dk, dv)).astype(np.float32)
    o, S = _run1(q, k, v, la, beta, S0, mask)
    o2, S2 = orc.chunked(q, k, v, la, beta, 16, S0, mask)
    np.testing.assert_allclose(o2, o, atol=1e-11)
    np.testing.assert_allclose(S2, S, atol=1e-11)


# ---------------------------------------------------------------- carry / resume
@pytest.mark.parametrize("split", [1, 31, 64, 99])
def test_split_sequence_with_carried_state(split):
    T, dk, dv = 128, 16, 12
    q, k, v, la, beta = _one(11, T, dk, dv)
    S0 = np.random.default_rng(12).normal(0, 0.1, (dk, dv)).astype(np.float32)
    o, S = _run1(q, k, v, la, beta, S0)
    oa, Sa = _run1(q[:split], k[:split], v[:split], la[:split], beta[:split], S0)
    # carry the fp64 state exactly: continue with the brute force from Sa
    ob, Sb = orc.brute_force(q[split:], k[split:], v[split:], la[split:], beta[split:], Sa)
    np.testing.assert_allclose(np.concatenate([oa, ob]), o, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(Sb, S, rtol=1e-12, atol=1e-13)


def test_prefill_then_decode_continuation():
    T, H, dk, dv = 40, 3, 8, 8
    c = gen.random_case(13, [T + 1], H, dk, dv, "f32", init_state=True)
    o, fs = orc.prefill(c["q"], c["k"], c["v"], c["log_alpha"], c["beta"], c["cu_seqlens"],
                        init_state=c["init_state"])
    o1, fs1 = orc.prefill(c["q"][:T], c["k"][:T], c["v"][:T], c["log_alpha"][:T],
                          c["beta"][:T], np.array([0, T], np.int32), init_state=c["init_state"])
    st = fs1.copy()
    od = orc.decode(c["q"][T:], c["k"][T:], c["v"][T:], c["log_alpha"][T:], c["beta"][T:], st)
    np.testing.assert_allclose(od[0], o[T], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(st, fs, rtol=1e-12, atol=1e-13)


def test_decode_mask_leaves_rows_untouched():
    B, H, d = 6, 2, 8
    c = gen.random_case(14, [1] * B, H, d, d, "f32", init_state=True)
    st = c["init_state"].astype(np.float64)
    before = st.copy()
    mask = np.array([1, 0, 1, 0, 0, 1], np.uint8)
    o = orc.decode(c["q"], c["k"], c["v"], c["log_alpha"], c["beta"], st, mask)
    assert np.all(o[mask == 0] == 0.0)
    np.testing.assert_array_equal(st[mask == 0], before[mask == 0])
    assert np.all(np.abs(st[mask == 1] - before[mask == 1]).max(axis=(1, 2, 3)) > 0)
    # active rows equal a one-token prefill per row
    o2, fs2 = orc.prefill(c["q"], c["k"], c["v"], c["log_alpha"], c["beta"], c["cu_seqlens"],
                          init_state=c["init_state"])
    np.testing.assert_allclose(o[mask == 1], o2[mask == 1], rtol=1e-13)
    np.testing.assert_allclose(st[mask == 1], fs2[mask == 1], rtol=1e-13)


# ---------------------------------------------------------------- packing and padding
def test_varlen_packing_equals_solo_runs():
    lengths = [1, 15, 16, 17, 50]
    H, dk, dv = 2, 8, 12
    c = gen.random_case(15, lengths, H, dk, dv, "f32", init_state=True)
    o, fs = orc.prefill(c["q"], c["k"], c["v"], c["log_alpha"], c["beta"], c["cu_seqlens"],
                        init_state=c["init_state"])
    cu = c["cu_seqlens"]
    for b in range(len(lengths)):
        sl = slice(cu[b], cu[b + 1])
        for h in range(H):
            ob, Sb = orc.brute_force(c["q"][sl, h], c["k"][sl, h], c["v"][sl, h],
                                     c["log_alpha"][sl, h], c["beta"][sl, h],
                                     c["init_state"][b, h])
            np.testing.assert_allclose(o[sl, h], ob, rtol=1e-12, atol=1e-13)
            np.testing.assert_allclose(fs[b, h], Sb, rtol=1e-12, atol=1e-13)


def _buggy_pads(q, k, v, la, beta, S0, mask):
    """A planted mistake (test-only): pads zero q/k/v but keep their gates."""
    q, k, v = q.copy(), k.copy(), v.copy()
    q[mask == 0] = 0
    k[mask == 0] = 0
    v[mask == 0] = 0
    return orc.brute_force(q, k, v, la, beta, S0)


@pytest.mark.parametrize("side", ["left", "right", "interior"])
def test_padding_equals_unpadded_run(side):
    """Cached continuation (6 cached positions), 3 valid + 2 pads, then 1 probe position.

    The shape follows the reproduction in "Transformers Community Reports Kimi
    Linear Cache Bug" (ainews): the baseline is the UNPADDED run, not a padded one.
    """
    dk = dv = 8
    q, k, v, la, beta = _one(16, 6 + 5 + 1, dk, dv)
    # cached prefix
    _, Sc = orc.brute_force(q[:6], k[:6], v[:6], la[:6], beta[:6])
    Sc32 = Sc.astype(np.float32)
    valid_idx = np.arange(6, 9)
    # padded continuation: 5 positions, pads where requested, zero q/k/v but random gates
    pad_pos = {"left": [0, 1], "right": [3, 4], "interior": [1, 3]}[side]
    mask = np.ones(5, np.uint8)
    mask[pad_pos] = 0
    qp, kp, vp = (np.zeros((5, dk), np.float32) for _ in range(3))
    slots = np.nonzero(mask)[0]
    qp[slots], kp[slots], vp[slots] = q[valid_idx], k[valid_idx], v[valid_idx]
    lap = -np.abs(np.random.default_rng(17).normal(size=(5, dk))).astype(np.float32)
    lap[slots] = la[valid_idx]
    bp = np.random.default_rng(18).uniform(0.2, 0.9, 5).astype(np.float32)
    bp[slots] = beta[valid_idx]
    o_pad, S_pad = _run1(qp, kp, vp, lap, bp, Sc32, mask)
    o_ref, S_ref = _run1(q[valid_idx], k[valid_idx], v[valid_idx], la[valid_idx],
                         beta[valid_idx], Sc32)
    np.testing.assert_array_equal(o_pad[mask == 0], 0.0)
    np.testing.assert_allclose(o_pad[slots], o_ref, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(S_pad, S_ref, rtol=1e-13, atol=1e-14)
    # the probe position after the continuation sees the same state
    probe = 11
    p_pad, _ = _run1(q[probe:], k[probe:], v[probe:], la[probe:], beta[probe:],
                     S_pad.astype(np.float32))
    p_ref, _ = _run1(q[probe:], k[probe:], v[probe:], la[probe:], beta[probe:],
                     S_ref.astype(np.float32))
    np.testing.assert_array_equal(p_pad, p_ref)
    # positive control: letting pads decay the state (the reported bug) is visible
    ob, Sb = _buggy_pads(qp, kp, vp, lap, bp, Sc32, mask)
    assert np.abs(Sb - S_ref).max() > 1e-3


# ---------------------------------------------------------------- invariants
def test_linearity_in_values_and_state():
    """o(a V1 + b V2, a S1 + b S2) = a o(V1, S1) + b o(V2, S2) for fixed q, k, gates."""
    T, dk, dv = 30, 8, 6
    q, k, v1, la, beta = _one(19, T, dk, dv)
    v1 = v1.astype(np.float64)
    rng = np.random.default_rng(20)
    v2 = rng.normal(size=v1.shape)
    S1, S2 = rng.normal(size=(dk, dv)), rng.normal(size=(dk, dv))
    a, b = 0.75, -1.5
    o1, F1 = orc.brute_force(q, k, v1, la, beta, S1)
    o2, F2 = orc.brute_force(q, k, v2, la, beta, S2)
    vm = (a * v1 + b * v2)
    Sm = (a * S1 + b * S2)
    om, Fm = orc.brute_force(q, k, vm, la, beta, Sm)
    np.testing.assert_allclose(om, a * o1 + b * o2, atol=1e-12)
    np.testing.assert_allclose(Fm, a * F1 + b * F2, atol=1e-12)
    # and the C oracle agrees on the mixed case (inputs exactly representable in fp32)
    vm32, Sm32 = vm.astype(np.float32), Sm.astype(np.float32)   # representable inputs
    oc, Fc = _run1(q, k, vm32, la, beta, Sm32)
    ob, Fb = orc.brute_force(q, k, vm32, la, beta, Sm32)
    np.testing.assert_allclose(oc, ob, atol=1e-12)


def test_contraction_bound():
    """||S_t||_F <= ||S_{t-1}||_F + |beta| ||k|| ||v|| for unit k, beta in [0,1], alpha <= 1."""
    T, dk, dv = 50, 8, 8
    q, k, v, la, beta = _one(21, T, dk, dv)
    S = np.random.default_rng(22).normal(size=(dk, dv))
    for t in range(T):
        prev = np.linalg.norm(S)
        _, S = orc.brute_force(q[t:t + 1], k[t:t + 1], v[t:t + 1], la[t:t + 1], beta[t:t + 1], S)
        bound = prev + abs(beta[t]) * np.linalg.norm(k[t]) * np.linalg.norm(v[t])
        assert np.linalg.norm(S) <= bound * (1 + 1e-12)


# ---------------------------------------------------------------- prefix invariance
def _leaky_chunked(q, k, v, la, beta, chunk):
    """Planted leak (test-only): every chunk after the first reads the sequence's
    FINAL state instead of its incoming state -- a reduction over the wrong chunk
    axis, the defect class of "The Mask Is Not the Model" (dev.to)."""
    _, S_final = orc.chunked(q, k, v, la, beta, chunk)
    o_ok, _ = orc.chunked(q, k, v, la, beta, chunk)
    T = q.shape[0]
    o = o_ok.copy()
    for c0 in range(chunk, T, chunk):
        g = np.cumsum(la[c0:c0 + chunk].astype(np.float64), axis=0)
        o[c0:c0 + chunk] += (q[c0:c0 + chunk] * np.exp(g)) @ S_final * 1e-3
    return o, S_final


@pytest.mark.parametrize("T", [16 * 3 + 1, 16 * 4 + 7])
def test_prefix_invariance_with_positive_control(T):
    """Perturbing position T-1 leaves o[0:T-1] unchanged; a planted leak is caught
    with onset equal to the chunk size (audit length T exceeds 3 chunks)."""
    C, dk, dv = 16, 8, 8
    q, k, v, la, beta = _one(23, T, dk, dv)
    rng = np.random.default_rng(24)

    def variant(which, fn):
        qq, kk, vv, ll, bb = q.copy(), k.copy(), v.copy(), la.copy(), beta.copy()
        if which:
            qq[T - 1] = rng.normal(size=dk)
            kk[T - 1] = rng.normal(size=dk)
            vv[T - 1] = rng.normal(size=dv)
            ll[T - 1] = -np.abs(rng.normal(size=dk))
            bb[T - 1] = 0.123
        return fn(qq, kk, vv, ll, bb)

    for fn in (lambda *a: _run1(*a)[0], lambda *a: orc.chunked(*a, C)[0]):
        leak, onset, d = orc.prefix_audit(lambda w: variant(w, fn), T, 1)
        assert not leak and d.max() == 0.0
    leak, onset, _ = orc.prefix_audit(lambda w: variant(w, lambda *a: _leaky_chunked(*a, C)[0]),
                                      T, 1)
    assert leak and onset == C


# ---------------------------------------------------------------- head-wise gate
def _run_head(q, k, v, la_head, beta, S0, H=2):
    """C oracle through its [N, H] gate entry: one sequence, the same inputs on H heads
    (head h uses la_head * (h + 1), so a broadcast over the wrong axis shows)."""
    T, dk = q.shape
    rep = lambda x: np.repeat(x[:, None], H, axis=1)
    la = np.stack([la_head * (h + 1) for h in range(H)], axis=1).astype(np.float32)
    o, fs = orc.prefill(rep(q), rep(k), rep(v), la, rep(beta), np.array([0, T], np.int32),
                        init_state=np.repeat(S0[None, None], H, axis=1))
    return o, fs[0]


def test_head_gate_zero_beta_closed_form():
    """One gate per token and head, beta = 0: S_T = exp(sum log_alpha) S0 (a scalar per
    head) and o_t = exp(cumsum_t) S0^T q_t."""
    T, dk, dv = 29, 10, 7
    q, k, v, _, _ = _one(21, T, dk, dv)
    la = -np.abs(np.random.default_rng(22).normal(0.2, 0.1, T)).astype(np.float32)
    S0 = np.random.default_rng(23).normal(0, 1, (dk, dv)).astype(np.float32)
    o, S = _run_head(q, k, v, la, np.zeros(T, np.float32), S0)
    for h in range(2):
        G = np.cumsum(la.astype(np.float64) * (h + 1))
        np.testing.assert_allclose(S[h], np.exp(G[-1]) * S0, rtol=1e-12, atol=1e-14)
        o_ref = np.stack([np.exp(G[t]) * (S0.T.astype(np.float64) @ q[t]) for t in range(T)])
        np.testing.assert_allclose(o[:, h], o_ref, rtol=1e-12, atol=1e-14)


def test_head_gate_brute_force():
    """Explicit transitions alpha_t (I - beta_t k_t k_t^T) (a scalar gate times the
    identity) vs the C oracle given the [N, H] gate."""
    rng = np.random.default_rng(31)
    T, dk, dv = 9, 4, 3
    q, k, v = (rng.normal(size=(T, d)).astype(np.float32) for d in (dk, dk, dv))
    la = -np.abs(rng.normal(size=T)).astype(np.float32)
    beta = rng.uniform(0, 1, size=T).astype(np.float32)
    S0 = rng.normal(size=(dk, dv)).astype(np.float32)
    o, S = _run_head(q, k, v, la, beta, S0, H=1)
    Sx = S0.astype(np.float64)
    for t in range(T):
        kk = k[t].astype(np.float64)
        A = np.exp(np.float64(la[t])) * (np.eye(dk) - np.float64(beta[t]) * np.outer(kk, kk))
        Sx = A @ Sx + np.float64(beta[t]) * np.outer(kk, v[t].astype(np.float64))
        np.testing.assert_allclose(o[t, 0], Sx.T @ q[t].astype(np.float64), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(S[0], Sx, rtol=1e-12, atol=1e-12)


def test_head_gate_rotation_invariance_with_positive_control():
    """A gate that is a scalar per head commutes with any rotation R of the key space:
    (q, k, S0) -> (R q, R k, R S0) gives S_t -> R S_t and the same o_t.  A per-channel
    gate does not commute with R, so the same check must fail for it."""
    T, dk, dv = 40, 8, 5
    q, k, v, la_ch, beta = _one(41, T, dk, dv)
    la_h = la_ch[:, 0].copy()
    S0 = np.random.default_rng(42).normal(0, 1, (dk, dv)).astype(np.float32)
    R, _ = np.linalg.qr(np.random.default_rng(43).normal(size=(dk, dk)))
    rot = lambda x: (x.astype(np.float64) @ R.T).astype(np.float32)   # rows x -> R x
    S0r = (R @ S0.astype(np.float64)).astype(np.float32)
    o1, S1 = _run_head(q, k, v, la_h, beta, S0, H=1)
    o2, S2 = _run_head(rot(q), rot(k), v, la_h, beta, S0r, H=1)
    tol = 1e-5 * max(1.0, np.abs(o1).max())        # float32 rounding of the rotated inputs
    np.testing.assert_allclose(o2, o1, rtol=0, atol=tol)
    np.testing.assert_allclose(S2[0], R @ S1[0], rtol=0, atol=tol)
    # positive control: per-channel gates break the invariance
    p1, _ = _run1(q, k, v, la_ch, beta, S0)
    p2, _ = _run1(rot(q), rot(k), v, la_ch, beta, S0r)
    assert np.abs(p2 - p1).max() > 100 * tol


# ---------------------------------------------------------------- short convolution
def _conv_case(seed, lengths, D, W, pads=0.0, state=True):
    rng = np.random.default_rng(seed)
    cu = np.zeros(len(lengths) + 1, np.int64)
    cu[1:] = np.cumsum(lengths)
    N = int(cu[-1])
    x = rng.normal(size=(N, D)).astype(np.float32)
    w = rng.normal(size=(D, W)).astype(np.float32)
    b = rng.normal(size=D).astype(np.float32)
    m = None if pads == 0 else (rng.uniform(size=N) >= pads).astype(np.uint8)
    s = rng.normal(size=(len(lengths), W - 1, D)).astype(np.float32) if state else None
    return x, w, b, cu, m, s


@pytest.mark.parametrize("W", [1, 2, 3, 4])
def test_conv_unpadded_equals_numpy_convolve(W):
    """No pads, zero state: each channel is numpy's full convolution with the reversed
    weights, truncated to the sequence (the causal window), plus the bias."""
    x, w, b, cu, _, _ = _conv_case(61, [37, 5, 64], 6, W, state=False)
    y, s = orc.short_conv(x, w, b, cu)
    for i in range(len(cu) - 1):
        a, e = int(cu[i]), int(cu[i + 1])
        for c in range(6):
            ref = np.convolve(x[a:e, c].astype(np.float64), w[c, ::-1].astype(np.float64))[:e - a] + b[c]
            np.testing.assert_allclose(y[a:e, c], ref, rtol=1e-12, atol=1e-12)
        # final state: the last W-1 inputs (zeros in front when the sequence is short)
        tail = np.concatenate([np.zeros((W - 1, 6)), x[a:e].astype(np.float64)])[-(W - 1):] if W > 1 else np.zeros((0, 6))
        np.testing.assert_array_equal(s[i], tail)


def test_conv_padding_equals_unpadded_run_with_positive_control():
    """Pads anywhere (edges and inside) give the unpadded run's outputs at the valid
    positions, 0 at the pads, and the same final state; a window that lets pads in
    (the reported bug) does not."""
    x, w, b, cu, m, s = _conv_case(62, [40, 3, 70], 5, 4, pads=0.3)
    m[38], m[39] = 0, 1            # a pad inside sequence 0's final window
    y, so = orc.short_conv(x, w, b, cu, m, s)
    keep = m.astype(bool)
    lens = [int(keep[cu[i]:cu[i + 1]].sum()) for i in range(len(cu) - 1)]
    cu2 = np.concatenate([[0], np.cumsum(lens)])
    y2, so2 = orc.short_conv(x[keep], w, b, cu2, None, s)
    np.testing.assert_array_equal(y[keep], y2)
    assert np.all(y[~keep] == 0.0)
    np.testing.assert_array_equal(so, so2)
    # positive control: pads as zero inputs inside the window
    xz = x.copy()
    xz[~keep] = 0.0
    y3, so3 = orc.short_conv(xz, w, b, cu, None, s)
    assert np.abs(y3[keep] - y2).max() > 1e-3 and np.abs(so3 - so2).max() > 1e-3


def test_conv_split_sequence_with_carried_state():
    """Two calls, the second starting from the first's state, equal one call."""
    x, w, b, _, m, s = _conv_case(63, [90], 7, 3, pads=0.2)
    cu = np.array([0, 90])
    y, so = orc.short_conv(x, w, b, cu, m, s)
    for cut in (1, 2, 45, 89):
        ya, sa = orc.short_conv(x[:cut], w, b, [0, cut], m[:cut], s)
        yb, sb = orc.short_conv(x[cut:], w, b, [0, 90 - cut], m[cut:], sa)
        np.testing.assert_allclose(np.concatenate([ya, yb]), y, rtol=0, atol=1e-12)
        np.testing.assert_array_equal(sb, so)


def test_conv_short_sequences_shift_the_state():
    """A sequence with n < W-1 valid inputs: the new state is the old one shifted by n
    rows with the n inputs appended; with only pads it is unchanged."""
    W, D = 4, 3
    rng = np.random.default_rng(64)
    s = rng.normal(size=(3, W - 1, D))
    x = rng.normal(size=(4, D))
    m = np.array([1, 0, 0, 1], np.uint8)         # seq0: 1 valid; seq1: 1 pad; seq2: 1 valid
    cu = [0, 1, 2, 4]
    y, so = orc.short_conv(x, np.ones((D, W)), None, cu, m, s)
    np.testing.assert_array_equal(so[0], np.concatenate([s[0][1:], x[0:1]]))
    np.testing.assert_array_equal(so[1], s[1])
    np.testing.assert_array_equal(so[2], np.concatenate([s[2][1:], x[3:4]]))
    np.testing.assert_allclose(y[0], s[0].sum(0) + x[0], rtol=1e-12)   # all-ones weights
    assert np.all(y[1] == 0) and np.all(y[2] == 0)


def test_conv_sampled_positions_match_window_form():
    x, w, b, cu, m, s = _conv_case(65, [33, 1, 120], 4, 4, pads=0.25)
    y, _ = orc.short_conv(x, w, b, cu, m, s)
    pos = np.array([0, 1, 5, 33, 34, 35, 100, 153])
    np.testing.assert_allclose(orc.short_conv_at(x, w, b, cu, pos, m, s), y[pos], rtol=0, atol=1e-12)


# ---------------------------------------------------------------- backward pass
def _loss_bf(q, k, v, la, be, S0, cu, m, do, dSf):
    """<o, do> + <S_final, dSf> through the fp64 brute force (explicit transitions),
    per sequence and head; la may be [N, H] (head-wise gate)."""
    tot = 0.0
    la_full = orc.head_gate_channels(la, q.shape[2])
    for b in range(len(cu) - 1):
        a, e = int(cu[b]), int(cu[b + 1])
        for h in range(q.shape[1]):
            o, S = orc.brute_force(q[a:e, h], k[a:e, h], v[a:e, h], la_full[a:e, h], be[a:e, h],
                                   S0[b, h], None if m is None else m[a:e])
            tot += (o * do[a:e, h]).sum() + (S * dSf[b, h]).sum()
    return tot


@pytest.mark.parametrize("head_gate", [False, True])
def test_backward_matches_central_differences(head_gate):
    """Every gradient of prefill_backward equals the central difference of the fp64
    brute-force loss <o, dO> + <S_T, dS_T> (step 1e-6), on two sequences with pads."""
    rng = np.random.default_rng(71)
    N, H, dk, dv = 9, 2, 3, 2
    q, k = rng.normal(size=(N, H, dk)), rng.normal(size=(N, H, dk))
    v = rng.normal(size=(N, H, dv))
    la = -np.abs(rng.normal(size=(N, H) if head_gate else (N, H, dk)))
    be = rng.uniform(-0.3, 1.2, (N, H))
    S0 = rng.normal(size=(2, H, dk, dv))
    cu = np.array([0, 4, 9])
    m = np.array([1, 1, 0, 1, 1, 0, 1, 1, 1], np.uint8)
    do, dSf = rng.normal(size=(N, H, dv)), rng.normal(size=(2, H, dk, dv))
    g = orc.prefill_backward(q, k, v, la, be, cu, do, dSf, m, S0)
    args = dict(q=q, k=k, v=v, la=la, be=be, S0=S0)
    keys = dict(q="dq", k="dk", v="dv", la="dlog_alpha", be="dbeta", S0="dS0")
    eps = 1e-6
    for name, x in list(args.items()):
        fd = np.zeros_like(x)
        for i in np.ndindex(x.shape):
            for sgn in (1, -1):
                xx = x.copy()
                xx[i] += sgn * eps
                fd[i] += sgn * _loss_bf(**dict(args, **{name: xx}), cu=cu, m=m, do=do, dSf=dSf)
        fd /= 2 * eps
        np.testing.assert_allclose(g[keys[name]], fd, rtol=1e-6, atol=1e-7, err_msg=name)
    # pads: zero input gradients
    for key in ("dq", "dk", "dv", "dlog_alpha", "dbeta"):
        assert np.all(g[key][m == 0] == 0.0)


def test_backward_zero_upstream_and_state_only():
    """dO = 0 and dS_T = 0 give all-zero gradients; with beta = 0 and dO = 0 the state
    gradient is the closed form dS0 = Diag(exp(sum log_alpha)) dS_T and
    dlog_alpha_t = rowsum(dS_T * S_T) for every t (each decay scales the final state)."""
    rng = np.random.default_rng(72)
    N, dk, dv = 6, 4, 3
    q, k, v = rng.normal(size=(N, 1, dk)), rng.normal(size=(N, 1, dk)), rng.normal(size=(N, 1, dv))
    la = -np.abs(rng.normal(size=(N, 1, dk)))
    S0 = rng.normal(size=(1, 1, dk, dv))
    cu = np.array([0, N])
    g = orc.prefill_backward(q, k, v, la, rng.uniform(size=(N, 1)), cu, np.zeros((N, 1, dv)),
                             None, None, S0)
    assert all(np.all(g[key] == 0) for key in ("dq", "dk", "dv", "dlog_alpha", "dbeta", "dS0"))
    dSf = rng.normal(size=(1, 1, dk, dv))
    g = orc.prefill_backward(q, k, v, la, np.zeros((N, 1)), cu, np.zeros((N, 1, dv)), dSf, None, S0)
    decay = np.exp(la[:, 0].sum(axis=0))
    np.testing.assert_allclose(g["dS0"][0, 0], decay[:, None] * dSf[0, 0], rtol=1e-12)
    ST = decay[:, None] * S0[0, 0]
    for t in range(N):
        np.testing.assert_allclose(g["dlog_alpha"][t, 0], (dSf[0, 0] * ST).sum(axis=1), rtol=1e-12)

