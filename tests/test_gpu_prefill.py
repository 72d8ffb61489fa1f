"""GPU parity tests for kda_prefill against the fp64 oracle (call through the C ABI).

Tolerance (normalised max-abs error of o and of the final state): 1e-4 for
fp32 inputs, 2e-2 for bf16 inputs.  Pad outputs must be exactly 0 and a
perturbation of the last position must leave every earlier output
bit-identical.
"""
import numpy as np
import pytest
import torch

from gated_delta_rule_148_b200 import inputs as gen
from gated_delta_rule_148_b200 import kda
from kda_testlib import TOL, dev_inputs, norm_err, to_np
from oracle import kda_oracle as orc

pytestmark = pytest.mark.gpu


def _gpu(inp, dtype, chunk=0, in_place=False):
    d = dev_inputs(inp, dtype)
    fs = None
    if in_place and "init_state" in d:
        fs = d["init_state"]
    o, fs = kda.prefill(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["cu_seqlens"],
                        pad_mask=d.get("pad_mask"), init_state=d.get("init_state"),
                        final_state=fs, chunk=chunk)
    torch.cuda.synchronize()
    assert kda.get_device_status() == kda.KDA_OK
    return o, fs


def _oracle(inp, heads=None):
    sel = slice(None) if heads is None else list(heads)
    s0 = inp.get("init_state")
    return orc.prefill(inp["q"][:, sel], inp["k"][:, sel], inp["v"][:, sel],
                       inp["log_alpha"][:, sel], inp["beta"][:, sel], inp["cu_seqlens"],
                       pad_mask=inp.get("pad_mask"),
                       init_state=None if s0 is None else s0[:, sel])


def _check(inp, dtype, o, fs, heads=None):
    o_ref, s_ref = _oracle(inp, heads)
    sel = slice(None) if heads is None else list(heads)
    eo = norm_err(to_np(o)[:, sel], o_ref)
    es = norm_err(to_np(fs)[:, sel], s_ref)
    assert eo <= TOL[dtype], f"o error {eo:.3e}"
    assert es <= TOL[dtype], f"state error {es:.3e}"
    return eo, es


def test_tiny_f32_chunk16():
    """B=1, H=2, T=128, d=64, chunk 16, fp32, zero initial state."""
    w = gen.tiny_f32()
    inp = gen.prefill_inputs(w)
    o, fs = _gpu(inp, "f32", chunk=16)
    _check(inp, "f32", o, fs)


@pytest.mark.parametrize("chunk", [16, 32, 64])
@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64), (128, 128)])
def test_f32_shapes_and_chunks(chunk, dk, dv):
    inp = gen.random_case(31, [1, chunk - 1, chunk, chunk + 1, 3 * chunk + 5], 2, dk, dv, "f32",
                          init_state=True)
    o, fs = _gpu(inp, "f32", chunk=chunk)
    _check(inp, "f32", o, fs)


@pytest.mark.parametrize("chunk", [16, 32, 64])
@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64), (128, 128)])
def test_bf16_shapes_and_chunks(chunk, dk, dv):
    inp = gen.random_case(32, [1, 63, 64, 65, 300], 3, dk, dv, "bf16", init_state=True)
    o, fs = _gpu(inp, "bf16", chunk=chunk)
    _check(inp, "bf16", o, fs)


def test_prefill_4k_h32_bf16():
    """B=1, H=32, T=4096, d=128, bf16 q/k/v, chunk 64, zero initial state (all heads)."""
    w = gen.prefill(4096)
    inp = gen.prefill_inputs(w)
    o, fs = _gpu(inp, "bf16")
    _check(inp, "bf16", o, fs)


def test_in_place_state_update():
    inp = gen.random_case(33, [100, 200], 2, 128, 128, "bf16", init_state=True)
    o, fs = _gpu(inp, "bf16", in_place=True)
    _check(inp, "bf16", o, fs)


def test_state_layout_needle():
    """d_k != d_v and a distinctive key->value written early, read back many chunks later
    with alpha ~ 1: a transposed or mis-strided state cannot return it."""
    for dk, dv in ((64, 128), (128, 64)):
        T = 64 * 20 + 17
        inp = gen.random_case(34, [T], 1, dk, dv, "bf16", init_state=True)
        inp["log_alpha"][:] = -1e-4
        inp["beta"][:] = 0.0
        key = np.zeros(dk, np.float32)
        key[5] = 1.0
        val = gen.round_bf16(np.linspace(-2, 2, dv).astype(np.float32))
        inp["k"][3, 0] = key
        inp["v"][3, 0] = val
        inp["beta"][3, 0] = 1.0
        inp["q"][T - 1, 0] = key
        o, fs = _gpu(inp, "bf16")
        _check(inp, "bf16", o, fs)
        o_ref, _ = _oracle(inp)
        assert np.abs(o_ref[T - 1, 0] - val).max() < 0.05 + 0.25 * np.abs(val).max()


def test_varlen_each_sequence_equals_solo_run():
    lengths = [1, 63, 64, 65, 700]
    inp = gen.random_case(35, lengths, 2, 128, 128, "bf16", init_state=True)
    o, fs = _gpu(inp, "bf16")
    cu = inp["cu_seqlens"]
    for b in range(len(lengths)):
        solo = {k: v[cu[b]:cu[b + 1]] for k, v in inp.items()
                if k in ("q", "k", "v", "log_alpha", "beta")}
        solo["cu_seqlens"] = np.array([0, lengths[b]], np.int32)
        solo["init_state"] = inp["init_state"][b:b + 1]
        o1, fs1 = _gpu(solo, "bf16")
        assert torch.equal(o[cu[b]:cu[b + 1]], o1)
        assert torch.equal(fs[b:b + 1], fs1)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_edge_pads_bit_identical_to_unpadded(dtype):
    """Cached continuation with 0-64 zero-valued pads (random gates) left or right per
    sequence: outputs and state equal the UNPADDED run bit for bit; pad outputs are 0."""
    w = gen.varlen_cached(H=4, n_seqs=6, lo=100, hi=700)
    w = gen.Workload(w.name, w.seed, w.H, w.dk, w.dv, dtype, 64, lengths=w.lengths,
                     init_state=True, pads=True)
    inp = gen.prefill_inputs(w)
    assert inp["pad_mask"].min() == 0
    un = gen.unpad(inp)
    o, fs = _gpu(inp, dtype)
    o_u, fs_u = _gpu(un, dtype)
    keep = torch.from_numpy(inp["pad_mask"].astype(bool)).cuda()
    assert torch.equal(o[keep], o_u)
    assert torch.equal(fs, fs_u)
    assert torch.all(o[~keep] == 0)
    _check(inp, dtype, o, fs)


def test_interior_pads_match_unpadded_within_tolerance():
    lengths = [300, 257]
    inp = gen.random_case(36, lengths, 2, 128, 128, "bf16", init_state=True)
    mask = np.ones(sum(lengths), np.uint8)
    mask[[5, 6, 64, 100, 101, 102, 299, 300, 420]] = 0
    inp["pad_mask"] = mask
    for key in ("q", "k", "v"):
        inp[key][mask == 0] = 0.0
    o, fs = _gpu(inp, "bf16")
    assert torch.all(o[torch.from_numpy(mask == 0).cuda()] == 0)
    _check(inp, "bf16", o, fs)


def test_cached_continuation_repro_shape():
    """Cache 6 positions, continue with 3 valid + 2 pads (left, then right), probe 1."""
    for side in ("left", "right"):
        inp = gen.random_case(37, [6 + 5 + 1], 1, 128, 128, "bf16")
        full = {k: v.copy() if isinstance(v, np.ndarray) else v for k, v in inp.items()}
        # cached prefix on the GPU
        pre = {k: full[k][:6] for k in ("q", "k", "v", "log_alpha", "beta")}
        pre["cu_seqlens"] = np.array([0, 6], np.int32)
        _, s6 = _gpu(pre, "bf16")
        cont = {k: full[k][6:11].copy() for k in ("q", "k", "v", "log_alpha", "beta")}
        mask = np.ones(5, np.uint8)
        mask[[0, 1] if side == "left" else [3, 4]] = 0
        for key in ("q", "k", "v"):
            cont[key][mask == 0] = 0.0
        cont["pad_mask"] = mask
        cont["cu_seqlens"] = np.array([0, 5], np.int32)
        cont["init_state"] = to_np(s6)
        o_p, s_p = _gpu(cont, "bf16")
        unp = {k: cont[k][mask == 1] for k in ("q", "k", "v", "log_alpha", "beta")}
        unp["cu_seqlens"] = np.array([0, 3], np.int32)
        unp["init_state"] = cont["init_state"]
        o_u, s_u = _gpu(unp, "bf16")
        assert torch.equal(o_p[torch.from_numpy(mask == 1).cuda()], o_u)
        assert torch.equal(s_p, s_u)
        probe = {k: full[k][11:12] for k in ("q", "k", "v", "log_alpha", "beta")}
        probe["cu_seqlens"] = np.array([0, 1], np.int32)
        probe["init_state"] = to_np(s_p)
        op, _ = _gpu(probe, "bf16")
        probe["init_state"] = to_np(s_u)
        ou, _ = _gpu(probe, "bf16")
        assert torch.equal(op, ou)


@pytest.mark.parametrize("dtype,T", [("bf16", 64 * 3 + 1), ("bf16", 64 * 4 + 30),
                                     ("f32", 16 * 3 + 1), ("f32", 16 * 5 + 9)])
def test_prefix_invariance_bit_identical(dtype, T):
    """Perturb q, k, v, log_alpha, beta at position T-1: o[0:T-1] is bit-identical.
    T spans at least 3 chunks; T-1 sits at a chunk start or mid-chunk (the audit
    length exceeds the chunk, "The Mask Is Not the Model", dev.to)."""
    inp = gen.random_case(38, [T], 4, 128, 128, dtype, init_state=True)
    chunk = 64 if dtype == "bf16" else 16
    rng = np.random.default_rng(39)

    def run(which):
        x = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in inp.items()}
        if which:
            x["q"][T - 1] = gen.round_bf16(rng.normal(size=x["q"][T - 1].shape).astype(np.float32))
            x["k"][T - 1] = gen.round_bf16(rng.normal(size=x["k"][T - 1].shape).astype(np.float32))
            x["v"][T - 1] = gen.round_bf16(rng.normal(size=x["v"][T - 1].shape).astype(np.float32))
            x["log_alpha"][T - 1] = -np.abs(rng.normal(size=x["log_alpha"][T - 1].shape))
            x["beta"][T - 1] = 0.77
        o, _ = _gpu(x, dtype, chunk=chunk)
        return to_np(o)

    leak, onset, d = orc.prefix_audit(run, T, 1)
    assert not leak, f"prefix leak, onset {onset}"
    assert d.max() == 0.0


def test_invalid_cu_seqlens_is_reported_and_nothing_written():
    inp = gen.random_case(40, [50, 60], 2, 64, 64, "bf16")
    d = dev_inputs(inp, "bf16")
    cu = torch.tensor([0, 70, 60], dtype=torch.int32, device="cuda")   # not non-decreasing
    o = torch.full((110, 2, 64), 7.0, dtype=torch.bfloat16, device="cuda")
    fs = torch.full((2, 2, 64, 64), 3.0, device="cuda")
    kda.prefill(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], cu, o=o, final_state=fs)
    assert kda.get_device_status() == kda.KDA_ERR_DEVICE_CHECK
    assert torch.all(o == 7.0) and torch.all(fs == 3.0)
    # the latch was cleared: a valid call works again
    o2, fs2 = _gpu(inp, "bf16")
    _check(inp, "bf16", o2, fs2)


def test_empty_sequences_keep_initial_state():
    inp = gen.random_case(41, [0, 5, 0], 2, 64, 64, "bf16", init_state=True)
    o, fs = _gpu(inp, "bf16")
    assert torch.equal(fs[0], torch.from_numpy(inp["init_state"][0]).cuda())
    assert torch.equal(fs[2], torch.from_numpy(inp["init_state"][2]).cuda())
    _check(inp, "bf16", o, fs)


def test_varlen_cached_continuation_full_size_sampled_heads():
    """8 sequences of 1024-16384 tokens, H=32, d=128, nonzero initial states, edge pads:
    the padded run equals the unpadded run bit for bit; heads 0, 13, 31 match the oracle."""
    w = gen.varlen_cached()
    inp = gen.prefill_inputs(w)
    o, fs = _gpu(inp, "bf16")
    un = gen.unpad(inp)
    o_u, fs_u = _gpu(un, "bf16")
    keep = torch.from_numpy(inp["pad_mask"].astype(bool)).cuda()
    assert torch.equal(o[keep], o_u) and torch.equal(fs, fs_u)
    assert torch.all(o[~keep] == 0)
    _check(inp, "bf16", o, fs, heads=[0, 13, 31])


def test_long_prefill_128k_sampled_heads():
    """B=1, H=32, T=131072, d=128, bf16, chunk 64: heads 0 and 21 against the oracle."""
    w = gen.long_prefill(131072)
    inp = gen.prefill_inputs(w)
    o, fs = _gpu(inp, "bf16")
    _check(inp, "bf16", o, fs, heads=[0, 21])
    assert torch.isfinite(o.float()).all()


@pytest.mark.parametrize("per_token", [-0.5, -1.1])
def test_strong_decay_within_tensor_core_range(per_token):
    """The tensor-core path forms e^{-g} inside a 64-token chunk; with a per-token
    log-decay of -0.5 (-32 per chunk) or -1.1 (-70 per chunk) on a quarter of the
    channels it must still match the oracle (the path's stated range is a chunk
    log-decay above about -80)."""
    inp = gen.random_case(61, [700, 64], 2, 128, 128, "bf16", init_state=True)
    la = inp["log_alpha"].copy()
    la[:, :, ::4] = per_token
    inp["log_alpha"] = la
    o, fs = _gpu(inp, "bf16")
    _check(inp, "bf16", o, fs)


def test_many_short_sequences_two_kernel_path():
    """3000 sequences of 1-40 tokens (most shorter than one chunk), H = 2, bf16, d = 128,
    pads, nonzero states: the chunk index over thousands of sequences and the many
    partial chunks of the two-kernel path."""
    rng = np.random.default_rng(77)
    lengths = [int(x) for x in rng.integers(1, 41, size=3000)]
    inp = gen.random_case(78, lengths, 2, 128, 128, "bf16", init_state=True)
    N = int(inp["cu_seqlens"][-1])
    m = (rng.uniform(size=N) > 0.1).astype(np.uint8)
    for key in ("q", "k", "v"):
        inp[key][m == 0] = 0.0
    inp["pad_mask"] = m
    o, fs = _gpu(inp, "bf16")
    _check(inp, "bf16", o, fs)
    assert np.all(to_np(o)[m == 0] == 0.0)


def test_state_slice_width_does_not_change_results():
    """One sequence of 32 heads runs its state pass in 32-column slices (128 chains fit the
    SMs); the same sequence next to a second one runs it in 64-column slices (256 chains).
    Columns of the state never mix, so the shared sequence's outputs and final state are
    bit-identical between the two."""
    lengths = [777, 300]
    inp = gen.random_case(81, lengths, 32, 128, 128, "bf16", init_state=True)
    o2, fs2 = _gpu(inp, "bf16")
    solo = {k: inp[k][:lengths[0]] for k in ("q", "k", "v", "log_alpha", "beta")}
    solo["cu_seqlens"] = np.array([0, lengths[0]], np.int32)
    solo["init_state"] = inp["init_state"][:1]
    o1, fs1 = _gpu(solo, "bf16")
    assert torch.equal(o2[:lengths[0]], o1)
    assert torch.equal(fs2[:1], fs1)
    _check(solo, "bf16", o1, fs1)
