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


def _run_path(inp, dtype, path, chunk=0):
    """Run one prefill path on the GPU: "split" (the full workspace: the two-kernel
    tensor-core path for bf16, d = 128, chunk 64), "fused" (a span-table workspace only:
    the single-kernel tensor-core path), "noalloc" (kda_prefill_noalloc) or "simt"
    (fp32 inputs: the CUDA-core path)."""
    d = dev_inputs(inp, dtype)
    N, H = d["q"].shape[0], d["q"].shape[1]
    B = d["cu_seqlens"].numel() - 1
    dv = d["v"].shape[2]
    dk = d["q"].shape[2]
    o = torch.full((N, H, dv), 9.0, dtype=d["q"].dtype, device="cuda")
    fs = torch.full((B, H, dk, dv), 9.0, dtype=torch.float32, device="cuda")
    args = (d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["cu_seqlens"])
    if path == "noalloc":
        kda.prefill_noalloc(*args, o, final_state=fs, pad_mask=d.get("pad_mask"),
                            init_state=d.get("init_state"), chunk=chunk)
    else:
        ws = None
        if path == "fused":
            ws = torch.empty(max(kda.prefill_workspace_bytes(B), 1), dtype=torch.uint8, device="cuda")
        kda.prefill(*args, pad_mask=d.get("pad_mask"), init_state=d.get("init_state"), o=o,
                    final_state=fs, chunk=chunk, workspace=ws)
    torch.cuda.synchronize()
    assert kda.get_device_status() == kda.KDA_OK
    return o, fs


_DECAYS = ["per_token_-0.5", "per_token_-1.1", "quarter_channels_-4", "spikes_-200"]


def _strong_decay(inp, pattern):
    la = inp["log_alpha"].copy()
    if pattern.startswith("per_token"):
        la[:, :, ::4] = float(pattern.split("_")[-1])
    elif pattern == "quarter_channels_-4":
        la[:, :, ::4] = -4.0          # -256 over a 64-token chunk
    else:                               # one -200 step mid-chunk: all channels, then half of them
        la[[30, 100, 357], :, :] = -200.0
        la[[500, 731], :, ::2] = -200.0
    inp["log_alpha"] = la
    return inp


@pytest.mark.parametrize("path", ["split", "fused"])
@pytest.mark.parametrize("pattern", _DECAYS)
def test_strong_decay_tensor_core_paths(path, pattern):
    """Every finite log_alpha <= 0 is in range: a quarter of the channels at -0.5 or -1.1 per
    token (inside the factorised range), at -4 per token (-256 per chunk), and single -200
    steps mid-chunk on all or half of the channels.  Both tensor-core paths match the oracle
    within the bf16 tolerance (channels beyond the factorised range take the exact Gram)."""
    inp = _strong_decay(gen.random_case(61, [700, 64, 130], 2, 128, 128, "bf16", init_state=True),
                        pattern)
    o, fs = _run_path(inp, "bf16", path)
    _check(inp, "bf16", o, fs)


@pytest.mark.parametrize("pattern", ["quarter_channels_-4", "spikes_-200"])
def test_strong_decay_cuda_core_path(pattern):
    inp = _strong_decay(gen.random_case(62, [700, 64, 130], 2, 128, 64, "f32", init_state=True),
                        pattern)
    o, fs = _run_path(inp, "f32", "simt", chunk=64)
    _check(inp, "f32", o, fs)


def _pad_case(seed, lengths, H, dtype, dv=128, interior=True, edges=True, garbage=True):
    """Edge and interior pads whose q, k, v, log_alpha and beta are random, large or not
    finite: none of it may reach the outputs or the state."""
    inp = gen.random_case(seed, lengths, H, 128, dv, dtype, init_state=True)
    cu = inp["cu_seqlens"]
    N = int(cu[-1])
    rng = np.random.default_rng(seed)
    mask = np.ones(N, np.uint8)
    for b in range(len(lengths)):
        a, e = int(cu[b]), int(cu[b + 1])
        if e - a < 8:
            continue
        if edges:
            mask[a:a + int(rng.integers(0, 5))] = 0
            mask[e - int(rng.integers(0, 5)):e] = 0
        if interior:
            inner = rng.choice(np.arange(a + 4, e - 4), size=min(9, e - a - 8), replace=False)
            mask[inner] = 0
    pads = np.nonzero(mask == 0)[0]
    if garbage and pads.size:
        big = lambda shape: gen.round_bf16((rng.normal(size=shape) * 1000.0).astype(np.float32))
        for key in ("q", "k", "v"):
            inp[key][pads] = big(inp[key][pads].shape)
        inp["log_alpha"][pads] = -np.abs(rng.normal(size=inp["log_alpha"][pads].shape) * 50.0)
        inp["beta"][pads] = (rng.normal(size=inp["beta"][pads].shape) * 10.0).astype(np.float32)
        inp["q"][pads[0]] = np.nan
        inp["v"][pads[-1]] = np.inf
        inp["k"][pads[len(pads) // 2]] = -np.inf
        inp["beta"][pads[0]] = np.nan
    inp["pad_mask"] = mask
    return inp


@pytest.mark.parametrize("path,dtype", [("split", "bf16"), ("fused", "bf16"), ("noalloc", "bf16"),
                                        ("simt", "f32")])
def test_pads_with_garbage_values_every_path(path, dtype):
    """Edge and interior pads carrying huge, random and non-finite q, k, v, log_alpha and
    beta: pad outputs are exactly 0, everything else matches the oracle run without the
    pads (which never reads the pad values)."""
    inp = _pad_case(63, [300, 17, 129, 700], 2, dtype)
    o, fs = _run_path(inp, dtype, path)
    keep = inp["pad_mask"] == 1
    assert torch.all(o[torch.from_numpy(~keep).cuda()] == 0)
    assert torch.isfinite(o.float()).all() and torch.isfinite(fs).all()
    _check(inp, dtype, o, fs)


@pytest.mark.parametrize("path", ["fused", "noalloc"])
def test_single_kernel_paths_match_oracle_with_pads(path):
    """The single-kernel tensor-core path (a span-table workspace, or the allocation-free
    entry point) with edge and interior pads and nonzero initial states, d_v = 128 and 64,
    against the oracle."""
    for dv in (128, 64):
        inp = _pad_case(64, [64, 1, 500, 90, 33, 250], 3, "bf16", dv=dv, garbage=False)
        o, fs = _run_path(inp, "bf16", path)
        assert torch.all(o[torch.from_numpy(inp["pad_mask"] == 0).cuda()] == 0)
        _check(inp, "bf16", o, fs)


@pytest.mark.parametrize("T", [64 * 3 + 1, 64 * 4 + 30])
def test_prefix_invariance_single_kernel_path(T):
    """The bit-identical prefix audit on the single-kernel tensor-core path."""
    inp = gen.random_case(38, [T], 4, 128, 128, "bf16", init_state=True)
    rng = np.random.default_rng(40)

    def run(which):
        x = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in inp.items()}
        if which:
            x["q"][T - 1] = gen.round_bf16(rng.normal(size=x["q"][T - 1].shape).astype(np.float32))
            x["k"][T - 1] = gen.round_bf16(rng.normal(size=x["k"][T - 1].shape).astype(np.float32))
            x["v"][T - 1] = gen.round_bf16(rng.normal(size=x["v"][T - 1].shape).astype(np.float32))
            x["log_alpha"][T - 1] = -np.abs(rng.normal(size=x["log_alpha"][T - 1].shape)) * 90.0
            x["beta"][T - 1] = 0.77
        o, _ = _run_path(x, "bf16", "fused")
        return to_np(o)

    leak, onset, d = orc.prefix_audit(run, T, 1)
    assert not leak, f"prefix leak, onset {onset}"
    assert d.max() == 0.0


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


def test_bounded_wait_runs_out_and_reports_timeout():
    """Failure detection without a GPU fault: with a planted fault the state pass issues no
    item loads, so its bounded waits (set to ~1 ms here) run out.  The call returns, the
    device status reads KDA_ERR_DEVICE_TIMEOUT, and the next normal call on the same context
    matches the oracle (the kernel left nothing in flight and released its tensor memory)."""
    inp = gen.random_case(91, [700, 130], 2, 128, 128, "bf16", init_state=True)
    d = dev_inputs(inp, "bf16")
    kda.debug_set_fault(kda.KDA_FAULT_STARVE_STATE_LOADS, 2_000_000)
    try:
        kda.prefill(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["cu_seqlens"],
                    init_state=d["init_state"])
        st = kda.get_device_status()
    finally:
        kda.debug_set_fault(0)
    assert st == kda.KDA_ERR_DEVICE_TIMEOUT, kda.status_string(st)
    assert kda.debug_timeout_site() == 11              # the state pass's item-load wait
    assert kda.get_device_status() == kda.KDA_OK       # the latch was cleared
    o, fs = _gpu(inp, "bf16")
    _check(inp, "bf16", o, fs)
