"""GPU parity of the tensor-core prefill with chunks of 128 and 256 rows (64-row items
merged into chunk items, then the state pass) against the fp64 oracle, through the C
ABI.  Same tolerances as the chunk-64 tests: 2e-2 normalised max-abs error for bf16,
pad outputs exactly 0, a perturbed last position leaves every earlier output
bit-identical.
"""
import numpy as np
import pytest
import torch

from gated_delta_rule_148_b200 import inputs as gen
from gated_delta_rule_148_b200 import kda
from kda_testlib import TOL, dev_inputs, norm_err, to_np
from oracle import kda_oracle as orc
from test_gpu_prefill import _pad_case, _strong_decay, _DECAYS

pytestmark = pytest.mark.gpu

CHUNKS = [128, 256]


def _run(inp, chunk, workspace=None):
    d = dev_inputs(inp, "bf16")
    N, H = d["q"].shape[0], d["q"].shape[1]
    B = d["cu_seqlens"].numel() - 1
    o = torch.full((N, H, 128), 9.0, dtype=torch.bfloat16, device="cuda")
    fs = torch.full((B, H, 128, 128), 9.0, dtype=torch.float32, device="cuda")
    kda.prefill(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["cu_seqlens"],
                pad_mask=d.get("pad_mask"), init_state=d.get("init_state"), o=o, final_state=fs,
                chunk=chunk, workspace=workspace)
    torch.cuda.synchronize()
    assert kda.get_device_status() == kda.KDA_OK
    return o, fs


def _check(inp, o, fs, heads=None):
    sel = slice(None) if heads is None else list(heads)
    s0 = inp.get("init_state")
    o_ref, s_ref = orc.prefill(inp["q"][:, sel], inp["k"][:, sel], inp["v"][:, sel],
                               inp["log_alpha"][:, sel], inp["beta"][:, sel], inp["cu_seqlens"],
                               pad_mask=inp.get("pad_mask"),
                               init_state=None if s0 is None else s0[:, sel])
    eo = norm_err(to_np(o)[:, sel], o_ref)
    es = norm_err(to_np(fs)[:, sel], s_ref)
    assert eo <= TOL["bf16"], f"o error {eo:.3e}"
    assert es <= TOL["bf16"], f"state error {es:.3e}"
    return eo, es


@pytest.mark.parametrize("chunk", CHUNKS)
def test_lengths_around_chunk_edges(chunk):
    """Sequences of 1 to 3 chunks with ragged tails, including odd numbers of 64-row
    sub-chunks (the last chunk then merges with identity rows) and empty sequences."""
    lengths = [1, 63, 64, 65, 127, 128, 129, 0, 255, 256, 257, 300, 700]
    inp = gen.random_case(91, lengths, 3, 128, 128, "bf16", init_state=True)
    o, fs = _run(inp, chunk)
    _check(inp, o, fs)
    assert torch.equal(fs[7], torch.from_numpy(inp["init_state"][7]).cuda())


@pytest.mark.parametrize("chunk", CHUNKS)
def test_zero_initial_state_and_many_heads(chunk):
    inp = gen.random_case(92, [1000, 513], 8, 128, 128, "bf16", init_state=False)
    o, fs = _run(inp, chunk)
    _check(inp, o, fs)


@pytest.mark.parametrize("chunk", CHUNKS)
@pytest.mark.parametrize("pattern", _DECAYS)
def test_strong_decay(chunk, pattern):
    """The decay patterns of the chunk-64 tests (-0.5, -1.1 and -4 per token on a quarter of
    the channels, single -200 steps): chunk items merge decay products that stay <= 1."""
    inp = _strong_decay(gen.random_case(93, [700, 64, 130], 2, 128, 128, "bf16", init_state=True),
                        pattern)
    o, fs = _run(inp, chunk)
    _check(inp, o, fs)


@pytest.mark.parametrize("chunk", CHUNKS)
def test_pads_with_garbage_values(chunk):
    """Edge and interior pads with huge and non-finite q, k, v, log_alpha, beta."""
    inp = _pad_case(94, [300, 17, 129, 700], 2, "bf16")
    o, fs = _run(inp, chunk)
    keep = inp["pad_mask"] == 1
    assert torch.all(o[torch.from_numpy(~keep).cuda()] == 0)
    assert torch.isfinite(o.float()).all() and torch.isfinite(fs).all()
    _check(inp, o, fs)


@pytest.mark.parametrize("chunk", CHUNKS)
def test_edge_pads_bit_identical_to_unpadded(chunk):
    w = gen.varlen_cached(H=4, n_seqs=6, lo=100, hi=700)
    w = gen.Workload(w.name, w.seed, w.H, w.dk, w.dv, "bf16", 64, lengths=w.lengths,
                     init_state=True, pads=True)
    inp = gen.prefill_inputs(w)
    un = gen.unpad(inp)
    o, fs = _run(inp, chunk)
    o_u, fs_u = _run(un, chunk)
    keep = torch.from_numpy(inp["pad_mask"].astype(bool)).cuda()
    assert torch.equal(o[keep], o_u)
    assert torch.equal(fs, fs_u)
    assert torch.all(o[~keep] == 0)
    _check(inp, o, fs)


@pytest.mark.parametrize("chunk", CHUNKS)
def test_head_gate(chunk):
    inp = gen.random_case(95, [1, 130, 300, 900], 3, 128, 128, "bf16", init_state=True)
    N = int(inp["cu_seqlens"][-1])
    inp["log_alpha"] = gen.head_gates(95, N, 3)
    o, fs = _run(inp, chunk)
    _check(inp, o, fs)


@pytest.mark.parametrize("chunk,T", [(128, 128 * 2 + 1), (128, 64 * 5 + 30), (256, 256 + 1),
                                     (256, 256 * 2 + 100)])
def test_prefix_invariance_bit_identical(chunk, T):
    """Perturb position T-1 (with a -90 gate step): o[0:T-1] stays bit-identical."""
    inp = gen.random_case(96, [T], 4, 128, 128, "bf16", init_state=True)
    rng = np.random.default_rng(97)

    def run(which):
        x = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in inp.items()}
        if which:
            x["q"][T - 1] = gen.round_bf16(rng.normal(size=x["q"][T - 1].shape).astype(np.float32))
            x["k"][T - 1] = gen.round_bf16(rng.normal(size=x["k"][T - 1].shape).astype(np.float32))
            x["v"][T - 1] = gen.round_bf16(rng.normal(size=x["v"][T - 1].shape).astype(np.float32))
            x["log_alpha"][T - 1] = -np.abs(rng.normal(size=x["log_alpha"][T - 1].shape)) * 90.0
            x["beta"][T - 1] = 0.77
        o, _ = _run(x, chunk)
        return to_np(o)

    leak, onset, d = orc.prefix_audit(run, T, 1)
    assert not leak, f"prefix leak, onset {onset}"
    assert d.max() == 0.0


def test_chunk_sizes_agree_within_rounding():
    """Chunk 64, 128 and 256 on the same input: all three match the oracle, and each pair
    differs by no more than the bf16 tolerance."""
    inp = gen.random_case(98, [2000, 333], 4, 128, 128, "bf16", init_state=True)
    res = {c: _run(inp, c) for c in (64, 128, 256)}
    for c in res:
        _check(inp, *res[c])
    ref = res[64][0].float()
    scale = ref.abs().max().item()
    for c in (128, 256):
        assert (res[c][0].float() - ref).abs().max().item() <= TOL["bf16"] * scale


def test_too_small_workspace_is_unsupported():
    """Chunks of 128 / 256 run only with the full workspace: a smaller one is refused."""
    inp = gen.random_case(99, [300], 2, 128, 128, "bf16")
    d = dev_inputs(inp, "bf16")
    need = kda.prefill_workspace_size_for(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                                          d["cu_seqlens"], chunk=128)
    assert need > kda.prefill_workspace_size_for(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"],
                                                 d["cu_seqlens"], chunk=64)
    ws = torch.empty(need - 1024, dtype=torch.uint8, device="cuda")
    with pytest.raises(kda.KdaError) as e:
        kda.prefill(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["cu_seqlens"],
                    chunk=128, workspace=ws)
    assert e.value.status == kda.KDA_ERR_UNSUPPORTED


@pytest.mark.parametrize("chunk", CHUNKS)
def test_varlen_cached_full_size_sampled_heads(chunk):
    """8 sequences of 1024-16384 tokens, H = 32, nonzero initial states, edge pads: heads
    0, 13, 31 against the oracle; the padded run equals the unpadded one bit for bit."""
    w = gen.varlen_cached()
    inp = gen.prefill_inputs(w)
    o, fs = _run(inp, chunk)
    un = gen.unpad(inp)
    o_u, fs_u = _run(un, chunk)
    keep = torch.from_numpy(inp["pad_mask"].astype(bool)).cuda()
    assert torch.equal(o[keep], o_u) and torch.equal(fs, fs_u)
    _check(inp, o, fs, heads=[0, 13, 31])


@pytest.mark.parametrize("chunk", CHUNKS)
def test_long_prefill_128k_sampled_heads(chunk):
    """B = 1, H = 32, T = 131072: heads 0 and 21 against the oracle."""
    inp = gen.prefill_inputs(gen.long_prefill(131072))
    o, fs = _run(inp, chunk)
    _check(inp, o, fs, heads=[0, 21])
    assert torch.isfinite(o.float()).all()


@pytest.mark.parametrize("chunk", CHUNKS)
def test_many_short_sequences_with_pads(chunk):
    """2000 sequences of 1-300 tokens (most shorter than one chunk, many with an odd number of
    64-row sub-chunks), H = 2, 10 % interior pads, nonzero states."""
    rng = np.random.default_rng(141)
    lengths = [int(x) for x in rng.integers(1, 301, size=2000)]
    inp = gen.random_case(142, lengths, 2, 128, 128, "bf16", init_state=True)
    N = int(inp["cu_seqlens"][-1])
    m = (rng.uniform(size=N) > 0.1).astype(np.uint8)
    for key in ("q", "k", "v"):
        inp[key][m == 0] = 0.0
    inp["pad_mask"] = m
    o, fs = _run(inp, chunk)
    _check(inp, o, fs)
    assert np.all(to_np(o)[m == 0] == 0.0)


def test_graph_replay_chunk_128():
    """The chunk-128 path (index, intra, merge, state kernels) captured in a CUDA graph and
    replayed: the same outputs as the eager call, bit for bit."""
    inp = gen.random_case(143, [700, 333], 4, 128, 128, "bf16", init_state=True)
    d = dev_inputs(inp, "bf16")
    ws = kda.prefill_workspace(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["cu_seqlens"], chunk=128)
    o = torch.empty((d["q"].shape[0], 4, 128), dtype=torch.bfloat16, device="cuda")
    fs = torch.empty((2, 4, 128, 128), dtype=torch.float32, device="cuda")
    run = lambda: kda.prefill(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["cu_seqlens"],
                              init_state=d["init_state"], o=o, final_state=fs, chunk=128, workspace=ws)
    run()
    torch.cuda.synchronize()
    o_ref, fs_ref = o.clone(), fs.clone()
    o.zero_()
    fs.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        run()
    g.replay()
    torch.cuda.synchronize()
    assert kda.get_device_status() == kda.KDA_OK
    assert torch.equal(o, o_ref) and torch.equal(fs, fs_ref)
    _check(inp, o, fs)


def test_bounded_wait_runs_out_in_the_ring_state_pass():
    """Failure detection without a GPU fault on the chunk-128 path: with the planted fault the
    state pass's producer issues no part loads, so the first waits on the ring's slots run out
    (after ~1 ms here); the call returns, the status reads KDA_ERR_DEVICE_TIMEOUT with an
    item-load site, and the next normal call on the same context matches the oracle."""
    inp = gen.random_case(144, [700, 130], 2, 128, 128, "bf16", init_state=True)
    d = dev_inputs(inp, "bf16")
    kda.debug_set_fault(kda.KDA_FAULT_STARVE_STATE_LOADS, 2_000_000)
    try:
        kda.prefill(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["cu_seqlens"],
                    init_state=d["init_state"], chunk=128)
        st = kda.get_device_status()
    finally:
        kda.debug_set_fault(0)
    assert st == kda.KDA_ERR_DEVICE_TIMEOUT, kda.status_string(st)
    assert kda.debug_timeout_site() in (11, 16)       # a tile slot or the U_v slot
    assert kda.get_device_status() == kda.KDA_OK
    o, fs = _run(inp, 128)
    _check(inp, o, fs)
