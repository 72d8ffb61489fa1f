"""kda_prefill_noalloc against kda_prefill and the fp64 oracle (GPU, through the C ABI).

The allocation-free entry point exists for callers that cannot call
cudaMalloc where they run the operator (memory owned up front by a host
framework, or loops where an allocation could synchronise the device).  It
must give the same results as the workspace entry point up to rounding (it
takes the single-kernel tensor-core path or the CUDA-core path, never the
two-kernel path that needs the large workspace), call after call, although
every call reuses the same fixed scratch array inside the library; and both
must match the oracle.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

from gated_delta_rule_148_b200 import inputs as gen
from gated_delta_rule_148_b200 import kda
from kda_testlib import TOL, dev_inputs, norm_err, to_np
from oracle import kda_oracle as orc

pytestmark = pytest.mark.gpu


def _padded_case(seed, lengths, dtype="bf16", pads=True):
    inp = gen.random_case(seed, lengths, 4, 128, 128, dtype, init_state=True)
    if not pads:
        return inp
    cu = inp["cu_seqlens"]
    mask = np.ones(int(cu[-1]), np.uint8)
    rng = np.random.default_rng(seed)
    for b in range(len(lengths)):
        n = int(cu[b + 1] - cu[b])
        if n < 4:
            continue
        mask[cu[b]:cu[b] + int(rng.integers(0, 3))] = 0            # left edge pads
        mask[cu[b + 1] - int(rng.integers(0, 3)):cu[b + 1]] = 0    # right edge pads
        mask[cu[b] + n // 2] = 0                                   # one interior pad
    for key in ("q", "k", "v"):
        inp[key][mask == 0] = 0.0
    inp["pad_mask"] = mask
    return inp


def _call(entry, d, N, B, workspace=None):
    o = torch.full((N, 4, 128), 5.0, dtype=d["q"].dtype, device="cuda")
    fs = torch.full((B, 4, 128, 128), 5.0, dtype=torch.float32, device="cuda")
    a = kda.prefill_args(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["cu_seqlens"],
                         d.get("pad_mask"), d["init_state"], o, fs, 0, workspace)
    st = getattr(kda.load(), entry)(ctypes.byref(a), ctypes.c_void_p(
        torch.cuda.current_stream().cuda_stream))
    assert st == kda.KDA_OK, kda.status_string(st)
    assert kda.get_device_status() == kda.KDA_OK
    return o, fs


def _oracle_check(inp, dtype, o, fs):
    o_ref, s_ref = orc.prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                               inp["cu_seqlens"], pad_mask=inp.get("pad_mask"),
                               init_state=inp["init_state"])
    assert norm_err(to_np(o), o_ref) <= TOL[dtype]
    assert norm_err(to_np(fs), s_ref) <= TOL[dtype]


@pytest.mark.parametrize("dtype,pads", [("bf16", True), ("bf16", False), ("f32", True)])
def test_noalloc_matches_workspace_entry_two_calls_in_a_row(dtype, pads):
    """Two different batches one after the other through the allocation-free entry point
    (the second reuses the scratch the first left behind): each equals kda_prefill with a
    workspace up to rounding and matches the oracle; pad outputs are exactly 0."""
    cases = [(70, [300, 17, 129]), (71, [64, 1, 500, 90, 33, 250])]
    for seed, lengths in cases:
        inp = _padded_case(seed, lengths, dtype, pads)
        d = dev_inputs(inp, dtype)
        N, B = int(inp["cu_seqlens"][-1]), len(lengths)
        ws = torch.empty(kda.prefill_workspace_size_for(d["q"], d["k"], d["v"], d["log_alpha"],
                                                        d["beta"], d["cu_seqlens"]),
                         dtype=torch.uint8, device="cuda")
        o_ref, fs_ref = _call("kda_prefill", d, N, B, ws)
        o, fs = _call("kda_prefill_noalloc", d, N, B)
        assert norm_err(to_np(o), to_np(o_ref)) <= TOL[dtype]
        assert norm_err(to_np(fs), to_np(fs_ref)) <= TOL[dtype]
        _oracle_check(inp, dtype, o, fs)
        _oracle_check(inp, dtype, o_ref, fs_ref)
        if pads:
            keep = torch.from_numpy(inp["pad_mask"] == 0).cuda()
            assert torch.all(o[keep] == 0)


def test_noalloc_rejects_more_sequences_than_its_scratch_holds():
    a = kda.PrefillArgs()
    a.dtype, a.num_seqs, a.total_tokens, a.H, a.dk, a.dv = (
        kda.KDA_BF16, kda.NOALLOC_MAX_SEQS + 1, kda.NOALLOC_MAX_SEQS + 1, 1, 64, 64)
    st = kda.load().kda_prefill_noalloc(ctypes.byref(a), None)
    assert st == kda.KDA_ERR_INVALID_ARG


def test_noalloc_refuses_chunks_of_128_and_256():
    """Chunks of 128 / 256 need the merged chunk items of the full workspace, which the
    fixed scratch cannot hold: the call is refused and writes nothing."""
    inp = _padded_case(123, [300, 77], pads=False)
    d = dev_inputs(inp, "bf16")
    N, H = d["q"].shape[0], d["q"].shape[1]
    o = torch.full((N, H, 128), 7.0, dtype=torch.bfloat16, device="cuda")
    for chunk in (128, 256):
        with pytest.raises(kda.KdaError) as e:
            kda.prefill_noalloc(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["cu_seqlens"], o,
                                chunk=chunk)
        assert e.value.status == kda.KDA_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert torch.all(o == 7.0)
