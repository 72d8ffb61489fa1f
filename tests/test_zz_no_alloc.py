"""kda_prefill_noalloc against kda_prefill (GPU, through the C ABI).

The allocation-free entry point exists for callers that cannot call
cudaMalloc where they run the operator (memory owned up front by a host
framework, or loops where an allocation could synchronise the device).  It
must give the same results as the workspace entry point, call after call,
although every call reuses the same fixed scratch array inside the library.
This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

from gated_delta_rule_148_b200 import inputs as gen
from gated_delta_rule_148_b200 import kda
from kda_testlib import TOL, dev_inputs, norm_err, to_np

pytestmark = pytest.mark.gpu


def _padded_case(seed, lengths):
    inp = gen.random_case(seed, lengths, 4, 128, 128, "bf16", init_state=True)
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
    o = torch.full((N, 4, 128), 5.0, dtype=torch.bfloat16, device="cuda")
    fs = torch.full((B, 4, 128, 128), 5.0, dtype=torch.float32, device="cuda")
    a = kda.prefill_args(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["cu_seqlens"],
                         d["pad_mask"], d["init_state"], o, fs, 0, workspace)
    st = getattr(kda.load(), entry)(ctypes.byref(a), ctypes.c_void_p(
        torch.cuda.current_stream().cuda_stream))
    assert st == kda.KDA_OK, kda.status_string(st)
    assert kda.get_device_status() == kda.KDA_OK
    return o, fs


def test_noalloc_matches_workspace_entry_two_calls_in_a_row():
    cases = [(70, [300, 17, 129]), (71, [64, 1, 500, 90, 33, 250])]
    for seed, lengths in cases:
        inp = _padded_case(seed, lengths)
        d = dev_inputs(inp, "bf16")
        N, B = int(inp["cu_seqlens"][-1]), len(lengths)
        ws = torch.empty(kda.prefill_workspace_bytes(B), dtype=torch.uint8, device="cuda")
        o_ref, fs_ref = _call("kda_prefill", d, N, B, ws)
        o, fs = _call("kda_prefill_noalloc", d, N, B)
        assert norm_err(to_np(o), to_np(o_ref)) <= TOL["bf16"]
        assert norm_err(to_np(fs), to_np(fs_ref)) <= TOL["bf16"]
        keep = torch.from_numpy(inp["pad_mask"] == 0).cuda()
        assert torch.all(o[keep] == 0)


def test_noalloc_rejects_more_sequences_than_its_scratch_holds():
    a = kda.PrefillArgs()
    a.dtype, a.num_seqs, a.total_tokens, a.H, a.dk, a.dv = (
        kda.KDA_BF16, kda.NOALLOC_MAX_SEQS + 1, kda.NOALLOC_MAX_SEQS + 1, 1, 64, 64)
    st = kda.load().kda_prefill_noalloc(ctypes.byref(a), None)
    assert st == kda.KDA_ERR_INVALID_ARG
