"""GPU parity of the head-wise gate (log_alpha [rows, H], one decay per token and
head: Gated DeltaNet's gating, the special case of KDA's per-channel gate)
against the fp64 oracle, on every path that takes it: the two-kernel tensor-core
prefill, the CUDA-core prefill (fp32 inputs, and bf16 without the full
workspace), the allocation-free entry point and decode.  Same tolerances as the
per-channel tests.
"""
import numpy as np
import pytest
import torch

from gated_delta_rule_148_b200 import inputs as gen
from gated_delta_rule_148_b200 import kda
from kda_testlib import TOL, dev_inputs, norm_err, to_np
from oracle import kda_oracle as orc

pytestmark = pytest.mark.gpu


def _case(seed, lengths, H, dk, dv, dtype, pads=False):
    inp = gen.random_case(seed, lengths, H, dk, dv, dtype, init_state=True)
    N = int(inp["cu_seqlens"][-1])
    inp["log_alpha"] = gen.head_gates(seed, N, H)
    if pads:
        rng = np.random.default_rng(seed)
        mask = (rng.uniform(size=N) > 0.1).astype(np.uint8)
        for key in ("q", "k", "v"):
            inp[key][mask == 0] = 0.0
        inp["pad_mask"] = mask
    return inp


def _check(inp, dtype, o, fs):
    o_ref, s_ref = orc.prefill(inp["q"], inp["k"], inp["v"], inp["log_alpha"], inp["beta"],
                               inp["cu_seqlens"], pad_mask=inp.get("pad_mask"),
                               init_state=inp["init_state"])
    eo, es = norm_err(to_np(o), o_ref), norm_err(to_np(fs), s_ref)
    assert eo <= TOL[dtype], f"o error {eo:.3e}"
    assert es <= TOL[dtype], f"state error {es:.3e}"
    if inp.get("pad_mask") is not None:
        assert np.all(to_np(o)[inp["pad_mask"] == 0] == 0.0)


@pytest.mark.parametrize("pads", [False, True])
def test_head_gate_two_kernel_path(pads):
    """bf16, d_k = d_v = 128, chunk 64 with the full workspace: the intra/state kernels."""
    inp = _case(71, [1, 63, 64, 65, 300, 2000], 3, 128, 128, "bf16", pads=pads)
    d = dev_inputs(inp, "bf16")
    assert d["log_alpha"].dim() == 2
    o, fs = kda.prefill(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["cu_seqlens"],
                        pad_mask=d.get("pad_mask"), init_state=d["init_state"])
    torch.cuda.synchronize()
    assert kda.get_device_status() == kda.KDA_OK
    _check(inp, "bf16", o, fs)


@pytest.mark.parametrize("chunk", [16, 64])
def test_head_gate_cuda_core_path_f32(chunk):
    inp = _case(72, [1, 17, 100, 257], 2, 64, 128, "f32")
    d = dev_inputs(inp, "f32")
    o, fs = kda.prefill(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["cu_seqlens"],
                        init_state=d["init_state"], chunk=chunk)
    torch.cuda.synchronize()
    assert kda.get_device_status() == kda.KDA_OK
    _check(inp, "f32", o, fs)


def test_head_gate_small_workspace_and_noalloc():
    """Without the two-kernel workspace a head-wise gate runs on the CUDA-core kernel;
    the allocation-free entry point takes that route too."""
    inp = _case(73, [5, 130, 700], 2, 128, 128, "bf16")
    d = dev_inputs(inp, "bf16")
    N, H = d["q"].shape[0], d["q"].shape[1]
    ws = torch.empty(kda.prefill_workspace_bytes(3), dtype=torch.uint8, device="cuda")
    o, fs = kda.prefill(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["cu_seqlens"],
                        init_state=d["init_state"], workspace=ws)
    o2 = torch.empty((N, H, 128), dtype=torch.bfloat16, device="cuda")
    fs2 = torch.empty_like(fs)
    kda.prefill_noalloc(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["cu_seqlens"], o2,
                        final_state=fs2, init_state=d["init_state"])
    torch.cuda.synchronize()
    assert kda.get_device_status() == kda.KDA_OK
    _check(inp, "bf16", o, fs)
    assert torch.equal(o, o2) and torch.equal(fs, fs2)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_head_gate_decode(dtype):
    B, H, dk, dv, steps = 10, 3, 128, 64, 12
    st0 = gen.random_case(74, [1] * B, H, dk, dv, dtype, init_state=True)["init_state"]
    state = torch.from_numpy(st0).cuda()
    ref = st0.astype(np.float64)
    rng = np.random.default_rng(75)
    for s in range(steps):
        tok = gen.random_case(76 + s, [1] * B, H, dk, dv, dtype)
        tok["log_alpha"] = gen.head_gates(76 + s, B, H)
        mask = (rng.uniform(size=B) > 0.25).astype(np.uint8)
        d = dev_inputs(tok, dtype)
        o = kda.decode(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], state,
                       mask=torch.from_numpy(mask).cuda())
        o_ref = orc.decode(tok["q"], tok["k"], tok["v"], tok["log_alpha"], tok["beta"], ref, mask)
        torch.cuda.synchronize()
        assert norm_err(to_np(o), o_ref) <= TOL[dtype]
    assert norm_err(to_np(state), ref) <= TOL[dtype]
    assert kda.get_device_status() == kda.KDA_OK


def test_head_gate_equals_broadcast_channel_gate():
    """Two-kernel path: the [N, H] gate and the same values broadcast to [N, H, d_k] give
    the same bits (the head-wise load only changes where the value is read from)."""
    inp = _case(77, [700, 64], 2, 128, 128, "bf16")
    d = dev_inputs(inp, "bf16")
    la3 = d["log_alpha"][:, :, None].expand(-1, -1, 128).contiguous()
    o1, f1 = kda.prefill(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["cu_seqlens"],
                         init_state=d["init_state"])
    o2, f2 = kda.prefill(d["q"], d["k"], d["v"], la3, d["beta"], d["cu_seqlens"],
                         init_state=d["init_state"])
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(f1, f2)


@pytest.mark.parametrize("pattern", ["per_token_-4", "spikes_-200"])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_head_gate_strong_decay(pattern, dtype):
    """Head-wise gates far outside the factorised range of the tensor-core Gram (-4 per
    token on one head: -256 per chunk; single -200 steps mid-chunk on every head): the
    two-kernel path (exact Gram terms for the key rows past the range, every channel at
    once) and the CUDA-core path match the oracle."""
    inp = _case(78, [700, 64, 130], 2, 128, 128, dtype)
    la = inp["log_alpha"].copy()
    if pattern == "per_token_-4":
        la[:, 0] = -4.0
    else:
        la[[30, 100, 357, 500], :] = -200.0
    inp["log_alpha"] = la
    d = dev_inputs(inp, dtype)
    o, fs = kda.prefill(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["cu_seqlens"],
                        init_state=d["init_state"])
    torch.cuda.synchronize()
    assert kda.get_device_status() == kda.KDA_OK
    _check(inp, dtype, o, fs)
