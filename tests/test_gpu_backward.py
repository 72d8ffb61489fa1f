"""GPU parity of kda_prefill_backward (blockwise, fp32) against the oracle's fp64
reverse-mode pass (itself pinned by central differences).  Tolerance: 1e-4 normalised
max-abs error for every gradient, bf16 inputs included (the backward computes in fp32
from the bf16 values); pad positions get exactly zero gradients.
"""
import numpy as np
import pytest
import torch

from gated_delta_rule_148_b200 import inputs as gen
from gated_delta_rule_148_b200 import kda
from kda_testlib import dev_inputs, norm_err, to_np
from oracle import kda_oracle as orc

pytestmark = pytest.mark.gpu
TOL = 1e-4


def _run(seed, lengths, H, dk, dv, dtype, pads=False, head_gate=False, state=True, dsf=True):
    c = gen.random_case(seed, lengths, H, dk, dv, dtype, init_state=state)
    N, B = int(c["cu_seqlens"][-1]), len(lengths)
    if head_gate:
        c["log_alpha"] = gen.head_gates(seed, N, H)
    rng = np.random.default_rng(seed + 1)
    if pads:
        m = (rng.uniform(size=N) > 0.15).astype(np.uint8)
        for key in ("q", "k", "v"):
            c[key][m == 0] = 0.0
        c["pad_mask"] = m
    do = rng.normal(size=(N, H, dv)).astype(np.float32)
    dsf_np = rng.normal(size=(B, H, dk, dv)).astype(np.float32) if dsf else None
    d = dev_inputs(c, dtype)
    g = kda.prefill_backward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["cu_seqlens"],
                             torch.from_numpy(do).cuda(),
                             None if dsf_np is None else torch.from_numpy(dsf_np).cuda(),
                             pad_mask=d.get("pad_mask"), init_state=d.get("init_state"))
    torch.cuda.synchronize()
    assert kda.get_device_status() == kda.KDA_OK
    ref = orc.prefill_backward(c["q"], c["k"], c["v"], c["log_alpha"], c["beta"], c["cu_seqlens"], do,
                               dsf_np, c.get("pad_mask"), c.get("init_state"))
    for key in ("dq", "dk", "dv", "dlog_alpha", "dbeta", "dS0"):
        err = norm_err(to_np(g[key]), ref[key])
        assert err <= TOL, f"{key}: {err:.3e}"
    if pads:
        m = c["pad_mask"] == 0
        for key in ("dq", "dk", "dv", "dlog_alpha", "dbeta"):
            assert np.all(to_np(g[key])[m] == 0.0), key
    return g


@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64), (128, 128)])
def test_backward_f32_shapes(dk, dv):
    _run(101, [1, 7, 70], 2, dk, dv, "f32", pads=True)


def test_backward_bf16_head_gate_and_without_state():
    _run(102, [33, 200], 2, 128, 128, "bf16", head_gate=True)
    _run(103, [50], 3, 128, 128, "bf16", state=False, dsf=False)


def test_backward_longer_sequences():
    """Two sequences of 1500 and 900 tokens, H = 4, d = 128, bf16, pads."""
    _run(104, [1500, 900], 4, 128, 128, "bf16", pads=True)


def test_backward_empty_and_one_token_sequences():
    """An empty sequence passes dS_final straight to dS0; one-token sequences."""
    _run(105, [0, 1, 5, 0], 2, 64, 128, "f32")
