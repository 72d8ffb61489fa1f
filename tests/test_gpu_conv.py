"""GPU parity of kda_short_conv (the padding-correct short causal convolution with a
carried state) against the oracle's window form.  fp32: 1e-5; bf16 (x, y in bf16,
fp32 accumulation, y rounded once): the bf16 tolerance.  Pad outputs are exactly 0;
the final state is a copy of input rows (or old state rows) and must match exactly.
"""
import numpy as np
import pytest
import torch

from gated_delta_rule_148_b200 import inputs as gen
from gated_delta_rule_148_b200 import kda
from kda_testlib import TOL, norm_err, to_np
from oracle import kda_oracle as orc

pytestmark = pytest.mark.gpu
CTOL = {"f32": 1e-5, "bf16": TOL["bf16"]}


def _dev(c, dtype):
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    d = {"x": torch.from_numpy(c["x"]).cuda().to(tdt),
         "weight": torch.from_numpy(c["weight"]).cuda(), "bias": torch.from_numpy(c["bias"]).cuda(),
         "cu_seqlens": torch.from_numpy(c["cu_seqlens"]).cuda()}
    d["pad_mask"] = None if c["pad_mask"] is None else torch.from_numpy(c["pad_mask"]).cuda()
    d["state"] = None if c["state"] is None else torch.from_numpy(c["state"]).cuda()
    return d


def _run(d, state_out=None):
    y = kda.short_conv(d["x"], d["weight"], d["cu_seqlens"], bias=d["bias"], pad_mask=d["pad_mask"],
                       state_in=d["state"], state_out=state_out)
    torch.cuda.synchronize()
    assert kda.get_device_status() == kda.KDA_OK
    return y


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("W", [1, 2, 3, 4])
@pytest.mark.parametrize("D", [72, 2056])
def test_conv_varlen_pads_state(dtype, W, D):
    lengths = [1, 2, 3, 255, 256, 257, 700]
    c = gen.conv_inputs(81 + W, lengths, D, W, dtype, pad_frac=0.2)
    d = _dev(c, dtype)
    so = torch.empty((len(lengths), W - 1, D), device="cuda") if W > 1 else None
    y = _run(d, so)
    y_ref, s_ref = orc.short_conv(c["x"], c["weight"], c["bias"], c["cu_seqlens"], c["pad_mask"], c["state"])
    assert norm_err(to_np(y), y_ref) <= CTOL[dtype]
    assert np.all(to_np(y)[c["pad_mask"] == 0] == 0.0)
    if W > 1:
        np.testing.assert_array_equal(to_np(so), s_ref.astype(np.float32))


def test_conv_state_in_place_and_no_state():
    c = gen.conv_inputs(90, [5, 300, 2], 64, 4, "bf16", pad_frac=0.1)
    d = _dev(c, "bf16")
    so = torch.empty_like(d["state"])
    y1 = _run(d, so)
    st = d["state"].clone()
    d2 = dict(d, state=st)
    y2 = _run(d2, st)                      # state_out is state_in
    assert torch.equal(y1, y2) and torch.equal(so, st)
    c0 = dict(c, state=None)
    y_ref, _ = orc.short_conv(c0["x"], c0["weight"], c0["bias"], c0["cu_seqlens"], c0["pad_mask"], None)
    y3 = _run(dict(d, state=None))
    assert norm_err(to_np(y3), y_ref) <= CTOL["bf16"]


def test_conv_decode_steps_in_place():
    """Decode: one token per row per call, the state updated in place, masked rows
    untouched; equals the oracle run over the rows' whole histories."""
    B, D, W, steps = 6, 128, 4, 9
    c = gen.conv_inputs(91, [steps] * B, D, W, "f32")
    rng = np.random.default_rng(92)
    masks = (rng.uniform(size=(steps, B)) > 0.3).astype(np.uint8)
    st = torch.from_numpy(c["state"]).cuda()
    wgt, bias = torch.from_numpy(c["weight"]).cuda(), torch.from_numpy(c["bias"]).cuda()
    cu1 = torch.arange(B + 1, dtype=torch.int32, device="cuda")
    ys = []
    for s in range(steps):
        rows = np.array([c["cu_seqlens"][b] + s for b in range(B)])
        x = torch.from_numpy(c["x"][rows]).cuda()
        ys.append(to_np(kda.short_conv(x, wgt, cu1, bias=bias, pad_mask=torch.from_numpy(masks[s]).cuda(),
                                       state_in=st, state_out=st)))
    torch.cuda.synchronize()
    full_mask = np.concatenate([masks[:, b] for b in range(B)])
    y_ref, s_ref = orc.short_conv(c["x"], c["weight"], c["bias"], c["cu_seqlens"], full_mask, c["state"])
    got = np.stack(ys, axis=1).reshape(B * steps, D)
    assert norm_err(got, y_ref) <= 1e-5
    np.testing.assert_array_equal(to_np(st), s_ref.astype(np.float32))


def test_conv_full_size_sampled():
    """N = 131072, D = 4096 (one of q, k, v of 32 heads x 128), W = 4, bf16, one
    sequence, 1 % pads: sampled outputs from the oracle's per-position window form, and
    the final state exactly."""
    N, D, W = 131072, 4096, 4
    c = gen.conv_inputs(93, [N], D, W, "bf16", pad_frac=0.01)
    d = _dev(c, "bf16")
    so = torch.empty((1, W - 1, D), device="cuda")
    y = _run(d, so)
    pos = np.concatenate([np.arange(0, 8), np.random.default_rng(94).integers(0, N, 48), np.arange(N - 8, N)])
    ref = orc.short_conv_at(c["x"], c["weight"], c["bias"], c["cu_seqlens"], pos, c["pad_mask"], c["state"])
    assert norm_err(to_np(y[torch.from_numpy(pos).cuda()]), ref) <= CTOL["bf16"]
    valid = np.nonzero(c["pad_mask"])[0][-(W - 1):]
    np.testing.assert_array_equal(to_np(so)[0], c["x"][valid])


def test_conv_empty_sequences_keep_state():
    """Zero-length sequences leave their state rows as they were (copied to state_out)."""
    c = gen.conv_inputs(95, [0, 7, 0, 3], 64, 4, "f32", pad_frac=0.3)
    d = _dev(c, "f32")
    so = torch.empty_like(d["state"])
    y = _run(d, so)
    y_ref, s_ref = orc.short_conv(c["x"], c["weight"], c["bias"], c["cu_seqlens"], c["pad_mask"], c["state"])
    assert norm_err(to_np(y), y_ref) <= CTOL["f32"]
    np.testing.assert_array_equal(to_np(so), s_ref.astype(np.float32))
    np.testing.assert_array_equal(to_np(so)[0], c["state"][0])


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_conv_long_spans_many_pads(dtype):
    """A packed batch long enough that each CTA's span of positions (about one wave of CTAs)
    exceeds one 256-position compaction pass, with 30 % pads, sequence boundaries inside
    spans and a carried state: every output and the new state against the oracle."""
    lengths = [40000, 1, 3, 65000, 257, 30000]
    D, W = 72, 4
    c = gen.conv_inputs(97, lengths, D, W, dtype, pad_frac=0.3)
    d = _dev(c, dtype)
    so = torch.empty((len(lengths), W - 1, D), device="cuda")
    y = _run(d, so)
    y_ref, s_ref = orc.short_conv(c["x"], c["weight"], c["bias"], c["cu_seqlens"], c["pad_mask"], c["state"])
    assert norm_err(to_np(y), y_ref) <= CTOL[dtype]
    assert np.all(to_np(y)[c["pad_mask"] == 0] == 0.0)
    np.testing.assert_array_equal(to_np(so), s_ref.astype(np.float32))
