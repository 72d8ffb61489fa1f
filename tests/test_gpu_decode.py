"""GPU parity tests for kda_decode (call through the C ABI) against the fp64 oracle."""
import numpy as np
import pytest
import torch

from gated_delta_rule_148_b200 import inputs as gen
from gated_delta_rule_148_b200 import kda
from kda_testlib import TOL, dev_inputs, norm_err, to_np
from oracle import kda_oracle as orc

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv", [(64, 64), (64, 128), (128, 64), (128, 128)])
def test_decode_steps_match_oracle(dtype, dk, dv):
    B, H, steps = 12, 3, 20
    st0 = gen.random_case(50, [1] * B, H, dk, dv, dtype, init_state=True)["init_state"]
    state = torch.from_numpy(st0).cuda()
    ref = st0.astype(np.float64)
    rng = np.random.default_rng(51)
    for s in range(steps):
        tok = gen.random_case(52 + s, [1] * B, H, dk, dv, dtype)
        mask = (rng.uniform(size=B) > 0.25).astype(np.uint8)
        d = dev_inputs(tok, dtype)
        m = torch.from_numpy(mask).cuda()
        before = state.clone()
        o = kda.decode(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], state, mask=m)
        o_ref = orc.decode(tok["q"], tok["k"], tok["v"], tok["log_alpha"], tok["beta"], ref, mask)
        torch.cuda.synchronize()
        mb = torch.from_numpy(mask == 0).cuda()
        assert torch.equal(state[mb], before[mb])     # masked rows: state bytes untouched
        assert torch.all(o[mb] == 0)
        assert norm_err(to_np(o), o_ref) <= TOL[dtype]
    assert norm_err(to_np(state), ref) <= TOL[dtype]
    assert kda.get_device_status() == kda.KDA_OK


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_decode_equals_one_token_prefill(dtype):
    """A decode step and a prefill of one-token sequences compute the same step.  fp32
    inputs run the fp32 CUDA-core prefill: agreement to fp32 rounding.  bf16 inputs run
    the tensor-core prefill, whose products take S as a bf16 operand: agreement to the
    bf16 tolerance, and both sides within it of the oracle."""
    B, H, d = 8, 2, 128
    c = gen.random_case(53, [1] * B, H, d, d, dtype, init_state=True)
    dd = dev_inputs(c, dtype)
    st = dd["init_state"].clone()
    o = kda.decode(dd["q"], dd["k"], dd["v"], dd["log_alpha"], dd["beta"], st)
    o2, fs2 = kda.prefill(dd["q"], dd["k"], dd["v"], dd["log_alpha"], dd["beta"],
                          dd["cu_seqlens"], init_state=dd["init_state"])
    torch.cuda.synchronize()
    ref = c["init_state"].astype(np.float64)
    o_ref = orc.decode(c["q"], c["k"], c["v"], c["log_alpha"], c["beta"], ref)
    bound = 1e-5 if dtype == "f32" else TOL["bf16"]
    assert norm_err(to_np(o), to_np(o2)) <= bound
    assert norm_err(to_np(st), to_np(fs2)) <= bound
    for got_o, got_s in ((o, st), (o2, fs2)):
        assert norm_err(to_np(got_o), o_ref) <= TOL[dtype]
        assert norm_err(to_np(got_s), ref) <= TOL[dtype]


def test_batched_decode_full_size_1000_steps():
    """256 rows x 32 heads x 128 x 128 fp32 state (537 MB), 1000 steps, 26 masked rows per
    step.  Every step: masked rows' state bytes unchanged and o = 0.  Rows 0-7 (all heads)
    are tracked by the fp64 oracle through all 1000 steps."""
    w = gen.batched_decode()
    state = torch.from_numpy(gen.decode_state(w)).cuda()
    track = list(range(8))
    ref = gen.decode_state(w)[track].astype(np.float64)
    pool = gen.decode_pool(w)
    dpool = [dev_inputs(t, "bf16") for t in pool]
    worst = 0.0
    for s in range(w.decode_steps):
        mask = gen.decode_mask(w, s)
        m = torch.from_numpy(mask).cuda()
        d = dpool[s % len(pool)]
        check = s % 50 == 0
        if check:
            masked_rows = torch.from_numpy(np.nonzero(mask == 0)[0]).cuda()
            before = state[masked_rows].clone()
        o = kda.decode(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], state, mask=m)
        t = pool[s % len(pool)]
        o_ref = orc.decode(t["q"][track], t["k"][track], t["v"][track], t["log_alpha"][track],
                           t["beta"][track], ref, mask[track])
        if check:
            assert torch.equal(state[masked_rows], before)
            assert torch.all(o[masked_rows] == 0)
            worst = max(worst, norm_err(to_np(o[track]), o_ref))
    torch.cuda.synchronize()
    assert worst <= TOL["bf16"]
    assert norm_err(to_np(state[track]), ref) <= TOL["bf16"]
    assert kda.get_device_status() == kda.KDA_OK


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_prefill_to_decode_handoff(dtype):
    """Prefill hands its final state to decode with no conversion (same [B,H,dk,dv] fp32
    layout, updated in place): prefill of T tokens then 5 decode steps equals the oracle's
    prefill of the T + 5 tokens, for the outputs of the decoded tokens and the final state."""
    H, d, T, steps = 2, 128, 300, 5
    lens = [T + steps, T + steps]
    c = gen.random_case(55, lens, H, d, d, dtype, init_state=True)
    B = len(lens)
    cu = c["cu_seqlens"]
    first = np.concatenate([np.arange(cu[b], cu[b] + T) for b in range(B)])
    pre = {k: c[k][first] for k in ("q", "k", "v", "log_alpha", "beta")}
    pre["cu_seqlens"] = np.array([0, T, 2 * T], np.int32)
    pre["init_state"] = c["init_state"]
    dd = dev_inputs(pre, dtype)
    _, state = kda.prefill(dd["q"], dd["k"], dd["v"], dd["log_alpha"], dd["beta"], dd["cu_seqlens"],
                           init_state=dd["init_state"])
    outs = []
    for s in range(steps):
        rows = np.array([cu[b] + T + s for b in range(B)])
        tok = {k: c[k][rows] for k in ("q", "k", "v", "log_alpha", "beta")}
        dt = dev_inputs(tok, dtype)
        outs.append(to_np(kda.decode(dt["q"], dt["k"], dt["v"], dt["log_alpha"], dt["beta"], state)))
    torch.cuda.synchronize()
    o_ref, s_ref = orc.prefill(c["q"], c["k"], c["v"], c["log_alpha"], c["beta"], cu,
                               init_state=c["init_state"])
    for s in range(steps):
        rows = np.array([cu[b] + T + s for b in range(B)])
        assert norm_err(outs[s], o_ref[rows]) <= TOL[dtype]
    assert norm_err(to_np(state), s_ref) <= TOL[dtype]
    assert kda.get_device_status() == kda.KDA_OK
