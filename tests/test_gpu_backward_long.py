"""The blockwise backward at a length the per-position form could not hold: one sequence
of 32768 tokens (512 chunks), H = 2, d = 128, bf16 inputs, with pads, a strong-decay
spike and a nonzero initial state, against the oracle's fp64 reverse-mode pass.  Same
tolerance as the other backward tests (1e-4 normalised max-abs error)."""
import numpy as np
import pytest
import torch

from gated_delta_rule_148_b200 import inputs as gen
from gated_delta_rule_148_b200 import kda
from kda_testlib import dev_inputs, norm_err, to_np
from oracle import kda_oracle as orc

pytestmark = pytest.mark.gpu


def test_backward_32k_tokens():
    T, H = 32768, 2
    c = gen.random_case(111, [T], H, 128, 128, "bf16", init_state=True)
    rng = np.random.default_rng(112)
    m = (rng.uniform(size=T) > 0.05).astype(np.uint8)
    c["pad_mask"] = m
    c["log_alpha"][[100, 5000, 20001], :, ::3] = -150.0
    do = rng.normal(size=(T, H, 128)).astype(np.float32)
    dsf = rng.normal(size=(1, H, 128, 128)).astype(np.float32)
    d = dev_inputs(c, "bf16")
    g = kda.prefill_backward(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["cu_seqlens"],
                             torch.from_numpy(do).cuda(), torch.from_numpy(dsf).cuda(),
                             pad_mask=d["pad_mask"], init_state=d["init_state"])
    torch.cuda.synchronize()
    assert kda.get_device_status() == kda.KDA_OK
    ref = orc.prefill_backward(c["q"], c["k"], c["v"], c["log_alpha"], c["beta"], c["cu_seqlens"], do,
                               dsf, m, c["init_state"])
    for key in ("dq", "dk", "dv", "dlog_alpha", "dbeta", "dS0"):
        err = norm_err(to_np(g[key]), ref[key])
        assert err <= 1e-4, f"{key}: {err:.3e}"
    for key in ("dq", "dk", "dv", "dlog_alpha", "dbeta"):
        assert np.all(to_np(g[key])[m == 0] == 0.0), key
