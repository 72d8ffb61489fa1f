"""The operator inside CUDA graphs: a captured prefill and a captured decode step,
replayed, give the same bits as the eager calls (launch-bound loops such as a decode
step can be replayed as one graph launch)."""
import numpy as np
import pytest
import torch

from gated_delta_rule_148_b200 import inputs as gen
from gated_delta_rule_148_b200 import kda
from kda_testlib import dev_inputs

pytestmark = pytest.mark.gpu


def test_decode_steps_in_a_cuda_graph():
    B, H, d, steps = 16, 4, 128, 8
    st0 = torch.from_numpy(gen.random_case(120, [1] * B, H, d, d, "bf16", init_state=True)["init_state"]).cuda()
    toks = [dev_inputs(gen.random_case(121 + s, [1] * B, H, d, d, "bf16"), "bf16") for s in range(steps)]
    mask = torch.from_numpy((np.arange(B) % 5 != 0).astype(np.uint8)).cuda()
    # eager
    se = st0.clone()
    oe = [kda.decode(t["q"], t["k"], t["v"], t["log_alpha"], t["beta"], se, mask=mask).clone() for t in toks]
    torch.cuda.synchronize()
    # one captured step, replayed with each step's inputs copied into its static buffers
    sg = st0.clone()
    static = {k: torch.empty_like(v) for k, v in toks[0].items() if k in ("q", "k", "v", "log_alpha", "beta")}
    og = torch.empty_like(oe[0])
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        kda.decode(toks[0]["q"], toks[0]["k"], toks[0]["v"], toks[0]["log_alpha"], toks[0]["beta"],
                   st0.clone(), mask=mask)            # warm-up outside the graph
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        kda.decode(static["q"], static["k"], static["v"], static["log_alpha"], static["beta"], sg,
                   mask=mask, o=og)
    outs = []
    for t in toks:
        for key in static:
            static[key].copy_(t[key])
        g.replay()
        outs.append(og.clone())
    torch.cuda.synchronize()
    for a, b in zip(outs, oe):
        assert torch.equal(a, b)
    assert torch.equal(sg, se)
    assert kda.get_device_status() == kda.KDA_OK


def test_prefill_in_a_cuda_graph():
    inp = gen.random_case(122, [700, 64, 129], 2, 128, 128, "bf16", init_state=True)
    d = dev_inputs(inp, "bf16")
    o1, f1 = kda.prefill(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["cu_seqlens"],
                         init_state=d["init_state"])
    torch.cuda.synchronize()
    ws = kda.prefill_workspace(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["cu_seqlens"])
    o2 = torch.empty_like(o1)
    f2 = torch.empty_like(f1)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        kda.prefill(d["q"], d["k"], d["v"], d["log_alpha"], d["beta"], d["cu_seqlens"],
                    init_state=d["init_state"], o=o2, final_state=f2, workspace=ws)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(f1, f2)
    assert kda.get_device_status() == kda.KDA_OK
