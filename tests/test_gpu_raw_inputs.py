"""The raw-input mode (GDR_RAW_INPUTS) against the fp64 oracle.

In this mode the kernels take q, k, beta (eta) and the gates as raw
projections and logits, and apply the input transforms on their load paths:
unit-norm q and k (KLA's keys excepted), sigmoid of beta / eta and of the GDN-2
gates, log g = -softplus of the decay logit.  The oracle is fed the same raw
values transformed in float64 (inputs.transform_raw), so each comparison
checks the fused transforms and the recurrence together.  Paths: the chunked
forward (chunk 0 and 65, including its segmented and pipelined schedules),
the per-token forward (chunk 1) and the decode kernel.
"""
import pytest
import torch

import gated_delta_rule_forward_b200 as gdr
import oracle
from gated_delta_rule_forward_b200.inputs import make_raw_inputs, random_state, transform_raw
from parity_util import assert_close, gate_kwargs, select, to_dev

pytestmark = pytest.mark.gpu
VARS = ["deltanet", "gdn", "kda", "gdn2", "kla"]


@pytest.mark.parametrize("chunk", [0, 1, 65])
@pytest.mark.parametrize("variant", VARS)
def test_raw_forward(variant, chunk):
    B, T, H = 2, 333, 3
    raw = make_raw_inputs(variant, B, T, H, seed=61)
    S0 = random_state(B, H, 128, 128, 62)
    d = to_dev(raw)
    o, S = gdr.forward(d["q"], d["k"], d["v"], variant=variant, **gate_kwargs(d), initial_state=S0.cuda(),
                       chunk=chunk, raw_inputs=True)
    gdr.device_status()
    o_ref, S_ref = oracle.forward(variant, **transform_raw(variant, raw), initial_state=S0)
    assert_close(o, o_ref, torch.bfloat16, "o")
    assert_close(S, S_ref, torch.bfloat16, "S")


@pytest.mark.parametrize("shape", [(1, 4100, 2), (4, 1531, 16)])
@pytest.mark.parametrize("variant", ["gdn", "kda"])
def test_raw_forward_rescheduled(variant, shape):
    """The segmented carry (few long sequences) and the pipelined sweep."""
    B, T, H = shape
    assert gdr.forward_launches(variant, torch.bfloat16, B, T, H, 128, 128, 0) == 4
    raw = make_raw_inputs(variant, B, T, H, seed=63)
    d = to_dev(raw)
    o, S = gdr.forward(d["q"], d["k"], d["v"], variant=variant, **gate_kwargs(d), raw_inputs=True)
    gdr.device_status()
    o_ref, S_ref = oracle.forward(variant, **transform_raw(variant, raw))
    assert_close(o, o_ref, torch.bfloat16, "o")
    assert_close(S, S_ref, torch.bfloat16, "S")


@pytest.mark.parametrize("variant", VARS)
def test_raw_decode(variant):
    N, H, steps = 5, 3, 6
    raw = make_raw_inputs(variant, N, steps, H, seed=64)
    S0 = random_state(N, H, 128, 128, 65)
    state = S0.cuda()
    d = to_dev(raw)
    outs = []
    for t in range(steps):
        s = select(d, t=t)
        outs.append(gdr.decode_step(s["q"], s["k"], s["v"], state, variant=variant, **gate_kwargs(s),
                                    raw_inputs=True))
    o_ref, S_ref = oracle.forward(variant, **transform_raw(variant, raw), initial_state=S0)
    assert_close(torch.stack(outs, 1), o_ref, torch.bfloat16, "o")
    assert_close(state, S_ref, torch.bfloat16, "state")
