"""Device-side failure detection, exercised without faulting the GPU.

The chunked kernels report two conditions through a device error word that
gdr_device_status() reads after synchronising the stream:

* GDR_ERR_RANGE: an fp16 operand of the chunked path (the residual E, the
  state, W, U') beyond 6e4.  Made here with ordinary host inputs: values
  scaled by 1e5.
* GDR_ERR_TIMEOUT: a bounded wait inside a kernel gave up.  Made here by
  host-side fault injection (GDR_FAULT=wait): the carry kernel's first CTA
  never issues the copy of one record (nor expects its bytes), so its waits
  give up after their limit (about a second); the kernel then drains its own
  MMAs and copies, frees its tensor memory and returns.

In both cases the kernel returns normally, the status is reported once (the
word is cleared when read), and the next call on the same context computes
correct results again.  No test traps, faults or hangs the GPU.
"""
import os

import numpy as np
import pytest
import torch

import gated_delta_rule_forward_b200 as gdr
import oracle
from gated_delta_rule_forward_b200.inputs import make_inputs, random_state
from parity_util import assert_close, gate_kwargs, to_dev

pytestmark = pytest.mark.gpu


def _forward(d, variant, S0=None, chunk=0):
    dd = to_dev(d)
    return gdr.forward(dd["q"], dd["k"], dd["v"], variant=variant, **gate_kwargs(dd),
                       initial_state=None if S0 is None else S0.cuda(), chunk=chunk)


def _status():
    try:
        gdr.device_status()
        return 0
    except gdr.GdrError as e:
        return e.status


def _clean_call_matches_oracle(variant, B, T, H, seed):
    d = make_inputs(variant, B, T, H, dtype=torch.bfloat16, seed=seed)
    S0 = random_state(B, H, 128, 128, seed + 1)
    o, S = _forward(d, variant, S0)
    assert _status() == 0
    o_ref, S_ref = oracle.forward(variant, **d, initial_state=S0)
    assert_close(o, o_ref, torch.bfloat16, "o after the fault")
    assert_close(S, S_ref, torch.bfloat16, "S after the fault")


@pytest.mark.parametrize("variant", ["gdn", "kda", "gdn2"])
def test_range_fault_is_reported(variant):
    """Values scaled by 1e5 push the fp16 operands of the chunked path past 6e4."""
    assert _status() == 0                     # nothing stale
    B, T, H = 1, 130, 1
    d = make_inputs(variant, B, T, H, dtype=torch.bfloat16, seed=3)
    d["v"] = (d["v"].float() * 1e5).to(torch.bfloat16)
    _forward(d, variant)
    assert _status() == 6                     # GDR_ERR_RANGE
    assert _status() == 0                     # reported once
    # the per-token kernel (fp32 state, no fp16 operands) has no such limit
    o, S = _forward(d, variant, chunk=1)
    assert _status() == 0
    o_ref, S_ref = oracle.forward(variant, **d)
    assert_close(o, o_ref, torch.bfloat16, "per-token o")
    _clean_call_matches_oracle(variant, 2, 200, 2, 5)


@pytest.mark.parametrize("shape", [(1, 300, 2), (1, 4100, 2), (4, 1531, 16)])
def test_timeout_is_reported_and_the_context_stays_usable(shape):
    """Serial sweep, segmented carry and pipelined sweep: the injected missing copy
    makes one CTA's wait give up; the call reports GDR_ERR_TIMEOUT and the next
    call (without the fault) matches the oracle."""
    B, T, H = shape
    assert _status() == 0
    d = make_inputs("gdn", B, T, H, dtype=torch.bfloat16, seed=7)
    os.environ["GDR_FAULT"] = "wait"
    try:
        _forward(d, "gdn")
        st = _status()
    finally:
        del os.environ["GDR_FAULT"]
    assert st == 5, st                        # GDR_ERR_TIMEOUT
    assert _status() == 0
    _clean_call_matches_oracle("gdn", B, min(T, 1000), H, 9)
