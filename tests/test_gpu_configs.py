"""GPU parity at the full workload sizes, in the launch configuration the
benchmark times (chunk = 0: the library's automatic kernel choice).

Workloads (synthetic, seeded; recipe in gated_delta_rule_forward_b200/inputs.py):
  350M-model layer: Gated DeltaNet and DeltaNet, bf16, B=8 T=2048 H=8 d=128
  1.3B-model layer: KDA and KLA, bf16, B=4 T=4096 H=16 d=128
  GDN-2 layer:      bf16, B=4 T=4096 H=16 d=128, plus tied gates == KDA
  long context:     Gated DeltaNet and KLA forward, B=1 T=65536 H=16 d=128
  decode:           256 sequences x 16 heads, fp32 state, 1024 steps from the
                    long-context final state (broadcast), inputs seeded per step

The fp64 oracle finishes the three layer workloads whole in seconds, so they
are compared on every output.  The long-context forward is compared whole
too, and the 1024-step decode on a sample of sequences at every
step (the GPU runs the full batch).
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_forward_b200 as gdr
import oracle
from gated_delta_rule_forward_b200.inputs import make_decode_inputs, make_inputs
from parity_util import assert_close, assert_gpu_close, gate_kwargs, to_dev

pytestmark = pytest.mark.gpu
BF16 = torch.bfloat16


def full_parity(variant, B, T, H, seed=0, **gen):
    d = make_inputs(variant, B, T, H, 128, 128, dtype=BF16, seed=seed, **gen)
    dd = to_dev(d)
    o, S = gdr.forward(dd["q"], dd["k"], dd["v"], variant=variant, **gate_kwargs(dd), chunk=0)
    gdr.device_status()          # no timeout / range flag raised by the kernel
    o_ref, S_ref = oracle.forward(variant, **d)
    e_o = assert_close(o, o_ref, BF16, f"{variant} o")
    e_s = assert_close(S, S_ref, BF16, f"{variant} S")
    return o, S, e_o, e_s


@pytest.mark.parametrize("variant", ["gdn", "deltanet"])
def test_350m_layer(variant):
    full_parity(variant, 8, 2048, 8)


@pytest.mark.parametrize("variant", ["kda", "kla"])
def test_1p3b_layer(variant):
    full_parity(variant, 4, 4096, 16)


def test_gdn2_layer_and_tied_reduction():
    full_parity("gdn2", 4, 4096, 16)
    # tied gates b = w = beta: equal to KDA on the same inputs
    o2, S2, _, _ = full_parity("gdn2", 4, 4096, 16, gdn2_tied=True)
    dk = to_dev(make_inputs("kda", 4, 4096, 16, dtype=BF16, seed=0))
    o1, S1 = gdr.forward(dk["q"], dk["k"], dk["v"], variant="kda", **gate_kwargs(dk), chunk=0)
    assert_gpu_close(o2, o1, "o")
    assert_gpu_close(S2, S1, "S")


@pytest.mark.parametrize("variant", ["gdn", "kla"])
def test_long_context_forward_and_decode(variant):
    B, T, H = 1, 65536, 16
    d = make_inputs(variant, B, T, H, 128, 128, dtype=BF16, seed=0)
    dd = to_dev(d)
    o, S = gdr.forward(dd["q"], dd["k"], dd["v"], variant=variant, **gate_kwargs(dd), chunk=0)
    torch.cuda.synchronize()
    o_ref_all, S_all = oracle.forward(variant, **d)
    assert_close(o, o_ref_all, BF16, "o")
    assert_close(S, S_all, BF16, "S")
    # decode: 256 sequences from the broadcast final state, 1024 seeded steps
    N, steps = 256, 1024
    # both sides start from the oracle's long-context final state [1,16,128,128]
    S_start = torch.from_numpy(S_all).float()
    state = S_start.expand(N, H, 128, 128).contiguous().cuda()
    sample = [0, 1, 128, 255]
    S_ref = np.broadcast_to(S_all, (len(sample), H, 128, 128)).copy()
    worst = 0.0
    for s in range(steps):
        di = make_decode_inputs(variant, N, H, s, dtype=BF16)
        dg = to_dev(di)
        out = gdr.decode_step(dg["q"], dg["k"], dg["v"], state, variant=variant, **gate_kwargs(dg))
        sub = {k: (None if v is None else v[sample].contiguous()) for k, v in di.items()}
        o_ref, S_ref = oracle.decode_step(variant, sub["q"], sub["k"], sub["v"], S_ref, **gate_kwargs(sub))
        worst = max(worst, assert_close(out[sample], o_ref, BF16, f"decode step {s}"))
    assert_close(state[sample], S_ref, BF16, "decode state")
