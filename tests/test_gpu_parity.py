"""GPU parity: the CUDA path, called through the C ABI, against the fp64 oracle.

Every case feeds the same seeded inputs (gated_delta_rule_forward_b200.inputs)
to both sides; the oracle sees the I/O-dtype-rounded values up-cast exactly.
Tolerances are in tests/parity_util.py.  ``chunk`` 1 is the per-token kernel,
65 the chunked tensor-core path (chunk-parallel preparation + carry); a case
is skipped where the library reports it does not cover it.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_forward_b200 as gdr
import oracle
from gated_delta_rule_forward_b200.inputs import make_decode_inputs, make_inputs, random_state
from parity_util import assert_close, assert_gpu_close, gate_kwargs, select, to_dev

pytestmark = pytest.mark.gpu
VARS = ["deltanet", "gdn", "kda", "gdn2", "kla"]


def kernel_or_skip(variant, dtype, B, T, H, dk, dv, chunk):
    name = gdr.forward_kernel_name(variant, dtype, B, T, H, dk, dv, chunk)
    if name == "none":
        pytest.skip(f"no kernel for chunk={chunk} {variant} {dtype} dk={dk} dv={dv}")
    return name


def run_both(variant, B, T, H, dk, dv, dtype, chunk, seed=0, s0=True, **gen):
    kernel_or_skip(variant, dtype, B, T, H, dk, dv, chunk)
    d = make_inputs(variant, B, T, H, dk, dv, dtype=dtype, seed=seed, **gen)
    S0 = random_state(B, H, dk, dv, seed + 1) if s0 else None
    dd = to_dev(d)
    o, S = gdr.forward(dd["q"], dd["k"], dd["v"], variant=variant, **gate_kwargs(dd),
                       initial_state=None if S0 is None else S0.cuda(), chunk=chunk)
    torch.cuda.synchronize()
    o_ref, S_ref = oracle.forward(variant, **d, initial_state=S0)
    return o, S, o_ref, S_ref


# ----------------------------------------------------------------- config 0 (fp32)
def test_config0_gdn_fp32():
    """GDN fp32, B=1 H=2 T=256 dk=dv=64, seed 0: max rel error 1e-4."""
    o, S, o_ref, S_ref = run_both("gdn", 1, 256, 2, 64, 64, torch.float32, chunk=0, s0=False)
    assert_close(o, o_ref, torch.float32, "o")
    assert_close(S, S_ref, torch.float32, "S")


# ----------------------------------------------------------------- small, ragged
@pytest.mark.parametrize("chunk", [1, 65])
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("variant", VARS)
def test_small_ragged(variant, dtype, chunk):
    o, S, o_ref, S_ref = run_both(variant, 2, 137, 3, 128, 128, dtype, chunk, seed=3)
    assert_close(o, o_ref, dtype, "o")
    assert_close(S, S_ref, dtype, "S")


@pytest.mark.parametrize("chunk", [1, 65])
@pytest.mark.parametrize("dkdv", [(64, 64), (64, 128), (128, 64)])
@pytest.mark.parametrize("variant", ["gdn", "kda", "gdn2"])
def test_head_dims(variant, dkdv, chunk):
    dk, dv = dkdv
    o, S, o_ref, S_ref = run_both(variant, 1, 100, 2, dk, dv, torch.bfloat16, chunk, seed=5)
    assert_close(o, o_ref, torch.bfloat16, "o")
    assert_close(S, S_ref, torch.bfloat16, "S")


@pytest.mark.parametrize("chunk", [1, 65])
@pytest.mark.parametrize("T", [1, 2, 63, 64, 65, 128, 191])
def test_sequence_lengths(T, chunk):
    for variant in ("gdn", "kda"):
        o, S, o_ref, S_ref = run_both(variant, 2, T, 2, 128, 128, torch.bfloat16, chunk, seed=T)
        assert_close(o, o_ref, torch.bfloat16, f"{variant} o")
        assert_close(S, S_ref, torch.bfloat16, f"{variant} S")


@pytest.mark.parametrize("chunk", [1, 65])
def test_zero_initial_state_and_no_final_state(chunk):
    kernel_or_skip("gdn", torch.bfloat16, 2, 70, 2, 128, 128, chunk)
    d = make_inputs("gdn", 2, 70, 2, dtype=torch.bfloat16, seed=9)
    dd = to_dev(d)
    o, S = gdr.forward(dd["q"], dd["k"], dd["v"], variant="gdn", **gate_kwargs(dd),
                       output_final_state=False, chunk=chunk)
    assert S is None
    o_ref, _ = oracle.forward("gdn", **d)
    assert_close(o, o_ref, torch.bfloat16, "o")


@pytest.mark.parametrize("chunk", [1, 65])
def test_state_in_place(chunk):
    """final_state may be the initial_state buffer."""
    kernel_or_skip("kda", torch.bfloat16, 2, 90, 2, 128, 128, chunk)
    d = make_inputs("kda", 2, 90, 2, dtype=torch.bfloat16, seed=12)
    S0 = random_state(2, 2, 128, 128, 13)
    dd = to_dev(d)
    buf = S0.cuda()
    o, S = gdr.forward(dd["q"], dd["k"], dd["v"], variant="kda", **gate_kwargs(dd),
                       initial_state=buf, final_state=buf, chunk=chunk)
    assert S.data_ptr() == buf.data_ptr()
    o_ref, S_ref = oracle.forward("kda", **d, initial_state=S0)
    assert_close(o, o_ref, torch.bfloat16, "o")
    assert_close(buf, S_ref, torch.bfloat16, "S")


def test_empty_sequence_copies_state():
    S0 = random_state(2, 3, 128, 128, 1).cuda()
    q = torch.empty(2, 0, 3, 128, device="cuda", dtype=torch.bfloat16)
    beta = torch.empty(2, 0, 3, device="cuda")
    o, S = gdr.forward(q, q, q, variant="gdn", beta=beta, log_g=beta, initial_state=S0)
    torch.cuda.synchronize()
    assert o.shape == (2, 0, 3, 128) and torch.equal(S, S0)
    o, S = gdr.forward(q, q, q, variant="gdn", beta=beta, log_g=beta)
    torch.cuda.synchronize()
    assert torch.count_nonzero(S).item() == 0


# ----------------------------------------------------------------- consistency
@pytest.mark.parametrize("chunk", [1, 65])
def test_deterministic(chunk):
    kernel_or_skip("gdn2", torch.bfloat16, 2, 300, 4, 128, 128, chunk)
    d = to_dev(make_inputs("gdn2", 2, 300, 4, dtype=torch.bfloat16, seed=2))
    a = gdr.forward(d["q"], d["k"], d["v"], variant="gdn2", **gate_kwargs(d), chunk=chunk)
    b = gdr.forward(d["q"], d["k"], d["v"], variant="gdn2", **gate_kwargs(d), chunk=chunk)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


@pytest.mark.parametrize("chunk", [1, 65])
@pytest.mark.parametrize("variant", VARS)
def test_resume_split(variant, chunk):
    """forward over [0,T) == forward over [0,T1) then [T1,T) from the carried state."""
    kernel_or_skip(variant, torch.bfloat16, 2, 200, 2, 128, 128, chunk)
    d = to_dev(make_inputs(variant, 2, 200, 2, dtype=torch.bfloat16, seed=4))
    o, S = gdr.forward(d["q"], d["k"], d["v"], variant=variant, **gate_kwargs(d), chunk=chunk)
    a = select(d, t=slice(0, 77))
    b = select(d, t=slice(77, 200))
    oa, Sa = gdr.forward(a["q"], a["k"], a["v"], variant=variant, **gate_kwargs(a), chunk=chunk)
    ob, Sb = gdr.forward(b["q"], b["k"], b["v"], variant=variant, **gate_kwargs(b), chunk=chunk,
                         initial_state=Sa)
    assert_gpu_close(torch.cat([oa, ob], 1), o, "o")
    assert_gpu_close(Sb, S, "S")


@pytest.mark.parametrize("variant", ["gdn", "kda", "kla", "gdn2"])
def test_segmented_carry(variant):
    """Few sequences, many chunks: the two-kernel path splits each sequence into
    segments (segment 0's end state and the other segments' affine maps in one
    launch, a chain of start states, then every segment from its start).
    B=1, H=2, T=4100 gives 65 chunks with a ragged tail (13 segments of 5);
    compared element by element with the oracle, with an initial state."""
    B, T, H = 1, 4100, 2
    launches = gdr.forward_launches(variant, torch.bfloat16, B, T, H, 128, 128, 0)
    assert launches == 4, f"expected the segmented carry (4 launches), got {launches}"
    o, S, o_ref, S_ref = run_both(variant, B, T, H, 128, 128, torch.bfloat16, 0, seed=21)
    assert_close(o, o_ref, torch.bfloat16, "o")
    assert_close(S, S_ref, torch.bfloat16, "S")


@pytest.mark.parametrize("variant", ["gdn", "deltanet", "kla", "kda", "gdn2"])
def test_pipelined_sweep(variant):
    """B*H = 64 sequences leave most SMs idle beside the carry, so the two-kernel
    path cuts the sweep in two: the second part's preparation runs beside the
    first part's carry, and the second carry starts from the first one's states
    (kept in the workspace).  24 chunks, the last one ragged; with an initial state."""
    B, T, H = 4, 1531, 16
    launches = gdr.forward_launches(variant, torch.bfloat16, B, T, H, 128, 128, 0)
    assert launches == 4, f"expected the pipelined sweep (4 launches), got {launches}"
    o, S, o_ref, S_ref = run_both(variant, B, T, H, 128, 128, torch.bfloat16, 0, seed=23)
    assert_close(o, o_ref, torch.bfloat16, "o")
    assert_close(S, S_ref, torch.bfloat16, "S")


@pytest.mark.parametrize("variant", ["gdn", "kda", "gdn2"])
def test_pipelined_sweep_dv64(variant):
    """The pipelined sweep at d_v = 64: the first carry's end states (32 KB per
    sequence) in the chunk-0 records of the smaller dv = 64 record layout."""
    B, T, H = 4, 1531, 16
    assert gdr.forward_launches(variant, torch.bfloat16, B, T, H, 128, 64, 0) == 4
    o, S, o_ref, S_ref = run_both(variant, B, T, H, 128, 64, torch.bfloat16, 0, seed=25)
    assert_close(o, o_ref, torch.bfloat16, "o")
    assert_close(S, S_ref, torch.bfloat16, "S")


def test_pipelined_sweep_no_states():
    """The pipelined sweep with neither an initial nor a final state: the middle
    states live in the workspace, so the output is unchanged."""
    B, T, H = 4, 1531, 16
    assert gdr.forward_launches("gdn", torch.bfloat16, B, T, H, 128, 128, 0) == 4
    d = make_inputs("gdn", B, T, H, 128, 128, dtype=torch.bfloat16, seed=24)
    dd = to_dev(d)
    o, S = gdr.forward(dd["q"], dd["k"], dd["v"], variant="gdn", **gate_kwargs(dd), output_final_state=False)
    torch.cuda.synchronize()
    assert S is None
    o_ref, _ = oracle.forward("gdn", **d)
    assert_close(o, o_ref, torch.bfloat16, "o")


@pytest.mark.parametrize("variant,s0", [("gdn", True), ("kla", True), ("kda", True), ("gdn2", True),
                                        ("gdn", False)])
def test_segmented_carry_finer_parts(variant, s0):
    """Phase 2 cut finer than phase 1's segments: B=1, H=17, T=7041 (111 chunks,
    the last of one token) runs the maps over 5 segments of 24 chunks and the
    carry with outputs over 7 parts of 16 (the last one 15).  Part starts fall
    inside segment 0 (chunk 16: the state itself), inside later segments
    (chunks 32, 64, 80: map and offset after the chunks before them, applied to
    the segment's start) and on segment starts (chunks 48, 96).  Compared
    element by element with the oracle."""
    B, T, H = 1, 7041, 17
    plan = gdr.forward_plan(variant, B, T, H, 128, 148)
    assert (plan["segments"], plan["segment_chunks"], plan["parts"], plan["part_chunks"]) == (5, 24, 7, 16)
    assert gdr.forward_launches(variant, torch.bfloat16, B, T, H, 128, 128, 0) == 4
    o, S, o_ref, S_ref = run_both(variant, B, T, H, 128, 128, torch.bfloat16, 0, seed=41, s0=s0)
    assert_close(o, o_ref, torch.bfloat16, "o")
    assert_close(S, S_ref, torch.bfloat16, "S")


@pytest.mark.parametrize("shape", [(1, 4100, 2), (1, 7041, 17)])
def test_segmented_carry_long_memory(shape):
    """The segmented carry where a segment's start state still shows at its
    end: DeltaNet (no decay) with beta scaled by 0.1, so that the maps M_g and
    M_g(j) keep most of a state over a segment (with the recipe's gates they
    fall below 1e-20 and a wrong map product would go unseen).  Both plans: 13
    segments of 5 chunks, and 5 segments of 24 with 7 parts of 16."""
    B, T, H = shape
    assert gdr.forward_launches("deltanet", torch.bfloat16, B, T, H, 128, 128, 0) == 4
    d = make_inputs("deltanet", B, T, H, 128, 128, dtype=torch.bfloat16, seed=47)
    d["beta"] = (0.1 * d["beta"]).contiguous()
    S0 = random_state(B, H, 128, 128, 48)
    dd = to_dev(d)
    o, S = gdr.forward(dd["q"], dd["k"], dd["v"], variant="deltanet", **gate_kwargs(dd), initial_state=S0.cuda(),
                       chunk=0)
    torch.cuda.synchronize()
    o_ref, S_ref = oracle.forward("deltanet", **d, initial_state=S0)
    assert_close(o, o_ref, torch.bfloat16, "o")
    assert_close(S, S_ref, torch.bfloat16, "S")


def test_segmented_carry_no_initial_state():
    """Segmented carry from a zero state, B=2 H=3 T=4480 (70 chunks, 12 segments
    of 6): segment 0 then starts from zeros like every other segment's offset."""
    B, T, H = 2, 4480, 3
    assert gdr.forward_launches("gdn", torch.bfloat16, B, T, H, 128, 128, 0) == 4
    o, S, o_ref, S_ref = run_both("gdn", B, T, H, 128, 128, torch.bfloat16, 0, seed=22, s0=False)
    assert_close(o, o_ref, torch.bfloat16, "o")
    assert_close(S, S_ref, torch.bfloat16, "S")


def test_kla_is_gdn_with_kaczmarz_beta():
    """KLA = Gated DeltaNet with beta_t = eta_t / (||k_t||^2 + eps) ("Kaczmarz Linear
    Attention", implementation: only the diagonal coefficient matrix changes)."""
    for chunk in (1, 65):
        if gdr.forward_kernel_name("kla", torch.bfloat16, 2, 150, 2, 128, 128, chunk) == "none":
            continue
        d = to_dev(make_inputs("kla", 2, 150, 2, dtype=torch.bfloat16, seed=8))
        o1, S1 = gdr.forward(d["q"], d["k"], d["v"], variant="kla", **gate_kwargs(d), eps=1e-6, chunk=chunk)
        kk = d["k"].float().pow(2).sum(-1)
        beta = (d["beta"] / (kk + 1e-6)).contiguous()
        o2, S2 = gdr.forward(d["q"], d["k"], d["v"], variant="gdn", beta=beta, log_g=d["log_g"], chunk=chunk)
        assert_gpu_close(o2, o1, "o", tol=1e-2)
        assert_gpu_close(S2, S1, "S", tol=1e-2)


def test_gdn2_tied_equals_kda_gpu():
    """GDN-2 with b_t = w_t = beta_t equals KDA ("Gated DeltaNet-2", what is new)."""
    for chunk in (1, 65):
        if gdr.forward_kernel_name("gdn2", torch.bfloat16, 2, 150, 2, 128, 128, chunk) == "none":
            continue
        dk = to_dev(make_inputs("kda", 2, 150, 2, dtype=torch.bfloat16, seed=6))
        d2 = to_dev(make_inputs("gdn2", 2, 150, 2, dtype=torch.bfloat16, seed=6, gdn2_tied=True))
        assert torch.equal(dk["q"], d2["q"]) and torch.equal(dk["log_g"], d2["log_g"])
        o1, S1 = gdr.forward(dk["q"], dk["k"], dk["v"], variant="kda", **gate_kwargs(dk), chunk=chunk)
        o2, S2 = gdr.forward(d2["q"], d2["k"], d2["v"], variant="gdn2", **gate_kwargs(d2), chunk=chunk)
        assert_gpu_close(o2, o1, "o", tol=1e-2)
        assert_gpu_close(S2, S1, "S", tol=1e-2)


@pytest.mark.parametrize("variant", VARS)
def test_forward_equals_decode_steps(variant):
    """A forward over T tokens equals T single-token decode steps."""
    B, T, H = 3, 20, 2
    d = to_dev(make_inputs(variant, B, T, H, dtype=torch.bfloat16, seed=10))
    S0 = random_state(B, H, 128, 128, 11).cuda()
    o, S = gdr.forward(d["q"], d["k"], d["v"], variant=variant, **gate_kwargs(d), initial_state=S0)
    state = S0.clone()
    outs = []
    for t in range(T):
        s = select(d, t=t)
        outs.append(gdr.decode_step(s["q"], s["k"], s["v"], state, variant=variant, **gate_kwargs(s)))
    assert_gpu_close(torch.stack(outs, 1), o, "o")
    assert_gpu_close(state, S, "S")


# ----------------------------------------------------------------- decode vs oracle
@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32])
@pytest.mark.parametrize("variant", VARS)
def test_decode_step_parity(variant, dtype):
    N, H = 7, 3
    S0 = random_state(N, H, 128, 128, 3)
    state = S0.cuda()
    S_ref = S0.double().numpy()
    for step in range(4):
        d = make_decode_inputs(variant, N, H, step, dtype=dtype)
        dd = to_dev(d)
        o = gdr.decode_step(dd["q"], dd["k"], dd["v"], state, variant=variant, **gate_kwargs(dd))
        o_ref, S_ref = oracle.decode_step(variant, d["q"], d["k"], d["v"], S_ref, **gate_kwargs(d))
        assert_close(o, o_ref, dtype, f"o step {step}")
    assert_close(state, S_ref, dtype, "state")


@pytest.mark.parametrize("dkdv", [(64, 64), (64, 128), (128, 64)])
def test_decode_head_dims(dkdv):
    dk, dv = dkdv
    S0 = random_state(5, 2, dk, dv, 4)
    state = S0.cuda()
    d = make_decode_inputs("gdn2", 5, 2, 0, dk=dk, dv=dv)
    dd = to_dev(d)
    o = gdr.decode_step(dd["q"], dd["k"], dd["v"], state, variant="gdn2", **gate_kwargs(dd))
    o_ref, S_ref = oracle.decode_step("gdn2", d["q"], d["k"], d["v"], S0, **gate_kwargs(d))
    assert_close(o, o_ref, torch.bfloat16, "o")
    assert_close(state, S_ref, torch.bfloat16, "state")


# ----------------------------------------------------------------- CLVR value routing
@pytest.mark.parametrize("routing", ["target", "mixed", "output"])
@pytest.mark.parametrize("variant", ["gdn", "deltanet"])
def test_cross_layer_value_routing(variant, routing):
    """Cross-layer value routing ("Linear Attention Architectures", the CLVR part):
    a lower layer hands its write target to a higher layer, which writes it in
    place of (or mixed with) its own value.  Only the value input changes, so the
    kernels take the routed tensor as v: here the upper layer's v is the lower
    layer's v ("target"), the mean of both ("mixed"), or the lower layer's output
    ("output", the routed tensor produced on the GPU by the call before), and the
    upper call is compared with the oracle fed the same routed values."""
    B, T, H = 2, 333, 3
    lower = make_inputs(variant, B, T, H, dtype=torch.bfloat16, seed=51)
    upper = make_inputs(variant, B, T, H, dtype=torch.bfloat16, seed=52)
    dl, du = to_dev(lower), to_dev(upper)
    o_low, _ = gdr.forward(dl["q"], dl["k"], dl["v"], variant=variant, **gate_kwargs(dl))
    if routing == "target":
        v_routed = dl["v"]
    elif routing == "mixed":
        v_routed = (0.5 * (dl["v"].float() + du["v"].float())).to(torch.bfloat16).contiguous()
    else:
        v_routed = o_low
    o, S = gdr.forward(du["q"], du["k"], v_routed, variant=variant, **gate_kwargs(du))
    torch.cuda.synchronize()
    ref_in = dict(upper)
    ref_in["v"] = v_routed.cpu()
    o_ref, S_ref = oracle.forward(variant, **ref_in)
    assert_close(o, o_ref, torch.bfloat16, f"{routing} o")
    assert_close(S, S_ref, torch.bfloat16, f"{routing} S")
