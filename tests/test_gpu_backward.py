"""GPU parity of the chunked backward (all five variants) against the fp64
reverse-mode oracle, through the C ABI.

The backward re-runs the forward's chunk products and carry, runs the
end-state-gradient recurrence on the forward's carry kernel over the chunks in
reverse, and computes each chunk's gradients in fp32.  Its carries use fp16
operands with fp32 accumulation, as the forward's chunked path does, so the
bar is the forward's (tests/parity_util.py): bf16 gradients (dq, dk, dv)
within 2e-2 of RMS beyond their own bf16 rounding (and 3.56e-2 plain on the
bulk), fp32 gradients (d beta / d eta, d log_g, the initial state's) within
2e-2 of RMS.  The oracle sees the bf16-rounded inputs up-cast exactly.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_forward_b200 as gdr
import oracle
from gated_delta_rule_forward_b200.inputs import make_inputs, random_output_grad, random_state
from parity_util import assert_close, assert_close_gate_grad, select, to_dev

pytestmark = pytest.mark.gpu
VARS = ["deltanet", "gdn", "kda", "gdn2", "kla"]


def run_backward(variant, B, T, H, dv=128, seed=0, s0=True, d_final=True, do_scale=1.0, scale=None, edit=None):
    dk = 128
    scale = dk ** -0.5 if scale is None else scale
    d = make_inputs(variant, B, T, H, dk, dv, dtype=torch.bfloat16, seed=seed)
    if edit is not None:
        edit(d)
    S0 = random_state(B, H, dk, dv, seed + 1) if s0 else None
    dS = random_state(B, H, dk, dv, seed + 2, scale=1.0) if d_final else None
    dO = random_output_grad(B, T, H, dv, seed + 3, scale=do_scale)
    dd = to_dev(d)
    g = gdr.backward(dd["q"], dd["k"], dd["v"], dO.cuda(), variant=variant, **gates(dd),
                     initial_state=None if S0 is None else S0.cuda(),
                     d_final_state=None if dS is None else dS.cuda(), scale=scale)
    gdr.device_status()
    ref = oracle.backward(variant, d["q"], d["k"], d["v"], dO, **gates(d), initial_state=S0, d_final=dS,
                          scale=scale)
    return g, ref


def gates(d):
    return {x: d[x] for x in ("beta", "log_g", "erase_b", "write_w")}


def check_grads(g, ref, variant, what=""):
    for name in ("q", "k", "v"):
        assert_close(g[name], ref[name], torch.bfloat16, f"{what} d{name}")
    if variant == "gdn2":
        assert_close_gate_grad(g["erase_b"], ref["erase_b"], f"{what} d erase_b")
        assert_close_gate_grad(g["write_w"], ref["write_w"], f"{what} d write_w")
    else:
        assert_close(g["beta"], ref["beta"], torch.bfloat16, f"{what} d{'eta' if variant == 'kla' else 'beta'}")
    if variant != "deltanet" and ref["log_g"] is not None:
        assert_close(g["log_g"], ref["log_g"], torch.bfloat16, f"{what} dlog_g")
    assert_close(g["initial_state"], ref["initial_state"], torch.bfloat16, f"{what} d initial state")


@pytest.mark.parametrize("dv", [128, 64])
@pytest.mark.parametrize("variant", VARS)
def test_backward_small_ragged(variant, dv):
    """Four chunks, the last one ragged (200 = 3 x 64 + 8), with an initial
    state and a final-state gradient."""
    g, ref = run_backward(variant, 2, 200, 3, dv=dv, seed=21)
    check_grads(g, ref, variant)


@pytest.mark.parametrize("T", [1, 37, 64, 65, 128])
def test_backward_short_sequences(T):
    """One partial chunk, one full chunk, one token past a chunk boundary."""
    g, ref = run_backward("gdn", 1, T, 2, seed=22)
    check_grads(g, ref, "gdn", f"T={T}")


@pytest.mark.parametrize("T", [1, 20, 37, 65])
@pytest.mark.parametrize("variant", ["kda", "gdn2"])
def test_backward_short_sequences_channel_decay(variant, T):
    """The channel-decay chunk products factor the decay around token 31 of a
    chunk, or around the last token of a shorter one: chunks of 1, 20 and 37
    tokens and a 1-token tail."""
    g, ref = run_backward(variant, 1, T, 2, seed=31)
    check_grads(g, ref, variant, f"T={T}")


def test_backward_without_states():
    """No initial state and no final-state gradient: the initial state's
    gradient is still returned (that of a zero initial state)."""
    g, ref = run_backward("gdn", 2, 150, 2, seed=23, s0=False, d_final=False)
    check_grads(g, ref, "gdn")


def test_backward_zero_length():
    """T = 0: no token gradients; the initial state's gradient is the final state's."""
    dS = random_state(1, 2, 128, 128, 5).cuda()
    z = torch.empty(1, 0, 2, 128, device="cuda", dtype=torch.bfloat16)
    beta = torch.empty(1, 0, 2, device="cuda")
    g = gdr.backward(z, z, z, z, variant="gdn", beta=beta, log_g=beta, d_final_state=dS)
    torch.cuda.synchronize()
    assert torch.equal(g["initial_state"], dS)


@pytest.mark.parametrize("do_scale", [1e-6, 1e4])
def test_backward_gradient_magnitudes(do_scale):
    """Output gradients far from unit scale: the internal power-of-two rescaling
    keeps the fp16 operands of the reverse carry in range."""
    g, ref = run_backward("kla", 2, 160, 2, seed=24, d_final=False, do_scale=do_scale)
    check_grads(g, ref, "kla", f"d_o x {do_scale:g}")


def test_backward_strong_decay():
    """A decay logit scaled by 6 (log g down to about -20 per token): decay
    enters only through factors at most 1, so nothing overflows."""
    def edit(d):
        d["log_g"] = (d["log_g"] * 6.0).contiguous()
    g, ref = run_backward("gdn", 1, 192, 2, seed=25, edit=edit)
    check_grads(g, ref, "gdn", "strong decay")


def chunk_span_log2(log_g):
    """Largest |gamma_t - gamma_31| within a 64-token chunk (log2 units), gamma the
    chunk-local cumulative log decay of each channel (zero-padded past T)."""
    B, T, H, dk = log_g.shape
    NC = (T + 63) // 64
    pad = np.zeros((B, NC * 64, H, dk))
    pad[:, :T] = log_g.double().numpy()
    g = np.cumsum(pad.reshape(B, NC, 64, H, dk), axis=2)
    return float(np.abs(g - g[:, :, 31:32]).max() / np.log(2.0))


@pytest.mark.parametrize("variant", ["kda", "gdn2"])
def test_backward_strong_channel_decay(variant):
    """Channel decay doubled: factors up to 2^90-2^120 within a chunk, inside
    the forward's factoring range (2^120)."""
    def edit(d):
        d["log_g"] = (d["log_g"] * 2.0).contiguous()
        span = chunk_span_log2(d["log_g"])
        assert 85.0 < span < 120.0, span
    g, ref = run_backward(variant, 1, 192, 2, seed=25, edit=edit)
    check_grads(g, ref, variant, "strong channel decay")


def test_backward_gdn2_tied_gates_is_kda():
    """GDN-2 with b = w = beta on every channel is KDA ("Gated DeltaNet-2", what
    is new): its q, k, v and log g gradients are KDA's, and the gate gradients
    summed over the channels, sum_i (d b_i + d w_i), are KDA's d beta."""
    B, T, H = 2, 200, 3
    d = make_inputs("gdn2", B, T, H, dtype=torch.bfloat16, seed=34, gdn2_tied=True)
    S0 = random_state(B, H, 128, 128, 35)
    dS = random_state(B, H, 128, 128, 36, scale=1.0)
    dO = random_output_grad(B, T, H, 128, 37)
    dd = to_dev(d)
    g = gdr.backward(dd["q"], dd["k"], dd["v"], dO.cuda(), variant="gdn2", **gates(dd), initial_state=S0.cuda(),
                     d_final_state=dS.cuda(), scale=128 ** -0.5)
    gdr.device_status()
    beta = d["erase_b"][..., 0].contiguous()
    ref = oracle.backward("kda", d["q"], d["k"], d["v"], dO, beta=beta, log_g=d["log_g"], initial_state=S0, d_final=dS,
                          scale=128 ** -0.5)
    for name in ("q", "k", "v"):
        assert_close(g[name], ref[name], torch.bfloat16, f"d{name}")
    assert_close(g["log_g"], ref["log_g"], torch.bfloat16, "dlog_g")
    assert_close(g["initial_state"], ref["initial_state"], torch.bfloat16, "d initial state")
    assert_close(g["erase_b"].sum(-1) + g["write_w"].sum(-1), ref["beta"], torch.bfloat16, "sum d b + d w = d beta")


@pytest.mark.parametrize("variant", ["kda", "gdn2"])
def test_backward_decay_beyond_the_guard_is_reported(variant):
    """A decay of e^-5 per token on every channel spans 2^230 within a chunk:
    the backward returns normally and reports GDR_ERR_RANGE."""
    d = to_dev(make_inputs(variant, 1, 130, 2, seed=32))
    d["log_g"] = torch.full_like(d["log_g"], -5.0)
    dO = random_output_grad(1, 130, 2, 128, 33).cuda()
    gdr.device_status()
    gdr.backward(d["q"], d["k"], d["v"], dO, variant=variant, **gates(d))
    with pytest.raises(gdr.GdrError) as e:
        gdr.device_status()
    assert e.value.status == 6, str(e.value)
    gdr.device_status()   # the flag is cleared once read


@pytest.mark.parametrize("variant", ["gdn", "kla", "kda", "gdn2"])
def test_backward_350m_layer_sampled(variant):
    """The 350M layer (B=8, T=2048, H=8, full size, in the launch configuration of
    a training step), checked against the oracle on two of its sequences."""
    B, T, H = 8, 2048, 8
    dk = dv = 128
    scale = dk ** -0.5
    d = make_inputs(variant, B, T, H, dk, dv, dtype=torch.bfloat16, seed=26)
    dO = random_output_grad(B, T, H, dv, 27)
    dd = to_dev(d)
    g = gdr.backward(dd["q"], dd["k"], dd["v"], dO.cuda(), variant=variant, **gates(dd), scale=scale)
    gdr.device_status()
    for b in (0, B - 1):
        s = select(d, b=slice(b, b + 1))
        ref = oracle.backward(variant, s["q"], s["k"], s["v"], dO[b:b + 1], **gates(s), scale=scale)
        gb = {k: (None if x is None else x[b:b + 1]) for k, x in g.items()}
        check_grads(gb, ref, variant, f"sequence {b}")


def test_backward_rejects_uncovered_cases():
    """fp32 I/O is not covered by the backward (GDR_ERR_UNSUPPORTED)."""
    d = to_dev(make_inputs("gdn", 1, 64, 1, dtype=torch.float32))
    dO = torch.zeros(1, 64, 1, 128, device="cuda", dtype=torch.float32)
    with pytest.raises(gdr.GdrError) as e:
        gdr.backward(d["q"], d["k"], d["v"], dO, variant="gdn", beta=d["beta"], log_g=d["log_g"])
    assert e.value.status == 2   # GDR_ERR_UNSUPPORTED


def test_backward_long_context_sampled():
    """The 65536-token sequence (B=1, H=16): 1024 chunks through both carries,
    checked against the oracle on two of its heads."""
    B, T, H = 1, 65536, 16
    scale = 128 ** -0.5
    d = make_inputs("gdn", B, T, H, dtype=torch.bfloat16, seed=28)
    dO = random_output_grad(B, T, H, 128, 29)
    dd = to_dev(d)
    g = gdr.backward(dd["q"], dd["k"], dd["v"], dO.cuda(), variant="gdn", beta=dd["beta"], log_g=dd["log_g"],
                     scale=scale)
    gdr.device_status()
    for h in (0, H - 1):
        s = select(d, h=slice(h, h + 1))
        ref = oracle.backward("gdn", s["q"], s["k"], s["v"], dO[:, :, h:h + 1], beta=s["beta"], log_g=s["log_g"],
                              scale=scale)
        gh = {k: (None if x is None else (x[:, h:h + 1] if k == "initial_state" else x[:, :, h:h + 1]))
              for k, x in g.items()}
        check_grads(gh, ref, "gdn", f"head {h}")


@pytest.mark.parametrize("variant", ["gdn", "kda", "gdn2"])
def test_backward_segmented_finer_parts(variant):
    """Both carries segmented with their second phase cut finer than the maps
    (B=1, H=17, T=7041: 5 segments of 24 chunks, 7 parts of 16); heads 0 and 16
    compared with the oracle.  The last chunk holds one token, whose d log g
    carries the whole <dS_T, S_T> term of the final-state gradient (57 RMS for
    GDN, 360 RMS for KDA on this input, each within 6e-4 of itself), so d log g
    takes the per-chunk metric that allows 2^-10 of a chunk's largest value."""
    B, T, H = 1, 7041, 17
    plan = gdr.forward_plan(variant, B, T, H, 128, 148)
    assert (plan["segments"], plan["parts"]) == (5, 7)
    scale = 128 ** -0.5
    d = make_inputs(variant, B, T, H, dtype=torch.bfloat16, seed=42)
    S0 = random_state(B, H, 128, 128, 43)
    dS = random_state(B, H, 128, 128, 44, scale=1.0)
    dO = random_output_grad(B, T, H, 128, 45)
    dd = to_dev(d)
    g = gdr.backward(dd["q"], dd["k"], dd["v"], dO.cuda(), variant=variant, **gates(dd), initial_state=S0.cuda(),
                     d_final_state=dS.cuda(), scale=scale)
    gdr.device_status()
    for h in (0, H - 1):
        s = select(d, h=slice(h, h + 1))
        ref = oracle.backward(variant, s["q"], s["k"], s["v"], dO[:, :, h:h + 1], **gates(s),
                              initial_state=S0[:, h:h + 1], d_final=dS[:, h:h + 1], scale=scale)
        gh = {k: (None if x is None else (x[:, h:h + 1] if k == "initial_state" else x[:, :, h:h + 1]))
              for k, x in g.items()}
        assert_close_gate_grad(gh["log_g"], ref["log_g"], f"head {h} dlog_g")
        check_grads({**gh, "log_g": None}, {**ref, "log_g": None}, variant, f"head {h}")


def test_backward_segmented_long_memory():
    """Both backward carries segmented (5 segments of 24 chunks, 7 parts of 16)
    where the maps keep most of a state over a segment: DeltaNet with beta
    scaled by 0.1 (see test_segmented_carry_long_memory); heads 0 and 16."""
    B, T, H = 1, 7041, 17
    scale = 128 ** -0.5
    d = make_inputs("deltanet", B, T, H, dtype=torch.bfloat16, seed=49)
    d["beta"] = (0.1 * d["beta"]).contiguous()
    S0 = random_state(B, H, 128, 128, 50)
    dS = random_state(B, H, 128, 128, 51, scale=1.0)
    dO = random_output_grad(B, T, H, 128, 52)
    dd = to_dev(d)
    g = gdr.backward(dd["q"], dd["k"], dd["v"], dO.cuda(), variant="deltanet", **gates(dd), initial_state=S0.cuda(),
                     d_final_state=dS.cuda(), scale=scale)
    gdr.device_status()
    for h in (0, H - 1):
        s = select(d, h=slice(h, h + 1))
        ref = oracle.backward("deltanet", s["q"], s["k"], s["v"], dO[:, :, h:h + 1], **gates(s),
                              initial_state=S0[:, h:h + 1], d_final=dS[:, h:h + 1], scale=scale)
        gh = {k: (None if x is None else (x[:, h:h + 1] if k == "initial_state" else x[:, :, h:h + 1]))
              for k, x in g.items()}
        check_grads(gh, ref, "deltanet", f"head {h}")


@pytest.mark.parametrize("variant", ["gdn", "kla", "kda", "gdn2"])
def test_backward_segmented(variant):
    """Few long sequences (B*H = 2, 65 chunks): both carries run in segments (13
    of 5 chunks) from an initial state and a final-state gradient."""
    assert gdr.forward_plan(variant, 1, 4100, 2, 128, 148)["segments"] == 13
    g, ref = run_backward(variant, 1, 4100, 2, seed=30)
    check_grads(g, ref, variant)
