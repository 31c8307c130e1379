"""Shared helpers of the GPU parity tests: error metrics and input plumbing.

Tolerances (written here once, used by every parity test):
  * fp32 I/O: max|gpu - ref| / max|ref| <= 1e-4, for o and, separately, for
    the final state;
  * bf16 I/O (fp32 state), with the oracle run on the bf16-rounded inputs
    up-cast exactly to fp64:
      - final state (fp32): max|gpu - ref| <= 2e-2 * RMS(ref);
      - o (stored as bf16): max(|gpu - ref| - 2^-8 |ref|) <= 2e-2 * RMS(ref).
    The 2^-8 |ref| term is the rounding of the output to bf16 itself (at most
    half an ulp, i.e. <= 2^-8 of the value), which no bf16-output kernel can
    avoid; the outputs are heavy-tailed (max|o| / RMS(o) reaches 20-50 on
    these workloads), so without it even the exact result rounded to bf16
    would exceed 2e-2 * RMS.  The bound on the arithmetic is unchanged.
      - o, bulk elements (|ref| <= 4 RMS(ref)), with no allowance at all:
        max|gpu - ref| <= (2e-2 + 4 * 2^-8) * RMS(ref) = 3.56e-2 * RMS(ref),
        the arithmetic budget plus the largest bf16 rounding such an element
        can have.  It is reported beside the first metric so that the
        rounding allowance cannot hide an error on the bulk of the output.
  * GDN-2's gate gradients (d erase_b, d write_w; fp32) in the backward, per
    64-token chunk: max|gpu - ref| <= 2e-2 * RMS(ref) + 2^-10 * max|ref| over
    the chunk.  The gradients inherit the relative error of the chunk states
    that the carries hold with fp16 operands (unit roundoff 2^-11; 2^-10 allows
    twice that) in proportion to the size of the terms a chunk's gradients
    are built from.  d erase_b is k times a difference of two such terms, which
    the final-state gradient dominates at the sequence's last tokens: under a
    random unit-scale d_final the last chunk's largest elements reach ~270
    RMS, and every element of that chunk carries an error of ~2^-11 of them.
    In every other chunk the allowance is a few 1e-3 RMS.
  * d log g under the same per-chunk metric where the last chunk holds one
    token: that token's d log g carries the whole <dS_T, S_T> term of the
    final-state gradient (57 RMS for GDN, 360 RMS for KDA in the segmented
    test with a one-token tail, each measured within 6e-4 of itself).
"""
import numpy as np
import torch

F32_TOL = 1e-4
BF16_TOL = 2e-2


def to_dev(d, device="cuda"):
    return {k: (None if v is None else v.to(device)) for k, v in d.items()}


def max_rel(gpu, ref):
    gpu = gpu.detach().double().cpu().numpy() if hasattr(gpu, "detach") else np.asarray(gpu)
    return float(np.max(np.abs(gpu - ref)) / max(np.max(np.abs(ref)), 1e-30))


def elem_rel(gpu, ref):
    """max |gpu - ref| / max(|ref|, 1e-6 max|ref|): the element-wise relative error,
    floored where the reference is near zero (reported next to the fp32 bar)."""
    gpu = gpu.detach().double().cpu().numpy() if hasattr(gpu, "detach") else np.asarray(gpu)
    floor = 1e-6 * max(float(np.max(np.abs(ref))), 1e-30)
    return float(np.max(np.abs(gpu - ref) / np.maximum(np.abs(ref), floor)))


def rms_rel(gpu, ref):
    gpu = gpu.detach().double().cpu().numpy() if hasattr(gpu, "detach") else np.asarray(gpu)
    return float(np.max(np.abs(gpu - ref)) / max(np.sqrt(np.mean(ref * ref)), 1e-30))


BF16_ROUND = 2.0 ** -8


def bf16_out_rel(gpu, ref):
    """max(|gpu - ref| - 2^-8 |ref|) / RMS(ref): error beyond the output's own bf16 rounding."""
    gpu = gpu.detach().double().cpu().numpy() if hasattr(gpu, "detach") else np.asarray(gpu)
    excess = np.abs(gpu - ref) - BF16_ROUND * np.abs(ref)
    return float(max(np.max(excess), 0.0) / max(np.sqrt(np.mean(ref * ref)), 1e-30))


BULK_RMS = 4.0
BULK_TOL = BF16_TOL + BULK_RMS * BF16_ROUND


def bulk_rel(gpu, ref):
    """max|gpu - ref| / RMS(ref) over the elements with |ref| <= 4 RMS(ref), plain."""
    gpu = gpu.detach().double().cpu().numpy() if hasattr(gpu, "detach") else np.asarray(gpu)
    rms = max(np.sqrt(np.mean(ref * ref)), 1e-30)
    bulk = np.abs(ref) <= BULK_RMS * rms
    if not bulk.any():
        return 0.0
    return float(np.max(np.abs(gpu - ref)[bulk]) / rms)


def assert_close(gpu, ref, dtype, what=""):
    """The parity bar for the I/O dtype (see module docstring).  A bf16 tensor
    is an output stored in bf16; an fp32 tensor in a bf16 run is the state."""
    if dtype == torch.float32:
        err = max_rel(gpu, ref)
        assert err <= F32_TOL, (f"{what}: max|err|/max|ref| = {err:.3e} > {F32_TOL} "
                                f"(element-wise, floored at 1e-6 max|ref|: {elem_rel(gpu, ref):.3e})")
    elif gpu.dtype == torch.bfloat16:
        err = bf16_out_rel(gpu, ref)
        bulk = bulk_rel(gpu, ref)
        assert err <= BF16_TOL, (f"{what}: max(|err| - 2^-8|ref|)/RMS(ref) = {err:.3e} > {BF16_TOL} "
                                 f"(plain max|err|/RMS = {rms_rel(gpu, ref):.3e}, on the bulk {bulk:.3e})")
        assert bulk <= BULK_TOL, (f"{what}: plain max|err|/RMS(ref) on |ref| <= 4 RMS = {bulk:.3e} > "
                                  f"{BULK_TOL:.4f} (rounding-aware metric {err:.3e})")
    else:
        err = rms_rel(gpu, ref)
        assert err <= BF16_TOL, f"{what}: max|err|/RMS(ref) = {err:.3e} > {BF16_TOL}"
    return err


CARRY_ROUND = 2.0 ** -10


def assert_close_gate_grad(gpu, ref, what="", chunk=64):
    """fp32 gate gradients [B,T,H] or [B,T,H,dk] whose values concentrate in a
    few chunks: GDN-2's gates (see module docstring), and d log g where a short
    last chunk takes the final-state gradient's whole term.  Per chunk,
    max(|err|) - 2^-10 max|ref| <= 2e-2 RMS(ref)."""
    gpu = gpu.detach().double().cpu().numpy() if hasattr(gpu, "detach") else np.asarray(gpu)
    rms = max(np.sqrt(np.mean(ref * ref)), 1e-30)
    err, T = 0.0, ref.shape[1]
    for c0 in range(0, T, chunk):
        e = np.abs(gpu[:, c0:c0 + chunk] - ref[:, c0:c0 + chunk]).max()
        err = max(err, (e - CARRY_ROUND * np.abs(ref[:, c0:c0 + chunk]).max()) / rms)
    assert err <= BF16_TOL, (f"{what}: max over chunks of (max|err| - 2^-10 max|ref|)/RMS(ref) = {err:.3e} > "
                             f"{BF16_TOL} (plain max|err|/RMS = {rms_rel(gpu, ref):.3e})")
    return err


def gate_kwargs(d):
    return {k: d[k] for k in ("beta", "log_g", "erase_b", "write_w")}


def select(d, b=None, t=None, h=None):
    """Slice every [B,T,H,...] tensor of an input dict (None entries pass through)."""
    out = {}
    for k, v in d.items():
        if v is None:
            out[k] = None
            continue
        x = v
        if b is not None:
            x = x[b]
        if t is not None:
            x = x[:, t]
        if h is not None:
            x = x[:, :, h]
        out[k] = x.contiguous()
    return out


def assert_gpu_close(a, b, what="", tol=BF16_TOL):
    """GPU-vs-GPU agreement of two results of the same quantity: for bf16
    tensors each side carries its own output rounding (allowance 2 * 2^-8 |b|);
    fp32 tensors are compared plainly.  Both against tol * RMS(b)."""
    a64, b64 = a.detach().double().cpu(), b.detach().double().cpu()
    allow = 2 * BF16_ROUND * b64.abs() if (a.dtype == torch.bfloat16 or b.dtype == torch.bfloat16) else 0.0
    excess = ((a64 - b64).abs() - allow).clamp_min(0).max().item()
    rms = b64.pow(2).mean().sqrt().item()
    assert excess <= tol * rms, f"{what}: excess {excess:.3e} > {tol} * RMS {rms:.3e}"
