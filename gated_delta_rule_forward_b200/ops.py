"""Python binding of libgdr: argument marshalling only.

Every step of the computation runs in the CUDA kernels behind the C ABI
(include/gdr.h).  These functions check devices, dtypes, shapes and
contiguity, allocate the outputs with PyTorch, and pass raw pointers and the
current CUDA stream.  There is no CPU path.
"""
from __future__ import annotations

import ctypes

import torch

from ._lib import BwdGrads, FwdArgs, check, lib

VARIANTS = {"deltanet": 0, "gdn": 1, "kda": 2, "gdn2": 3, "kla": 4}
RAW_INPUTS = 0x100   # GDR_RAW_INPUTS (include/gdr.h)
_DTYPES = {torch.float32: 0, torch.bfloat16: 1}
CHANNEL_DECAY = ("kda", "gdn2")


def variant_id(variant) -> int:
    if isinstance(variant, int):
        return variant
    try:
        return VARIANTS[variant]
    except KeyError:
        raise ValueError(f"unknown variant {variant!r}; one of {sorted(VARIANTS)}") from None


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need(t, name, shape, dtype, device):
    if t is None:
        raise ValueError(f"{name} is required")
    if t.device != device:
        raise ValueError(f"{name} must be on {device}")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _gates(vid, lead, dk, device, beta, log_g, erase_b, write_w):
    name = [k for k, v in VARIANTS.items() if v == vid][0]
    f32 = torch.float32
    if name != "gdn2":
        _need(beta, "beta", lead, f32, device)
    else:
        beta = None
    if name == "deltanet":
        log_g = None
    elif name in CHANNEL_DECAY:
        _need(log_g, "log_g", lead + (dk,), f32, device)
    else:
        _need(log_g, "log_g", lead, f32, device)
    if name == "gdn2":
        _need(erase_b, "erase_b", lead + (dk,), f32, device)
        _need(write_w, "write_w", lead + (dk,), f32, device)
    else:
        erase_b = write_w = None
    return beta, log_g, erase_b, write_w


def _stream(stream, device):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def forward(q, k, v, *, variant, beta=None, log_g=None, erase_b=None, write_w=None,
            initial_state=None, output_final_state=True, eps=1e-6, scale=1.0, chunk=0,
            out=None, final_state=None, stream=None, raw_inputs=False):
    """Gated delta-rule forward over whole sequences.

    q, k: [B,T,H,dk]; v: [B,T,H,dv]; bf16 or fp32 (all the same), CUDA,
    contiguous.  Gates fp32: beta [B,T,H] (eta for KLA); log_g [B,T,H]
    (gdn, kla) or [B,T,H,dk] (kda, gdn2); erase_b / write_w [B,T,H,dk] (gdn2).
    initial_state: fp32 [B,H,dk,dv] or None.  Returns (o, final_state or None).
    ``chunk``: 0 auto, 1 per-token kernel, 65 chunked path (preparation +
    carry; workspace allocated here).  ``raw_inputs``: q, k, beta and the gates
    are raw projections and logits; the kernels normalise q and k (not KLA's k)
    and apply sigmoid / -softplus themselves (GDR_RAW_INPUTS).
    """
    vid = variant_id(variant)
    if q.dim() != 4:
        raise ValueError("q must be [B,T,H,dk]")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("inputs must be CUDA tensors (there is no CPU path)")
    if q.dtype not in _DTYPES:
        raise ValueError("q, k, v must be bf16 or fp32")
    _need(q, "q", (B, T, H, dk), q.dtype, dev)
    _need(k, "k", (B, T, H, dk), q.dtype, dev)
    _need(v, "v", (B, T, H, dv), q.dtype, dev)
    beta, log_g, erase_b, write_w = _gates(vid, (B, T, H), dk, dev, beta, log_g, erase_b, write_w)
    if initial_state is not None:
        _need(initial_state, "initial_state", (B, H, dk, dv), torch.float32, dev)
    if out is None:
        out = torch.empty(B, T, H, dv, device=dev, dtype=q.dtype)
    else:
        _need(out, "out", (B, T, H, dv), q.dtype, dev)
    if output_final_state and final_state is None:
        final_state = torch.empty(B, H, dk, dv, device=dev, dtype=torch.float32)
    elif final_state is not None:
        _need(final_state, "final_state", (B, H, dk, dv), torch.float32, dev)
    a = FwdArgs(q=q.data_ptr(), k=k.data_ptr(), v=v.data_ptr(),
                beta=None if beta is None else beta.data_ptr(),
                log_g=None if log_g is None else log_g.data_ptr(),
                erase_b=None if erase_b is None else erase_b.data_ptr(),
                write_w=None if write_w is None else write_w.data_ptr(),
                initial_state=None if initial_state is None else initial_state.data_ptr(),
                final_state=None if final_state is None else final_state.data_ptr(),
                o=out.data_ptr())
    L = lib()
    dt = _DTYPES[q.dtype]
    vflag = vid | (RAW_INPUTS if raw_inputs else 0)
    ws = L.gdr_forward_workspace_size(vflag, dt, B, T, H, dk, dv, chunk)
    workspace = torch.empty(ws, device=dev, dtype=torch.uint8) if ws else None
    check(L.gdr_forward_chunked(vflag, dt, B, T, H, dk, dv, ctypes.byref(a), float(eps), float(scale),
                                int(chunk), _ptr(workspace), ws, _stream(stream, dev)))
    return out, final_state


def backward(q, k, v, d_o, *, variant, beta=None, log_g=None, erase_b=None, write_w=None, initial_state=None,
             d_final_state=None, eps=1e-6, scale=1.0, stream=None):
    """Gradients of <d_o, o> + <d_final_state, S_T> for the forward over the
    same inputs: the chunked backward (all five variants; bf16 q, k, v, d_o
    with dk = 128, dv 64 or 128; gates fp32 as for forward()).  Returns a dict
    keyed by the inputs: q, k, v (bf16), beta (d beta, or d eta for KLA; None
    for GDN-2), log_g (shaped as log_g; None for DeltaNet), erase_b and
    write_w (GDN-2, else None) and initial_state (fp32 [B,H,dk,dv]; the
    gradient of the initial state, zero-initial-state runs included)."""
    vid = variant_id(variant)
    if q.dim() != 4:
        raise ValueError("q must be [B,T,H,dk]")
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("inputs must be CUDA tensors (there is no CPU path)")
    if q.dtype not in _DTYPES:
        raise ValueError("q, k, v must be bf16 or fp32")
    _need(k, "k", (B, T, H, dk), q.dtype, dev)
    _need(v, "v", (B, T, H, dv), q.dtype, dev)
    _need(d_o, "d_o", (B, T, H, dv), q.dtype, dev)
    beta, log_g, erase_b, write_w = _gates(vid, (B, T, H), dk, dev, beta, log_g, erase_b, write_w)
    f32 = torch.float32
    if initial_state is not None:
        _need(initial_state, "initial_state", (B, H, dk, dv), f32, dev)
    if d_final_state is not None:
        _need(d_final_state, "d_final_state", (B, H, dk, dv), f32, dev)
    g = {"q": torch.empty_like(q), "k": torch.empty_like(k), "v": torch.empty_like(v),
         "beta": None if beta is None else torch.empty(B, T, H, device=dev, dtype=f32),
         "log_g": None if log_g is None else torch.empty(log_g.shape, device=dev, dtype=f32),
         "erase_b": None if erase_b is None else torch.empty_like(erase_b),
         "write_w": None if write_w is None else torch.empty_like(write_w),
         "initial_state": torch.empty(B, H, dk, dv, device=dev, dtype=f32)}
    opt = lambda x: None if x is None else x.data_ptr()
    a = FwdArgs(q=q.data_ptr(), k=k.data_ptr(), v=v.data_ptr(), beta=opt(beta), log_g=opt(log_g),
                erase_b=opt(erase_b), write_w=opt(write_w), initial_state=opt(initial_state))
    gr = BwdGrads(dq=g["q"].data_ptr(), dk=g["k"].data_ptr(), dv=g["v"].data_ptr(), dbeta=opt(g["beta"]),
                  dlog_g=opt(g["log_g"]), d_initial_state=g["initial_state"].data_ptr(),
                  d_erase_b=opt(g["erase_b"]), d_write_w=opt(g["write_w"]))
    L = lib()
    dt = _DTYPES[q.dtype]
    ws = L.gdr_backward_workspace_size(vid, dt, B, T, H, dk, dv)
    workspace = torch.empty(max(ws, 16), device=dev, dtype=torch.uint8)
    check(L.gdr_backward(vid, dt, B, T, H, dk, dv, ctypes.byref(a), _ptr(d_o),
                         _ptr(d_final_state), ctypes.byref(gr), float(eps), float(scale),
                         _ptr(workspace), ws, _stream(stream, dev)))
    return g


def decode_step(q, k, v, state, *, variant, beta=None, log_g=None, erase_b=None, write_w=None,
                eps=1e-6, scale=1.0, out=None, stream=None, raw_inputs=False):
    """One decode token for N sequences: q, k [N,H,dk]; v [N,H,dv]; state fp32
    [N,H,dk,dv] updated in place.  Returns o [N,H,dv].  ``raw_inputs`` as for
    forward()."""
    vid = variant_id(variant)
    N, H, dk = q.shape
    dv = v.shape[-1]
    dev = q.device
    if dev.type != "cuda":
        raise ValueError("inputs must be CUDA tensors (there is no CPU path)")
    if q.dtype not in _DTYPES:
        raise ValueError("q, k, v must be bf16 or fp32")
    _need(k, "k", (N, H, dk), q.dtype, dev)
    _need(v, "v", (N, H, dv), q.dtype, dev)
    _need(state, "state", (N, H, dk, dv), torch.float32, dev)
    beta, log_g, erase_b, write_w = _gates(vid, (N, H), dk, dev, beta, log_g, erase_b, write_w)
    if out is None:
        out = torch.empty(N, H, dv, device=dev, dtype=q.dtype)
    else:
        _need(out, "out", (N, H, dv), q.dtype, dev)
    check(lib().gdr_decode_step(vid | (RAW_INPUTS if raw_inputs else 0), _DTYPES[q.dtype], N, H, dk, dv,
                                _ptr(q), _ptr(k), _ptr(v),
                                _ptr(beta), _ptr(log_g), _ptr(erase_b), _ptr(write_w), _ptr(state),
                                _ptr(out), float(eps), float(scale), _stream(stream, dev)))
    return out


def device_status(stream=None, device=None) -> None:
    """Synchronise and raise GdrError if a kernel reported a timeout or a range fault."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    check(lib().gdr_device_status(_stream(stream, dev)))


def forward_launches(variant, dtype, B, T, H, dk, dv, chunk=0) -> int:
    """Kernel launches one forward call makes (host-only query)."""
    return int(lib().gdr_forward_launches(variant_id(variant), _DTYPES[dtype], B, T, H, dk, dv, chunk))


def forward_kernel_name(variant, dtype, B, T, H, dk, dv, chunk=0) -> str:
    return lib().gdr_forward_kernel_name(variant_id(variant), _DTYPES[dtype], B, T, H, dk, dv, chunk).decode()


def forward_plan(variant, B, T, H, dv, sms) -> dict:
    """How the two-kernel chunked path schedules this problem on a device with
    ``sms`` SMs (host-only): segments per sequence and chunks per segment (the
    segmented carry's maps), the parts per sequence and chunks per part of its
    carry with outputs, and the chunk where the pipelined sweep cuts each
    sequence (0: serial)."""
    g, lc, cs, pa, pc = (ctypes.c_int() for _ in range(5))
    check(lib().gdr_forward_plan(variant_id(variant), B, T, H, dv, sms, ctypes.byref(g), ctypes.byref(lc),
                                 ctypes.byref(cs)))
    check(lib().gdr_forward_segment_parts(variant_id(variant), B, T, H, dv, sms, ctypes.byref(pa), ctypes.byref(pc)))
    return {"segments": g.value, "segment_chunks": lc.value, "parts": pa.value, "part_chunks": pc.value,
            "split_chunk": cs.value}
