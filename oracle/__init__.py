"""Gated delta-rule oracle: plain fp64 CPU recurrence (C, OpenMP) behind ctypes.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  It shares no code
with the CUDA library (``gated_delta_rule_forward_b200``) and imports nothing
from it; both sides receive the same arrays from the seeded input generator.

The arithmetic lives in ``gdr_oracle.c``; its header states what is computed
and which passages of the pages each step follows ("Kaczmarz Linear
Attention", KLA update rule; "Gated DeltaNet-2: Decoupling Erase and Write in
Linear Attention", technical core).  Everything here is marshalling: up-cast
to contiguous float64, call, return float64 arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdr_oracle.c")
_BUILD = os.path.join(_HERE, "_build")

VARIANTS = {"deltanet": 0, "gdn": 1, "kda": 2, "gdn2": 3, "kla": 4}
_SCALAR_DECAY = ("gdn", "kla")
_CHANNEL_DECAY = ("kda", "gdn2")

_lock = threading.Lock()
_libs: dict[int, ctypes.CDLL] = {}


def lib_path(mutant: int = 0) -> str:
    name = "liboracle.so" if mutant == 0 else f"liboracle_m{mutant}.so"
    return os.path.join(_BUILD, name)


def build(mutant: int = 0, force: bool = False) -> str:
    """Compile the oracle (gcc -O2 -fopenmp).  ``mutant`` > 0 plants a mistake."""
    out = lib_path(mutant)
    if (not force and os.path.exists(out)
            and os.path.getmtime(out) >= os.path.getmtime(_SRC)):
        return out
    os.makedirs(_BUILD, exist_ok=True)
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c99", "-o", tmp, _SRC, "-lm"]
    if mutant:
        cmd.insert(1, f"-DORACLE_MUTANT={mutant}")
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def _load(mutant: int = 0) -> ctypes.CDLL:
    with _lock:
        if mutant not in _libs:
            lib = ctypes.CDLL(build(mutant))
            dp = ctypes.POINTER(ctypes.c_double)
            i = ctypes.c_int
            d = ctypes.c_double
            lib.oracle_forward.argtypes = [i, i, i, i, i, i, dp, dp, dp, dp, dp, dp, dp,
                                           dp, dp, dp, d, d, i]
            lib.oracle_forward.restype = i
            lib.oracle_decode_step.argtypes = [i, i, i, i, i, dp, dp, dp, dp, dp, dp, dp,
                                               dp, dp, d, d, i]
            lib.oracle_decode_step.restype = i
            lib.oracle_backward.argtypes = [i, i, i, i, i, i] + [dp] * 18 + [d, d, i]
            lib.oracle_backward.restype = i
            lib.oracle_max_threads.argtypes = []
            lib.oracle_max_threads.restype = i
            _libs[mutant] = lib
        return _libs[mutant]


def _f64(x):
    """Exact up-cast of a numpy array or torch tensor to contiguous float64."""
    if x is None:
        return None
    if hasattr(x, "detach"):          # torch tensor: bf16/fp32 -> fp64 is exact
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def _check_gates(variant, beta, log_g, erase_b, write_w, lead, dk):
    if variant not in VARIANTS:
        raise ValueError(f"unknown variant {variant!r}")
    if variant in _SCALAR_DECAY:
        if log_g is None or log_g.shape != lead:
            raise ValueError(f"{variant}: log_g must have shape {lead}")
    if variant in _CHANNEL_DECAY:
        if log_g is None or log_g.shape != lead + (dk,):
            raise ValueError(f"{variant}: log_g must have shape {lead + (dk,)}")
    if variant == "gdn2":
        for name, g in (("erase_b", erase_b), ("write_w", write_w)):
            if g is None or g.shape != lead + (dk,):
                raise ValueError(f"gdn2: {name} must have shape {lead + (dk,)}")
    elif beta is None or beta.shape != lead:
        raise ValueError(f"{variant}: beta must have shape {lead}")


def forward(variant, q, k, v, beta=None, log_g=None, erase_b=None, write_w=None,
            initial_state=None, eps=1e-6, scale=1.0, threads=0, mutant=0):
    """Token-by-token fp64 forward.  Returns (o [B,T,H,dv], final_state [B,H,dk,dv])."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    beta, log_g, erase_b, write_w = _f64(beta), _f64(log_g), _f64(erase_b), _f64(write_w)
    initial_state = _f64(initial_state)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if k.shape != (B, T, H, dk) or v.shape != (B, T, H, dv):
        raise ValueError("q, k, v must be [B,T,H,dk], [B,T,H,dk], [B,T,H,dv]")
    _check_gates(variant, beta, log_g, erase_b, write_w, (B, T, H), dk)
    if variant == "deltanet":
        log_g = None
    if variant == "gdn2":
        beta = None
    if initial_state is not None and initial_state.shape != (B, H, dk, dv):
        raise ValueError("initial_state must be [B,H,dk,dv]")
    o = np.zeros((B, T, H, dv), np.float64)
    S = np.zeros((B, H, dk, dv), np.float64)
    rc = _load(mutant).oracle_forward(
        VARIANTS[variant], B, T, H, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(beta),
        _ptr(log_g), _ptr(erase_b), _ptr(write_w), _ptr(initial_state), _ptr(o), _ptr(S),
        float(eps), float(scale), int(threads))
    if rc != 0:
        raise ValueError("oracle_forward rejected its arguments")
    return o, S


def decode_step(variant, q, k, v, state, beta=None, log_g=None, erase_b=None,
                write_w=None, eps=1e-6, scale=1.0, threads=0, mutant=0):
    """One token for N sequences.  Returns (o [N,H,dv], new state [N,H,dk,dv])."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    beta, log_g, erase_b, write_w = _f64(beta), _f64(log_g), _f64(erase_b), _f64(write_w)
    S = _f64(state).copy()
    N, H, dk = q.shape
    dv = v.shape[-1]
    if S.shape != (N, H, dk, dv):
        raise ValueError("state must be [N,H,dk,dv]")
    _check_gates(variant, beta, log_g, erase_b, write_w, (N, H), dk)
    if variant == "deltanet":
        log_g = None
    if variant == "gdn2":
        beta = None
    o = np.zeros((N, H, dv), np.float64)
    rc = _load(mutant).oracle_decode_step(
        VARIANTS[variant], N, H, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(log_g),
        _ptr(erase_b), _ptr(write_w), _ptr(S), _ptr(o), float(eps), float(scale), int(threads))
    if rc != 0:
        raise ValueError("oracle_decode_step rejected its arguments")
    return o, S


def backward(variant, q, k, v, d_o, beta=None, log_g=None, erase_b=None, write_w=None,
             initial_state=None, d_final=None, eps=1e-6, scale=1.0, threads=0, mutant=0):
    """Gradients of <d_o, o> + <d_final, S_T> with respect to every input of
    ``forward`` (reverse mode through the same fp64 recurrence).  Returns a dict
    with keys q, k, v, beta, log_g, erase_b, write_w, initial_state (None for
    inputs the variant does not take; ``beta`` is d/d eta for KLA)."""
    q, k, v, d_o = _f64(q), _f64(k), _f64(v), _f64(d_o)
    beta, log_g, erase_b, write_w = _f64(beta), _f64(log_g), _f64(erase_b), _f64(write_w)
    initial_state, d_final = _f64(initial_state), _f64(d_final)
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    if k.shape != (B, T, H, dk) or v.shape != (B, T, H, dv) or d_o.shape != (B, T, H, dv):
        raise ValueError("q, k, v, d_o must be [B,T,H,dk], [B,T,H,dk], [B,T,H,dv], [B,T,H,dv]")
    _check_gates(variant, beta, log_g, erase_b, write_w, (B, T, H), dk)
    for name, st in (("initial_state", initial_state), ("d_final", d_final)):
        if st is not None and st.shape != (B, H, dk, dv):
            raise ValueError(f"{name} must be [B,H,dk,dv]")
    if variant == "deltanet":
        log_g = None
    if variant == "gdn2":
        beta = None
    g = {"q": np.zeros_like(q), "k": np.zeros_like(k), "v": np.zeros_like(v),
         "beta": None if beta is None else np.zeros_like(beta),
         "log_g": None if log_g is None else np.zeros_like(log_g),
         "erase_b": None if variant != "gdn2" else np.zeros_like(erase_b),
         "write_w": None if variant != "gdn2" else np.zeros_like(write_w),
         "initial_state": np.zeros((B, H, dk, dv), np.float64)}
    rc = _load(mutant).oracle_backward(
        VARIANTS[variant], B, T, H, dk, dv, _ptr(q), _ptr(k), _ptr(v), _ptr(beta), _ptr(log_g),
        _ptr(erase_b), _ptr(write_w), _ptr(initial_state), _ptr(d_o), _ptr(d_final),
        _ptr(g["q"]), _ptr(g["k"]), _ptr(g["v"]), _ptr(g["beta"]), _ptr(g["log_g"]),
        _ptr(g["erase_b"]), _ptr(g["write_w"]), _ptr(g["initial_state"]),
        float(eps), float(scale), int(threads))
    if rc != 0:
        raise ValueError("oracle_backward rejected its arguments")
    return g
