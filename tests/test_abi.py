"""Host-side checks of the C ABI (no GPU work).

Every call that passes validation here runs with GDR_FAULT=launch, which makes
the library return GDR_ERR_CUDA before any CUDA call; pointer values are
placeholders that are never dereferenced, and no test launches a kernel.
"""
import ctypes
import os
import re

import pytest
import torch

from gated_delta_rule_forward_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
FAKE = 0x10000            # 16-byte aligned placeholder address, never dereferenced
MISALIGNED = 0x10008


@pytest.fixture(autouse=True)
def _no_launch(monkeypatch):
    monkeypatch.setenv("GDR_FAULT", "launch")
    yield


@pytest.fixture(scope="module")
def L():
    return _lib.lib()


def declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(gdr_[a-z0-9_]+)\s*\(", text))
    return names


def test_library_exports_every_declared_symbol(L):
    syms = declared_symbols()
    assert {"gdr_forward_chunked", "gdr_decode_step", "gdr_status_string"} <= syms
    for s in sorted(syms):
        assert hasattr(L, s), f"{s} declared in include/ but not exported"
    assert set(_lib.EXPORTS) == syms


def test_status_strings(L):
    for code, name in _lib.STATUS.items():
        assert L.gdr_status_string(code).decode() == name
    assert L.gdr_version() >= 100


def args(**over):
    a = dict(q=FAKE, k=FAKE, v=FAKE, beta=FAKE, log_g=FAKE, erase_b=FAKE, write_w=FAKE,
             initial_state=None, final_state=FAKE, o=FAKE)
    a.update(over)
    return _lib.FwdArgs(**a)


def fwd(L, variant=1, dtype=1, B=2, T=8, H=2, dk=128, dv=128, a=None, eps=1e-6, chunk=0):
    a = a if a is not None else args()
    return L.gdr_forward_chunked(variant, dtype, B, T, H, dk, dv, ctypes.byref(a), eps, 1.0, chunk,
                                 None, 0, None)


def test_valid_call_reaches_launch(L):
    # passes validation, stops at the injected launch failure
    assert fwd(L) == 4
    assert "injected" in L.gdr_last_error().decode()


@pytest.mark.parametrize("over,code", [
    (dict(variant=7), 1), (dict(variant=-1), 1), (dict(dtype=5), 1),
    (dict(dk=96), 2), (dict(dv=256), 2), (dict(B=-1), 1), (dict(T=-3), 1),
    (dict(chunk=32), 1), (dict(eps=-1.0), 1),
])
def test_bad_arguments(L, over, code):
    assert fwd(L, **over) == code
    assert L.gdr_last_error().decode()


@pytest.mark.parametrize("field", ["q", "k", "v", "o"])
def test_missing_tensor(L, field):
    assert fwd(L, a=args(**{field: None})) == 1


@pytest.mark.parametrize("field", ["q", "k", "v", "o", "beta", "log_g", "final_state"])
def test_misaligned(L, field):
    assert fwd(L, a=args(**{field: MISALIGNED})) == 3


@pytest.mark.parametrize("variant,field", [
    (0, "beta"), (1, "beta"), (1, "log_g"), (2, "log_g"), (3, "erase_b"), (3, "write_w"),
    (3, "log_g"), (4, "beta"), (4, "log_g")])
def test_required_gates(L, variant, field):
    assert fwd(L, variant=variant, a=args(**{field: None})) == 1


def test_unused_gates_may_be_null(L):
    assert fwd(L, variant=0, a=args(log_g=None, erase_b=None, write_w=None)) == 4
    assert fwd(L, variant=3, a=args(beta=None)) == 4


def test_empty_batch_is_a_noop(L):
    assert fwd(L, B=0) == 0
    assert fwd(L, H=0, a=args(q=None, k=None, v=None, o=None)) == 0


def test_chunk_selection(L):
    # the per-token kernel exists for every shape and dtype
    for v in range(5):
        for dt in (0, 1):
            assert L.gdr_forward_kernel_name(v, dt, 2, 100, 2, 64, 128, 1).decode().startswith("token")
            assert L.gdr_forward_launches(v, dt, 2, 100, 2, 64, 128, 1) == 1
    # fp32 I/O never takes the tensor-core kernel; chunk=64 (a one-kernel path) is not built
    assert fwd(L, dtype=0, chunk=65) == 2
    assert fwd(L, chunk=64) == 2
    assert L.gdr_forward_kernel_name(1, 1, 8, 2048, 8, 128, 128, 64).decode() == "none"
    assert L.gdr_forward_kernel_name(1, 0, 8, 2048, 8, 128, 128, 0).decode() == "token_f32io"
    assert L.gdr_forward_launches(1, 1, 8, 2048, 8, 128, 128, 7) == 0


def test_decode_validation(L):
    i = ctypes.c_void_p
    def dec(variant=1, dtype=1, N=4, H=2, dk=128, dv=128, q=FAKE, state=FAKE, beta=FAKE, log_g=FAKE,
            eb=FAKE, ww=FAKE):
        return L.gdr_decode_step(variant, dtype, N, H, dk, dv, i(q) if q else None, i(FAKE), i(FAKE),
                                 i(beta) if beta else None, i(log_g) if log_g else None,
                                 i(eb) if eb else None, i(ww) if ww else None,
                                 i(state) if state else None, i(FAKE), 1e-6, 1.0, None)
    assert dec() == 4
    assert dec(N=0) == 0
    assert dec(state=None) == 1
    assert dec(state=MISALIGNED) == 3
    assert dec(q=MISALIGNED) == 3
    assert dec(dk=32) == 2
    assert dec(variant=3, eb=None) == 1
    assert dec(variant=2, log_g=None) == 1
    assert dec(variant=0, log_g=None) == 4


def test_workspace_sizes(L):
    # two-kernel path: one record per (b, h, 64-token chunk): -W, Qg, Kt (16 KB each),
    # P (8 KB), U'^T (8 KB per 64 value columns) and Gamma_C (16 bytes)
    assert L.gdr_forward_workspace_size(1, 1, 8, 2048, 8, 128, 128, 0) == 8 * 8 * 32 * (57344 + 16384 + 16)
    assert L.gdr_forward_workspace_size(1, 1, 2, 65, 3, 128, 64, 65) == 2 * 3 * 2 * (57344 + 8192 + 16)
    assert L.gdr_forward_workspace_size(1, 1, 8, 2048, 8, 128, 128, 64) == 0   # not built
    assert L.gdr_forward_workspace_size(1, 0, 8, 2048, 8, 128, 128, 0) == 0    # fp32: per-token
    # KDA: the same record with Gamma_C a vector of 128 floats
    assert L.gdr_forward_workspace_size(2, 1, 8, 2048, 8, 128, 128, 0) == 8 * 8 * 32 * (57344 + 16384 + 512)
    # GDN-2: the channel-decay record, then (P^d V)^T and (Dt^T V)^T (8 + 16 KB per 64 values)
    assert L.gdr_forward_workspace_size(3, 1, 8, 2048, 8, 128, 128, 0) == 8 * 8 * 32 * (57344 + 16384 + 512 + 49152)
    assert L.gdr_forward_kernel_name(3, 1, 8, 2048, 8, 128, 128, 0).decode() == "chunk64_split"
    assert L.gdr_forward_kernel_name(1, 1, 8, 2048, 8, 128, 128, 0).decode() == "chunk64_split"
    # preparation + carry; with a device whose idle SMs pay for it, the pipelined
    # sweep (two of each) -- without one, as here, the serial pair
    assert L.gdr_forward_launches(1, 1, 8, 2048, 8, 128, 128, 0) == (4 if torch.cuda.is_available() else 2)
    assert L.gdr_forward_kernel_name(2, 1, 8, 2048, 8, 128, 128, 0).decode() == "chunk64_split"


def test_split_needs_workspace(L):
    assert fwd(L, chunk=65) == 1                      # no workspace passed
    a = args()
    assert L.gdr_forward_chunked(1, 1, 2, 8, 2, 128, 128, ctypes.byref(a), 1e-6, 1.0, 65,
                                 ctypes.c_void_p(FAKE), 1 << 20, None) == 4   # reaches the launch
    assert L.gdr_forward_chunked(1, 1, 2, 8, 2, 128, 128, ctypes.byref(a), 1e-6, 1.0, 65,
                                 ctypes.c_void_p(MISALIGNED), 1 << 20, None) == 3


def _plan(L, variant, B, T, H, dv=128, sms=148):
    g, lc, cs = ctypes.c_int(-1), ctypes.c_int(-1), ctypes.c_int(-1)
    st = L.gdr_forward_plan(variant, B, T, H, dv, sms, ctypes.byref(g), ctypes.byref(lc), ctypes.byref(cs))
    assert st == 0, L.gdr_last_error()
    return g.value, lc.value, cs.value


def test_two_kernel_schedule_on_a_148_sm_device(L):
    """The schedules the benchmark workloads get on B200 (148 SMs), and the edge cases."""
    assert _plan(L, 1, 8, 2048, 8) == (1, 32, 20)      # 350M GDN: pipelined, cut at chunk 20 of 32
    assert _plan(L, 0, 8, 2048, 8) == (1, 32, 20)      # DeltaNet: the same kernels
    assert _plan(L, 4, 4, 4096, 16) == (1, 64, 39)     # 1.3B KLA
    assert _plan(L, 2, 4, 4096, 16) == (1, 64, 53)     # 1.3B KDA
    assert _plan(L, 3, 4, 4096, 16) == (1, 64, 51)     # 1.3B GDN-2
    assert _plan(L, 1, 1, 65536, 16) == (6, 183, 0)    # 64k: six segments of 183 chunks (phase 1)
    assert _plan(L, 1, 1, 4100, 2) == (13, 5, 0)       # the segmented GPU test: 13 segments of 5
    assert _plan(L, 1, 2, 4480, 3) == (12, 6, 0)       # and its other shape: 12 of 6
    for v in range(5):                                  # the pipelined GPU tests (24 chunks)
        assert _plan(L, v, 4, 1531, 16)[2] > 0
        assert _plan(L, v, 4, 1531, 16, dv=64)[2] > 0
    assert _plan(L, 1, 2, 130, 3) == (1, 3, 0)         # three chunks: serial
    assert _plan(L, 1, 16, 2048, 16) == (1, 32, 0)     # B*H = 256 > SMs: serial
    assert _plan(L, 1, 1, 65536, 16, dv=64)[0] == 1    # segmenting needs dv = 128
    assert _plan(L, 1, 0, 5000, 8) == (1, 79, 0)       # no sequences: nothing to divide by
    assert _plan(L, 1, 4, 4096, 16, sms=0) == (1, 64, 0)


def _parts(L, variant, B, T, H, dv=128, sms=148):
    pa, pc = ctypes.c_int(-1), ctypes.c_int(-1)
    st = L.gdr_forward_segment_parts(variant, B, T, H, dv, sms, ctypes.byref(pa), ctypes.byref(pc))
    assert st == 0, L.gdr_last_error()
    return pa.value, pc.value


def test_segment_parts_on_a_148_sm_device(L):
    """The segmented carry's second phase: one CTA per part, so it may cut finer
    than the maps' segments (B200, 148 SMs)."""
    assert _parts(L, 1, 1, 65536, 16) == (9, 114)     # 64k: nine parts, 144 CTAs
    assert _parts(L, 1, 1, 7041, 17) == (7, 16)       # the finer-parts GPU test (5 segments of 24)
    assert _plan(L, 1, 1, 7041, 17) == (5, 24, 0)
    assert _parts(L, 1, 1, 5000, 12) == (7, 12)       # a short sequence: the chain's products cost more
    assert _parts(L, 1, 1, 4100, 2) == (13, 5)        # the segmented GPU test: the segments themselves
    assert _parts(L, 1, 8, 2048, 8) == (1, 32)        # not segmented: one part
    assert _parts(L, 1, 1, 65536, 16, dv=64) == (1, 1024)
    assert _parts(L, 1, 1, 1 << 20, 1) == (61, 269)   # at most 64 parts
    g = ctypes.c_int()
    assert L.gdr_forward_segment_parts(9, 1, 64, 1, 128, 148, ctypes.byref(g), ctypes.byref(g)) == 1
    assert L.gdr_forward_segment_parts(1, 1, 64, 1, 128, -1, ctypes.byref(g), ctypes.byref(g)) == 1
    assert L.gdr_forward_segment_parts(1, 1, 64, 1, 128, 148, ctypes.byref(g), None) == 1


def test_segment_plan_invariants(L):
    """Every segmented plan over a grid of shapes and device sizes: the segments
    and the parts each cover the sequence with a ragged last one; phase 1
    (2G - 3 CTAs per sequence) and phase 2 (one per part) fit the SMs; and no part
    starts strictly inside the last segment, which phase 1 does not run (its
    start states come from the maps after the chunks before them)."""
    n = 0
    for sms in (132, 148, 160):
        for B, H in ((1, 1), (1, 2), (1, 3), (2, 3), (1, 5), (1, 8), (1, 12), (1, 16), (2, 8), (1, 24), (1, 40)):
            for T in (4033, 4100, 5000, 8150, 12345, 40000, 65536, 100000, 1 << 20):
                NC = (T + 63) // 64
                G, Lc, _ = _plan(L, 1, B, T, H, sms=sms)
                P, Lp = _parts(L, 1, B, T, H, sms=sms)
                if G == 1:
                    assert (P, Lp) == (1, Lc)
                    continue
                n += 1
                bh = B * H
                assert G >= 3 and (G - 1) * Lc < NC <= G * Lc
                assert (P - 1) * Lp < NC <= P * Lp
                assert (2 * G - 3) * bh <= sms and P * bh <= sms and P <= max(G, 64)
                assert (P - 1) * Lp <= (G - 1) * Lc
                assert P >= G and (P == G) == (Lp == Lc)
    assert n > 100


def test_two_kernel_schedule_rejects_bad_arguments(L):
    g = ctypes.c_int()
    assert L.gdr_forward_plan(9, 1, 64, 1, 128, 148, ctypes.byref(g), ctypes.byref(g), ctypes.byref(g)) == 1
    assert L.gdr_forward_plan(1, 1, 64, 1, 96, 148, ctypes.byref(g), ctypes.byref(g), ctypes.byref(g)) == 1
    assert L.gdr_forward_plan(1, -1, 64, 1, 128, 148, ctypes.byref(g), ctypes.byref(g), ctypes.byref(g)) == 1
    assert L.gdr_forward_plan(1, 1, 64, 1, 128, 148, None, ctypes.byref(g), ctypes.byref(g)) == 1


def test_empty_batch_workspace_query(L):
    """B * H = 0 with a long T is a valid no-op call; its workspace query must not divide by B * H."""
    assert L.gdr_forward_workspace_size(1, 1, 0, 5000, 8, 128, 128, 0) == 0


def test_forward_plan_binding():
    import gated_delta_rule_forward_b200 as gdr
    assert gdr.forward_plan("gdn", 8, 2048, 8, 128, 148) == {"segments": 1, "segment_chunks": 32, "parts": 1,
                                                             "part_chunks": 32, "split_chunk": 20}
    assert gdr.forward_plan("kla", 1, 65536, 16, 128, 148) == {"segments": 6, "segment_chunks": 183, "parts": 9,
                                                               "part_chunks": 114, "split_chunk": 0}
    with pytest.raises(gdr.GdrError):
        gdr.forward_plan("gdn", 8, 2048, 8, 96, 148)


def test_raw_input_flag_is_accepted_everywhere(L):
    RAW = 0x100                                      # GDR_RAW_INPUTS
    for v in range(5):
        assert fwd(L, variant=v | RAW, a=args()) == 4                 # validated, reaches the launch
        assert L.gdr_forward_kernel_name(v | RAW, 1, 8, 2048, 8, 128, 128, 0).decode() == \
            L.gdr_forward_kernel_name(v, 1, 8, 2048, 8, 128, 128, 0).decode()
        assert L.gdr_forward_workspace_size(v | RAW, 1, 8, 2048, 8, 128, 128, 0) == \
            L.gdr_forward_workspace_size(v, 1, 8, 2048, 8, 128, 128, 0)
    assert fwd(L, variant=5 | RAW) == 1                               # the flag does not hide a bad variant
    i = ctypes.c_void_p
    assert L.gdr_decode_step(1 | RAW, 1, 4, 2, 128, 128, i(FAKE), i(FAKE), i(FAKE), i(FAKE), i(FAKE), None,
                             None, i(FAKE), i(FAKE), 1e-6, 1.0, None) == 4


def bwd_call(L, variant=1, dtype=1, B=2, T=130, H=3, dk=128, dv=128, ws=None, d_o=FAKE, grads=None, a=None,
             eps=1e-6):
    a = a or args(initial_state=FAKE)
    g = grads or _lib.BwdGrads(dq=FAKE, dk=FAKE, dv=FAKE, dbeta=FAKE, dlog_g=FAKE, d_initial_state=FAKE)
    need = L.gdr_backward_workspace_size(variant, dtype, B, T, H, dk, dv)
    return L.gdr_backward(variant, dtype, B, T, H, dk, dv, ctypes.byref(a), d_o, FAKE, ctypes.byref(g),
                          eps, 1.0, FAKE, need if ws is None else ws, None)


def test_backward_validation(L):
    assert bwd_call(L) == 4                                  # valid: reaches the (injected) launch failure
    for v in (0, 1, 2, 4):
        assert bwd_call(L, variant=v) == 4
    assert bwd_call(L, variant=3) == 1                                       # GDN-2 needs its gate gradients
    g2 = _lib.BwdGrads(dq=FAKE, dk=FAKE, dv=FAKE, dbeta=None, dlog_g=FAKE, d_initial_state=FAKE,
                       d_erase_b=FAKE, d_write_w=FAKE)
    a2 = args(beta=None, erase_b=FAKE, write_w=FAKE, initial_state=FAKE)
    assert bwd_call(L, variant=3, grads=g2, a=a2) == 4                       # ... and takes no dbeta
    assert bwd_call(L, variant=3, grads=g2, a=args(beta=None, erase_b=None, initial_state=FAKE)) == 1   # needs the gates
    assert bwd_call(L, variant=1 | 0x100) == 2                               # raw inputs: unsupported
    assert bwd_call(L, dtype=0) == 2 and bwd_call(L, dk=64) == 2             # fp32 I/O, dk = 64
    assert bwd_call(L, dv=96) == 2
    assert bwd_call(L, variant=9) == 1 and bwd_call(L, T=-1) == 1
    assert bwd_call(L, ws=16) == 1                                           # workspace too small
    assert bwd_call(L, d_o=None) == 1
    assert bwd_call(L, d_o=MISALIGNED) == 3
    g = _lib.BwdGrads(dq=FAKE, dk=FAKE, dv=FAKE, dbeta=FAKE, dlog_g=None, d_initial_state=None)
    assert bwd_call(L, grads=g) == 1                                         # GDN needs dlog_g
    assert bwd_call(L, variant=0, grads=g) == 4                              # DeltaNet does not
    assert bwd_call(L, a=args(log_g=None, initial_state=FAKE)) == 1          # GDN needs log_g
    assert bwd_call(L, eps=-1.0) == 1
    assert bwd_call(L, B=0) == 0                                             # empty batch: nothing to do


def test_backward_workspace_sizes(L):
    # forward records + reverse records + two fp32 states per chunk + two states
    B, T, H, NC, bh = 8, 2048, 8, 32, 64
    rec, rev = 57344 + 8192 * 2 + 16, 57344 + 8192 * 2 + 512 + 24576 * 2
    up = lambda x: (x + 255) // 256 * 256
    # chunk start states in fp16 (fp32 for KDA), end-state gradients in fp32
    want = up(bh * NC * rec) + up(bh * NC * rev) + up(bh * NC * 128 * 128 * 2) + up(bh * NC * 128 * 128 * 4) + \
        2 * up(bh * 128 * 128 * 4) + 256
    assert L.gdr_backward_workspace_size(1, 1, B, T, H, 128, 128) == want
    rec_kda = rec + 512 - 16                                                 # Gamma_C as 128 floats
    want_kda = up(bh * NC * rec_kda) + up(bh * NC * rev) + 2 * up(bh * NC * 128 * 128 * 4) + 2 * up(bh * 128 * 128 * 4) + 256
    assert L.gdr_backward_workspace_size(2, 1, B, T, H, 128, 128) == want_kda
    assert L.gdr_backward_workspace_size(3, 1, B, T, H, 128, 128) == \
        up(bh * NC * rev) + up(bh * NC * rev) + 2 * up(bh * NC * 128 * 128 * 4) + 2 * up(bh * 128 * 128 * 4) + 256
    assert L.gdr_backward_workspace_size(1, 0, B, T, H, 128, 128) == 0       # fp32 I/O
    assert L.gdr_backward_workspace_size(1, 1, B, 0, H, 128, 128) == 0
