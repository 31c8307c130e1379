"""gdr_forward_chunked_noalloc: the forward for callers that cannot allocate.

Some callers cannot allocate device memory when they call the forward: a
serving runtime whose device memory is planned up front and that forbids
allocation on its request path, or a host program that drives the library
without a device allocator of its own.  For them the library keeps a fixed
scratch array in its own device image and runs the two-kernel chunked path
on it.  These tests call that entry point through the C ABI, twice in a row
(the array keeps the previous call's contents), and check each result:

  * against the regular entry point (gdr_forward_chunked with a
    caller-allocated workspace), on a short ragged shape, all five variants;
  * against the fp64 oracle, on the three schedules the two-kernel path has
    for shapes that fit the array: the segmented carry (few long sequences),
    the pipelined sweep (a mid-size number of sequences), and the
    unsegmented sweep that replaces the segmented one when its maps do not
    fit beside the records.

The file is collected last so that a failure here cannot hide the other
tests in a run that stops at the first failure.
"""
import ctypes

import pytest
import torch

import gated_delta_rule_forward_b200 as gdr
import oracle
from gated_delta_rule_forward_b200 import _lib
from gated_delta_rule_forward_b200.inputs import make_inputs, random_state
from parity_util import assert_close, assert_gpu_close, gate_kwargs, to_dev

pytestmark = pytest.mark.gpu
VARIANT_IDS = {"deltanet": 0, "gdn": 1, "kda": 2, "gdn2": 3, "kla": 4}
FIXED_SCRATCH = 32 << 20


def call_noalloc(variant, d, S0, B, T, H, dv):
    o = torch.empty(B, T, H, dv, device="cuda", dtype=torch.bfloat16)
    S = torch.empty(B, H, 128, dv, device="cuda", dtype=torch.float32)
    ptr = lambda name: None if d.get(name) is None else d[name].data_ptr()
    a = _lib.FwdArgs(q=d["q"].data_ptr(), k=d["k"].data_ptr(), v=d["v"].data_ptr(),
                     beta=ptr("beta"), log_g=ptr("log_g"), erase_b=ptr("erase_b"),
                     write_w=ptr("write_w"), initial_state=S0.data_ptr(),
                     final_state=S.data_ptr(), o=o.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = _lib.lib().gdr_forward_chunked_noalloc(VARIANT_IDS[variant], 1, B, T, H, 128, dv, ctypes.byref(a),
                                                1e-6, 1.0, stream)
    _lib.check(st)
    return o, S


def plan(variant, B, T, H, dv):
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    a, b, c = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    _lib.check(_lib.lib().gdr_forward_plan(VARIANT_IDS[variant], B, T, H, dv, sms, ctypes.byref(a),
                                           ctypes.byref(b), ctypes.byref(c)))
    return sms, a.value, c.value


@pytest.mark.parametrize("variant,dv", [("gdn", 128), ("kla", 64), ("deltanet", 128), ("kda", 128),
                                        ("gdn2", 64)])
def test_noalloc_matches_workspace_path_twice(variant, dv):
    B, T, H = 2, 333, 3                     # ragged tail; 2 * 3 * 6 = 36 records
    d = to_dev(make_inputs(variant, B, T, H, 128, dv, dtype=torch.bfloat16, seed=41))
    S0 = random_state(B, H, 128, dv, 42).cuda()
    o_ref, S_ref = gdr.forward(d["q"], d["k"], d["v"], variant=variant, **gate_kwargs(d),
                               initial_state=S0, chunk=65)
    for _ in range(2):                      # the shared scratch keeps the last call's contents
        o, S = call_noalloc(variant, d, S0, B, T, H, dv)
        gdr.device_status()
        assert_gpu_close(o, o_ref, "o")
        assert_gpu_close(S, S_ref, "S")


# (variant, B, T, H): the schedule each shape takes on a 148-SM B200
SCHEDULES = {
    "segmented": ("gdn", 1, 4096, 2),       # 128 records + maps of 16 segments, ~9 MB
    "pipelined": ("kda", 2, 1000, 8),       # 256 records, cut at chunk 10 of 16 (ragged tail)
    "unsegmented": ("gdn", 1, 4033, 7),     # 448 records fill the array; the maps would not fit
}


@pytest.mark.parametrize("schedule", list(SCHEDULES))
def test_noalloc_schedules_against_oracle_twice(schedule):
    variant, B, T, H = SCHEDULES[schedule]
    dv = 128
    record = _lib.lib().gdr_forward_workspace_size(VARIANT_IDS[variant], 1, 1, 64, 1, 128, dv, 65)
    records = B * H * ((T + 63) // 64)
    assert records * record <= FIXED_SCRATCH
    full = _lib.lib().gdr_forward_workspace_size(VARIANT_IDS[variant], 1, B, T, H, 128, dv, 65)
    sms, segments, split = plan(variant, B, T, H, dv)
    if sms == 148:
        if schedule == "segmented":
            assert segments > 1 and full <= FIXED_SCRATCH, (segments, full)
        elif schedule == "pipelined":
            assert segments == 1 and split > 0, (segments, split)
        else:
            assert segments > 1 and full > FIXED_SCRATCH, (segments, full)
    d = make_inputs(variant, B, T, H, 128, dv, dtype=torch.bfloat16, seed=43)
    S0 = random_state(B, H, 128, dv, 44)
    o_ref, S_ref = oracle.forward(variant, **d, initial_state=S0)
    dd, S0d = to_dev(d), S0.cuda()
    for call in range(2):
        o, S = call_noalloc(variant, dd, S0d, B, T, H, dv)
        gdr.device_status()
        assert_close(o, o_ref, torch.bfloat16, f"{schedule} call {call} o")
        assert_close(S, S_ref, torch.bfloat16, f"{schedule} call {call} S")


def test_noalloc_rejects_problems_beyond_the_fixed_scratch():
    B, T, H = 8, 8192, 8                    # 8 * 8 * 128 records, more than 32 MiB holds
    record = _lib.lib().gdr_forward_workspace_size(1, 1, 1, 64, 1, 128, 128, 65)
    limit = FIXED_SCRATCH // record
    assert B * H * (T // 64) > limit
    q = torch.empty(1, device="cuda", dtype=torch.bfloat16)
    a = _lib.FwdArgs(q=q.data_ptr(), k=q.data_ptr(), v=q.data_ptr(), beta=q.data_ptr(),
                     log_g=q.data_ptr(), erase_b=None, write_w=None, initial_state=None,
                     final_state=None, o=q.data_ptr())
    st = _lib.lib().gdr_forward_chunked_noalloc(1, 1, B, T, H, 128, 128, ctypes.byref(a), 1e-6, 1.0, None)
    assert st == 2
    msg = _lib.lib().gdr_last_error().decode()
    assert f"at most {limit} " in msg and str(FIXED_SCRATCH) in msg, msg
