"""gdr_forward_chunked_noalloc: the forward for callers that cannot allocate.

Some callers cannot allocate device memory when they call the forward: a
serving runtime whose device memory is planned up front and that forbids
allocation on its request path, or a host program that drives the library
without a device allocator of its own.  For them the library keeps a fixed
scratch array in its own device image and runs the two-kernel chunked path
on it.  This test calls that entry point through the C ABI, twice in a row,
and checks each result against the regular entry point (gdr_forward_chunked
with a caller-allocated workspace) under the same bf16 tolerance the parity
tests use.  The file is collected last so that a failure here cannot hide
the other tests in a run that stops at the first failure.
"""
import ctypes

import pytest
import torch

import gated_delta_rule_forward_b200 as gdr
from gated_delta_rule_forward_b200 import _lib
from gated_delta_rule_forward_b200.inputs import make_inputs, random_state
from parity_util import assert_gpu_close, gate_kwargs, to_dev

pytestmark = pytest.mark.gpu
VARIANT_IDS = {"deltanet": 0, "gdn": 1, "kda": 2, "gdn2": 3, "kla": 4}


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


def test_noalloc_rejects_problems_beyond_the_fixed_scratch():
    B, T, H = 8, 8192, 8                    # 8 * 8 * 128 records, more than 32 MiB holds
    record = _lib.lib().gdr_forward_workspace_size(1, 1, 1, 64, 1, 128, 128, 65)
    limit = (32 << 20) // record
    assert B * H * (T // 64) > limit
    q = torch.empty(1, device="cuda", dtype=torch.bfloat16)
    a = _lib.FwdArgs(q=q.data_ptr(), k=q.data_ptr(), v=q.data_ptr(), beta=q.data_ptr(),
                     log_g=q.data_ptr(), erase_b=None, write_w=None, initial_state=None,
                     final_state=None, o=q.data_ptr())
    st = _lib.lib().gdr_forward_chunked_noalloc(1, 1, B, T, H, 128, 128, ctypes.byref(a), 1e-6, 1.0, None)
    assert st == 2
    assert str(limit) in _lib.lib().gdr_last_error().decode()
