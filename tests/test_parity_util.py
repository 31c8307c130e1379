"""The parity metrics themselves, on plain arrays (CPU)."""
import numpy as np
import pytest
import torch

from parity_util import (BF16_TOL, BULK_RMS, BULK_TOL, F32_TOL, assert_close, bf16_out_rel, bulk_rel, elem_rel,
                          max_rel, rms_rel)


def test_metrics_on_known_arrays():
    ref = np.array([1.0, -2.0, 0.0, 4.0])
    gpu = ref + np.array([1e-5, 0.0, 2e-6, -4e-5])
    assert max_rel(gpu, ref) == pytest.approx(1e-5)
    assert rms_rel(gpu, ref) == pytest.approx(4e-5 / np.sqrt(21 / 4))
    # element-wise: the zero entry is measured against the floor 1e-6 * 4
    assert elem_rel(gpu, ref) == pytest.approx(2e-6 / 4e-6)


def test_bf16_output_metric_discounts_the_output_rounding():
    ref = np.linspace(-3, 3, 101)
    rounded = torch.from_numpy(ref).to(torch.bfloat16)
    assert bf16_out_rel(rounded, ref) == 0.0          # the exact result, rounded, passes
    assert assert_close(rounded, ref, torch.bfloat16) == 0.0


def test_fp32_bar_fails_with_both_ratios_in_the_message():
    ref = np.array([1.0, 2.0, 0.0])
    gpu = torch.tensor(ref + np.array([0.0, 1e-3, 0.0]), dtype=torch.float32)
    with pytest.raises(AssertionError, match="element-wise"):
        assert_close(gpu, ref, torch.float32, "o")
    assert F32_TOL == 1e-4 and BF16_TOL == 2e-2


def test_bulk_metric_catches_an_error_the_rounding_allowance_forgives():
    # a heavy tail (one element at 50 RMS) and an arithmetic error of 0.1 RMS on a bulk element
    rng = np.random.default_rng(0)
    ref = rng.standard_normal(4096)
    ref[0] = 50.0 * np.sqrt(np.mean(ref * ref))
    rms = np.sqrt(np.mean(ref * ref))
    bad = ref.copy()
    bad[1] = ref[1] + 0.1 * rms                        # |ref[1]| is well inside 4 RMS
    bad_t = torch.from_numpy(bad).to(torch.bfloat16)
    assert bulk_rel(bad_t, ref) > BULK_TOL
    with pytest.raises(AssertionError):
        assert_close(bad_t, ref, torch.bfloat16, "o")
    # the exact result rounded to bf16 passes both metrics
    ok = torch.from_numpy(ref).to(torch.bfloat16)
    assert bulk_rel(ok, ref) <= BULK_RMS * 2 ** -8 + 1e-12
