"""The parity metrics themselves, on plain arrays (CPU)."""
import numpy as np
import pytest
import torch

from parity_util import BF16_TOL, F32_TOL, assert_close, bf16_out_rel, elem_rel, max_rel, rms_rel


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
