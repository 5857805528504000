"""The parity gate of the GPU tests, checked on the CPU with hand-made
outputs on both sides of its rounding allowance."""
import numpy as np
import pytest
import torch

from tests import hta_testlib as H


def _gate(out_vals, ref_vals, dtype=torch.bfloat16):
    D = len(out_vals)
    out = torch.tensor([out_vals], dtype=torch.float64).to(dtype)
    ref = np.array([ref_vals], dtype=np.float64)
    lse = torch.zeros(1, dtype=torch.float32)
    return H.assert_parity(out, lse, ref, np.zeros(1), "gate")


def test_exact_bf16_rounding_passes_below_4():
    # the nearest bf16 of 3.0039 is 3.0 (spacing 2^-6 at [2, 4)): error 0.0039
    _gate([3.0] + [0.0] * 127, [3.0039] + [0.0] * 127)


def test_one_bf16_step_fails_below_4():
    # 3.015625 is the next bf16 above 3: 0.0156 > 1e-2, no allowance below 4
    with pytest.raises(AssertionError):
        _gate([3.015625] + [0.0] * 127, [3.0] + [0.0] * 127)


def test_error_between_1e2_and_allowance_fails_below_4_passes_above():
    # 0.014 off: over the strict bound at |x| = 3, inside 1e-2 + 2^-6 at |x| = 5
    with pytest.raises(AssertionError):
        _gate([3.0] + [0.0] * 127, [3.014] + [0.0] * 127)
    _gate([5.0] + [0.0] * 127, [5.014] + [0.0] * 127)


def test_one_bf16_step_fails_above_4():
    # 5.03125 is the next bf16 above 5: 0.031 > 1e-2 + 2^-6
    with pytest.raises(AssertionError):
        _gate([5.03125] + [0.0] * 127, [5.0] + [0.0] * 127)


def test_fp32_outputs_get_no_allowance():
    with pytest.raises(AssertionError):
        _gate([5.0] + [0.0] * 127, [5.014] + [0.0] * 127, dtype=torch.float32)
