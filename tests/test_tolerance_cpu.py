"""The parity helpers themselves (CPU): bf16 rounding of the storage floor and
the scale rule of the gradient check."""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

from tests import tolerance


def test_bf16_rounding_matches_torch_on_float32_values():
    # float32 inputs round once either way, so the direct rounding must agree
    # with torch's float32 -> bfloat16 conversion (round to nearest, ties to even)
    x32 = (torch.randn(200000, generator=torch.Generator().manual_seed(1)) * 7).float()
    ours = tolerance.bf16_rne(x32.double().numpy())
    ref = x32.to(torch.bfloat16).double().numpy()
    assert np.array_equal(ours, ref)


def test_bf16_rounding_ties_and_exact_values():
    v = np.array([1.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -3.0, 4.0 + 2.0 ** -6, 0.0])
    assert tolerance.bf16_rne(v).tolist() == [1.0, 1.0, 1.0 + 2.0 ** -6, -3.0, 4.0, 0.0]


def test_storage_floor_is_the_bf16_rounding_error():
    o = np.array([4.0 + 2.0 ** -6 + 1e-9, 0.5, -2.0])  # just above a tie at |o| in [4, 8)
    assert tolerance.storage_floor(o) == pytest.approx(2.0 ** -6 - 1e-9, abs=1e-15)
    assert tolerance.storage_floor(np.array([1.0, 2.0])) == 0.0


def test_o_allowance_is_counted_not_silent():
    tolerance.O_RECORDS.clear()
    ref = np.full(100, 0.25)
    ref[0] = 5.0 + 2.0 ** -6 * 0.9
    got = tolerance.bf16_rne(ref)  # error 0.014 > 1e-2 at the first element, within half an ulp
    st = tolerance.check_o(got, ref, "allowance")
    assert st["n_floor"] == 1 and tolerance.O_RECORDS[-1]["n_floor"] == 1
    assert any("allowance 1" in line for line in tolerance.o_summary())
    bad = ref.copy()
    bad[0] += 0.03
    with pytest.raises(AssertionError):
        tolerance.check_o(bad, ref, "beyond the allowance")


def test_gradient_scale_comes_from_the_given_oracle_maximum():
    ref = np.array([0.1, -0.2])
    # the sample's own max would give 0.05 / 0.2 = 0.25; the oracle's maximum over
    # all samples (100) makes the same error 5e-4
    tolerance.check_grad("dv", ref + 0.05, ref, "sample", ref_max=100.0)
    with pytest.raises(AssertionError):
        tolerance.check_grad("dv", ref + 0.05, ref, "sample")


def test_lse_bound_covers_the_rounded_row_sum_and_is_nearly_tight():
    """The lse tolerance is the worst case of summing bf16-rounded weights:
    random rows of few keys stay inside it, and weights placed just above a
    power of two (each rounded down by almost 2^-8 of its value) come within a
    few percent of it."""
    rng = np.random.default_rng(5)
    worst = 0.0
    for n in (2, 3, 4, 8, 64):
        z = rng.normal(size=(20000, n)) * 3
        p = np.exp2(z - z.max(axis=1, keepdims=True) + rng.uniform(0, 8, size=(20000, 1)))  # lazy max: p up to 2^8
        l, lt = p.sum(axis=1), tolerance.bf16_rne(p).sum(axis=1)
        worst = max(worst, float(np.abs(np.log(lt) - np.log(l)).max()))
    assert worst <= tolerance.LSE_ABS
    # adversarial: every weight just above a power of two, one ulp-half minus a hair
    p = np.ldexp(1.0 + 2.0 ** -8 - 2.0 ** -20, rng.integers(-8, 8, size=16))
    gap = abs(np.log(tolerance.bf16_rne(p).sum()) - np.log(p.sum()))
    assert 0.95 * math.log1p(2.0 ** -8) < gap <= tolerance.LSE_ABS
