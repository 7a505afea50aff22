"""The exp2 polynomial fit script reproduces its recorded coefficients and error.

The prefill kernel keeps this fit for evaluating 2^x on the FMA pipes; the
recorded constants must be what the script's minimax fit gives, and their fp32
evaluation must stay well inside bf16 precision.
"""

import pytest

from ragged_paged_kv_rope_b200 import exp2_poly_fit as F


def test_fit_reproduces_recorded_coefficients():
    pytest.importorskip("scipy")
    got = F.fit()
    for a, b in zip(got, F.COEFFS):
        assert abs(a - b) <= 2e-7 * max(1.0, abs(b))


def test_fit_error_is_far_below_bf16_rounding():
    assert F.max_rel_error(F.COEFFS) < 1.1e-4
    assert F.max_rel_error(F.COEFFS) < 2.0 ** -9 / 10
