"""The parity metric itself (CPU): max arithmetic error net of the GPU value's own bf16 rounding."""
import numpy as np
import pytest

import workloads as W
from tests.helpers import bf16_half_ulp, compare


def _bits(v):
    return W.f32_to_bf16_bits(np.asarray(v, np.float32))


def test_half_ulp():
    assert bf16_half_ulp(np.array([1.0]))[0] == 2.0 ** -8          # ulp of [1, 2) is 2^-7
    assert bf16_half_ulp(np.array([3.0]))[0] == 2.0 ** -7
    assert bf16_half_ulp(np.array([-0.75]))[0] == 2.0 ** -9


def test_rounding_alone_is_not_an_arithmetic_error():
    ref = np.array([[1.0 + 2.0 ** -8, 3.0 - 2.0 ** -9, 0.5, -2.0]])   # first: a bf16 midpoint
    rel, cos, rms, raw = compare(_bits(ref), ref)
    assert rel == 0.0 and raw > 0.0 and cos == pytest.approx(1.0)


def test_one_ulp_off_counts_half_an_ulp():
    ref = np.array([[1.0, 1.0, 1.0, 1.0]])
    g = _bits(ref)
    g[0, 0] += 1                                                       # 1 + 2^-7
    rel, _, rms, raw = compare(g, ref)
    assert raw == pytest.approx(2.0 ** -7 / rms) and rel == pytest.approx(2.0 ** -8 / rms)
