"""CPU: the parity helper's tolerances do what the test suite relies on.

bf16 outputs must be within max-abs-error 1e-2 and max-rel-error 2e-2 of the float64
oracle.  The helper reads the absolute bar as 1e-2 wherever bf16 can resolve it and as
half a bf16 ulp plus the fp32 slack where it cannot (|r| >= 4), and the relative bar as
elementwise |g - r| / max(|r|, 1e-3).  These cases pin both readings: a correctly rounded
output passes everywhere, and errors that either bar must catch fail.
"""

import numpy as np
import pytest
import torch

import workloads
from _parity import BF16_REL, F32_SLACK, abs_bar, assert_close, bf16_ulp, errors

W_BF16 = workloads.independent([1], dtype="bf16")
W_F32 = workloads.independent([1], dtype="f32")


def _bf16(x):
    """Round float64 values to bfloat16 (nearest even) and back, as a torch tensor."""
    return torch.from_numpy(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)


def test_bf16_ulp_and_bar():
    assert bf16_ulp(1.0) == 2.0 ** -7
    assert bf16_ulp(3.99) == 2.0 ** -6
    assert bf16_ulp(-4.0) == 2.0 ** -5
    # below |r| = 4 half an ulp is at most 2^-7 < 1e-2: the literal bar
    assert abs_bar(3.99) == 1e-2
    # from 4 up, half an ulp (2^-6) plus the slack
    assert abs_bar(4.5) == pytest.approx(2.0 ** -6 + F32_SLACK)
    # two rounded outputs compared with each other: twice that
    assert abs_bar(4.5, exact_ref=False) == pytest.approx(2.0 ** -5 + 2 * F32_SLACK)


def test_correctly_rounded_outputs_pass():
    rng = np.random.default_rng(0)
    r = np.concatenate([rng.standard_normal((4, 8, 128)) * s for s in (1e-4, 0.03, 1.0, 3.0)])
    r[0, 0, :5] = [4.26526, -4.26526, 7.99, -5.5, 0.0]   # |r| >= 4: half an ulp > 1e-2
    res = assert_close(W_BF16, _bf16(r), r)
    assert res["abs"] > 1e-2            # 4.26526 rounds to 4.25: 0.0153 off
    assert res["abs_bar"] <= 1.0


def test_one_ulp_off_fails_where_half_an_ulp_is_the_bar():
    r = np.full((1, 1, 8), 4.26526)
    g = _bf16(r).double().numpy() + 2.0 ** -5          # the next bf16 number up
    with pytest.raises(AssertionError):
        assert_close(W_BF16, torch.from_numpy(g), r)


def test_relative_bar_catches_small_outputs():
    r = np.full((1, 1, 8), 0.01)
    g = r * 1.03                                        # 3e-4 abs: passes the abs bar
    res = errors(torch.from_numpy(g), r, bf16=True)
    assert res["abs_bar"] <= 1.0 and res["rel"] > BF16_REL
    with pytest.raises(AssertionError):
        assert_close(W_BF16, torch.from_numpy(g), r)
    # near zero the floor makes it an absolute bar of 2e-5
    r0 = np.zeros((1, 1, 8))
    r0[0, 0, 0] = 1e-6
    g0 = r0.copy()
    g0[0, 0, 0] = 1.5e-5
    assert assert_close(W_BF16, torch.from_numpy(g0), r0)["rel"] < BF16_REL
    g0[0, 0, 0] = 3e-5
    with pytest.raises(AssertionError):
        assert_close(W_BF16, torch.from_numpy(g0), r0)


def test_zero_rows_must_be_exactly_zero():
    r = np.zeros((2, 1, 8))
    r[1] = 1.0
    g = r.copy()
    g[0, 0, 3] = 1e-7
    with pytest.raises(AssertionError):
        errors(torch.from_numpy(g), r, bf16=True)


def test_fp32_bar():
    r = np.ones((1, 1, 4))
    assert_close(W_F32, torch.from_numpy(r + 9e-5), r)
    with pytest.raises(AssertionError):
        assert_close(W_F32, torch.from_numpy(r + 2e-4), r)


def test_figures_reported():
    r = np.full((1, 2, 4), 0.5)
    g = r.copy()
    g[0, 1, 0] = 0.5 + 4e-3
    res = errors(torch.from_numpy(g), r, bf16=True)
    assert res["rel"] == pytest.approx(8e-3, rel=1e-5)
    assert res["rel_unfloored"] == pytest.approx(8e-3, rel=1e-5)
    assert res["rel_row"] == pytest.approx(8e-3, rel=1e-5)
    assert res["abs"] == pytest.approx(4e-3, rel=1e-5)
