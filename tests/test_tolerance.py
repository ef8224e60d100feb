"""The GPU parity bound's rounding helpers, checked against torch's bf16 (CPU).

``tests/_gpu.compare`` requires |out - exact| <= 1e-2 per element, except
that where |exact| >= 2 an element may be the correctly rounded bf16 value of
a number within 1e-2 of the exact result (|out - exact| <= 1e-2 + half an ulp
of out).  The half-ulp helper must therefore be exactly half the gap between
neighbouring bf16 numbers, and ``bf16_round`` (used to report how many such
elements are the correctly rounded value itself) exactly round-to-nearest-even
to 8 significant bits.
"""
import numpy as np
import pytest
import torch

from tests._gpu import bf16_half_ulp, bf16_round, compare


def test_half_ulp_bounds_bf16_rounding():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.normal(0, 3, 20000), rng.uniform(-9, 9, 20000),
                        [0.0, 1.0, -1.0, 2.0, 4.0, 3.999, 7.99, 1e-30, -1e-5]])
    r = torch.from_numpy(x).to(torch.bfloat16).double().numpy()
    assert np.all(np.abs(r - x) <= bf16_half_ulp(x))


def test_half_ulp_is_half_the_bf16_gap():
    # v are bf16 numbers; the next bf16 number above |v| is |v| + gap
    def bf16(x):
        return torch.tensor([x], dtype=torch.float64).to(torch.bfloat16).double().item()

    for v, gap in [(1.0, 2.0 ** -7), (1.5, 2.0 ** -7), (2.0, 2.0 ** -6), (4.0, 2.0 ** -5),
                   (5.5, 2.0 ** -5), (-6.0, 2.0 ** -5), (0.3125, 2.0 ** -9)]:
        assert bf16(v) == v
        assert bf16_half_ulp(np.float64(v)) == gap / 2
        assert bf16(abs(v) + gap) == abs(v) + gap
        assert bf16(abs(v) + 0.4 * gap) == abs(v)  # nothing representable in between


def test_bf16_round_matches_torch_on_fp32_values():
    # torch rounds fp32 to bf16 to nearest, ties to even, in one step: on
    # values that are exact fp32 numbers the two must agree bit for bit
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.normal(0, 3, 50000), rng.uniform(-9, 9, 50000)]).astype(np.float32)
    # ties: bf16 values plus exactly half their spacing
    b = torch.from_numpy(x).to(torch.bfloat16).double().numpy()
    ties = (b + bf16_half_ulp(b) * np.sign(b)).astype(np.float32)
    for v in (x, ties):
        want = torch.from_numpy(v).to(torch.bfloat16).double().numpy()
        assert np.array_equal(bf16_round(v.astype(np.float64)), want)


def test_bf16_round_is_the_nearest_bf16_by_brute_force():
    # for fp64 inputs (no fp32 step): the result is a bf16 number and no bf16
    # number lies nearer; on ties the even significand wins
    rng = np.random.default_rng(2)
    x = np.concatenate([rng.normal(0, 4, 3000), [4.0 + 2.0 ** -6, 4.0 + 3 * 2.0 ** -6,
                                                 -6.0 - 2.0 ** -6, 0.0]])
    r = bf16_round(x)
    for xi, ri in zip(x, r):
        lo = torch.tensor([xi], dtype=torch.float64).to(torch.float32).to(torch.bfloat16)
        cand = set()
        for d in (-2, -1, 0, 1, 2):
            c = (lo.view(torch.int16) + d).view(torch.bfloat16).double().item()
            cand.add(c)
        best = min(abs(c - xi) for c in cand)
        assert abs(ri - xi) == best
        assert torch.tensor([ri]).to(torch.bfloat16).double().item() == ri
    assert bf16_round(np.float64(4.0 + 2.0 ** -6)) == 4.0  # tie: even significand 128
    assert bf16_round(np.float64(4.0 + 3 * 2.0 ** -6)) == 4.0 + 2.0 ** -4  # tie: even 130


class _Cpu:
    """A stand-in for a device tensor of bf16 values (compare calls .float().cpu())."""

    def __init__(self, a):
        self.t = torch.from_numpy(np.asarray(a, dtype=np.float32)).to(torch.bfloat16)

    def float(self):
        return self.t.float()


def test_compare_allows_only_the_output_rounding_and_only_above_two():
    # exact 2.004897, out 2.015625: 1.07e-2 off, but the bf16 rounding of
    # 2.008 (within 1e-2 of exact) -- the prefill case that motivated the allowance
    exact = np.array([[2.004897, 1.0, 0.5]])
    compare(_Cpu([[2.015625, 1.0, 0.5]]), None, exact, None, mean_abs=1e-2)
    # the next bf16 value up is no rounding of anything within 1e-2
    with pytest.raises(AssertionError):
        compare(_Cpu([[2.03125, 1.0, 0.5]]), None, exact, None, mean_abs=1e-2)
    # below |exact| = 2 there is no allowance: 1.2e-2 off fails
    with pytest.raises(AssertionError):
        compare(_Cpu([[1.0 + 2.0 ** -6, 1.0, 0.5]]), None,
                np.array([[1.0 + 2.0 ** -6 - 1.2e-2, 1.0, 0.5]]), None, mean_abs=1e-2)
    # above 4: the correctly rounded value passes, the far neighbour does not
    exact = np.array([[4.0 + 0.0150, 1.0, 2.5]])
    compare(_Cpu([[4.0 + 2.0 ** -5, 1.0, 2.5]]), None, exact, None, mean_abs=1e-2)
    with pytest.raises(AssertionError):
        compare(_Cpu([[4.0 + 2 * 2.0 ** -5, 1.0, 2.5]]), None, exact, None, mean_abs=1e-2)
