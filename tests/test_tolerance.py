"""The GPU parity bound's rounding helpers, checked against torch's bf16 (CPU).

``tests/_gpu.compare`` admits an element that misses max-abs 1e-2 of the
exact value only if it is within 1e-2 of the correctly rounded bf16 value,
``bf16_round(exact)``, which must therefore be exactly round-to-nearest-even
to 8 significant bits.  The half-ulp helper must be what rounding to bf16 can
cost: never less than the rounding error of any value, and half the gap
between neighbouring bf16 numbers.
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


def test_compare_admits_only_the_correctly_rounded_value_above_four():
    exact = np.array([[4.0 + 0.0150, 1.0, 2.5]])
    # out = bf16_round(exact): 4.0 is 0.015 from the exact value, > 1e-2
    compare(_Cpu([[4.0, 1.0, 2.5]]), None, exact, None, mean_abs=1e-2)
    # the other bf16 neighbour of a value above 4 is refused
    with pytest.raises(AssertionError):
        compare(_Cpu([[4.0 + 2.0 ** -5, 1.0, 2.5]]), None, exact, None, mean_abs=1e-2)
    # below 4 the rounded value is always within 1e-2: an element 1.2e-2 off fails
    with pytest.raises(AssertionError):
        compare(_Cpu([[4.0, 1.0 + 2.0 ** -6, 2.5]]), None,
                np.array([[4.0, 1.0 + 2.0 ** -6 - 1.2e-2, 2.5]]), None, mean_abs=1e-2)
