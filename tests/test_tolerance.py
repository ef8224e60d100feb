"""The GPU parity bound's rounding allowance, checked against torch's bf16 (CPU).

``tests/_gpu.compare`` allows, per element, max-abs 1e-2 plus half a bf16
ulp of the exact value.  The half-ulp helper must be exactly what rounding to
bf16 can cost: never less than the rounding error of any value, and equal to
half the gap between neighbouring bf16 numbers.
"""
import numpy as np
import torch

from tests._gpu import bf16_half_ulp


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
