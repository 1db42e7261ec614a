"""The constants of the softmax's FMA-pipe exponential, pinned on the host to the definition
the kernel's comment gives: the cubic that interpolates 2^f at the four Chebyshev nodes of
[-1/2, 1/2].  The device evaluation is checked against float64 in tests/test_approx_gpu.py."""
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "mla_latent_kv_attn_b200", "csrc", "exp2.cuh")


def kernel_constants() -> np.ndarray:
    text = open(HEADER).read()
    vals = [float(re.search(r"kExp2C%d = ([0-9.eE+-]+)f;" % i, text).group(1)) for i in range(4)]
    return np.array(vals, dtype=np.float32).astype(np.float64)


def chebyshev_interpolant() -> np.ndarray:
    nodes = 0.5 * np.cos((2 * np.arange(4) + 1) * np.pi / 8)      # roots of T_4 on [-1/2, 1/2]
    return np.linalg.solve(np.vander(nodes, 4, increasing=True), 2.0 ** nodes)


def interpolation_error(coef: np.ndarray) -> float:
    f = np.linspace(-0.5, 0.5, 2_000_001)
    p = np.polyval(coef[::-1], f)
    return float(np.max(np.abs(p - 2.0 ** f) / 2.0 ** f))


def test_constants_are_the_chebyshev_interpolant_of_exp2():
    c = kernel_constants()
    ref = chebyshev_interpolant()
    # float32 constants: within a float32 rounding of the float64 interpolant
    np.testing.assert_allclose(c, ref, rtol=2.0 ** -23)


def test_interpolant_error_is_below_the_stated_bound():
    err = interpolation_error(kernel_constants())
    assert err < 1.0e-4
    # the error equioscillates: it is nowhere near zero at the ends of the interval
    assert err > 9.0e-5


def test_a_plausible_slip_in_the_constants_is_caught():
    # interpolating at equally spaced nodes (instead of Chebyshev ones) gives another cubic
    nodes = np.linspace(-0.5, 0.5, 4)
    wrong = np.linalg.solve(np.vander(nodes, 4, increasing=True), 2.0 ** nodes)
    assert not np.allclose(wrong, chebyshev_interpolant(), rtol=2.0 ** -23)
    # and a Taylor cubic around 0 misses the bound at the interval's ends
    taylor = np.array([1.0, np.log(2), np.log(2) ** 2 / 2, np.log(2) ** 3 / 6])
    assert interpolation_error(taylor) > 1.0e-4
