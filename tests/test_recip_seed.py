"""The device reciprocal used in place of 1 / d on the FMA pipe, restated on the CPU.

Its method: the bit pattern of a positive float approximates a scaled, shifted log2, so an
integer subtraction from a constant approximates 1 / d (Blinn, "Floating-point tricks",
IEEE Computer Graphics and Applications, 1997); two Newton-Raphson steps r <- r + r (1 - d r)
refine it. These checks pin the claims the kernels' comment makes about the constant
0x7EF311C2: the seed's relative error equioscillates at 5.051% over a binade, and after
two steps it is at most 6.6e-6 from 2^-126 to 2^125. The device function itself is
compared with 1 / d in tests/test_gpu_debug_hooks.py.
"""
import numpy as np

MAGIC = 0x7EF311C2


def _seed(d):
    return (np.int32(MAGIC) - np.asarray(d, np.float32).view(np.int32)).view(np.float32)


def _fma32(a, b, c):
    """round_to_float32(a * b + c): the product of two float32 is exact in float64."""
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def recip_newton2(d):
    d = np.asarray(d, np.float32)
    one = np.ones_like(d)
    r = _seed(d)
    r = _fma32(r, _fma32(-d, r, one), r)
    return _fma32(r, _fma32(-d, r, one), r)


def _binade(e, step=1):
    m = np.arange(0x3F800000, 0x40000000, step, dtype=np.int64).astype(np.int32).view(np.float32)
    return (m.astype(np.float64) * 2.0 ** e).astype(np.float32)


def test_seed_error_equioscillates_at_five_percent():
    d = _binade(0)
    rel = _seed(d).astype(np.float64) * d - 1.0
    assert abs(rel.max() - 0.05051) < 5e-5 and abs(rel.min() + 0.05051) < 5e-5


def test_two_newton_steps_reach_6p6e_minus_6_in_every_binade():
    worst = 0.0
    for e in range(-126, 125, 7):
        d = _binade(e, step=61)
        worst = max(worst, float(np.max(np.abs(recip_newton2(d).astype(np.float64) * d - 1.0))))
    d = _binade(0)  # every float of one binade
    worst = max(worst, float(np.max(np.abs(recip_newton2(d).astype(np.float64) * d - 1.0))))
    assert 6.0e-6 < worst <= 6.6e-6


def test_the_bound_fails_above_2_to_the_125():
    """Where the comment says it stops: the seed goes subnormal."""
    d = _binade(125, step=61)
    assert np.max(np.abs(recip_newton2(d).astype(np.float64) * d - 1.0)) > 1e-5
