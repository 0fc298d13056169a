"""The rounding bound the large-bank screen relies on (CPU, numpy emulation).

The screen sums d^2 = sum_i (q_i - x_i)^2 in fp32 the way the kernel does:
four lanes per stored entry, lane s taking the 16-byte chunks d = 4 s + 16 j
(n = dim / 4 terms per lane) in order, each term as one rounded subtraction
and one fused multiply-add, then two additions joining the lanes. Its
decision (the smallest computed value is the exact argmin when the runner-up
exceeds it by more than 4e-5 relative at dim 512) assumes the computed value
is within (n + 4) u of the exact one, u = 2^-24. Here the emulated fp32 sums
are compared with exact sums for random and for badly scaled inputs.
"""
import numpy as np

U = 2.0 ** -24


def _fma32(a, b, c):
    # fp32 fused multiply-add: a*b is exact in fp64 for fp32 a, b; the fp64
    # sum is rounded to fp32 (one extra fp64 rounding, far below the bound)
    return np.float32(np.float64(a) * np.float64(b) + np.float64(c))


def _screen_d2(q, x):
    dim = q.shape[0]
    lanes = []
    for sub in range(4):
        acc = np.float32(0.0)
        for d in range(4 * sub, dim, 16):
            for e in range(4):
                df = np.float32(q[d + e] - x[d + e])      # fp32 subtraction
                acc = _fma32(df, df, acc)
        lanes.append(acc)
    # butterfly: lanes (0,1) and (2,3) joined, then the pairs
    a = np.float32(lanes[0] + lanes[1])
    b = np.float32(lanes[2] + lanes[3])
    return np.float32(a + b)


def _exact_d2(q, x):
    from fractions import Fraction
    return float(sum((Fraction(float(a)) - Fraction(float(b))) ** 2 for a, b in zip(q, x)))


def test_screen_sum_stays_within_its_bound():
    rng = np.random.default_rng(7)
    worst = 0.0
    for dim in (64, 128, 512):
        n = dim // 4
        for trial in range(12):
            scale = [2.0, 1e-3, 300.0][trial % 3]
            q = (scale * rng.standard_normal(dim)).astype(np.float32)
            x = (scale * rng.standard_normal(dim)).astype(np.float32)
            if trial % 4 == 3:
                # near duplicates: small differences, heavy cancellation in q - x
                x = (q + np.float32(1e-4) * rng.standard_normal(dim).astype(np.float32)).astype(
                    np.float32)
            got = float(_screen_d2(q, x))
            want = _exact_d2(q, x)
            rel = abs(got - want) / want
            assert rel <= (n + 4) * U, (dim, trial, rel, (n + 4) * U)
            worst = max(worst, rel / ((n + 4) * U))
    # the bound is not vacuous: observed errors reach a visible part of it
    assert worst > 1e-3, worst
