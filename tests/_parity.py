"""Element-wise parity bound shared by the GPU parity tests.

A value output y passes against the fp64 oracle value y_ref when
    |y - y_ref| <= 2**-7 * |y_ref| + 1e-4 * S
where S is the sum of |term| over the output's reduction index (k for Y, n
for dX, m for dW; masked-out terms are zero).  Outputs whose S is zero (an
empty block row or column) must be exactly zero.  The 2**-7 term is twice
the largest relative error of rounding the fp32 accumulator to bf16 (2**-8);
fp32 accumulation over K terms adds about sqrt(K) * 2**-24 * S, far below
1e-4 * S.
"""
import numpy as np

REL = 2.0 ** -7
ABS = 1e-4


def parity_violations(got, ref, refabs):
    got = np.asarray(got, dtype=np.float64)
    bound = REL * np.abs(ref) + ABS * refabs
    bad = np.abs(got - ref) > bound
    bad |= (refabs == 0) & (got != 0)
    bad |= ~np.isfinite(got)
    return bad


def assert_parity(got, ref, refabs, what=""):
    bad = parity_violations(got, ref, refabs)
    if bad.any():
        idx = np.argwhere(bad)[:5]
        got = np.asarray(got, dtype=np.float64)
        detail = ", ".join(f"{tuple(i)}: got {got[tuple(i)]!r} ref {ref[tuple(i)]!r} S {refabs[tuple(i)]!r}"
                           for i in idx)
        raise AssertionError(f"{what}: {int(bad.sum())} of {bad.size} outside bound; first: {detail}")
