"""The attention acceptance check shared by the GPU tests.

Two bars, both required, element by element against the fp64 oracle run on
the same index rows:

1. The stated tolerance: |g - o| <= 2e-2 + 1e-2 |o|.

2. A bound derived from the arithmetic of a bf16 kernel, which scales with
   the output.  This is what makes the check able to fail at the Gaussian
   workloads' scales, where |o| is about 2e-3 and bar 1 alone would accept
   an all-zero output.
   bf16 keeps 8 significant bits, so rounding to nearest has a relative
   error of at most u = 2^-8.
   - The output is rounded to bf16, a relative error of at most u.  The
     first term allows 2u |o| = 2^-7 |o|.
   - The softmax weights enter the P.V product in bf16.  Each weight then
     carries an independent relative error of at most u (standard deviation
     at most u/sqrt(3)).  That moves o by a random amount of standard
     deviation at most u/sqrt(3) * spread, where
     spread = sqrt(sum_s p_s^2 V[s]^2) comes from oracle.attn_weight_spread.
     The second term allows 6u * spread, about ten such deviations.
   - fp32 accumulation and ex2.approx (relative error near 2^-22) add
     orders of magnitude less.
   - A floor of 1e-6 covers outputs whose every selected V value is zero.

   So |g - o| <= 2^-7 |o| + 6 * 2^-8 * spread + 1e-6.

tests/test_attn_checker.py shows on the CPU that bar 2 rejects the
oracle's own output, rounded to bf16, after one key is dropped, one index
is moved to a key outside the set, one V row is read from the wrong
position, or all keys of the second half are dropped.  It checks both
near-uniform and peaked softmax rows at the full workloads' scales.
"""
import numpy as np

import oracle

ATT_ATOL, ATT_RTOL = 2e-2, 1e-2
OUT_REL = 2.0 ** -7
SPREAD_K = 6 * 2.0 ** -8
ABS_FLOOR = 1e-6


def bars(got, ref, spread):
    """Boolean arrays (bar 1, bar 2) over the elements."""
    got = np.asarray(got, np.float64)
    err = np.abs(got - ref)
    return (err <= ATT_ATOL + ATT_RTOL * np.abs(ref),
            err <= OUT_REL * np.abs(ref) + SPREAD_K * spread + ABS_FLOOR)


def passes(got, ref, spread) -> bool:
    b1, b2 = bars(got, ref, spread)
    return bool(b1.all() and b2.all())


def assert_attention(got, ref, spread, what=""):
    got = np.asarray(got, np.float64)
    b1, b2 = bars(got, ref, spread)
    err = np.abs(got - ref)
    assert b1.all(), "%s: stated tolerance, max err %.3g" % (what, float(err.max()))
    if not b2.all():
        bad = np.argwhere(~b2)[0]
        i = tuple(bad)
        raise AssertionError(
            "%s: rounding bound failed at %s: got %.6g want %.6g (err %.3g, spread %.3g); "
            "%d of %d elements" % (what, i, got[i], ref[i], err[i], spread[i], int((~b2).sum()),
                                   b2.size))


def error_in_spreads(got, ref, spread):
    """max over elements of (|g - o| - 2^-8 |o|) / (2^-8 spread): the error
    beyond one output rounding, in units of u * spread (for reports)."""
    got = np.asarray(got, np.float64)
    ex = np.abs(got - ref) - 2.0 ** -8 * np.abs(ref)
    return float(np.max(ex / (2.0 ** -8 * spread + 1e-30)))


def check(got, Q, K, V, idx, rows=None, rows_per_seq=0, q_is_rows=False, scale=None, what=""):
    """Runs the oracle (output and weight spread) on the given index rows and
    asserts both bars on `got` ([nrows, Hq, d])."""
    ref = oracle.sparse_attn(Q, K, V, idx, rows=rows, rows_per_seq=rows_per_seq,
                             q_is_rows=q_is_rows, scale=scale)
    spread = oracle.attn_weight_spread(Q, K, V, idx, rows=rows, rows_per_seq=rows_per_seq,
                                       q_is_rows=q_is_rows, scale=scale)
    assert_attention(got, ref, spread, what)
    return ref, spread
