"""Pins for the oracle's FP8 linear passes (fwd, dgrad, wgrad) with unscale.

  * brute force with exact rationals (fractions.Fraction) on small,
    deliberately non-square shapes, every index written out by explicit loops,
    for all three passes — a transposed operand, a swapped index, a dropped
    term, a wrong sign of the unscale exponent all fail here;
  * the sampled-entry path equals the full path;
  * structural identities between the passes: dgrad(dY, W) is the forward of
    dY against W transposed; wgrad(dY, X) is the forward of dY^T against X^T.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle

E4, E5 = oracle.E4M3, oracle.E5M2


def _rand_codes(rng, shape, fmt):
    """Random finite FP8 codes (NaN / inf codes excluded)."""
    table = oracle.fp8_decode_table(fmt)
    finite = np.nonzero(np.isfinite(table))[0].astype(np.uint8)
    return rng.choice(finite, size=shape)


def _frac(code, fmt):
    return Fraction(float(oracle.fp8_decode([code], fmt)[0]))


def _brute(pass_, A, fa, ba, B, fb, bb, T, In, Out):
    scale = Fraction(2) ** (-(ba + bb))
    if pass_ == oracle.FWD:          # Y[t,o] = sum_i X[t,i] W[o,i]
        R, C = T, Out
        f = lambda r, c: sum(_frac(A[r, i], fa) * _frac(B[c, i], fb) for i in range(In))
    elif pass_ == oracle.DGRAD:      # dX[t,i] = sum_o dY[t,o] W[o,i]
        R, C = T, In
        f = lambda r, c: sum(_frac(A[r, o], fa) * _frac(B[o, c], fb) for o in range(Out))
    else:                            # dW[o,i] = sum_t dY[t,o] X[t,i]
        R, C = Out, In
        f = lambda r, c: sum(_frac(A[t, r], fa) * _frac(B[t, c], fb) for t in range(T))
    return [[f(r, c) * scale for c in range(C)] for r in range(R)]


SHAPES = [(3, 5, 4), (4, 4, 4), (1, 7, 2), (6, 2, 5)]


@pytest.mark.parametrize("T,In,Out", SHAPES)
def test_brute_force_all_passes(T, In, Out):
    rng = np.random.default_rng(T * 100 + In * 10 + Out)
    X = _rand_codes(rng, (T, In), E4)
    W = _rand_codes(rng, (Out, In), E4)
    dY = _rand_codes(rng, (T, Out), E5)
    bx, bw, bdy = 5, -2, 17
    cases = [(oracle.FWD, X, E4, bx, W, E4, bw),
             (oracle.DGRAD, dY, E5, bdy, W, E4, bw),
             (oracle.WGRAD, dY, E5, bdy, X, E4, bx)]
    for pass_, A, fa, ba, B, fb, bb in cases:
        val, av = oracle.linear(pass_, A, fa, ba, B, fb, bb, T, In, Out)
        ref = _brute(pass_, A, fa, ba, B, fb, bb, T, In, Out)
        for r in range(val.shape[0]):
            for c in range(val.shape[1]):
                # FP8 x FP8 products and short sums are exact in fp64
                assert Fraction(val[r, c]) == ref[r][c], (pass_, r, c)
                assert av[r, c] >= abs(val[r, c])


def test_unscale_sign_and_output_shapes():
    rng = np.random.default_rng(0)
    X = _rand_codes(rng, (2, 3), E4)
    W = _rand_codes(rng, (4, 3), E4)
    v0 = oracle.linear(oracle.FWD, X, E4, 0, W, E4, 0, 2, 3, 4, with_abs=False)
    v1 = oracle.linear(oracle.FWD, X, E4, 3, W, E4, 2, 2, 3, 4, with_abs=False)
    assert v0.shape == (2, 4)
    np.testing.assert_array_equal(v1, v0 / 32.0)          # bias 3+2 divides by 2^5


@pytest.mark.parametrize("pass_", [oracle.FWD, oracle.DGRAD, oracle.WGRAD])
def test_entries_equal_full(pass_):
    rng = np.random.default_rng(42 + pass_)
    T, In, Out = 37, 48, 32
    X = _rand_codes(rng, (T, In), E4)
    W = _rand_codes(rng, (Out, In), E4)
    dY = _rand_codes(rng, (T, Out), E5)
    A, fa, B, fb = {oracle.FWD: (X, E4, W, E4), oracle.DGRAD: (dY, E5, W, E4),
                    oracle.WGRAD: (dY, E5, X, E4)}[pass_]
    full, fabs_ = oracle.linear(pass_, A, fa, 4, B, fb, -1, T, In, Out)
    R, C = full.shape
    rows = rng.integers(0, R, 500)
    cols = rng.integers(0, C, 500)
    v, av = oracle.linear_entries(pass_, A, fa, 4, B, fb, -1, T, In, Out, rows, cols)
    np.testing.assert_array_equal(v, full[rows, cols])
    np.testing.assert_array_equal(av, fabs_[rows, cols])


def test_pass_identities():
    rng = np.random.default_rng(9)
    T, In, Out = 9, 16, 12
    X = _rand_codes(rng, (T, In), E4)
    W = _rand_codes(rng, (Out, In), E4)
    dY = _rand_codes(rng, (T, Out), E5)
    # dgrad(dY, W) == fwd(x=dY, w=W^T) with in'=Out, out'=In
    dg = oracle.linear(oracle.DGRAD, dY, E5, 2, W, E4, 1, T, In, Out, with_abs=False)
    fw = oracle.linear(oracle.FWD, dY, E5, 2, np.ascontiguousarray(W.T), E4, 1, T, Out, In,
                       with_abs=False)
    np.testing.assert_array_equal(dg, fw)
    # wgrad(dY, X) == fwd(x=dY^T [Out,T], w=X^T [In,T]) with T'=Out, in'=T, out'=In
    wg = oracle.linear(oracle.WGRAD, dY, E5, 2, X, E4, 1, T, In, Out, with_abs=False)
    fw2 = oracle.linear(oracle.FWD, np.ascontiguousarray(dY.T), E5, 2, np.ascontiguousarray(X.T),
                        E4, 1, Out, T, In, with_abs=False)
    np.testing.assert_array_equal(wg, fw2)
