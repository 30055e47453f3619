"""Pins of the float64 oracle by exact algebraic invariants of

    Y[m][n] = gscale * sum_k x[m][k] * e2m1(q[n][k]) * e4m3(s[n][k/16]),

checked on seeded random inputs of the synthetic recipe.  None of them
retypes the oracle's formula; each one fails for a specific plausible
mistake in it (checked by planting each mistake in a copy of the oracle):

- flipping every code's sign bit negates Y exactly (a wrong E2M1 sign rule);
- flipping every scale's sign bit negates Y exactly (a dropped E4M3 sign);
- one more E4M3 exponent step on every scale doubles Y exactly (a wrong
  exponent field or bias);
- keeping only the low nibbles equals zeroing X's odd columns, and keeping
  only the high nibbles equals zeroing its even columns (swapped nibble
  order);
- doubling the scales of one block changes Y by exactly that block's own
  partial product (a wrong scale index k/16);
- doubling gscale or X doubles Y exactly (a dropped or misplaced factor).
"""
import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle
from nvfp4_weight_streaming_decode_b200 import synth

SHAPES = [(1, 16), (3, 48), (8, 64), (5, 80), (17, 32)]


def _case(seed, shape, M):
    N, K = shape
    g = synth.rng(900 + M, seed)
    return synth.codes(g, N, K), synth.scales(g, N, K), synth.activations(g, M, K)


def _close(Y1, Y0, A):
    # same terms, another summation order: float64 rounding only
    assert np.all(np.abs(Y1 - Y0) <= 1e-12 * A + 1e-300)


common = settings(max_examples=30, deadline=None)
inputs = (st.integers(0, 100_000), st.sampled_from(SHAPES), st.integers(1, 4))


@common
@given(*inputs)
def test_code_sign_flip_negates(seed, shape, M):
    q, s, X = _case(seed, shape, M)
    Y, _ = oracle.gemm(X, q, s, synth.GSCALE)
    Yn, _ = oracle.gemm(X, q ^ np.uint8(0x88), s, synth.GSCALE)
    assert np.array_equal(Yn, -Y)


@common
@given(*inputs)
def test_scale_sign_flip_negates(seed, shape, M):
    q, s, X = _case(seed, shape, M)
    Y, _ = oracle.gemm(X, q, s, synth.GSCALE)
    Yn, _ = oracle.gemm(X, q, s ^ np.uint8(0x80), synth.GSCALE)
    assert np.array_equal(Yn, -Y)


@common
@given(*inputs)
def test_scale_exponent_step_doubles(seed, shape, M):
    q, s, X = _case(seed, shape, M)
    # the recipe's scale exponents are -4..2 (fields 3..9): one more step stays finite
    assert ((s >> 3) & 15).max() <= 9
    Y, _ = oracle.gemm(X, q, s, synth.GSCALE)
    Y2, _ = oracle.gemm(X, q, (s + np.uint8(8)).astype(np.uint8), synth.GSCALE)
    assert np.array_equal(Y2, 2 * Y)


@common
@given(*inputs)
def test_low_nibbles_carry_the_even_columns(seed, shape, M):
    q, s, X = _case(seed, shape, M)
    # zero codes in every high nibble == zero X in every odd column: both leave the even-k terms only
    Y1, _ = oracle.gemm(X, (q & np.uint8(15)).astype(np.uint8), s, synth.GSCALE)
    Xe = X.copy()
    Xe[:, 1::2] = 0
    Y2, _ = oracle.gemm(Xe, q, s, synth.GSCALE)
    assert np.array_equal(Y1, Y2)
    # and the high nibbles carry the odd columns
    Y3, _ = oracle.gemm(X, (q & np.uint8(0xF0)).astype(np.uint8), s, synth.GSCALE)
    Xo = X.copy()
    Xo[:, 0::2] = 0
    Y4, _ = oracle.gemm(Xo, q, s, synth.GSCALE)
    assert np.array_equal(Y3, Y4)


@common
@given(*inputs, st.integers(0, 1_000))
def test_one_scale_block_moves_only_its_columns(seed, shape, M, pick):
    q, s, X = _case(seed, shape, M)
    N, K = shape
    b = pick % (K // 16)
    Y, A = oracle.gemm(X, q, s, synth.GSCALE)
    s2 = s.copy()
    s2[:, b] = s2[:, b] + np.uint8(8)       # that block's scales doubled
    Y2, _ = oracle.gemm(X, q, s2, synth.GSCALE)
    Xb = np.zeros_like(X)
    Xb[:, 16 * b:16 * b + 16] = X[:, 16 * b:16 * b + 16]
    Yb, _ = oracle.gemm(Xb, q, s, synth.GSCALE)
    # Y2 - Y is block b's own partial product, and nothing else
    _close(Y2 - Y, Yb, A)


@common
@given(*inputs)
def test_doubling_gscale_or_x_doubles(seed, shape, M):
    q, s, X = _case(seed, shape, M)
    Y, _ = oracle.gemm(X, q, s, synth.GSCALE)
    Yg, _ = oracle.gemm(X, q, s, 2 * synth.GSCALE)
    assert np.array_equal(Yg, 2 * Y)
    xf = (X.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    X2 = synth.bf16_bits_from_f64(2 * xf)
    Yx, _ = oracle.gemm(X2, q, s, synth.GSCALE)
    assert np.array_equal(Yx, 2 * Y)
