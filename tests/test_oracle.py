"""Pins of the float64 oracle against facts that do not come from the oracle.

Sources of truth used here: the E2M1 value list of the standard element
format (tests/golden/e2m1_values.txt), torch's float8_e4m3fn decoder and
ml_dtypes' float4_e2m1fn / float8_e4m3fn decoders (library routines),
scipy's expit, numpy's matmul and sum, a hand-worked example
(tests/golden/worked_example.txt), and closed forms that hold for
structured weights.  Each would fail for a plausible mistake in the oracle:
a wrong bias or subnormal rule (tables), swapped nibbles or a wrong scale
index (probes, worked example), a dropped scale or global scale (closed
forms), a transposed operand (rank-1 and permutation checks).
"""
import os

import numpy as np
import pytest
import torch
from scipy.special import expit

import oracle
from nvfp4_weight_streaming_decode_b200 import synth

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _read_golden(name):
    out = {}
    with open(os.path.join(GOLD, name)) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                key, *vals = line.split()
                out[key] = vals
    return out


def _e2m1_golden():
    vals = np.zeros(16)
    with open(os.path.join(GOLD, "e2m1_values.txt")) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                c, v = line.split()
                vals[int(c)] = float(v)
    return vals


def _e4m3_torch():
    return torch.arange(256, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn) \
        .to(torch.float64).numpy()


def _bf16_to_f64(bits):
    return (np.asarray(bits, np.uint32) << 16).view(np.float32).astype(np.float64)


def _dense_weights(q, s):
    """Dequantise with independent decoders: golden E2M1 list, torch E4M3."""
    e2 = _e2m1_golden()
    e4 = _e4m3_torch()
    lo = q & 15
    hi = q >> 4
    codes = np.empty((q.shape[0], q.shape[1] * 2), np.int64)
    codes[:, 0::2] = lo
    codes[:, 1::2] = hi
    sc = np.repeat(e4[s], 16, axis=1)
    return e2[codes] * sc


# ---------------------------------------------------------------- tables

def test_e2m1_table_matches_standard_values():
    e2, _ = oracle.tables()
    gold = _e2m1_golden()
    assert np.array_equal(e2, gold)
    assert np.array_equal(np.signbit(e2), np.signbit(gold))  # code 8 is -0


def test_e4m3_table_matches_torch_float8():
    _, e4 = oracle.tables()
    ref = _e4m3_torch()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(e4), nan)
    assert sorted(np.nonzero(nan)[0].tolist()) == [0x7F, 0xFF]
    assert np.array_equal(e4[~nan], ref[~nan])
    assert np.array_equal(np.signbit(e4[~nan]), np.signbit(ref[~nan]))


def test_tables_match_ml_dtypes():
    # a second library decoder for both formats (ml_dtypes' float4_e2m1fn and
    # float8_e4m3fn, one code per byte), independent of the golden list and torch
    ml_dtypes = pytest.importorskip("ml_dtypes")
    e2, e4 = oracle.tables()
    ref2 = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    assert np.array_equal(e2, ref2) and np.array_equal(np.signbit(e2), np.signbit(ref2))
    ref4 = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    nan = np.isnan(ref4)
    assert np.array_equal(np.isnan(e4), nan)
    assert np.array_equal(e4[~nan], ref4[~nan]) and np.array_equal(np.signbit(e4[~nan]), np.signbit(ref4[~nan]))


def test_table_invariants():
    e2, e4 = oracle.tables()
    for c in range(16):
        assert e2[c ^ 8] == -e2[c] and np.signbit(e2[c ^ 8]) != np.signbit(e2[c])
    pos = e4[:0x7F]
    assert np.all(np.diff(pos) > 0), "E4M3 must increase over 0x00..0x7E"
    assert e4[0x7E] == 448.0 and e4[0x01] == 2.0 ** -9 and e4[0x08] == 2.0 ** -6
    assert np.array_equal(e4[0x80:0xFF], -e4[0x00:0x7F])


def test_nan_scale_count():
    s = np.array([[0x7F, 0x38], [0xFF, 0xFE]], np.uint8)
    assert oracle.count_nan_scales(s) == 2


# ---------------------------------------------------------------- layout

def test_single_nonzero_probes_pin_nibble_order_and_scale_index():
    N, K = 8, 64
    for n in range(N):
        for k in range(K):
            q = np.zeros((N, K // 2), np.uint8)
            s = np.full((N, K // 16), 0x38, np.uint8)
            q[n, k // 2] = 0x2 << (4 * (k % 2))
            W = oracle.dequant(q, s, 1.0)
            hot = np.zeros((N, K), np.float32)
            hot[n, k] = 1.0
            assert np.array_equal(W, hot), (n, k)
    # scale indexing: a 2.0 scale on block b of row n doubles exactly k in [16b, 16b+16)
    q = np.full((N, K // 2), 0x22, np.uint8)
    for n in range(N):
        for b in range(K // 16):
            s = np.full((N, K // 16), 0x38, np.uint8)
            s[n, b] = 0x40
            W = oracle.dequant(q, s, 1.0)
            exp = np.ones((N, K), np.float32)
            exp[n, 16 * b:16 * b + 16] = 2.0
            assert np.array_equal(W, exp), (n, b)


def test_worked_example_by_hand():
    g = _read_golden("worked_example.txt")
    N, K = int(g["N"][0]), int(g["K"][0])
    gscale = float(g["gscale"][0])
    x = np.array([float(v) for v in g["x"]])
    X = synth.bf16_bits_from_f64(x[None, :])
    q = np.array([[int(b, 16) for b in g["q0"]], [int(b, 16) for b in g["q1"]]], np.uint8)
    s = np.array([[int(g["s0"][0], 16)], [int(g["s1"][0], 16)]], np.uint8)
    Y, _ = oracle.gemm(X, q, s, gscale)
    assert Y.tolist() == [[float(v) for v in g["y"]]]
    W = oracle.dequant(q, s, gscale)
    assert W[1, :4].tolist() == [float(v) for v in g["w1_head"]]
    assert N == 2 and K == 16


# ---------------------------------------------------------------- dequant

def test_dequant_matches_independent_decoders():
    q, s = synth.matrix(0, 0, 64, 256)
    s[0, 0] = 0x01   # a subnormal scale
    s[1, 1] = 0x7E   # the largest scale
    s[2, 2] = 0x00   # zero
    s[3, 3] = 0x80   # negative zero
    s[4, 4] = 0xB9   # a negative scale
    gscale = 1.0 / 64
    W = oracle.dequant(q, s, gscale)
    ref = (_dense_weights(q, s) * gscale).astype(np.float32)
    assert np.array_equal(W.view(np.uint32), ref.view(np.uint32))


# ---------------------------------------------------------------- GEMM

def test_gemm_brute_force_against_numpy_matmul():
    for M in range(1, 9):
        for (N, K) in [(1, 16), (3, 48), (17, 128), (64, 96)]:
            g = synth.rng(100 + M, N * 1000 + K)
            q = synth.codes(g, N, K)
            s = synth.scales(g, N, K)
            X = synth.activations(g, M, K)
            Y, A = oracle.gemm(X, q, s, 1.0 / 64)
            Wd = _dense_weights(q, s)
            Xf = _bf16_to_f64(X)
            ref = (Xf @ Wd.T) / 64
            assert np.allclose(Y, ref, rtol=1e-12, atol=1e-12), (M, N, K)
            assert np.allclose(A, np.abs(Xf) @ np.abs(Wd.T / 64).astype(np.float32).astype(np.float64),
                               rtol=1e-12, atol=1e-15)


@pytest.mark.parametrize("M", [9, 16, 17, 33, 64])
def test_gemm_brute_force_at_verify_widths(M):
    # the verify widths (lanes x (1 + drafts), up to 64 rows) use the same oracle
    for (N, K) in [(5, 32), (33, 208)]:
        g = synth.rng(300 + M, N * 1000 + K)
        q = synth.codes(g, N, K)
        s = synth.scales(g, N, K)
        X = synth.activations(g, M, K)
        Y, A = oracle.gemm(X, q, s, 1.0 / 64)
        Wd = _dense_weights(q, s)
        Xf = _bf16_to_f64(X)
        assert np.allclose(Y, (Xf @ Wd.T) / 64, rtol=1e-12, atol=1e-12), (M, N, K)
        rows = np.array([N - 1, 0, N // 2])
        Yr, Ar = oracle.gemm_rows(X, q, s, 1.0 / 64, rows)
        assert np.array_equal(Yr, Y[:, rows]) and np.array_equal(Ar, A[:, rows])


def test_gemm_identity_weights_at_64_rows():
    K = 128
    q, s = _identity_planes(K)
    X = synth.activations(synth.rng(12, 12), 64, K)
    Y, _ = oracle.gemm(X, q, s, 1.0)
    assert np.array_equal(Y, _bf16_to_f64(X))


@pytest.mark.parametrize("c,sb", [(0x2, 0x38), (0x7, 0x7E), (0xB, 0x30), (0x1, 0x01), (0x0, 0x40)])
def test_gemm_constant_code_closed_form(c, sb):
    M, N, K = 3, 5, 160
    q = np.full((N, K // 2), c | (c << 4), np.uint8)
    s = np.full((N, K // 16), sb, np.uint8)
    X = synth.activations(synth.rng(7, 7), M, K)
    gscale = 0.25
    Y, _ = oracle.gemm(X, q, s, gscale)
    e2 = _e2m1_golden()[c]
    e4 = _e4m3_torch()[sb]
    rowsum = _bf16_to_f64(X).sum(axis=1)
    ref = np.repeat((e2 * e4 * gscale * rowsum)[:, None], N, axis=1)
    assert np.allclose(Y, ref, rtol=1e-13, atol=1e-300)


def _identity_planes(K, perm=None):
    q = np.zeros((K, K // 2), np.uint8)
    cols = np.arange(K) if perm is None else perm
    for n in range(K):
        k = cols[n]
        q[n, k // 2] |= 0x2 << (4 * (k % 2))
    s = np.full((K, K // 16), 0x38, np.uint8)
    return q, s


def test_gemm_identity_weights_reproduce_x_exactly():
    K = 64
    q, s = _identity_planes(K)
    X = synth.activations(synth.rng(8, 8), 4, K)
    Y, _ = oracle.gemm(X, q, s, 1.0)
    assert np.array_equal(Y, _bf16_to_f64(X))


def test_gemm_permutation_weights_permute_x_exactly():
    K = 96
    perm = np.random.default_rng(3).permutation(K)
    q, s = _identity_planes(K, perm)
    X = synth.activations(synth.rng(9, 9), 2, K)
    Y, _ = oracle.gemm(X, q, s, 1.0)
    assert np.array_equal(Y, _bf16_to_f64(X)[:, perm])


def test_gemm_rank1_picks_a_column_of_the_weights():
    N, K = 24, 80
    q, s = synth.matrix(10, 0, N, K)
    W = oracle.dequant(q, s, 1.0).astype(np.float64)
    for k in (0, 1, 15, 16, 47, 79):
        x = np.zeros((1, K))
        x[0, k] = 1.0
        Y, _ = oracle.gemm(synth.bf16_bits_from_f64(x), q, s, 1.0)
        assert np.array_equal(Y[0], W[:, k]), k


def test_gemm_rows_matches_full_gemm():
    N, K, M = 40, 128, 5
    q, s = synth.matrix(11, 0, N, K)
    X = synth.activations(synth.rng(11, 1), M, K)
    Y, A = oracle.gemm(X, q, s, 1.0 / 64)
    rows = np.array([0, 7, 39, 3])
    Yr, Ar = oracle.gemm_rows(X, q, s, 1.0 / 64, rows)
    assert np.array_equal(Yr, Y[:, rows]) and np.array_equal(Ar, A[:, rows])


# ---------------------------------------------------------------- fused MLP

def test_gateup_silu_against_expit_and_matmul():
    M, Nff, K = 4, 48, 64
    qg, sg = synth.matrix(12, 0, Nff, K)
    qu, su = synth.matrix(12, 1, Nff, K)
    X = synth.activations(synth.rng(12, 2), M, K)
    G, U, H, AG, AU = oracle.gateup_silu(X, qg, sg, 1.0 / 64, qu, su, 1.0 / 32)
    Xf = _bf16_to_f64(X)
    g = Xf @ _dense_weights(qg, sg).T / 64
    u = Xf @ _dense_weights(qu, su).T / 32
    assert np.allclose(G, g, rtol=1e-12) and np.allclose(U, u, rtol=1e-12)
    assert np.allclose(H, g * expit(g) * u, rtol=1e-12, atol=1e-300)


def test_gateup_silu_constant_code_closed_form():
    M, Nff, K = 2, 3, 32
    qg = np.full((Nff, K // 2), 0x22, np.uint8)   # +1.0
    qu = np.full((Nff, K // 2), 0xAA, np.uint8)   # -1.0
    s = np.full((Nff, K // 16), 0x38, np.uint8)   # 1.0
    X = synth.bf16_bits_from_f64(np.array([[0.5] * K, [-0.25] * K]))
    _, _, H, _, _ = oracle.gateup_silu(X, qg, s, 1.0, qu, s, 1.0)
    for m, xv in enumerate((0.5, -0.25)):
        g = K * xv
        u = -K * xv
        h = g / (1.0 + np.exp(-g)) * u
        assert np.allclose(H[m], h, rtol=1e-14)


def test_tolerance_helpers():
    A = np.array([0.0, 1.0, 1000.0])
    assert np.allclose(oracle.gemm_tolerance(A), [1e-6, 2e-3 + 1e-6, 2.0 + 1e-6])
    b = oracle.silu_tolerance(np.zeros(1), np.ones(1), np.zeros(1), np.zeros(1))
    assert b[0] > 0


# ---------------------------------------------------------------- input generators

def test_bf16_rounding_matches_torch():
    a = np.random.default_rng(0).standard_normal(10000) * np.array([1e-30, 1.0, 1e30]).repeat(
        [3000, 4000, 3000])
    mine = synth.bf16_bits_from_f64(a)
    ref = torch.from_numpy(a).to(torch.float32).to(torch.bfloat16).view(torch.int16).numpy() \
        .view(np.uint16)
    assert np.array_equal(mine, ref)


def test_scale_recipe_ranges():
    s = synth.scales(synth.rng(1, 1), 64, 1024, synth.EXP_LOGU_M6_4)
    _, e4 = oracle.tables()
    v = e4[s]
    assert v.min() >= 2.0 ** -6 and v.max() <= 1.875 * 2.0 ** 4
    e = (s >> 3).astype(int) - 7
    assert set(np.unique(e)) == set(range(-6, 5))
    assert set(np.unique(s & 7)) == set(range(8))
