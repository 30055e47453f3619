"""Pins of the oracle's top-k (ignis README, "What sets it apart",
"Speculative decoding (DFlash2)": the row-split top-k after the output head).

The oracle is checked against hand-derived cases (tests/golden/topk_cases.txt),
against numpy's lexsort and stable argsort on finite data, against closed forms
(constant rows, k = V), and against the defining invariants of a top-k."""
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "topk_cases.txt")


def _cases():
    out = []
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        k, bits, exp = (p.strip() for p in line.split(";"))
        row = np.array([int(b, 16) for b in bits.split()], np.uint32).view(np.float32)
        out.append((int(k), row, [int(e) for e in exp.split()]))
    return out


@pytest.mark.parametrize("case", range(len(_cases())))
def test_golden_cases(case):
    k, row, expect = _cases()[case]
    vals, idx = oracle.topk(row[None, :], k)
    assert idx[0].tolist() == expect
    # values are the inputs at those indices, bit for bit
    assert np.array_equal(vals[0].view(np.uint32), row[expect].view(np.uint32))


@pytest.mark.parametrize("M,V,k", [(1, 1000, 1), (3, 4099, 7), (8, 20000, 8), (2, 513, 64), (5, 64, 64)])
def test_matches_numpy_lexsort(M, V, k):
    rng = np.random.default_rng(M * 7919 + V)
    # coarse values so that ties occur, plus a continuous part
    x = np.where(rng.random((M, V)) < 0.5, rng.integers(-20, 20, (M, V)) / 4.0,
                 rng.standard_normal((M, V))).astype(np.float32)
    vals, idx = oracle.topk(x, k)
    for m in range(M):
        order = np.lexsort((np.arange(V), -x[m].astype(np.float64)))[:k]
        assert idx[m].tolist() == order.tolist()
        assert np.array_equal(vals[m], x[m][order])


def test_full_sort_is_stable_argsort():
    rng = np.random.default_rng(3)
    x = (rng.integers(-5, 5, 300) / 2.0).astype(np.float32)
    x[::7] = -0.0
    vals, idx = oracle.topk(x[None, :], 300)
    ref = np.argsort(-x.astype(np.float64), kind="stable")
    assert idx[0].tolist() == ref.tolist()


def test_constant_row_takes_lowest_indices():
    x = np.full((4, 1000), 1.25, np.float32)
    vals, idx = oracle.topk(x, 17)
    assert (idx == np.arange(17)).all() and (vals == 1.25).all()


def test_columns_past_v_are_ignored():
    rng = np.random.default_rng(5)
    x = rng.standard_normal((3, 128)).astype(np.float32)
    x[:, 100:] = 1e30
    vals, idx = oracle.topk(x, 5, V=100)
    assert (idx < 100).all()
    ref_vals, ref_idx = oracle.topk(np.ascontiguousarray(x[:, :100]), 5)
    assert np.array_equal(idx, ref_idx) and np.array_equal(vals, ref_vals)


def test_invariants_on_large_row():
    rng = np.random.default_rng(11)
    V, k = 151936, 64
    x = rng.standard_normal((2, V)).astype(np.float32)
    vals, idx = oracle.topk(x, k)
    for m in range(2):
        assert len(set(idx[m].tolist())) == k
        assert np.all(np.diff(vals[m].astype(np.float64)) <= 0)
        rest = np.delete(x[m], idx[m])
        assert rest.max() <= vals[m][-1]
        assert np.array_equal(x[m][idx[m]], vals[m])


@pytest.mark.parametrize("k,V,ldv", [(0, 10, 10), (11, 10, 10), (1, 10, 9)])
def test_bad_arguments(k, V, ldv):
    x = np.zeros((1, max(ldv, 1)), np.float32)
    with pytest.raises(ValueError):
        oracle.topk(x[:, :ldv] if ldv < x.shape[1] else x, k, V=V)
