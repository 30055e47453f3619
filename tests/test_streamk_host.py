"""CPU check of the split-K ("stream-K") work assignment the GEMM kernels use:
every unit is owned by exactly one warp, the owner formula inverts the range
formula, each partial tile's contributors are counted right, and no two
partial tiles share a counter or a partial-sum slot.  These are the integer
formulas of the kernel (range_begin / range_owner / slot choice), replayed
in Python over many grid sizes.  Also the X row each lane block loads at
widths 1..32: always a row of X, and the lane's own row where it has one."""
import itertools

import pytest


def begin(U, TW, w):
    return U * w // TW


def owner(U, TW, x):
    return ((x + 1) * TW - 1) // U


@pytest.mark.parametrize("n_tiles,k_chunks,TW", list(itertools.product(
    [1, 2, 8, 80, 160], [1, 4, 8, 40, 80, 136], [8, 64, 1184, 2368, 4736])))
def test_stream_k_assignment(n_tiles, k_chunks, TW):
    U = n_tiles * k_chunks
    TW = min(TW, max(8, -(-U // 8) * 8))          # the host never launches more CTAs than units need
    seen = [0] * U
    for w in range(TW):
        for u in range(begin(U, TW, w), begin(U, TW, w + 1)):
            seen[u] += 1
            assert owner(U, TW, u) == w
    assert all(c == 1 for c in seen)
    counters, slots = {}, {}
    for tile in range(n_tiles):
        ts, te = tile * k_chunks, (tile + 1) * k_chunks
        glo, ghi = owner(U, TW, ts), owner(U, TW, te - 1)
        contributors = [w for w in range(glo, ghi + 1) if begin(U, TW, w) < begin(U, TW, w + 1)]
        assert contributors and contributors[0] == glo and contributors[-1] == ghi
        full = len(contributors) == 1 and begin(U, TW, glo) <= ts and begin(U, TW, glo + 1) >= te
        if full:
            continue
        assert len(contributors) >= 2
        assert glo not in counters, "two partial tiles share a counter"
        counters[glo] = tile
        for w in contributors:
            slot = 0 if begin(U, TW, w) // k_chunks == tile else 1
            key = (w, slot)
            assert key not in slots, "two partial tiles share a slot"
            slots[key] = tile
            assert w < TW and slot in (0, 1)


def x_row(M, g, b):
    """Row of X that lane group g of lane block b loads in the decode kernel:
    block 0's row g % M plus the block's offset ((8b + g) % M - g % M)."""
    return g % M + ((8 * b + g) % M - g % M)


@pytest.mark.parametrize("M", range(1, 33))
def test_lane_block_x_rows_stay_inside_x(M):
    # NB = ceil(M / 8) blocks of 8 lanes; a lane whose row 8b + g is a real
    # row reads exactly that row, and every other lane reads some row of X
    # (its MMA column is dropped), never one past the last
    NB = -(-M // 8)
    for b in range(NB):
        for g in range(8):
            r = x_row(M, g, b)
            assert 0 <= r < M, (M, g, b, r)
            if 8 * b + g < M:
                assert r == 8 * b + g
