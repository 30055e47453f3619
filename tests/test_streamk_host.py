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


def _combine_plan(n_tiles, k_chunks, TW, W, POOL):
    """Replay, for every warp, what the decode kernel does when it is done
    with its part of a tile (the flush site and finish_tile), in the kernel's
    integer formulas.  Returns the writes (location -> (tile, writer)), the
    epilogues run per tile, and the reads and waits of every finisher."""
    U = n_tiles * k_chunks

    def cta_range(c):
        return begin(U, TW, c * W), begin(U, TW, min((c + 1) * W, TW))

    def cta_slot(c, tile):
        _, uc1 = cta_range(c)
        return ("slot", c * W + (0 if tile == (uc1 - 1) // k_chunks else 1), 1)

    writes, epilogues, finishes = {}, {}, []

    def write(loc, tile, gw):
        assert loc not in writes, f"{loc} written twice"
        writes[loc] = (tile, gw)

    for gw in range(TW):
        c = gw // W
        uc, uc1 = cta_range(c)
        u0, u1 = begin(U, TW, gw), begin(U, TW, gw + 1)
        for tile in sorted({u // k_chunks for u in range(u0, u1)}):
            ts, te = tile * k_chunks, (tile + 1) * k_chunks
            a, b = max(ts, uc), min(te, uc1)
            alone = a >= u0 and b <= u1
            if alone and ts >= uc and te <= uc1:
                epilogues[tile] = epilogues.get(tile, 0) + 1
            elif u1 > b:                       # leaves the tile in mid-range
                ps = tile - uc // k_chunks     # its slot in the CTA's shared-memory pool
                if alone:
                    write(cta_slot(c, tile), tile, gw)
                elif ps < POOL:
                    write(("pool", c, ps), tile, gw)
                else:
                    write(("slot", gw, 0), tile, gw)
            else:                              # its range ends in the tile
                write(("ring", gw), tile, gw)
                whi = owner(U, TW, b - 1)
                fin = whi - 1 if begin(U, TW, whi + 1) > b else whi
                if gw != fin:
                    continue
                wlo = owner(U, TW, a)
                reads, waits = [], []
                for v in range(wlo, whi + 1):
                    if v == whi and begin(U, TW, whi + 1) > b:
                        ps = tile - uc // k_chunks
                        reads.append(("pool", c, ps) if ps < POOL else ("slot", whi, 0))
                    else:
                        reads.append(("ring", v))
                        if v != gw:
                            waits.append(v)              # its shared-memory flag
                clo, chi = owner(U, TW, ts) // W, owner(U, TW, te - 1) // W
                if clo != chi and c != clo:
                    write(cta_slot(c, tile), tile, gw)
                else:
                    if clo != chi:
                        reads += [cta_slot(cc, tile) for cc in range(clo + 1, chi + 1)]
                    epilogues[tile] = epilogues.get(tile, 0) + 1
                finishes.append((tile, gw, reads, waits))
    return U, writes, epilogues, finishes


@pytest.mark.parametrize("n_tiles,k_chunks,TW,W,POOL", [c[:4] + (p,) for c in itertools.product(
    [1, 3, 8, 80, 160, 480], [1, 2, 8, 40, 80, 272], [8, 64, 1184, 2368], [16, 12, 8]) for p in (0, 2, 8)])
def test_designated_finisher_plan(n_tiles, k_chunks, TW, W, POOL):
    U = n_tiles * k_chunks
    ctas = min(-(-U // W), max(1, TW // W))
    TW = min(ctas * W, U)
    U, writes, epilogues, finishes = _combine_plan(n_tiles, k_chunks, TW, W, POOL)
    # every tile is finished exactly once
    assert sorted(epilogues) == list(range(n_tiles)) and all(n == 1 for n in epilogues.values()), epilogues
    for tile, gw, reads, waits in finishes:
        for loc in reads:
            assert loc in writes and writes[loc][0] == tile, (tile, gw, loc)
        # a finisher waits only for warps whose range ends in the tile and that finish nothing themselves
        for v in waits:
            assert writes.get(("ring", v)) == (tile, v)
            assert all(f[1] != v for f in finishes)
    # every partial published in the workspace is read by exactly one finisher
    readers = {}
    for tile, gw, reads, _ in finishes:
        for loc in reads:
            readers[loc] = readers.get(loc, 0) + 1
    for loc, (tile, gw) in writes.items():
        if loc[0] in ("slot", "pool"):
            assert readers.get(loc) == 1, (loc, tile, gw)
        if loc[0] == "slot":
            assert loc[1] < -(-TW // W) * W    # inside the grid's slots
        if loc[0] == "pool":
            assert 0 <= loc[2] < POOL
