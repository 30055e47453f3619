"""CPU replay of the verify-width kernel's work plan (no GPU).

The tcgen05 kernel splits the (256-row group, pair of 64-column chunks) units
of a call contiguously over its CTAs (stream-K); a group whose units span CTAs
is finished by the last CTA to count in, which adds every contributor's
partial in CTA order.  This replays, from the library's own geometry
(nvfp4_verify_geometry), the index arithmetic each CTA runs and checks what
the kernel relies on: every unit once, in bounds copies, at most one partial
per slot and CTA, the count each group's last arriver expects, and that the
finisher reads each contributor's partial from the slot it was written to."""
import pytest

from nvfp4_weight_streaming_decode_b200 import abi

SLICES = 8   # 32-row slices per group (two 128-row MMA tiles)
SMS = 148


@pytest.fixture(scope="module")
def lib():
    from nvfp4_weight_streaming_decode_b200 import build
    build.build()
    return abi.load()


def _begin(U, T, i):
    return U * i // T


def _owner(U, T, x):
    return ((x + 1) * T - 1) // U


def _plan(M, N, K):
    st, ctas, units, nl = abi.nvfp4_verify_geometry(M, N, K, SMS)
    assert st == abi.NVFP4_OK
    n_tiles = -(-N // 32)
    n_groups = -(-n_tiles // SLICES)
    KC = -(-K // 64)
    KP = -(-KC // 2)
    assert units == n_groups * KP
    U, T = units, ctas
    covered = [0] * U
    written = {}       # (cta, slot) -> group
    contributors = {}  # group -> list of ctas
    for c in range(T):
        u0, u1 = _begin(U, T, c), _begin(U, T, c + 1)
        n = u1 - u0
        assert n >= 1
        for j in range(n):
            x = u0 + j
            covered[x] += 1
            g, pr = divmod(x, KP)
            nch = 2 if 2 * pr + 1 < KC else 1
            # the bulk copies of every slice of the group stay inside the planes and X
            for s in range(SLICES):
                t32 = g * SLICES + s
                if t32 < n_tiles:
                    assert t32 * KC + 2 * pr + nch - 1 < n_tiles * KC
            assert 2 * pr + nch - 1 < KC
            if pr == KP - 1 or j == n - 1:  # the group's end in this CTA
                ps = g * KP
                whole = ps >= u0 and ps + KP <= u1
                contributors.setdefault(g, []).append(c)
                if not whole:
                    slot = 0 if ps <= u0 else 1
                    assert (c, slot) not in written, (c, slot)
                    written[(c, slot)] = g
    assert all(v == 1 for v in covered)
    for g, cs in contributors.items():
        ps = g * KP
        glo, ghi = _owner(U, T, ps), _owner(U, T, ps + KP - 1)
        assert cs == list(range(glo, ghi + 1)), (g, cs, glo, ghi)
        if glo == ghi:
            continue
        # the last of the (ghi - glo + 1) count-ins sees ghi - glo before its own
        assert len(cs) - 1 == ghi - glo
        glo_slot = 0 if _begin(U, T, glo) >= ps else 1
        for ci in cs:
            sl = glo_slot if ci == glo else 0
            assert written.get((ci, sl)) == g, (g, ci, sl)
    return ctas, units, nl


@pytest.mark.parametrize("M", [33, 40, 48, 64])
@pytest.mark.parametrize("N,K", [(32, 64), (300, 1040), (5120, 5120), (5120, 17408), (15360, 5120),
                                 (151936, 5120), (1000, 16), (257, 8256), (4096, 64 * 149)])
def test_verify_plan(lib, M, N, K):
    ctas, units, nl = _plan(M, N, K)
    assert 1 <= ctas <= SMS


def test_verify_plan_many_shapes(lib):
    import numpy as np
    rng = np.random.default_rng(7)
    for _ in range(300):
        N = int(rng.integers(1, 40000))
        K = 16 * int(rng.integers(1, 1200))
        _plan(int(rng.integers(33, 65)), N, K)
