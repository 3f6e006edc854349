"""Layout properties of the decode kernel's shared-memory reads, checked on the host.

A tile's weights sit in shared memory as [unit pair][16 rows][128 B], written by TMA with
the 128-byte swizzle (16-byte chunk c of the 128-byte line of row r lands at chunk
c ^ (r % 8)). Lane (g = lane / 4, t = lane % 4) of a warp reads, for its unit slot, the
16 bytes at chunk t of the unit's half-line in rows gr and gr + 8 of the tile. A 128-bit
shared load serves 8 lanes per wavefront, and is one wavefront per quarter-warp only when
those 8 addresses fall in 8 different 16-byte bank groups."""
import pytest


def swz128(lin):
    return lin ^ ((lin >> 3) & 0x70)


def wavefronts(row_of_g, us, hi):
    worst = 0
    for quarter in range(4):
        lanes = range(8 * quarter, 8 * quarter + 8)
        groups = {}
        for lane in lanes:
            g, t = lane >> 2, lane & 3
            row = row_of_g(g) + (8 if hi else 0)
            lin = ((us >> 1) * 16 + row) * 128 + (us & 1) * 64 + 16 * t
            addr = swz128(lin)
            groups.setdefault((addr >> 4) & 7, set()).add(addr)
        worst = max(worst, max(len(v) for v in groups.values()))
    return worst


@pytest.mark.parametrize("us", range(16))
@pytest.mark.parametrize("hi", [False, True])
def test_permuted_rows_make_weight_loads_conflict_free(us, hi):
    # MMA row g reads tile row (g >> 1) | ((g & 1) << 2): a quarter-warp reads rows q, q + 4
    assert wavefronts(lambda g: (g >> 1) | ((g & 1) << 2), us, hi) == 1


@pytest.mark.parametrize("us", range(16))
def test_identity_rows_would_conflict(us):
    # rows g and g + 1 of a quarter-warp share a bank half under the swizzle: 2-way conflict
    assert wavefronts(lambda g: g, us, False) == 2


def test_permutation_covers_each_row_once():
    rows = sorted((g >> 1) | ((g & 1) << 2) for g in range(8))
    assert rows == list(range(8))
