"""Host replay of the grouped-expert (MoE) schedule.

Device side (act_quant.cuh group_prologue_kernel, round_kernel.cuh moe_round_kernel):
the prologue turns expert offsets into tile_prefix[g] = sum over g' < g of
ceil(rows_g' / 128) and chunk_prefix[g] = sum over g' < g of ceil(tiles_g' / 2).
The persistent kernel's work items are (unit, 128-row weight band) pairs; a unit is a
chunk of up to two 128-row tiles of one expert (plain linear) or one tile (fused
SwiGLU).  Unit u belongs to the last expert e whose prefix entry is <= u (binary
search) and covers rows [offsets[e] + 128 t, offsets[e+1]) clipped to its tiles; its
scale rows are groups tile_prefix[e] + t of the grouped quantizer's padded SF layout.
These replays check, for many offset patterns (empty experts, single rows, multiples
of 128, one huge expert), that every expert row is computed exactly once, by a unit
of its own expert, that no unit reaches into another expert, and that every scale
group is read by exactly one tile.
"""
import numpy as np
import pytest


def tile_prefix(offsets):
    counts = np.diff(offsets)
    tiles = np.where(counts > 0, (counts + 127) // 128, 0)
    return np.concatenate([[0], np.cumsum(tiles)])


def owner(prefix, E, t):
    lo, hi = 0, E - 1
    while lo < hi:                       # last expert whose first tile <= t
        mid = (lo + hi + 1) >> 1
        if prefix[mid] <= t:
            lo = mid
        else:
            hi = mid - 1
    return lo


def replay(offsets):
    """Single-tile units (fused SwiGLU items)."""
    E = len(offsets) - 1
    M = int(offsets[-1])
    prefix = tile_prefix(offsets)
    assert prefix[E] <= (M + 127) // 128 + E
    cover = np.zeros(M, dtype=np.int64)
    for t in range(prefix[E]):
        e = owner(prefix, E, t)
        m0 = offsets[e] + (t - prefix[e]) * 128
        m1 = min(m0 + 128, offsets[e + 1])
        assert offsets[e] <= m0 < m1 <= offsets[e + 1], (t, e, m0, m1)
        cover[m0:m1] += 1
    assert np.all(cover == 1)


def patterns():
    yield [0, 0]
    yield [0, 1]
    yield [0, 128]
    yield [0, 129]
    yield [0, 0, 0, 5, 5, 300, 300]                        # empty experts first, between, last
    yield [0, 256, 256, 257, 1000, 1000]
    rng = np.random.default_rng(0)
    for E in (1, 2, 7, 128):
        for _ in range(20):
            counts = rng.choice([0, 0, 1, 16, 127, 128, 129, 255, 256, 1841], size=E)
            yield np.concatenate([[0], np.cumsum(counts)]).tolist()


def chunk_prefix(offsets):
    tiles = np.diff(tile_prefix(offsets))
    return np.concatenate([[0], np.cumsum((tiles + 1) // 2)])


def replay_chunks(offsets):
    """Units of up to two tiles (plain linear items): unit c belongs to the last expert e
    with chunk_prefix[e] <= c and runs the expert's tiles 2 (c - chunk_prefix[e]) and the
    next one if the expert has it, scale groups tile_prefix[e] + those tile numbers."""
    E = len(offsets) - 1
    M = int(offsets[-1])
    tp, cp = tile_prefix(offsets), chunk_prefix(offsets)
    assert cp[E] <= (M + 255) // 256 + E
    cover = np.zeros(M, dtype=np.int64)
    groups = np.zeros(tp[E], dtype=np.int64)
    for c in range(cp[E]):
        e = owner(cp, E, c)
        k = c - cp[e]
        nt = min(2, tp[e + 1] - tp[e] - 2 * k)
        assert nt >= 1, (c, e)
        for t in range(nt):
            m0 = offsets[e] + (2 * k + t) * 128
            m1 = min(m0 + 128, offsets[e + 1])
            assert offsets[e] <= m0 < m1 <= offsets[e + 1], (c, e, t, m0, m1)
            cover[m0:m1] += 1
            groups[tp[e] + 2 * k + t] += 1
    assert np.all(cover == 1)
    assert np.all(groups == 1)           # every scale group read by exactly one tile


@pytest.mark.parametrize("offsets", list(patterns()))
def test_every_row_once(offsets):
    replay(np.asarray(offsets, dtype=np.int64))


@pytest.mark.parametrize("offsets", list(patterns()))
def test_every_row_once_in_chunks(offsets):
    replay_chunks(np.asarray(offsets, dtype=np.int64))


def test_zipf_routing_of_the_moe_workload():
    from vector_quantized_mx_b200 import synth
    _, off = synth.config4_routing()
    replay(np.asarray(off, dtype=np.int64))
    replay_chunks(np.asarray(off, dtype=np.int64))
