"""Host checks of the split-K work layouts of the output projection and the down-projection + append
(out_proj.cuh, down_proj.cuh): U units laid out M tile by M tile, CTA c of G takes units
[floor(c U / G), floor((c + 1) U / G)), its partial of each M tile it touches goes to slot c (its
first segment) or G_max + m - 1 (the segment of tile m it starts after crossing into it), and the
sum kernel reads the partials of tile m from CTAs ceil((u + 1) G / U) - 1 for the tile's first and
last units.  These are the invariants the kernels rely on: every unit belongs to exactly one CTA,
a CTA crosses at most one tile boundary (two TMEM segments), the CTAs of a tile fit the sum
kernel's unrolled loads, and no two segments share a slot."""
import pytest

# (units, units per M tile, largest G, the sum kernel's CTA cap), as the kernels define them
LAYOUTS = {
    "output projection, 256-row units": (2560, 128, 160, 16),
    "output projection, 128-row units": (2560, 64, 160, 16),
    "down-projection + append": (200, 40, 100, 22),
}


def unit0(c, G, U):
    return c * U // G


def cta_of(u, G, U):
    return ((u + 1) * G + U - 1) // U - 1


@pytest.mark.parametrize("name", sorted(LAYOUTS))
def test_split_layout_invariants(name):
    U, per_tile, g_max, cap = LAYOUTS[name]
    tiles = U // per_tile
    g_min = max(tiles, -(-U // per_tile))   # the launchers' lower bound on G
    for G in range(g_min, g_max + 1):
        owner = {}
        slots = {}
        for c in range(G):
            u0, u1 = unit0(c, G, U), unit0(c + 1, G, U)
            for u in range(u0, u1):
                assert u not in owner
                owner[u] = c
            if u1 == u0:
                continue
            m_first, m_last = u0 // per_tile, (u1 - 1) // per_tile
            assert m_last - m_first <= 1, (name, G, c)
            for seg, m in enumerate(range(m_first, m_last + 1)):
                slot = c if seg == 0 else g_max + m - 1
                assert slot not in slots, (name, G, c, m)
                slots[slot] = (c, m)
        assert sorted(owner) == list(range(U))
        for m in range(tiles):
            lo, hi = cta_of(m * per_tile, G, U), cta_of(m * per_tile + per_tile - 1, G, U)
            assert lo == owner[m * per_tile] and hi == owner[m * per_tile + per_tile - 1]
            assert hi - lo + 1 <= cap, (name, G, m)
            # the segment index the sum kernel computes for each contributing CTA names its slot
            for c in range(lo, hi + 1):
                seg = m - unit0(c, G, U) // per_tile
                slot = c if seg == 0 else g_max + m - 1
                assert slots[slot] == (c, m)
