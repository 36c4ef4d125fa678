"""The windowed attention kernel's schedule, restated and checked on the CPU.

The kernel deals "pair items" (two neighbouring 128-query tiles 2p, 2p+1 of
one clip and head) to its persistent CTAs round by round, heaviest pairs
first, in alternating directions; each query tile visits the 64-key tiles
kt0 .. kt0 + n - 1, and the pair's K/V ring carries their union once.
Checked for many (T, W, B, H, grid): every (clip, head, query tile) is
processed exactly once; the visited key tiles hold every key of every row's
window (i - W < j <= i, causal) and each of them holds a key of some row's
window; the union range covers both tiles' ranges with no gap; the rounds
are dealt heaviest first.  The streaming kernel's slot-order mask over the
ring is checked against the window rule as well."""
import pytest

KEY_TILE = 64


def _pair_item(T, W, p):
    """(q0, kt0, n) of the two query tiles of pair p (q0 = -1: no tile), and
    the union's first key tile and tile count."""
    tiles = []
    for X in range(2):
        q0 = (2 * p + X) * 128
        if q0 >= T:
            tiles.append((-1, 0, 0))
            continue
        kt0 = max(0, q0 - W + 1) // KEY_TILE
        n = min(T - 1, q0 + 127) // KEY_TILE - kt0 + 1
        tiles.append((q0, kt0, n))
    u0 = tiles[0][1]
    end = tiles[1][1] + tiles[1][2] if tiles[1][2] > 0 else tiles[0][1] + tiles[0][2]
    return tiles, u0, end - u0


def _deal(B, H, T, grid):
    """Items of each CTA in processing order: (clip, head, pair)."""
    np_ = ((T + 127) // 128 + 1) // 2
    n_items = np_ * H * B
    out = [[] for _ in range(grid)]
    for x in range(grid):
        r = 0
        while True:
            pos = r * grid + (grid - 1 - x if r & 1 else x)
            if pos >= n_items:
                break
            rest = pos % (H * B)
            out[x].append((rest // H, rest % H, np_ - 1 - pos // (H * B)))
            r += 1
    return out


@pytest.mark.parametrize("B,H,T,grid", [(1, 2, 64, 148), (1, 32, 1500, 148), (8, 32, 6000, 148), (2, 3, 1000, 7),
                                        (1, 1, 129, 1), (3, 5, 4097, 148), (4, 32, 3000, 148)])
def test_every_query_tile_once(B, H, T, grid):
    seen = {}
    for items in _deal(B, H, T, grid):
        for b, h, p in items:
            tiles, _, _ = _pair_item(T, 16, p)
            for X, (q0, _, _) in enumerate(tiles):
                if q0 >= 0:
                    key = (b, h, q0 // 128)
                    assert key not in seen, f"query tile {key} dealt twice"
                    seen[key] = True
    n_qt = (T + 127) // 128
    assert len(seen) == B * H * n_qt


@pytest.mark.parametrize("B,H,T,grid", [(1, 32, 1500, 148), (8, 32, 6000, 148), (2, 3, 1000, 7)])
def test_rounds_are_heaviest_first(B, H, T, grid):
    # A pair's key-tile count never decreases with its index, and every CTA
    # takes pairs in non-increasing index order.
    for items in _deal(B, H, T, grid):
        ps = [p for _, _, p in items]
        assert ps == sorted(ps, reverse=True)


@pytest.mark.parametrize("W", [1, 16, 63, 64, 65, 128, 191, 192, 750, 5000])
@pytest.mark.parametrize("T", [1, 64, 127, 128, 129, 300, 1500, 3000])
def test_key_tiles_cover_exactly_the_windows(T, W):
    for p in range((((T + 127) // 128) + 1) // 2):
        tiles, u0, nu = _pair_item(T, W, p)
        covered = set()
        for q0, kt0, n in tiles:
            if q0 < 0:
                assert n == 0
                continue
            covered |= set(range(kt0, kt0 + n))
            lo, hi = kt0 * KEY_TILE, (kt0 + n) * KEY_TILE
            rows = range(q0, min(q0 + 128, T))
            for i in rows:   # every key of the row's window is visited
                assert lo <= max(0, i - W + 1) and i < hi
            for t in range(kt0, kt0 + n):   # every visited tile is needed by some row
                assert any(max(0, i - W + 1) < (t + 1) * KEY_TILE and i >= t * KEY_TILE for i in rows)
        assert covered == set(range(u0, u0 + nu)), "the union has a gap or extra tiles"


@pytest.mark.parametrize("W", [1, 2, 5, 16, 64, 65, 750])
def test_ring_slot_mask_is_the_window(W):
    # The streaming kernel walks the ring in slot order and keeps slot j as a
    # key of new frame p + r (r < n_new) iff j < min(p, W), d >= r + 1 and
    # p - W + d >= 0, with d = (j - p) mod W.  By the ring rule (frame f in
    # slot f mod W, frames max(0, p - W) .. p - 1 cached) that must be the set
    # of cached frames in the window of p + r: p + r - W < f <= p + r, f < p.
    for p in list(range(0, 3 * W + 3)) + [1000, 1003]:
        nslots = min(p, W)
        cached = {f % W: f for f in range(max(0, p - W), p)}
        for r in range(8):
            got = set()
            for j in range(W):
                d = (j - p) % W
                if j < nslots and d >= r + 1 and p - W + d >= 0:
                    got.add(p - W + d)
                    assert cached.get(j) == p - W + d, "slot holds another frame"
            want = {f for f in cached.values() if p + r - W < f <= p + r}
            assert got == want, (p, r)
