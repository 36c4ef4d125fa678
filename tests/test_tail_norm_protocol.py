"""A model of the RMSNorm run in a residual GEMM's tail (the CTA-pair GEMM
with one K split and d = 1280), run under random interleavings of its
epilogue warps.

Each CTA pair walks its work units (unit = pair + k * pairs) in the order the
kernel decodes them; CTA r of the pair stores rows m0 + 128 r .. + 127 of the
256-row tile, epilogue warp w the 32 rows of group (m0 + 128 r) / 32 + (w mod
4) and half of the tile's columns (w < 4: first half).  After storing, a warp
publishes its group (one increment of that group's counter; rows past M are
not published).  Once its CTA's tiles are done, every epilogue warp takes
rows two at a time from a shared work counter and waits until their group's
counter reaches 2 x (column tiles), then normalises them.  The last CTA to
finish sets every counter back to zero.

Checks: no row is normalised before every column tile of it was stored;
every row is normalised exactly once; nothing deadlocks; the counters are
zero at the end (so the next launch starts clean).  The grouped work order
is also checked to visit every (row panel, column tile) exactly once."""
import random

import pytest

GROUP_ROWS = 4   # row panels per group of the grouped order


def _unit_coords(u, m_tiles, n_tiles, order):
    """(mt, nt) of work unit u: "m" = M-fastest, "n" = N-fastest, "g" = groups
    of GROUP_ROWS row panels, M-fastest inside a group (one K split)."""
    if order == "g":
        per = GROUP_ROWS * n_tiles
        g, r = divmod(u, per)
        gm = min(m_tiles - g * GROUP_ROWS, GROUP_ROWS)
        return g * GROUP_ROWS + r % gm, r // gm
    if order == "n":
        return u // n_tiles, u % n_tiles
    return u % m_tiles, u // m_tiles


@pytest.mark.parametrize("order", ["m", "n", "g"])
@pytest.mark.parametrize("m_tiles,n_tiles", [(1, 5), (3, 5), (5, 10), (47, 5), (6, 40), (9, 3)])
def test_unit_orders_visit_every_tile_once(order, m_tiles, n_tiles):
    seen = [_unit_coords(u, m_tiles, n_tiles, order) for u in range(m_tiles * n_tiles)]
    assert sorted(seen) == [(m, n) for m in range(m_tiles) for n in range(n_tiles)]


def _run(M, n_tiles, pairs, order, seed):
    rnd = random.Random(seed)
    m_tiles = (M + 255) // 256
    units = m_tiles * n_tiles
    ngroups = (M + 31) // 32
    target = 2 * n_tiles
    counter = [0] * ngroups
    work = [0]
    finished = [0]
    stored = {}          # (row group, column tile, half) -> stored
    normed = [0] * M
    grid = 2 * min(units, pairs)
    P = grid // 2

    # One process per epilogue warp: a list of steps, each a function that
    # returns False while it must wait.
    procs = []
    cta_left = {}   # CTA -> epilogue warps not yet done

    for cta in range(grid):
        pair, rank = divmod(cta, 2)
        tiles = [_unit_coords(u, m_tiles, n_tiles, order) for u in range(pair, units, P)]
        cta_left[cta] = 8
        for w in range(8):
            steps = []
            for mt, nt in tiles:
                grp = (mt * 256 + 128 * rank) // 32 + (w % 4)

                def store(grp=grp, nt=nt, w=w):
                    stored[(grp, nt, w // 4)] = True
                    if grp < ngroups:
                        counter[grp] += 1
                    return True
                steps.append(store)
            state = {"r0": None}

            def norm(state=state):
                if state["r0"] is None:
                    state["r0"] = work[0]
                    work[0] += 2
                r0 = state["r0"]
                if r0 >= M:
                    return True
                if counter[r0 // 32] < target:
                    return False
                for r in range(r0, min(r0 + 2, M)):
                    g = r // 32
                    assert all(stored.get((g, nt, h)) for nt in range(n_tiles) for h in (0, 1)), \
                        f"row {r} normalised before its tiles were stored"
                    normed[r] += 1
                state["r0"] = None
                return "again"

            def finish(cta=cta):
                cta_left[cta] -= 1
                return True

            def end(cta=cta):
                if cta_left[cta] > 0:      # __syncthreads of the CTA
                    return False
                finished[0] += 1
                if finished[0] == grid:    # the last CTA resets the counters
                    for g in range(ngroups):
                        counter[g] = 0
                    work[0] = 0
                    finished[0] = 0
                return True
            steps += [norm, finish]
            if w == 0:
                steps.append(end)
            procs.append(steps)

    pcs = [0] * len(procs)
    for _ in range(10 ** 7):
        live = [i for i in range(len(procs)) if pcs[i] < len(procs[i])]
        if not live:
            break
        rnd.shuffle(live)
        moved = False
        for i in live:
            r = procs[i][pcs[i]]()
            if r is True:
                pcs[i] += 1
                moved = True
                break
            if r == "again":
                moved = True
                break
        assert moved, "deadlock"
    else:
        raise AssertionError("did not finish")
    assert normed == [1] * M
    assert counter == [0] * ngroups and work[0] == 0 and finished[0] == 0


@pytest.mark.parametrize("M,n_tiles,pairs", [(1500, 5, 74), (1500, 10, 74), (12000, 5, 74), (300, 5, 3),
                                             (64, 10, 74), (4100, 5, 7)])
@pytest.mark.parametrize("order", ["m", "g"])
def test_tail_norm_waits_for_every_tile(M, n_tiles, pairs, order):
    for seed in range(3):
        _run(M, n_tiles, pairs, order, seed)
