"""CPU check of the work split of the pipelined per-channel NHWC backward
(chan_nhwc_bwd_pipe_kernel), restated from its index arithmetic:

* tiles of `consumers * UT` units; block b takes tiles b, b + grid, ... below
  piped = floor(tiles / grid) * grid, through the shared-memory stages;
* the rest of the units (the last tiles mod grid whole tiles and the partial
  tile) form rows of `consumers` units, row r going to block r mod grid,
  whose units a consumer holds in a register array of UT entries.

The kernel relies on two facts checked here over many unit counts and
grids: every unit is taken exactly once, and no block gets more than UT
rows of the remainder.
"""
import pytest


def split(nunits, consumers, ut, grid):
    tile = consumers * ut
    piped = nunits // tile // grid * grid
    r0 = piped * tile
    taken = [0] * nunits
    rows_per_block = []
    for b in range(grid):
        for t in range(b, piped, grid):
            for i in range(t * tile, (t + 1) * tile):
                taken[i] += 1
        rows = 0
        q = 0
        while r0 + (b + q * grid) * consumers < nunits:
            start = r0 + (b + q * grid) * consumers
            for i in range(start, min(start + consumers, nunits)):
                taken[i] += 1
            rows += 1
            q += 1
        rows_per_block.append(rows)
    return taken, rows_per_block


def grid_of(nunits, consumers, ut, cap=296):
    """The launcher's grid: one block per whole tile up to the cap, at least one."""
    tiles = nunits // (consumers * ut)
    return max(1, min(tiles, cap))


@pytest.mark.parametrize("consumers,ut", [(288, 4), (288, 2), (32, 4), (96, 2)])
def test_every_unit_once_and_at_most_ut_rows(consumers, ut):
    tile = consumers * ut
    cases = [1, consumers - 1, consumers, tile - 1, tile, tile + 1, 3 * tile + 7]
    cases += [k * tile + extra for k in (5, 17, 33) for extra in (0, 1, consumers, tile - 1)]
    for nunits in cases:
        for grid in {grid_of(nunits, consumers, ut, cap) for cap in (3, 8, 16)}:
            taken, rows = split(nunits, consumers, ut, grid)
            assert all(c == 1 for c in taken), (nunits, grid)
            assert max(rows) <= ut, (nunits, grid, max(rows))


def test_full_workload_shape():
    """[128, 56, 56, 144] bf16: 12,544 tiles over 296 blocks leave 112 tiles,
    448 rows: one or two per block."""
    nunits = 128 * 56 * 56 * 144 // 4
    tile = 288 * 4
    assert nunits // tile == 12544
    piped = nunits // tile // 296 * 296
    remainder_rows = (nunits - piped * tile + 287) // 288
    assert remainder_rows == 448
    assert -(-remainder_rows // 296) == 2
