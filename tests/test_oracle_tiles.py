"""Pins of the oracle's 3D tile blockings (SPADE, arXiv 2608.03335, Pith
verdict page, key_machinery (i): spatial, temporal and mixed 3D blocking
candidates; order ids 6-11 of oracle/paro_ref.py).

* hand-derived orders on two small grids, one with partial edge tiles
  (tests/golden/tile_order_2x2x4.txt);
* an independent construction by a stable sort on the key (tile
  coordinates, then f, h, w) on ragged grids and every tile shape;
* on grids the tile divides, every block of the order is exactly one
  tile's token set;
* bijection, and inverse after forward is the identity for every id;
* SICS of a tile blocking equals the pairwise brute force over its blocks.
"""

import itertools
import os

import numpy as np
import pytest

from oracle import paro_ref as ref
from oracle import selection_ref as sel


def golden(golden_dir):
    vals = {}
    with open(os.path.join(golden_dir, "tile_order_2x2x4.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                key, *rest = line.split()
                vals[key] = [int(x) for x in rest]
    return vals


def test_tile_order_golden(golden_dir):
    g = golden(golden_dir)
    assert ref.tile_order(tuple(g["grid"]), tuple(g["tile"])).tolist() == g["order"]
    assert ref.tile_order(tuple(g["grid2"]), tuple(g["tile2"])).tolist() == g["order2"]


def sort_order(grid, shape):
    """Tokens sorted by (f // tf, h // th, w // tw, f, h, w): the tile-major
    order built by a stable sort rather than by loops."""
    F, H, W = grid
    tf, th, tw = shape
    f, h, w = np.meshgrid(np.arange(F), np.arange(H), np.arange(W), indexing="ij")
    f, h, w = f.ravel(), h.ravel(), w.ravel()
    keys = (w, h, f, w // tw, h // th, f // tf)  # np.lexsort: last key is primary
    return (f * H * W + h * W + w)[np.lexsort(keys)]


@pytest.mark.parametrize("block", [64, 128])
@pytest.mark.parametrize("grid", [(5, 7, 9), (21, 30, 52), (3, 16, 24), (17, 5, 33)])
def test_tile_order_matches_sort_construction(grid, block):
    for shape in ref.TILE_SHAPES[block]:
        assert (ref.tile_order(grid, shape) == sort_order(grid, shape)).all(), shape


@pytest.mark.parametrize("block", [64, 128])
def test_blocks_are_tiles_when_the_tile_divides_the_grid(block):
    for shape in ref.TILE_SHAPES[block]:
        tf, th, tw = shape
        grid = (2 * tf, 3 * th, 2 * tw)
        F, H, W = grid
        order = ref.tile_order(grid, shape)
        for i in range(order.size // block):
            n = order[i * block:(i + 1) * block]
            f, h, w = n // (H * W), (n // W) % H, n % W
            # one tile: each coordinate spans exactly one tile's range
            assert len(set(f // tf)) == len(set(h // th)) == len(set(w // tw)) == 1
            assert len(set(zip(f, h, w))) == block


@pytest.mark.parametrize("block", [64, 128])
def test_reorder_inverse_identity_for_every_id(block):
    rng = np.random.default_rng(7)
    grid = (3, 11, 13)
    N = 3 * 11 * 13
    x = rng.standard_normal((N, 5))
    for pid in range(ref.N_ORDERS):
        xp = ref.reorder_head(x, grid, pid, block)
        assert xp.shape[0] == -(-N // block) * block
        assert (xp[N:] == 0).all()
        assert (ref.inverse_reorder_head(xp, grid, pid, block) == x).all()
        if pid >= 6:
            order = ref.tile_order(grid, ref.TILE_SHAPES[block][pid - 6])
            assert sorted(order.tolist()) == list(range(N))  # a bijection
            assert (xp[:N] == x[order]).all()


def brute_sics(rows):
    rows = np.asarray(rows, dtype=np.float64)
    tot = 0.0
    for s, t in itertools.permutations(range(len(rows)), 2):
        ns, nt = np.linalg.norm(rows[s]), np.linalg.norm(rows[t])
        if ns > 0 and nt > 0:
            tot += float(rows[s] @ rows[t]) / (ns * nt)
    return tot


def test_sics_of_a_tile_blocking_brute_force():
    """Block 64 (so the candidates include tile ids), a small ragged grid:
    SICS of each tile candidate equals the sum over its blocks (runs of 64
    positions of the tile-major order) of the pairwise cosine sums, taken
    here over tokens listed by the sort construction."""
    rng = np.random.default_rng(11)
    grid = (3, 6, 9)
    N = 3 * 6 * 9
    x = rng.standard_normal((N, 4))
    x[5] = 0.0
    for t, shape in enumerate(ref.TILE_SHAPES[64]):
        order = sort_order(grid, shape)
        want = sum(brute_sics(x[order[i:i + 64]]) for i in range(0, N, 64))
        got = sel.sics_order(x, grid, 6 + t, 64)
        assert abs(got - want) < 1e-9 * max(1.0, abs(want)), shape


def test_candidate_names_and_counts():
    assert ref.n_candidates(128) == ref.n_candidates(64) == 12
    assert ref.n_candidates(8) == 6
    assert ref.order_name(8, 128) == "T2x8x8" and ref.order_name(0, 128) == "FHW"
    for block, shapes in ref.TILE_SHAPES.items():
        assert len(shapes) == 6 and all(a * b * c == block for a, b, c in shapes)
        assert len(set(shapes)) == 6


def test_sics_picks_the_clustered_tile_blocking_closed_form():
    """Rows equal up to scale inside each 2x8x8 tile (one random direction
    per tile): only the mixed candidate 2x8x8 (id 8 at block 128) puts every
    tile in one block, so each of its blocks has all 128 * 127 ordered pairs
    at cosine 1 and it must win; q and k add their scores."""
    F, H, W, d = 4, 16, 16, 16
    rng = np.random.default_rng(9)
    f, h, w = np.meshgrid(np.arange(F), np.arange(H), np.arange(W), indexing="ij")
    tile = (f // 2, h // 8, w // 8)
    xs = []
    for _ in range(2):
        dirs = rng.standard_normal((F // 2, H // 8, W // 8, d))
        scale = rng.uniform(0.5, 2.0, size=(F * H * W, 1))
        xs.append(dirs[tile].reshape(F * H * W, d) * scale)
    scores = np.array([sel.sics_order(xs[0], (F, H, W), o, 128)
                       + sel.sics_order(xs[1], (F, H, W), o, 128)
                       for o in range(ref.N_ORDERS)])
    nblocks = F * H * W // 128
    assert abs(scores[8] - 2 * nblocks * 128 * 127) < 1e-9 * scores[8]
    assert scores[8] > np.delete(scores, 8).max()
    assert int(np.argmax(scores)) == 8
