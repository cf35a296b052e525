"""Pins of the oracle's mean-pooled block scores (SPADE, arXiv 2608.03335,
review: MEAN summariser and intra-estimation from block summaries).

Closed form: by bilinearity, q_bar_i . k_bar_j / sqrt(d) equals the mean of
the dense score matrix Q K^T / sqrt(d) over the valid rows of query block i
and the valid columns of key block j.  The dense matrix is computed here by
explicit loops over the natural-order tokens, using positions found by
enumeration, so the pin does not reuse the oracle's reorder.
"""

import itertools
import math

import numpy as np
import pytest

from oracle import paro_ref as ref


def positions(grid, pid):
    """Permuted position of every natural token, by enumeration."""
    F, H, W = grid
    names = ref.ORDER_NAMES[pid]
    sizes = dict(zip("FHW", grid))
    pos = np.empty(F * H * W, dtype=int)
    for p, c in enumerate(itertools.product(*[range(sizes[a]) for a in names])):
        co = dict(zip(names, c))
        pos[co["F"] * H * W + co["H"] * W + co["W"]] = p
    return pos


@pytest.mark.parametrize("grid,block", [((2, 3, 5), 4), ((3, 4, 4), 8), ((2, 2, 2), 3)])
def test_pooled_score_is_tile_mean(grid, block):
    rng = np.random.default_rng(7)
    N = grid[0] * grid[1] * grid[2]
    nh, d = 6, 6
    q = rng.standard_normal((1, nh, N, d))
    k = rng.standard_normal((1, nh, N, d))
    perms = list(range(6))
    qb, kb, s = ref.pooled_scores(q, k, grid, perms, block)
    nb = -(-N // block)
    assert s.shape == (1, nh, nb, nb)
    for h in range(nh):
        pos = positions(grid, perms[h])
        blk = pos // block
        dense = np.zeros((N, N))
        for r in range(N):
            for c in range(N):
                dense[r, c] = sum(q[0, h, r, t] * k[0, h, c, t] for t in range(d)) / math.sqrt(d)
        for i in range(nb):
            for j in range(nb):
                tile = dense[np.ix_(blk == i, blk == j)]
                assert abs(tile.mean() - s[0, h, i, j]) < 1e-12


def test_pool_uses_valid_rows_only():
    # 5 tokens, block 4: the last block holds one real row and 3 pad rows
    x = np.arange(5, dtype=np.float64).reshape(1, 1, 5, 1) + 1.0
    xp = ref.reorder(x, (1, 1, 5), [0], block=4)
    pooled = ref.block_pool(xp, 5, 4)
    assert pooled[0, 0, 0, 0] == 2.5
    assert pooled[0, 0, 1, 0] == 5.0


def test_constant_block_pools_to_constant():
    x = np.full((1, 1, 24, 3), 0.75)
    xp = ref.reorder(x, (2, 3, 4), [5], block=8)
    assert (ref.block_pool(xp, 24, 8) == 0.75).all()
