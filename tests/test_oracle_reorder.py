"""Pins of the oracle's per-head reorder (PAROAttention, arXiv 2506.16054,
review key_machinery: a per-head permutation of the flattened token sequence
among the six axis orders of [F, H, W]).

Pinned against: hand-derived tables (tests/golden/orders_2x2x3.txt), brute
force enumeration with nested loops, and the identity / bijection invariants.
"""

import itertools
import os

import numpy as np
import pytest

from oracle import paro_ref as ref

GRIDS = [(2, 2, 3), (3, 4, 5), (4, 1, 6), (1, 5, 2)]


def brute_order(grid, names):
    """Natural index at each permuted position, by nested loops."""
    sizes = dict(zip("FHW", grid))
    F, H, W = grid
    seq = []
    for c in itertools.product(*[range(sizes[a]) for a in names]):
        coord = dict(zip(names, c))
        seq.append(coord["F"] * H * W + coord["H"] * W + coord["W"])
    return np.array(seq)


def test_golden_tables(golden_dir):
    rows = {}
    with open(os.path.join(golden_dir, "orders_2x2x3.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            name, *vals = line.split()
            rows[name] = np.array([int(v) for v in vals])
    assert sorted(rows) == sorted(ref.ORDER_NAMES)
    grid = (2, 2, 3)
    for pid, name in enumerate(ref.ORDER_NAMES):
        x = np.arange(12, dtype=np.float64)[:, None]
        got = ref.reorder_head(x, grid, pid, block=4)[:12, 0].astype(int)
        assert (got == rows[name]).all(), name


@pytest.mark.parametrize("grid", GRIDS)
@pytest.mark.parametrize("pid", range(6))
def test_matches_nested_loops(grid, pid):
    N = grid[0] * grid[1] * grid[2]
    x = np.arange(N, dtype=np.float64)[:, None]
    got = ref.reorder_head(x, grid, pid, block=7)[:N, 0].astype(int)
    assert (got == brute_order(grid, ref.ORDER_NAMES[pid])).all()


@pytest.mark.parametrize("grid", GRIDS)
@pytest.mark.parametrize("pid", range(6))
def test_bijection_pad_and_inverse(grid, pid):
    rng = np.random.default_rng(1)
    N = grid[0] * grid[1] * grid[2]
    d = 5
    for block in (1, 4, 7, N, N + 3):
        x = rng.standard_normal((N, d))
        xp = ref.reorder_head(x, grid, pid, block)
        nb = -(-N // block)
        assert xp.shape == (nb * block, d)
        assert (xp[N:] == 0).all()
        # each row of x appears exactly once
        perm = ref.reorder_head(np.arange(N, dtype=np.float64)[:, None], grid, pid,
                                block)[:N, 0].astype(int)
        assert sorted(perm.tolist()) == list(range(N))
        assert (ref.inverse_reorder_head(xp, grid, pid) == x).all()


def test_fhw_is_identity():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((1, 2, 60, 3))
    xp = ref.reorder(x, (3, 4, 5), [0, 0], block=16)
    assert (xp[:, :, :60] == x).all()


def test_batched_matches_per_head():
    rng = np.random.default_rng(3)
    grid = (3, 4, 5)
    x = rng.standard_normal((2, 6, 60, 4))
    perms = list(range(6))
    xp = ref.reorder(x, grid, perms, block=8)
    for b in range(2):
        for h in range(6):
            assert (xp[b, h] == ref.reorder_head(x[b, h], grid, perms[h], 8)).all()
    assert (ref.inverse_reorder(xp, grid, perms) == x).all()
