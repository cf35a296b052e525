"""Pins of the oracle's top-k block selection (PASA, arXiv 2604.12219,
Figure 2: each query block keeps at most k key blocks; SPADE, arXiv
2608.03335, review core_discovery: Top-K filter) and of the static-mask
bitmask format (PAROAttention, arXiv 2506.16054, review key_machinery:
static masks stored as bitmasks).

Brute force: a greedy pure-Python selection that repeatedly takes the best
remaining block under the stated order (diagonal first, then score
descending, then lower index), and an exhaustive search over all subsets on
tiny rows.
"""

import itertools
import math

import numpy as np
import pytest

from oracle import paro_ref as ref


def key(s, j):
    v = s[j]
    if math.isnan(v):
        v = -math.inf
    return (v, -j)


def greedy(s, i, k):
    nb = len(s)
    chosen = [i]
    rest = [j for j in range(nb) if j != i]
    while len(chosen) < min(k, nb):
        best = rest[0]
        for j in rest[1:]:
            if key(s, j) > key(s, best):
                best = j
        chosen.append(best)
        rest.remove(best)
    return sorted(chosen)


def exhaustive(s, i, k):
    nb = len(s)
    best, best_keys = None, None
    for sub in itertools.combinations([j for j in range(nb) if j != i], min(k, nb) - 1):
        keys = sorted((key(s, j) for j in sub), reverse=True)
        if best is None or keys > best_keys:
            best, best_keys = sub, keys
    return sorted((i,) + best)


@pytest.mark.parametrize("nb", [1, 2, 5, 8])
def test_matches_brute_force(nb):
    rng = np.random.default_rng(nb)
    for trial in range(40):
        if trial % 2:
            s = rng.integers(-2, 3, size=nb).astype(np.float64)  # many ties
        else:
            s = rng.standard_normal(nb)
        if trial % 5 == 0 and nb > 2:
            s[rng.integers(nb)] = np.nan
        if trial % 7 == 0 and nb > 1:
            s[rng.integers(nb)] = -np.inf
        for i in range(nb):
            for k in range(1, nb + 1):
                got = ref.select_topk_row(s, i, k).tolist()
                assert got == greedy(s, i, k)
                if nb <= 6:
                    assert got == exhaustive(s, i, k)


def test_invariants_and_ties():
    rng = np.random.default_rng(11)
    nb, k = 37, 9
    s = rng.integers(0, 4, size=(1, 2, nb, nb)).astype(np.float64)
    s[0, 0, 3, 5] = -0.0
    s[0, 0, 3, 4] = 0.0
    idx = ref.select_topk(s, k)
    assert idx.shape == (1, 2, nb, k) and idx.dtype == np.int32
    for h in range(2):
        for i in range(nb):
            row = idx[0, h, i]
            assert len(set(row.tolist())) == k
            assert (np.diff(row) > 0).all()
            assert i in row
            # every unchosen block is worse than every chosen non-diagonal one
            chosen = [j for j in row if j != i]
            worst = min(key(s[0, h, i], j) for j in chosen)
            for j in range(nb):
                if j not in row:
                    assert key(s[0, h, i], j) < worst


def test_signed_zero_is_a_tie():
    s = np.array([5.0, -0.0, 0.0, -1.0])
    assert ref.select_topk_row(s, 0, 2).tolist() == [0, 1]
    s = np.array([5.0, 0.0, -0.0, -1.0])
    assert ref.select_topk_row(s, 0, 2).tolist() == [0, 1]


def test_k_for_density_values():
    # NB and k of the five workloads: ceil(density * NB)
    assert ref.k_for_density(4, 0.5) == 2
    assert ref.k_for_density(32, 0.30) == 10
    assert ref.k_for_density(256, 0.25) == 64
    assert ref.k_for_density(591, 0.15) == 89
    assert ref.k_for_density(929, 0.20) == 186
    assert ref.k_for_density(591, 1.0) == 591
    assert ref.k_for_density(10, 0.3) == 3  # 0.3*10 is 3.0000000000000004 in binary
    assert ref.k_for_density(100, 1e-6) == 1
    assert ref.k_for_density(7, 3.0) == 7


def test_bitmask_round_trip():
    rng = np.random.default_rng(5)
    nb = 70
    idx = np.zeros((1, 2, nb, 12), dtype=np.int32)
    for h in range(2):
        for i in range(nb):
            idx[0, h, i] = np.sort(rng.choice(nb, 12, replace=False))
    bm = ref.bitmask_from_idx(idx, nb)
    assert bm.shape == (1, 2, nb, 3) and bm.dtype == np.uint32
    # word/bit layout: bit j%32 of word j//32
    j = int(idx[0, 1, 4, 0])
    assert (int(bm[0, 1, 4, j // 32]) >> (j % 32)) & 1
    full, counts = ref.compact_mask(bm, nb)
    assert (counts == 12).all()
    assert (full[..., :12] == idx).all()
    assert (full[..., 12:] == -1).all()
