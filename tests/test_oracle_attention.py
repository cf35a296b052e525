"""Pins of the oracle's block-sparse attention.

* brute force: a per-row, per-key loop in the natural token order, with the
  mask found from positions computed by enumeration (no reorder, no BLAS);
* library routine: at density 1.0 the result equals
  torch.nn.functional.scaled_dot_product_attention in float64 on the CPU,
  whatever the per-head orders (dense attention does not depend on them);
* closed forms: V = 1 gives O = 1; V = identity gives the probability rows,
  which sum to 1 and are exactly 0 on masked keys; the hand-worked example in
  tests/golden/attn_2x1x2_whf.txt.

Mask semantics: SPADE (arXiv 2608.03335), review minor comment on section
2.2, Eq. (2) -- an additive mask, 0 on kept block pairs and -inf elsewhere.
"""

import math
import os

import numpy as np
import pytest
import torch

from oracle import paro_ref as ref
from test_oracle_scores import positions


def random_idx(rng, nh, nb, kmax, variable=True):
    idx = np.full((1, nh, nb, nb), -1, dtype=np.int32)
    counts = np.zeros((1, nh, nb), dtype=np.int32)
    for h in range(nh):
        for i in range(nb):
            c = int(rng.integers(1, kmax + 1)) if variable else kmax
            others = [j for j in range(nb) if j != i]
            pick = sorted([i] + list(rng.choice(others, c - 1, replace=False)))
            idx[0, h, i, :c] = pick
            counts[0, h, i] = c
    return idx, counts


def brute_attention(q, k, v, grid, perms, block, idx, counts):
    _, nh, N, d = q.shape
    out = np.zeros_like(q)
    for h in range(nh):
        blk = positions(grid, perms[h]) // block
        for r in range(N):
            kept = set(int(j) for j in idx[0, h, blk[r], :counts[0, h, blk[r]]])
            scores = {}
            for c in range(N):
                if blk[c] in kept:
                    scores[c] = sum(q[0, h, r, t] * k[0, h, c, t] for t in range(d)) / math.sqrt(d)
            m = max(scores.values())
            z = sum(math.exp(s - m) for s in scores.values())
            for t in range(d):
                out[0, h, r, t] = sum(math.exp(s - m) * v[0, h, c, t] for c, s in scores.items()) / z
    return out


@pytest.mark.parametrize("grid,block", [((2, 4, 4), 8), ((3, 2, 5), 7)])
def test_matches_brute_force(grid, block):
    rng = np.random.default_rng(21)
    N = grid[0] * grid[1] * grid[2]
    nh, d = 6, 4
    nb = -(-N // block)
    q, k, v = (rng.standard_normal((1, nh, N, d)) for _ in range(3))
    perms = list(range(6))
    idx, counts = random_idx(rng, nh, nb, max(1, nb - 1))
    got = ref.attention(q, k, v, grid, perms, block, idx, counts)
    want = brute_attention(q, k, v, grid, perms, block, idx, counts)
    assert np.abs(got - want).max() < 1e-12
    # the sampled-row evaluator agrees too
    rows = [(0, h, n) for h in range(nh) for n in range(0, N, 5)]
    sub = ref.attention_rows(q, k, v, grid, perms, block, idx, rows, counts)
    assert np.abs(sub - np.stack([want[0, h, n] for (_, h, n) in rows])).max() < 1e-12


def test_density_one_is_dense_sdpa():
    rng = np.random.default_rng(4)
    grid, block = (3, 4, 5), 8
    N, nh, d = 60, 6, 8
    nb = -(-N // block)
    q, k, v = (rng.standard_normal((1, nh, N, d)) for _ in range(3))
    idx = np.tile(np.arange(nb, dtype=np.int32), (1, nh, nb, 1))
    got = ref.attention(q, k, v, grid, list(range(6)), block, idx)
    t = lambda a: torch.from_numpy(a)
    want = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v)).numpy()
    assert np.abs(got - want).max() < 1e-12


def test_v_ones_and_identity():
    rng = np.random.default_rng(9)
    grid, block = (2, 3, 4), 5
    N, nh = 24, 3
    nb = 5
    q = rng.standard_normal((1, nh, N, 4))
    k = rng.standard_normal((1, nh, N, 4))
    idx, counts = random_idx(rng, nh, nb, 3)
    perms = [1, 3, 5]
    o = ref.attention(q, k, np.ones((1, nh, N, 4)), grid, perms, block, idx, counts)
    assert np.abs(o - 1).max() < 1e-14
    eye = np.tile(np.eye(N)[None, None], (1, nh, 1, 1))
    # d of V may differ from d of Q/K in the definition; use N columns
    p = ref.attention(q, k, eye, grid, perms, block, idx, counts)
    assert np.abs(p.sum(-1) - 1).max() < 1e-13
    for h in range(nh):
        blk = positions(grid, perms[h]) // block
        for r in range(N):
            kept = set(idx[0, h, blk[r], :counts[0, h, blk[r]]].tolist())
            for c in range(N):
                if blk[c] in kept:
                    assert p[0, h, r, c] > 0
                else:
                    assert p[0, h, r, c] == 0


def test_golden_hand_worked(golden_dir):
    vals = {}
    with open(os.path.join(golden_dir, "attn_2x1x2_whf.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            name, *rest = line.split()
            vals[name] = rest
    grid = tuple(int(x) for x in vals["grid"])
    pid = ref.ORDER_NAMES.index(vals["order"][0])
    block = int(vals["block"][0])
    N = 4
    q = np.ones((1, 1, N, 1))
    k = np.log(np.arange(1, N + 1, dtype=np.float64)).reshape(1, 1, N, 1)
    v = np.arange(1, N + 1, dtype=np.float64).reshape(1, 1, N, 1)
    idx = np.full((1, 1, 2, 2), -1, dtype=np.int32)
    counts = np.zeros((1, 1, 2), dtype=np.int32)
    for i in range(2):
        row = [int(x) for x in vals[f"idx{i}"]]
        idx[0, 0, i, :len(row)] = row
        counts[0, 0, i] = len(row)
    got = ref.attention(q, k, v, grid, [pid], block, idx, counts)[0, 0, :, 0]
    want = np.array([float(x) for x in vals["out"]])
    assert np.abs(got - want).max() < 1e-14
