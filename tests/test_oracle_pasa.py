"""Pins of the compensated block-sparse attention oracle (PASA, arXiv
2604.12219, Pith review page, Figure 2 caption: grouped first-order
compensation of the unselected key blocks; readings P1-P3 in
oracle/pasa_ref.py).

* brute force: per row and per key, in the natural token order, with block
  membership found by enumeration and the block means summed by loops;
* library routine: with every block kept there is nothing to compensate and
  the result equals torch's scaled_dot_product_attention in float64;
* closed forms: a block whose keys are all equal and whose values are all
  equal contributes exactly n_j e^{s} v, so with such blocks the
  compensated output is dense attention exactly (ragged tail included, which
  fixes n_j); unselected blocks whose scores underflow leave the
  block-sparse output unchanged;
* the error law that makes it first order: with equal values in a block and
  keys spread by eps about their mean, the error is O(eps^2) (halving eps
  quarters it), where an expansion about any other point than the mean
  would leave an O(eps) term;
* a hand-worked example (tests/golden/pasa_2x1x2_whf.txt): 7/2 - sqrt(2)/2.
"""

import math

import numpy as np
import pytest
import torch

from oracle import paro_ref as ref
from oracle import pasa_ref as pasa
from test_oracle_attention import random_idx
from test_oracle_scores import positions


def brute_compensated(q, k, v, grid, perms, block, idx, counts):
    _, nh, N, d = q.shape
    nb = -(-N // block)
    out = np.zeros_like(q)
    for h in range(nh):
        blk = positions(grid, perms[h]) // block
        members = {j: [c for c in range(N) if blk[c] == j] for j in range(nb)}
        for r in range(N):
            kept = set(int(j) for j in idx[0, h, blk[r], :counts[0, h, blk[r]]])
            terms = []  # (log weight, value vector)
            for j in range(nb):
                keys = members[j]
                if not keys:
                    continue
                if j in kept:
                    for c in keys:
                        s = sum(q[0, h, r, t] * k[0, h, c, t] for t in range(d)) / math.sqrt(d)
                        terms.append((s, [v[0, h, c, t] for t in range(d)]))
                else:
                    kb = [sum(k[0, h, c, t] for c in keys) / len(keys) for t in range(d)]
                    vb = [sum(v[0, h, c, t] for c in keys) / len(keys) for t in range(d)]
                    s = sum(q[0, h, r, t] * kb[t] for t in range(d)) / math.sqrt(d)
                    terms.append((s + math.log(len(keys)), vb))
            m = max(s for s, _ in terms)
            z = sum(math.exp(s - m) for s, _ in terms)
            for t in range(d):
                out[0, h, r, t] = sum(math.exp(s - m) * vv[t] for s, vv in terms) / z
    return out


@pytest.mark.parametrize("grid,block", [((2, 4, 4), 8), ((3, 2, 5), 7)])
def test_matches_brute_force(grid, block):
    rng = np.random.default_rng(41)
    N = grid[0] * grid[1] * grid[2]
    nh, d = 6, 4
    nb = -(-N // block)
    q, k, v = (rng.standard_normal((1, nh, N, d)) for _ in range(3))
    perms = list(range(6))
    idx, counts = random_idx(rng, nh, nb, max(1, nb - 2))
    got = pasa.attention_compensated(q, k, v, grid, perms, block, idx, counts)
    want = brute_compensated(q, k, v, grid, perms, block, idx, counts)
    assert np.abs(got - want).max() < 1e-12


def sdpa(q, k, v):
    return torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q), torch.from_numpy(k), torch.from_numpy(v)).numpy()


def test_all_blocks_kept_is_dense_attention():
    rng = np.random.default_rng(42)
    grid, block = (3, 4, 5), 8  # N = 60, ragged tail of 4
    N, nh, d = 60, 6, 8
    nb = 8
    q, k, v = (rng.standard_normal((1, nh, N, d)) for _ in range(3))
    idx = np.tile(np.arange(nb, dtype=np.int32), (1, nh, nb, 1))
    got = pasa.attention_compensated(q, k, v, grid, list(range(6)), block, idx)
    assert np.abs(got - sdpa(q, k, v)).max() < 1e-12


def constant_block_inputs(rng, grid, perms, block, d, spread=0.0, equal_values=True):
    """Natural-order q, k, v whose permuted blocks have equal keys (plus
    spread * a zero-mean deviation) and, if equal_values, equal values."""
    F, H, W = grid
    N = F * H * W
    nb = -(-N // block)
    nh = len(perms)
    q = rng.standard_normal((1, nh, N, d))
    k = np.zeros((1, nh, N, d))
    v = np.zeros((1, nh, N, d))
    for h, pid in enumerate(perms):
        kp = np.zeros((nb * block, d))
        vp = np.zeros((nb * block, d))
        for j in range(nb):
            lo, hi = j * block, min((j + 1) * block, N)
            dev = rng.standard_normal((hi - lo, d))
            dev -= dev.mean(axis=0)  # zero mean: kbar_j is the expansion point
            kp[lo:hi] = rng.standard_normal(d) + spread * dev
            vp[lo:hi] = rng.standard_normal(d) if equal_values else rng.standard_normal((hi - lo, d))
        k[0, h] = ref.inverse_reorder_head(kp, grid, pid)
        v[0, h] = ref.inverse_reorder_head(vp, grid, pid)
    return q, k, v


@pytest.mark.parametrize("grid,block", [((2, 4, 4), 8), ((3, 3, 5), 8)])
def test_equal_keys_and_values_make_it_exact(grid, block):
    rng = np.random.default_rng(43)
    perms = [0, 3, 5]
    N = grid[0] * grid[1] * grid[2]
    nb = -(-N // block)
    q, k, v = constant_block_inputs(rng, grid, perms, block, 8)
    idx, counts = random_idx(rng, len(perms), nb, 2)
    got = pasa.attention_compensated(q, k, v, grid, perms, block, idx, counts)
    assert np.abs(got - sdpa(q, k, v)).max() < 1e-12
    # and the uncompensated block-sparse output is not dense attention here
    plain = ref.attention(q, k, v, grid, perms, block, idx, counts)
    assert np.abs(plain - sdpa(q, k, v)).max() > 1e-3


def test_error_is_second_order_in_the_key_spread():
    rng = np.random.default_rng(44)
    grid, block, perms, d = (2, 4, 4), 8, [1, 4], 8
    nb = 4
    errs = []
    for eps in (0.04, 0.02, 0.01):
        q, k, v = constant_block_inputs(np.random.default_rng(45), grid, perms, block, d,
                                        spread=eps)
        idx, counts = random_idx(np.random.default_rng(46), len(perms), nb, 2)
        got = pasa.attention_compensated(q, k, v, grid, perms, block, idx, counts)
        errs.append(np.abs(got - sdpa(q, k, v)).max())
    assert errs[0] > 1e-7
    for a, b in zip(errs, errs[1:]):
        assert 3.6 < a / b < 4.4, errs


def test_underflowing_unselected_blocks_leave_sparse_output():
    # every query is the same vector u; unselected blocks' keys point along -u
    # far enough that exp of their mean score underflows to 0 in float64
    rng = np.random.default_rng(47)
    grid, block, d = (2, 4, 4), 8, 8
    N, nb = 32, 4
    u = rng.standard_normal(d)
    u /= np.linalg.norm(u)
    qp = np.tile(u, (N, 1))
    kp = rng.standard_normal((N, d))
    vp = rng.standard_normal((N, d))
    for j in (1, 3):
        kp[j * block:(j + 1) * block] = -3000.0 * u + 0.1 * rng.standard_normal((block, d))
    idx = np.tile(np.array([0, 2], dtype=np.int32), (nb, 1))
    got = pasa.compensated_permuted(qp, kp, vp, N, block, idx)
    want = ref.attention_permuted(qp, kp, vp, N, block, idx)
    assert np.abs(got - want).max() < 1e-12


def test_block_counts_ragged_tail():
    assert pasa.block_counts(60, 8, 8).tolist() == [8] * 7 + [4]
    assert pasa.block_counts(64, 8, 8).tolist() == [8] * 8


@pytest.mark.parametrize("grid,block", [((2, 4, 4), 8), ((3, 2, 5), 7)])
def test_row_evaluator_matches_whole_head(grid, block):
    rng = np.random.default_rng(48)
    N = grid[0] * grid[1] * grid[2]
    nh, d = 3, 4
    nb = -(-N // block)
    q, k, v = (rng.standard_normal((2, nh, N, d)) for _ in range(3))
    perms = [0, 4, 5]
    idx = np.full((2, nh, nb, nb), -1, dtype=np.int32)
    counts = np.zeros((2, nh, nb), dtype=np.int32)
    for b in range(2):
        i1, c1 = random_idx(rng, nh, nb, max(1, nb - 2))
        idx[b], counts[b] = i1[0], c1[0]
    counts[1, 2, 0] = 0  # an empty kept list: compensation alone
    whole = pasa.attention_compensated(q, k, v, grid, perms, block, idx, counts)
    rows = [(b, h, n) for b in range(2) for h in range(nh) for n in range(N)]
    got = pasa.compensated_rows(q, k, v, grid, perms, block, idx, rows, counts)
    want = np.stack([whole[b, h, n] for (b, h, n) in rows])
    assert np.abs(got - want).max() < 1e-12


def test_golden_hand_worked():
    import os
    vals = {}
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden",
                        "pasa_2x1x2_whf.txt")
    with open(path) as f:
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
    got = pasa.attention_compensated(q, k, v, grid, [pid], block, idx, counts)[0, 0, :, 0]
    want = np.array([float(x) for x in vals["out"]])
    assert np.abs(got - want).max() < 1e-14
    assert abs(want[0] - (3.5 - math.sqrt(2) / 2)) < 1e-15
