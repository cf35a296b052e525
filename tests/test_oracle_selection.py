"""Pins of the selection-variant oracle (SPADE, arXiv 2608.03335, Pith
verdict page: SICS blocking score, key_machinery (ii) and the note on
Eq. (5); Top-K / Top-P and local-window filters, core_discovery).

SICS: brute force over ordered pairs of rows, closed forms (one direction ->
n(n-1); orthonormal rows -> 0), scale invariance, and a grid built so that
exactly the frame-major orders put each frame into one block.
Top-P: brute force from the definition (explicit normalised softmax and a
scan for the shortest prefix), the limits p -> 0 and p = 1, ties, and the
non-finite conventions.  Hybrid: union and order invariants.
"""

import itertools
import math

import numpy as np
import pytest

from oracle import paro_ref as ref
from oracle import selection_ref as sel


def brute_sics(rows):
    rows = np.asarray(rows, dtype=np.float64)
    tot = 0.0
    for s, t in itertools.permutations(range(len(rows)), 2):
        ns, nt = np.linalg.norm(rows[s]), np.linalg.norm(rows[t])
        if ns > 0 and nt > 0:
            tot += float(rows[s] @ rows[t]) / (ns * nt)
    return tot


def test_sics_block_matches_pairwise_brute_force():
    rng = np.random.default_rng(1)
    for n, d in [(1, 4), (2, 3), (7, 5), (16, 8)]:
        x = rng.standard_normal((n, d))
        if n > 2:
            x[1] = 0.0  # a zero row has no direction
        assert abs(sel.sics_block(x) - brute_sics(x)) < 1e-10


def test_sics_block_closed_forms():
    v = np.array([0.3, -1.2, 2.0])
    same = np.outer([1.0, 2.5, 0.1, 7.0], v)  # one direction, positive scales
    assert abs(sel.sics_block(same) - 4 * 3) < 1e-12
    assert abs(sel.sics_block(np.eye(5)) - 0.0) < 1e-12
    opp = np.stack([v, -v])
    assert abs(sel.sics_block(opp) - (-2.0)) < 1e-12
    rng = np.random.default_rng(2)
    x = rng.standard_normal((9, 6))
    scale = rng.uniform(0.1, 10.0, size=(9, 1))
    assert abs(sel.sics_block(x * scale) - sel.sics_block(x)) < 1e-10


def test_sics_order_picks_the_frame_blocking():
    # grid 4 x 2 x 4, block 8 = H*W: orders with F outermost (FHW, FWH) put
    # each frame in its own block; every frame's tokens share a direction
    F, H, W, d = 4, 2, 4, 6
    rng = np.random.default_rng(3)
    dirs = rng.standard_normal((F, d))
    x = np.repeat(dirs, H * W, axis=0) * rng.uniform(0.5, 2.0, size=(F * H * W, 1))
    per = [sel.sics_order(x, (F, H, W), o, 8) for o in range(6)]
    assert abs(per[0] - F * 8 * 7) < 1e-9 and abs(per[1] - F * 8 * 7) < 1e-9
    assert max(per[2:]) < per[0] - 1.0
    s = sel.sics_scores(x[None, None], x[None, None], (F, H, W), 8)
    assert sel.select_orders(s)[0, 0] == 0  # tie FHW / FWH -> lower id
    # brute force over the permuted blocks agrees
    for o in range(6):
        xp = ref.reorder_head(x, (F, H, W), o, 8)
        bf = sum(brute_sics(xp[i * 8:(i + 1) * 8]) for i in range(4))
        assert abs(per[o] - bf) < 1e-9


def brute_topp(s, p):
    s = np.asarray(s, dtype=np.float64)
    key = np.where(np.isnan(s), -np.inf, s)
    if p <= 0 or key.max() == -np.inf:
        return []
    if key.max() == np.inf:
        w = [1.0 if v == np.inf else 0.0 for v in key]
    else:
        w = [math.exp(v - key.max()) for v in key]
    order = sorted(range(len(key)), key=lambda j: (-key[j], j))
    total = 0.0
    for j in order:
        total += w[j]
    acc = 0.0
    for n, j in enumerate(order):
        acc += w[j]
        if acc >= p * total:
            return sorted(order[:n + 1])
    return sorted(order)


@pytest.mark.parametrize("p", [0.0, 1e-9, 0.3, 0.5, 0.9, 0.999, 1.0])
def test_topp_matches_brute_force(p):
    rng = np.random.default_rng(int(p * 1000) + 5)
    for nb in [1, 5, 17, 40]:
        s = rng.standard_normal(nb) * 2.0
        assert sel.topp_row(s, p).tolist() == brute_topp(s, p)


def test_topp_limits_ties_and_non_finite():
    s = np.array([0.5, 3.0, -1.0, 3.0, 2.0])
    assert sel.topp_row(s, 1e-12).tolist() == [1]  # the largest, lower index
    assert sel.topp_row(s, 1.0).tolist() == [0, 1, 2, 3, 4]
    uniform = np.zeros(6)
    assert sel.topp_row(uniform, 0.5).tolist() == [0, 1, 2]  # ties -> lower idx
    assert sel.topp_row(uniform, 0.51).tolist() == [0, 1, 2, 3]
    assert sel.topp_row(np.array([np.nan, 1.0, -np.inf]), 0.99).tolist() == [1]
    assert sel.topp_row(np.array([-np.inf, np.nan]), 0.5).tolist() == []
    assert sel.topp_row(np.array([np.inf, 0.0, np.inf]), 0.5).tolist() == [0]
    assert sel.topp_row(np.array([np.inf, 0.0, np.inf]), 0.9).tolist() == [0, 2]
    # p = 1 stops at the last block of nonzero weight (-inf / NaN weigh 0)
    s3 = np.array([0.3, -np.inf, 1.7, np.nan, -2.0, 0.9], dtype=np.float32)
    assert sel.topp_row(s3, 1.0).tolist() == [0, 2, 4, 5]
    # the mass of two equal leaders covers p = 2 / (2 + e^-3)
    s2 = np.array([0.0, 0.0, -3.0])
    lead = 2.0 / (2.0 + math.exp(-3.0))
    assert sel.topp_row(s2, lead * (1 - 1e-9)).tolist() == [0, 1]
    assert sel.topp_row(s2, min(1.0, lead * (1 + 1e-9))).tolist() == [0, 1, 2]


def test_window_rows():
    assert sel.window_row(0, 2, 10).tolist() == [0, 1, 2]
    assert sel.window_row(9, 1, 10).tolist() == [8, 9]
    assert sel.window_row(4, 0, 10).tolist() == [4]
    assert sel.window_row(4, -1, 10).tolist() == []


def test_hybrid_union_and_reductions():
    rng = np.random.default_rng(7)
    nb = 23
    s = rng.standard_normal((1, 2, nb, nb)).astype(np.float32)
    idx, cnt = sel.hybrid_select(s, 4, 0.6, 1)
    for h in range(2):
        for i in range(nb):
            row = idx[0, h, i, :cnt[0, h, i]]
            assert (np.diff(row) > 0).all() and i in row
            assert (idx[0, h, i, cnt[0, h, i]:] == -1).all()
            want = set(ref.select_topk_row(s[0, h, i], i, 4)) | set(sel.window_row(i, 1, nb)) \
                | set(sel.topp_row(s[0, h, i], 0.6))
            assert set(row.tolist()) == want
    # pure top-k: equals the top-k oracle with constant counts
    idx_k, cnt_k = sel.hybrid_select(s, 5, 0.0, -1)
    assert (cnt_k == 5).all()
    assert (idx_k[..., :5] == ref.select_topk(s, 5)).all()
    # k = 0, p = 0, no window: only the diagonal
    idx_d, cnt_d = sel.hybrid_select(s, 0, 0.0, -1)
    assert (cnt_d == 1).all() and (idx_d[0, 0, :, 0] == np.arange(nb)).all()
    # k = NB keeps everything
    _, cnt_all = sel.hybrid_select(s, nb, 0.0, -1)
    assert (cnt_all == nb).all()
