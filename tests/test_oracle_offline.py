"""Pins of the PAROAttention offline-stage oracle (PAROAttention, arXiv
2506.16054, Pith verdict page: key_machinery — permutation metric from block
sparsifiability and block incoherence, static mask by block-sum
thresholding; referee note on Eq. (1): n^{<eps}_{ij}).

Brute force: entry-by-entry loops for the map and the block statistics on
tiny grids.  Closed forms: rows of the map sum to 1, so a block row's sums
add to its number of valid rows; a uniform map has incoherence 1; a map
that lives inside frames is block diagonal exactly for the frame-major
orders, which must then win the metric and give diagonal-only masks.
"""

import math

import numpy as np

from oracle import paro_offline_ref as off
from oracle import paro_ref as ref


def brute_map(q, k):
    N, d = q.shape
    p = np.zeros((N, N))
    for r in range(N):
        s = [float(q[r] @ k[c]) / math.sqrt(d) for c in range(N)]
        m = max(s)
        e = [math.exp(v - m) for v in s]
        z = sum(e)
        p[r] = [x / z for x in e]
    return p


def test_attention_map_matches_brute_force():
    rng = np.random.default_rng(0)
    q, k = rng.standard_normal((2, 24, 8))
    p = off.attention_map(q, k)
    assert np.abs(p - brute_map(q, k)).max() < 1e-12
    assert np.abs(p.sum(axis=1) - 1).max() < 1e-12


def test_block_stats_brute_force_and_row_sums():
    rng = np.random.default_rng(1)
    grid, block = (3, 2, 5), 4  # N = 30: ragged tail block of 2
    q, k = rng.standard_normal((2, 30, 8)) * 2.0
    p = off.attention_map(q, k)
    for o in range(6):
        st = off.block_stats(p, grid, o, block, eps=0.02)
        pos = ref.reorder_head(np.arange(30.0)[:, None], grid, o, 1)[:30, 0].astype(int)
        nb = 8
        for i in range(nb):
            for j in range(nb):
                vals = [p[pos[r], pos[c]] for r in range(i * block, min(30, (i + 1) * block))
                        for c in range(j * block, min(30, (j + 1) * block))]
                assert st["count"][i, j] == sum(v < 0.02 for v in vals)
                assert abs(st["total"][i, j] - sum(vals)) < 1e-12
                assert st["peak"][i, j] == max(vals)
                assert st["size"][i, j] == len(vals)
        rows = np.array([min(block, 30 - i * block) for i in range(nb)])
        assert np.abs(st["total"].sum(axis=1) - rows).max() < 1e-12


def test_uniform_map_statistics():
    grid, block = (2, 4, 4), 8
    q = np.zeros((32, 8))
    k = np.random.default_rng(2).standard_normal((32, 8))
    p = off.attention_map(q, k)  # every entry 1/32
    st = off.block_stats(p, grid, 3, block, eps=1e-3)
    assert abs(off.incoherence(st) - 1.0) < 1e-12
    assert off.sparse_fraction(st) == 0.0  # 1/32 > eps
    st2 = off.block_stats(p, grid, 3, block, eps=0.05)
    assert off.sparse_fraction(st2) == 1.0  # every entry below 0.05
    idx, cnt = off.static_mask_rows(st["total"], sigma=0.5)
    # equal sums: blocks 0 and 1 reach half (ties to the lower index), plus
    # the diagonal
    assert cnt.tolist() == [2, 2, 3, 3]
    assert idx[0, :2].tolist() == [0, 1] and idx[3, :3].tolist() == [0, 1, 3]


def test_frame_local_attention_picks_a_frame_major_order():
    # q = k = a large vector per frame: each token attends (almost) only to
    # its own frame; with block = H*W the frame-major orders are block diagonal
    F, H, W, d = 4, 2, 4, 8
    rng = np.random.default_rng(3)
    dirs = np.linalg.qr(rng.standard_normal((d, d)))[0][:F] * 12.0
    x = np.repeat(dirs, H * W, axis=0)
    p = off.attention_map(x, x)
    metric, sf, inc = off.permutation_metric(x, x, (F, H, W), 8)
    assert off.choose_order(metric) == 0  # FHW, tied with FWH, lower id
    assert abs(metric[0] - metric[1]) < 1e-12 and metric[0] < metric[2:].min()
    assert sf[0] == sf[1] == 0.75 and sf[2:].max() < 0.75  # off-diagonal blocks empty
    st = off.block_stats(p, (F, H, W), 0, 8)
    idx, cnt = off.static_mask_rows(st["total"], sigma=0.9)
    assert (cnt == 1).all() and (idx[:, 0] == np.arange(F)).all()
