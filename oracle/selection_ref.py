"""Float64 CPU oracle of the SPADE-style selection variants: the SICS
blocking-scheme score and the hybrid Top-K / Top-P / local-window block
filter.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's
CPU-baseline / reference legs may import this module.  It shares no code
with the CUDA library; it reuses this oracle's own reorder and top-k
(oracle/paro_ref.py).

Sources (SPADE, arXiv 2608.03335, Pith verdict page):
* key_machinery (ii) and the referee's note on Eq. (5): each candidate
  blocking of the Q/K token grid is scored by the Sum of Intra-block Cosine
  Similarities, the sum of all pairwise cosine similarities inside a block,
  which the identity  sum_{s != t} xh_s . xh_t = |sum_t xh_t|^2 - sum_t |xh_t|^2
  (xh = x / |x|) turns into a single pass over the block's rows; the blocking
  with the highest score is selected per head.
* core_discovery: only blocks that pass a head-wise Top-K / Top-P and
  local-window filter are attended.

Readings where the page is silent:

S1. Candidate blockings: the six axis orders of [F, H, W] and six 3D tile
    blockings (key_machinery (i): spatial, temporal and mixed candidates),
    ids 6-11, tiles of tf x th x tw = block tokens in tile-major order
    (oracle/paro_ref.py TILE_SHAPES: for block 128 spatial 1x8x16 and
    1x16x8, mixed 2x8x8 and 4x4x8, temporal 8x4x4 and 16x2x4); in every
    case the blocks are runs of ``block`` consecutive tokens of the
    candidate's order (the blocks the attention kernel runs).
S2. "Pairwise" counts ordered pairs s != t (the identity above); a zero row
    has no direction and contributes nothing (xh = 0).  Pad rows are zero.
S3. The score of a candidate is SICS over Q's blocks plus SICS over K's
    blocks (the same token sets); the selected one is the argmax, ties to
    the lower id; a head's pick sums its score over the batch.
S4. Top-P on a query-block row: weights w_j = exp(s_j - max_j s_j) over all
    key blocks (NaN scores weigh 0 and sort as -inf); blocks in order of
    decreasing score, ties to the lower index; keep the shortest prefix
    whose running sum reaches p times the full running sum (the total is
    the last prefix sum, so that p = 1 stops at the last block of nonzero
    weight whatever the rounding); all blocks if none does; none if
    p <= 0 or every score is -inf / NaN.  A row whose maximum is +inf gives
    weight 1 to its +inf entries and 0 to the rest.
S5. The kept set of row i is the union of the diagonal block, the local
    window {j : |i - j| <= w} (w >= 0; w < 0 adds nothing), the Top-K set of
    paro_ref.select_topk_row (k >= 1; k = 0 adds nothing) and the Top-P set;
    stored ascending with a per-row count.

Parity: every function is pinned by tests/test_oracle_selection.py (brute
force, closed forms, invariants); none is "parity unpinned".
"""

from __future__ import annotations

import numpy as np

from . import paro_ref as ref


# ------------------------------------------------------------------ SICS --

def sics_block(rows: np.ndarray) -> float:
    """Sum over ordered pairs s != t of cos(x_s, x_t) for one block's rows,
    by the identity |sum xh|^2 - sum |xh|^2 (readings S2)."""
    x = np.asarray(rows, dtype=np.float64)
    nrm = np.sqrt((x * x).sum(axis=1))
    xh = np.zeros_like(x)
    nz = nrm > 0
    xh[nz] = x[nz] / nrm[nz, None]
    tot = xh.sum(axis=0)
    return float(tot @ tot - (xh * xh).sum())


def sics_order(x: np.ndarray, grid: tuple, perm_id: int, block: int) -> float:
    """SICS of one head's [N, d] rows under the blocking of order perm_id:
    the sum of sics_block over the permuted blocks (reading S1)."""
    xp = ref.reorder_head(np.asarray(x, dtype=np.float64), grid, perm_id, block)
    nb = xp.shape[0] // block
    return float(sum(sics_block(xp[i * block:(i + 1) * block]) for i in range(nb)))


def sics_scores(q, k, grid: tuple, block: int) -> np.ndarray:
    """[B, h, N, d] q, k -> [B, h, 12] scores, SICS(Q) + SICS(K) per
    candidate blocking: the six axis orders and the six 3D tile blockings
    (readings S1, S3)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    B, nh = q.shape[:2]
    nc = ref.n_candidates(block)
    out = np.zeros((B, nh, nc), dtype=np.float64)
    for b in range(B):
        for h in range(nh):
            for o in range(nc):
                out[b, h, o] = (sics_order(q[b, h], grid, o, block)
                                + sics_order(k[b, h], grid, o, block))
    return out


def select_orders(scores: np.ndarray) -> np.ndarray:
    """[B, h, C] -> [B, h] int8 argmax candidate ids, ties to the lower id
    (np.argmax returns the first maximum)."""
    return np.argmax(np.asarray(scores), axis=-1).astype(np.int8)


def head_picks(scores: np.ndarray) -> np.ndarray:
    """[B, h, C] -> [h] int8: each head's blocking, the argmax of its score
    summed over the batch (a head has one blocking), ties to the lower id
    (reading S3)."""
    return np.argmax(np.asarray(scores, dtype=np.float64).sum(axis=0), axis=-1).astype(np.int8)


# ------------------------------------------------------------ filters --

def topp_row(s: np.ndarray, p: float) -> np.ndarray:
    """Top-P set of one row of block scores (reading S4), ascending."""
    v = np.asarray(s, dtype=np.float64)
    nb = v.shape[0]
    key = np.where(np.isnan(v), -np.inf, v)
    if p <= 0 or nb == 0:
        return np.zeros(0, dtype=np.int32)
    m = key.max()
    if m == -np.inf:
        return np.zeros(0, dtype=np.int32)
    if m == np.inf:
        w = (key == np.inf).astype(np.float64)
    else:
        w = np.exp(key - m)
    j = np.arange(nb)
    order = np.lexsort((j, -key))  # score descending, then index ascending
    cum = np.cumsum(w[order])
    target = p * cum[-1]  # the total as the same left-to-right sum
    reach = np.nonzero(cum >= target)[0]
    length = int(reach[0]) + 1 if reach.size else nb
    return np.sort(order[:length]).astype(np.int32)


def window_row(i: int, w: int, nb: int) -> np.ndarray:
    """Local window {j : |i - j| <= w} (none for w < 0), ascending."""
    if w < 0:
        return np.zeros(0, dtype=np.int32)
    return np.arange(max(0, i - w), min(nb, i + w + 1), dtype=np.int32)


def hybrid_row(s: np.ndarray, i: int, k: int, p: float, w: int) -> np.ndarray:
    """Kept set of query-block row i (reading S5), ascending."""
    nb = s.shape[0]
    parts = [np.array([i], dtype=np.int32), window_row(i, w, nb), topp_row(s, p)]
    if k >= 1:
        parts.append(ref.select_topk_row(s, i, k))
    return np.unique(np.concatenate(parts)).astype(np.int32)


def hybrid_select(scores: np.ndarray, k: int, p: float, w: int):
    """[B, h, NB, NB] scores -> (idx [B, h, NB, NB] int32 ascending, padded
    with -1; counts [B, h, NB] int32)."""
    B, nh, nb, _ = scores.shape
    idx = np.full((B, nh, nb, nb), -1, dtype=np.int32)
    counts = np.zeros((B, nh, nb), dtype=np.int32)
    for b in range(B):
        for h in range(nh):
            for i in range(nb):
                kept = hybrid_row(scores[b, h, i], i, k, p, w)
                counts[b, h, i] = kept.size
                idx[b, h, i, :kept.size] = kept
    return idx, counts
