"""Float64 CPU oracle of PAROAttention's offline stage: the per-head
permutation metric and the static block mask, both from block statistics of
the dense post-softmax attention map.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's
CPU-baseline / reference legs may import this module.  It shares no code
with the CUDA library; it reuses this oracle's own reorder (paro_ref.py).

Sources (PAROAttention, arXiv 2506.16054, Pith verdict page):
* key_machinery: the permutation is chosen offline per head among the six
  axis orders by a metric that balances block sparsifiability (the fraction
  of blocks that are mostly below a small threshold) against quantisation
  incoherence (max over mean absolute value inside each block); the static
  mask is chosen by block-sum thresholding.
* referee minor comment on Eq. (1): n^{<eps}_{ij} counts the entries of
  block (i, j) below eps; the report gives eps = 1e-3 and sigma = 90% as the
  example values, and leaves the weight alpha of Eq. (3) unstated.

Readings where the page is silent:

R1. The map is P = softmax(Q K^T / sqrt(d)) over the N valid tokens of a
    head, rows and columns both permuted by the candidate order; block
    (i, j) holds the valid rows of permuted block i and valid columns of
    permuted block j (size n_i * n_j; the tail blocks are partial).
R2. A block is sparse when at least rho = sigma = 0.9 of its entries are
    below eps = 1e-3 (n^{<eps}_{ij} >= 0.9 n_i n_j).
R3. Block incoherence = max(P_blk) / mean(P_blk) (P >= 0); a head's
    incoherence is the mean over its blocks of positive mean.
R4. M(order) = alpha * (1 - sparse fraction) / max over orders of the same
    + (1 - alpha) * incoherence / max over orders of the same, alpha = 0.5;
    the chosen order is the argmin, ties to the lower order id (each term
    normalised by its largest value over the six orders, so that the two
    scales can be weighed; a term that is 0 for every order contributes 0).
R5. Static mask of query-block row i (block-sum thresholding at sigma):
    blocks in decreasing block sum (ties to the lower index), the shortest
    run whose running sum reaches sigma of the row's running total, plus
    the diagonal block.  This is the Top-P rule of selection_ref.topp_row
    with weights equal to the block sums (scores = log block sums).

Parity: every function is pinned by tests/test_oracle_offline.py (brute
force block loops, closed forms of the map and of the statistics, a grid
built so that one order is block-diagonal); none is "parity unpinned".
"""

from __future__ import annotations

import math

import numpy as np

from . import paro_ref as ref
from . import selection_ref as sel


def attention_map(q: np.ndarray, k: np.ndarray) -> np.ndarray:
    """Dense post-softmax map of one head, natural order: [N, N] float64."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    s = q @ k.T / math.sqrt(q.shape[1])
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    return p / p.sum(axis=1, keepdims=True)


def permuted_map(p: np.ndarray, grid: tuple, perm_id: int) -> np.ndarray:
    """Rows and columns of the map in the order's token sequence (no pad)."""
    N = p.shape[0]
    pos = ref.reorder_head(np.arange(N, dtype=np.float64)[:, None], grid, perm_id,
                           1)[:N, 0].astype(np.int64)
    return p[np.ix_(pos, pos)]


def block_stats(p: np.ndarray, grid: tuple, perm_id: int, block: int, eps: float = 1e-3):
    """Per block of the permuted map (reading R1): dict of [NB, NB] arrays
    count (entries < eps), total (sum), peak (max), size (n_i * n_j)."""
    pp = permuted_map(p, grid, perm_id)
    N = pp.shape[0]
    nb = -(-N // block)
    out = {key: np.zeros((nb, nb)) for key in ("count", "total", "peak", "size")}
    for i in range(nb):
        r = slice(i * block, min(N, (i + 1) * block))
        for j in range(nb):
            c = slice(j * block, min(N, (j + 1) * block))
            blk = pp[r, c]
            out["count"][i, j] = np.count_nonzero(blk < eps)
            out["total"][i, j] = blk.sum()
            out["peak"][i, j] = blk.max()
            out["size"][i, j] = blk.size
    return out


def sparse_fraction(st, rho: float = 0.9) -> float:
    """Fraction of blocks with count >= rho * size (reading R2)."""
    return float(np.mean(st["count"] >= rho * st["size"]))


def incoherence(st) -> float:
    """Mean over blocks of positive mean of max / mean (reading R3)."""
    mean = st["total"] / st["size"]
    ok = mean > 0
    return float(np.mean(st["peak"][ok] / mean[ok])) if ok.any() else 0.0


def permutation_metric(q, k, grid: tuple, block: int, eps: float = 1e-3, rho: float = 0.9,
                       alpha: float = 0.5):
    """One head: (M [6], sparse fraction [6], incoherence [6]) (reading R4)."""
    p = attention_map(q, k)
    sf = np.zeros(6)
    inc = np.zeros(6)
    for o in range(6):
        st = block_stats(p, grid, o, block, eps)
        sf[o] = sparse_fraction(st, rho)
        inc[o] = incoherence(st)
    dense = 1.0 - sf

    def norm(x):
        m = x.max()
        return x / m if m > 0 else np.zeros_like(x)

    return alpha * norm(dense) + (1 - alpha) * norm(inc), sf, inc


def choose_order(metric: np.ndarray) -> int:
    """argmin, ties to the lower order id."""
    return int(np.argmin(metric))


def static_mask_rows(total: np.ndarray, sigma: float = 0.9):
    """Kept lists of every query-block row from the block sums (reading R5):
    (idx [NB, NB] ascending, -1 padded; counts [NB])."""
    nb = total.shape[0]
    idx = np.full((nb, nb), -1, dtype=np.int32)
    counts = np.zeros(nb, dtype=np.int32)
    with np.errstate(divide="ignore"):
        logs = np.log(total)
    for i in range(nb):
        kept = np.unique(np.concatenate(([i], sel.topp_row(logs[i], sigma)))).astype(np.int32)
        counts[i] = kept.size
        idx[i, :kept.size] = kept
    return idx, counts
