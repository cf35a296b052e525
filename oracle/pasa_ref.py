"""Float64 CPU oracle of PASA's grouped first-order compensation: block-sparse
attention in which every unselected key block still enters the softmax, as
a single pooled term, instead of being dropped.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's
CPU-baseline / reference legs may import this module.  It shares no code
with the CUDA library; it reuses this oracle's own reorder and pooling
(paro_ref.py).

Source (PASA, arXiv 2604.12219, Pith review page): the Figure 2 caption
(the unselected set of a query's key blocks gets a grouped first-order
compensation; keys outside the kept set are handled by coarse
approximations; the caption runs into the heading of section 3.3, a Taylor
expansion approximation for sparse attention) and the abstract (grouped
approximations aligned to the hardware, i.e. to the kernel's tiles).  No
formula is printed, so the three readings below are this oracle's:

P1. The groups are the key blocks of the permuted sequence, the same blocks
    the selection ranks.  A query row r of query block i attends exactly to
    the valid keys of its kept blocks idx[i]; every other key block j that
    holds at least one valid key (the unselected set U_i) enters through
    its n_j valid keys' mean kbar_j and values' mean vbar_j.
P2. First order: exp is expanded about the block's mean score
    sbar_rj = q_r . kbar_j / sqrt(d): exp(s_rt) ~ exp(sbar_rj) (1 + s_rt -
    sbar_rj).  Summed over the block's keys the linear term is zero (the
    scores' deviations from sbar_rj sum to q_r . sum_t (k_t - kbar_j) = 0),
    and the values are grouped the same way (v_t -> vbar_j), so block j adds
    n_j exp(sbar_rj) to the softmax denominator and n_j exp(sbar_rj) vbar_j
    to the numerator.  The error is second order in the keys' spread about
    kbar_j when a block's values are equal.
P3. O_r = (sum_{t kept} e^{s_rt} v_t + sum_{j in U_i} n_j e^{sbar_rj} vbar_j)
        / (sum_{t kept} e^{s_rt} + sum_{j in U_i} n_j e^{sbar_rj}),
    pad keys excluded everywhere, one max subtracted over both parts.

Parity: the arithmetic of P1-P3 is pinned by tests/test_oracle_pasa.py
(brute-force loops; all blocks kept = dense softmax attention; blocks with
equal keys and values = dense attention exactly; the second-order error
law); whether P1-P3 is PASA's own section 3.3 the page cannot say (the
caption is all it prints), so that reading is parity unpinned against the
paper.
"""

from __future__ import annotations

import math

import numpy as np

from . import paro_ref as ref


def block_counts(N: int, block: int, nb: int) -> np.ndarray:
    """n_j: valid (non-pad) keys of each permuted block, [NB] float64."""
    return np.array([max(0, min(block, N - j * block)) for j in range(nb)], dtype=np.float64)


def compensated_permuted(qp, kp, vp, N: int, block: int, idx, counts=None):
    """Readings P1-P3 in the permuted domain of one head.

    qp/kp/vp: [Np, d] (upcast to float64); idx [NB, k] kept lists (counts
    [NB] or None for full rows).  Returns [Np, d] (pad rows zero)."""
    qp = np.asarray(qp, dtype=np.float64)
    kp = np.asarray(kp, dtype=np.float64)
    vp = np.asarray(vp, dtype=np.float64)
    Np, d = qp.shape
    nb = Np // block
    scale = 1.0 / math.sqrt(d)
    kbar = ref.block_pool(kp[None, None], N, block)[0, 0]  # [NB, d]
    vbar = ref.block_pool(vp[None, None], N, block)[0, 0]
    n = block_counts(N, block, nb)
    out = np.zeros((Np, vp.shape[1]), dtype=np.float64)
    for i in range(nb):
        lo, hi = i * block, min((i + 1) * block, N)
        if hi <= lo:
            continue
        c = idx.shape[1] if counts is None else int(counts[i])
        kept = sorted({int(j) for j in idx[i, :c] if 0 <= int(j) < nb})
        unsel = [j for j in range(nb) if j not in kept and n[j] > 0]
        cols = (np.concatenate([np.arange(j * block, min((j + 1) * block, N)) for j in kept])
                if kept else np.zeros(0, dtype=np.int64))
        s = qp[lo:hi] @ kp[cols].T * scale                 # exact scores, kept keys
        sb = qp[lo:hi] @ kbar[unsel].T * scale             # mean scores, unselected blocks
        m = np.max(np.concatenate([s, sb], axis=1), axis=1, keepdims=True)
        if s.shape[1] + sb.shape[1] == 0:
            continue  # no valid key at all: output stays 0
        p = np.exp(s - m)
        w = n[unsel][None, :] * np.exp(sb - m)
        num = p @ vp[cols] + w @ vbar[unsel]
        den = p.sum(axis=1, keepdims=True) + w.sum(axis=1, keepdims=True)
        out[lo:hi] = num / den
    return out


def attention_compensated(q, k, v, grid, perms, block, idx, counts=None):
    """Reorder -> compensated block-sparse attention -> inverse reorder.
    q/k/v [B, h, N, d] natural order; idx [B, h, NB, k]; returns
    [B, h, N, d] float64."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, nh, N, d = q.shape
    out = np.zeros((B, nh, N, v.shape[-1]), dtype=np.float64)
    for b in range(B):
        for h in range(nh):
            qp = ref.reorder_head(q[b, h], grid, perms[h], block)
            kp = ref.reorder_head(k[b, h], grid, perms[h], block)
            vp = ref.reorder_head(v[b, h], grid, perms[h], block)
            cnt = None if counts is None else counts[b, h]
            op = compensated_permuted(qp, kp, vp, N, block, idx[b, h], cnt)
            out[b, h] = ref.inverse_reorder_head(op, grid, perms[h], block)
    return out


def compensated_rows(q, k, v, grid, perms, block, idx, rows, counts=None):
    """Outputs of selected natural-order query rows only: ``rows`` is a list
    of (b, h, n).  The same definition as :func:`attention_compensated`
    (readings P1-P3), one row at a time, for full-size checks where the
    whole output is too costly.  Block means are taken per (b, h) once."""
    F, H, W = grid
    N = F * H * W
    d = np.asarray(q[0, 0, 0]).shape[-1]
    nb = -(-N // block)
    n = block_counts(N, block, nb)
    res = np.zeros((len(rows), d), dtype=np.float64)
    perm_cache, pool_cache = {}, {}
    for r, (b, h, tok) in enumerate(rows):
        pid = int(perms[h])
        if pid not in perm_cache:
            perm_rows = ref.reorder_head(np.arange(N, dtype=np.float64)[:, None], grid, pid,
                                         block)[:N, 0].astype(np.int64)
            pos = np.empty(N, dtype=np.int64)
            pos[perm_rows] = np.arange(N)
            perm_cache[pid] = (perm_rows, pos)
        perm_rows, pos = perm_cache[pid]
        if (b, h) not in pool_cache:
            kp = ref.reorder_head(np.asarray(k[b, h], dtype=np.float64), grid, pid, block)
            vp = ref.reorder_head(np.asarray(v[b, h], dtype=np.float64), grid, pid, block)
            pool_cache[(b, h)] = (ref.block_pool(kp[None, None], N, block)[0, 0],
                                  ref.block_pool(vp[None, None], N, block)[0, 0])
        kbar, vbar = pool_cache[(b, h)]
        i = pos[tok] // block
        c = idx.shape[-1] if counts is None else int(counts[b, h, i])
        kept = sorted({int(j) for j in idx[b, h, i, :c] if 0 <= int(j) < nb})
        unsel = [j for j in range(nb) if j not in kept and n[j] > 0]
        cols = (perm_rows[np.concatenate([np.arange(j * block, min((j + 1) * block, N))
                                          for j in kept])]
                if kept else np.zeros(0, dtype=np.int64))
        qr = np.asarray(q[b, h, tok], dtype=np.float64)
        s = np.asarray(k[b, h][cols], dtype=np.float64) @ qr / math.sqrt(d)
        sb = kbar[unsel] @ qr / math.sqrt(d)
        m = max(s.max() if s.size else -np.inf, sb.max() if sb.size else -np.inf)
        if m == -np.inf:
            continue
        p = np.exp(s - m)
        w = n[unsel] * np.exp(sb - m)
        num = p @ np.asarray(v[b, h][cols], dtype=np.float64) + w @ vbar[unsel]
        res[r] = num / (p.sum() + w.sum())
    return res
