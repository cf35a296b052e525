"""Float64 CPU oracle of per-head block-sparse attention over a token grid.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the bench's
CPU-baseline / reference legs may import this module.  It shares no code with
the CUDA library and never imports it; both sides only share the seeded
input generator.

Every function is the plain definition of one step, written with NumPy in
float64 (except where the INT8 path fixes float32 rounding), with no
blocking, fusion or reordering beyond what the step itself states.  Sources:

* PAROAttention (arXiv 2506.16054), Pith verdict page, "key_machinery" and
  "core_discovery": a per-head permutation of the flattened sequence among
  the six orders of [F, H, W]; a static block mask; block-wise INT8
  quantisation of Q/K and of the post-softmax map P, with groups aligned to
  the FlashAttention block.
* SPADE (arXiv 2608.03335), Pith verdict page, "key_machinery" (iii) and the
  referee's minor comments on section 3.1 (MEAN summariser) and section 2.2,
  Eq. (2) (the mask is additive: 0 on kept block pairs, -inf on pruned ones),
  and "core_discovery" (Top-K filter); flash block-sparse attention with an
  online softmax.
* PASA (arXiv 2604.12219), Pith page, Figure 2 caption: each query block
  attends to at most k key blocks, cost O(S k) instead of O(S^2).

Readings where the pages are silent:

1. An order's letters list the axes outermost -> innermost; FHW is the
   natural flattening n = f*H*W + h*W + w.  Ids: 0 FHW, 1 FWH, 2 HFW,
   3 HWF, 4 WFH, 5 WHF.
2. Blocks are runs of ``block`` consecutive tokens of the permuted order;
   the permuted sequence is zero-padded at its tail to N_p = NB*block.
3. Block summary = mean of the block's valid (non-pad) rows; block score
   = q_bar . k_bar / sqrt(d) (no softmax: it would not change a row's top-k).
4. k = ceil(density * NB) clamped to [1, NB] (product rounded to 9 decimals
   first); the diagonal block always kept and counts toward k; the other
   k-1 are the largest scores, ties to the lower block index, NaN read as
   -inf.  Selected indices are returned in ascending order.
5. Pad keys are masked with -inf; pad query rows are never output.
6. Softmax scale 1/sqrt(d).
7. INT8: Q, K, V per-block symmetric codes (:func:`quantize_int8`); P read
   as the pages state it, the exactly normalised post-softmax map quantised
   per (query block, key block) tile with the tile's own absmax / 127
   (:func:`attention_int8`, mode "tile", the default).  The one-pass
   replays of a flash kernel's order ("online", "rowmax") are kept as
   named diagnostics.

Parity status: every function here is pinned by the tests under
``tests/test_oracle_*.py`` (brute force, library routines, closed forms);
none is "parity unpinned".
"""

from __future__ import annotations

import math

import numpy as np

# Axis letters of each order id, outermost first.
ORDER_NAMES = ("FHW", "FWH", "HFW", "HWF", "WFH", "WHF")

# Order ids 6 .. 11: SPADE's 3D blockings (SPADE, arXiv 2608.03335, Pith
# verdict page, key_machinery (i): spatial, temporal and mixed 3D blocking
# candidates of the token grid).  Reading: a blocking by tiles of
# tf x th x tw tokens (tf*th*tw = the block size) orders the tokens tile by
# tile -- tiles in (f, h, w) order of their tile coordinates, tokens inside a
# tile in (f, h, w) order -- and the executor's blocks are runs of ``block``
# consecutive positions of that order (tiles on the far edges of a grid that
# the tile does not divide are partial, so blocks then straddle tiles).  Two
# of each kind per block size: spatial (tf = 1), mixed, temporal (tf >= 8).
TILE_SHAPES = {
    128: ((1, 8, 16), (1, 16, 8), (2, 8, 8), (4, 4, 8), (8, 4, 4), (16, 2, 4)),
    64: ((1, 8, 8), (1, 4, 16), (2, 4, 8), (4, 4, 4), (8, 2, 4), (16, 2, 2)),
}
N_ORDERS = 12  # ids 0-5 axis orders, 6-11 tile blockings (blocks 64 and 128)


def n_candidates(block: int) -> int:
    """Blocking candidates of a block size: the six axis orders, plus the six
    tile blockings where a tile table exists."""
    return N_ORDERS if block in TILE_SHAPES else 6


def order_name(perm_id: int, block: int) -> str:
    if perm_id < 6:
        return ORDER_NAMES[perm_id]
    return "T%dx%dx%d" % TILE_SHAPES[block][perm_id - 6]


# ---------------------------------------------------------------- reorder --

def order_axes(perm_id: int) -> tuple:
    """(outer, middle, inner) axis indices of order ``perm_id`` (0=F,1=H,2=W)."""
    return tuple("FHW".index(c) for c in ORDER_NAMES[int(perm_id)])


def tile_order(grid: tuple, shape: tuple) -> np.ndarray:
    """Natural indices n = f*H*W + h*W + w of the tokens in tile-major order
    for tiles of ``shape`` = (tf, th, tw): tiles in (f, h, w) order, tokens
    inside a tile in (f, h, w) order, partial tiles at the far edges."""
    F, H, W = grid
    tf, th, tw = shape
    seq = []
    for f0 in range(0, F, tf):
        for h0 in range(0, H, th):
            for w0 in range(0, W, tw):
                for f in range(f0, min(f0 + tf, F)):
                    for h in range(h0, min(h0 + th, H)):
                        for w in range(w0, min(w0 + tw, W)):
                            seq.append(f * H * W + h * W + w)
    return np.asarray(seq, dtype=np.int64)


def reorder_head(x: np.ndarray, grid: tuple, perm_id: int, block: int) -> np.ndarray:
    """One head's [N, d] rows in natural FHW order -> [N_p, d] in the head's
    order, zero rows appended at the tail (PAROAttention review,
    key_machinery: the six axis orders of [F, H, W]; ids 6-11: SPADE's 3D
    tile blockings, see TILE_SHAPES)."""
    F, H, W = grid
    N, d = x.shape
    assert N == F * H * W
    if int(perm_id) < 6:
        ax = order_axes(perm_id)
        y = x.reshape(F, H, W, d).transpose(ax + (3,)).reshape(N, d)
    else:
        y = x[tile_order(grid, TILE_SHAPES[block][int(perm_id) - 6])]
    nb = -(-N // block)
    out = np.zeros((nb * block, d), dtype=x.dtype)
    out[:N] = y
    return out


def inverse_reorder_head(xp: np.ndarray, grid: tuple, perm_id: int,
                         block: int | None = None) -> np.ndarray:
    """Inverse of :func:`reorder_head`: drop the pad rows, undo the order
    (``block`` names the tile shape of ids 6-11)."""
    F, H, W = grid
    N = F * H * W
    d = xp.shape[1]
    if int(perm_id) >= 6:
        order = tile_order(grid, TILE_SHAPES[block][int(perm_id) - 6])
        out = np.zeros((N, d), dtype=xp.dtype)
        out[order] = xp[:N]
        return out
    ax = order_axes(perm_id)
    sizes = tuple((F, H, W)[a] for a in ax)
    y = xp[:N].reshape(sizes + (d,))
    inv = tuple(int(i) for i in np.argsort(ax)) + (3,)
    return y.transpose(inv).reshape(N, d)


def reorder(x: np.ndarray, grid: tuple, perms, block: int) -> np.ndarray:
    """[B, h, N, d] -> [B, h, N_p, d], per-head order ``perms[h]``."""
    B, nh, N, d = x.shape
    nb = -(-N // block)
    out = np.zeros((B, nh, nb * block, d), dtype=x.dtype)
    for b in range(B):
        for h in range(nh):
            out[b, h] = reorder_head(x[b, h], grid, perms[h], block)
    return out


def inverse_reorder(xp: np.ndarray, grid: tuple, perms, block: int | None = None) -> np.ndarray:
    """[B, h, N_p, d] -> [B, h, N, d]."""
    B, nh, _, d = xp.shape
    N = grid[0] * grid[1] * grid[2]
    out = np.zeros((B, nh, N, d), dtype=xp.dtype)
    for b in range(B):
        for h in range(nh):
            out[b, h] = inverse_reorder_head(xp[b, h], grid, perms[h], block)
    return out


# ------------------------------------------------------- pooled scores --

def block_pool(xp: np.ndarray, N: int, block: int) -> np.ndarray:
    """Mean of each block's valid rows (SPADE review, MEAN summariser).
    xp: [B, h, N_p, d] permuted; returns [B, h, NB, d] float64."""
    B, nh, Np, d = xp.shape
    nb = Np // block
    out = np.zeros((B, nh, nb, d), dtype=np.float64)
    for i in range(nb):
        lo, hi = i * block, min((i + 1) * block, N)
        out[:, :, i] = xp[:, :, lo:hi].astype(np.float64).mean(axis=2)
    return out


def block_scores(q_pool: np.ndarray, k_pool: np.ndarray) -> np.ndarray:
    """S_bar[i, j] = q_bar_i . k_bar_j / sqrt(d)  (SPADE review, key_machinery
    (iii), intra-estimation from the summaries).  [B, h, NB, NB] float64."""
    d = q_pool.shape[-1]
    return np.einsum("bhid,bhjd->bhij", q_pool, k_pool) / math.sqrt(d)


def pooled_scores(q, k, grid, perms, block):
    """Reorder -> mean-pool -> block score, from natural-order Q and K."""
    N = grid[0] * grid[1] * grid[2]
    qp = reorder(np.asarray(q, dtype=np.float64), grid, perms, block)
    kp = reorder(np.asarray(k, dtype=np.float64), grid, perms, block)
    qb = block_pool(qp, N, block)
    kb = block_pool(kp, N, block)
    return qb, kb, block_scores(qb, kb)


# ---------------------------------------------------------------- top-k --

def k_for_density(nb: int, density: float) -> int:
    """ceil(density * NB) clamped to [1, NB]; the product is rounded to 9
    decimals first so that binary round-off cannot add a block."""
    if nb <= 0:
        return 0
    return int(min(nb, max(1, math.ceil(round(density * nb, 9)))))


def select_topk_row(s: np.ndarray, i: int, k: int) -> np.ndarray:
    """One query-block row: the diagonal block, then the k-1 largest other
    scores, ties to the lower index, NaN as -inf; ascending indices
    (PASA review, Figure 2: at most k key blocks per query block; SPADE
    review, core_discovery: Top-K filter)."""
    nb = s.shape[0]
    k = min(k, nb)
    v = np.where(np.isnan(s), -np.inf, s.astype(np.float64))
    j = np.arange(nb)
    others = j[j != i]
    # lexsort: the last key is the primary one -> score descending, then index
    order = np.lexsort((others, -v[others]))
    chosen = np.concatenate(([i], others[order[:k - 1]]))
    return np.sort(chosen).astype(np.int32)


def select_topk(scores: np.ndarray, k: int) -> np.ndarray:
    """[B, h, NB, NB] scores -> [B, h, NB, k] int32 kept block indices."""
    B, nh, nb, _ = scores.shape
    k = min(k, nb)
    out = np.zeros((B, nh, nb, k), dtype=np.int32)
    for b in range(B):
        for h in range(nh):
            for i in range(nb):
                out[b, h, i] = select_topk_row(scores[b, h, i], i, k)
    return out


# ---------------------------------------------------------- static masks --

def bitmask_from_idx(idx: np.ndarray, nb: int, counts=None) -> np.ndarray:
    """Kept-index lists -> bitmask [B, h, NB, ceil(NB/32)] uint32, bit j%32 of
    word j//32 set when key block j is kept (PAROAttention review,
    key_machinery: static masks stored as bitmasks)."""
    B, nh, rows, kk = idx.shape
    words = -(-nb // 32)
    out = np.zeros((B, nh, rows, words), dtype=np.uint32)
    for b in range(B):
        for h in range(nh):
            for i in range(rows):
                c = kk if counts is None else int(counts[b, h, i])
                for j in idx[b, h, i, :c]:
                    out[b, h, i, j // 32] |= np.uint32(1 << (int(j) % 32))
    return out


def compact_mask(bitmask: np.ndarray, nb: int):
    """Bitmask -> (idx [B, h, NB, NB] int32 ascending, padded with -1;
    counts [B, h, NB] int32)."""
    B, nh, rows, _ = bitmask.shape
    idx = np.full((B, nh, rows, nb), -1, dtype=np.int32)
    counts = np.zeros((B, nh, rows), dtype=np.int32)
    for b in range(B):
        for h in range(nh):
            for i in range(rows):
                js = [j for j in range(nb)
                      if (int(bitmask[b, h, i, j // 32]) >> (j % 32)) & 1]
                counts[b, h, i] = len(js)
                idx[b, h, i, :len(js)] = js
    return idx, counts


# ------------------------------------------------------------- attention --

def attention_permuted(qp, kp, vp, N: int, block: int, idx, counts=None):
    """Block-sparse softmax(Q K^T / sqrt(d) + M) V in the permuted domain.

    M is the additive block mask (SPADE review, section 2.2, Eq. (2)): 0 where
    key block j is in query block i's kept list and the key is a real token,
    -inf elsewhere.  Rows are processed one query block at a time with a
    max-subtracted softmax; only kept key blocks are gathered.
    qp/kp/vp: [Np, d] float64; idx [NB, k] (counts [NB] or None).
    Returns [Np, d] (pad rows zero).
    """
    Np, d = qp.shape
    nb = Np // block
    out = np.zeros((Np, vp.shape[1]), dtype=np.float64)
    scale = 1.0 / math.sqrt(d)
    for i in range(nb):
        lo, hi = i * block, min((i + 1) * block, N)
        if hi <= lo:
            continue
        c = idx.shape[1] if counts is None else int(counts[i])
        kept = [int(j) for j in idx[i, :c]]
        cols = np.concatenate([np.arange(j * block, min((j + 1) * block, N))
                               for j in kept]) if kept else np.zeros(0, dtype=np.int64)
        if cols.size == 0:
            continue  # a row with no valid key: output stays 0
        s = qp[lo:hi] @ kp[cols].T * scale
        m = s.max(axis=1, keepdims=True)
        p = np.exp(s - m)
        out[lo:hi] = (p @ vp[cols]) / p.sum(axis=1, keepdims=True)
    return out


def attention(q, k, v, grid, perms, block, idx, counts=None):
    """Reorder -> block-sparse attention over the kept tiles -> inverse
    reorder.  q/k/v [B, h, N, d] natural order (any float dtype, upcast to
    float64); idx [B, h, NB, k]; returns [B, h, N, d] float64."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    B, nh, N, d = q.shape
    out = np.zeros((B, nh, N, v.shape[-1]), dtype=np.float64)
    for b in range(B):
        for h in range(nh):
            qp = reorder_head(q[b, h], grid, perms[h], block)
            kp = reorder_head(k[b, h], grid, perms[h], block)
            vp = reorder_head(v[b, h], grid, perms[h], block)
            cnt = None if counts is None else counts[b, h]
            op = attention_permuted(qp, kp, vp, N, block, idx[b, h], cnt)
            out[b, h] = inverse_reorder_head(op, grid, perms[h], block)
    return out


def attention_rows(q, k, v, grid, perms, block, idx, rows, counts=None):
    """Outputs of selected natural-order query rows only: ``rows`` is a list
    of (b, h, n).  Same definition as :func:`attention`, one row at a time,
    for full-size checks where the whole output is too costly."""
    q = np.asarray(q)
    F, H, W = grid
    N = F * H * W
    d = q.shape[-1]
    res = np.zeros((len(rows), d), dtype=np.float64)
    pos_cache = {}
    for r, (b, h, n) in enumerate(rows):
        pid = int(perms[h])
        if pid not in pos_cache:
            perm_rows = reorder_head(np.arange(N, dtype=np.float64)[:, None], grid,
                                     pid, block)[:N, 0].astype(np.int64)
            pos = np.empty(N, dtype=np.int64)
            pos[perm_rows] = np.arange(N)
            pos_cache[pid] = (perm_rows, pos)
        perm_rows, pos = pos_cache[pid]
        i = pos[n] // block
        c = idx.shape[-1] if counts is None else int(counts[b, h, i])
        kept = [int(j) for j in idx[b, h, i, :c]]
        cols_p = np.concatenate([np.arange(j * block, min((j + 1) * block, N))
                                 for j in kept])
        cols = perm_rows[cols_p]
        qr = np.asarray(q[b, h, n], dtype=np.float64)
        kk = np.asarray(k[b, h][cols], dtype=np.float64)
        vv = np.asarray(v[b, h][cols], dtype=np.float64)
        s = kk @ qr / math.sqrt(d)
        p = np.exp(s - s.max())
        res[r] = (p @ vv) / p.sum()
    return res


# ------------------------------------------------------------------ INT8 --

def quantize_int8(xp: np.ndarray, N: int, block: int, qmax: int = 127):
    """Per-block symmetric INT8 quantisation (PAROAttention review,
    key_machinery: block-wise INT8 with groups aligned to the FlashAttention
    block; QK^T in INT8 as in its SageAttention baseline).  ``qmax = 7`` is
    the 4-bit variant (INT4 PV, same review: block-wise INT8/INT4
    quantisation of the post-softmax map and PV), codes in [-7, 7].

    Defined in float32 with IEEE round-to-nearest on every operation
    (Q = qmax):
      absmax = max |x| over the block's valid rows,
      inv    = fl32(Q / absmax),
      q      = clamp(round_half_even(fl32(x * inv)), -Q, Q),
      scale  = fl32(absmax / Q);
    a block with absmax 0 gets q = 0 and scale 0.  Pad rows quantise to 0.
    xp: [B, h, N_p, d] permuted (values exactly representable in float32).
    Returns q [B, h, N_p, d] int8 and scales [B, h, NB] float32.
    """
    x32 = np.asarray(xp, dtype=np.float32)
    B, nh, Np, d = x32.shape
    nb = Np // block
    q = np.zeros((B, nh, Np, d), dtype=np.int8)
    sc = np.zeros((B, nh, nb), dtype=np.float32)
    for b in range(B):
        for h in range(nh):
            for i in range(nb):
                lo, hi = i * block, min((i + 1) * block, N)
                blk = x32[b, h, lo:hi]
                amax = np.float32(np.abs(blk).max()) if hi > lo else np.float32(0)
                if amax == 0:
                    continue
                qf = np.float32(qmax)
                inv = np.float32(qf / amax)
                y = np.rint(blk * inv)  # float32 multiply, then half-even
                q[b, h, lo:hi] = np.clip(y, -qmax, qmax).astype(np.int8)
                sc[b, h, i] = np.float32(amax / qf)
    return q, sc


def _int8_tiles(qi, ki, sq_i, sk, N, block, kept):
    """Score tiles of some query rows (integer codes ``qi`` [r, d] as float64,
    block scale ``sq_i``) against the kept key blocks, in the order listed:
    [(j, klo, khi, s)] with s = (q8 k8^T, exact) * s_q * s_k[j] / sqrt(d).
    The integer products are summed in float64, exactly: |q8 k8| <= 127^2
    per term, so every partial sum stays far below 2^53."""
    d = qi.shape[1]
    inv_sqrt_d = 1.0 / math.sqrt(d)
    tiles = []
    for j in kept:
        klo, khi = j * block, min((j + 1) * block, N)
        if khi <= klo:
            continue
        s_int = qi @ ki[klo:khi].T
        tiles.append((j, klo, khi, s_int * (float(sq_i) * float(sk[j]) * inv_sqrt_d)))
    return tiles


def _int8_block_tilewise(qi, ki, vi, sq_i, sk, sv, N, block, kept, quantize_p, p_levels):
    """Mode "tile" for all valid rows of one query block (the rows share each
    tile's P scale, so they are evaluated together).

    P is the exactly normalised softmax of every row over all its kept keys;
    then each (query block, key block) tile of P is quantised symmetrically
    with its own scale absmax/p_levels (absmax over the tile's valid rows and
    keys), codes round_half_even(P / scale); the tile contributes
    (codes V8) * scale * s_v[j].  A tile whose P is all zero contributes 0."""
    rows = qi.shape[0]
    tiles = _int8_tiles(qi, ki, sq_i, sk, N, block, kept)
    if not tiles:
        return np.zeros((rows, vi.shape[1]), dtype=np.float64)
    m = np.max([t[3].max(axis=1) for t in tiles], axis=0)[:, None]
    l = np.zeros((rows, 1))
    for (_, _, _, s) in tiles:
        l = l + np.exp(s - m).sum(axis=1, keepdims=True)
    out = np.zeros((rows, vi.shape[1]))
    for (j, klo, khi, s) in tiles:
        p = np.exp(s - m) / l
        if quantize_p:
            amax = p.max()
            if amax == 0.0:
                continue
            scale = amax / p_levels
            codes = np.clip(np.rint(p / scale), -p_levels, p_levels)
            out = out + (codes @ vi[klo:khi]) * (scale * float(sv[j]))
        else:
            out = out + (p @ vi[klo:khi]) * float(sv[j])
    return out


def _int8_query_rows(qi, ki, vi, sq_i, sk, sv, N, block, kept, mode, quantize_p, p_levels=127):
    """Modes "online" and "rowmax" of INT8 attention for some query rows of
    one query block, over the kept key blocks in the order listed.  Every
    step is row-wise, so any subset of a block's rows gets the same values
    as the whole block.  Returns [r, d] float64."""
    tiles = _int8_tiles(qi, ki, sq_i, sk, N, block, kept)
    rows = qi.shape[0]
    if not tiles:
        return np.zeros((rows, vi.shape[1]), dtype=np.float64)
    if mode == "rowmax":
        m_row = np.max([t[3].max(axis=1) for t in tiles], axis=0)[:, None]
    m = np.full((rows, 1), -np.inf)
    l = np.zeros((rows, 1))
    acc = np.zeros((rows, vi.shape[1]))
    for (j, klo, khi, s) in tiles:
        if mode == "online":
            m_new = np.maximum(m, s.max(axis=1, keepdims=True))
            alpha = np.exp(m - m_new)
        else:
            m_new = m_row
            alpha = np.ones((rows, 1))
        pt = np.exp(s - m_new)
        pq = np.rint(p_levels * pt) / p_levels if quantize_p else pt
        l = l * alpha + pt.sum(axis=1, keepdims=True)
        acc = acc * alpha + (pq @ vi[klo:khi]) * float(sv[j])
        m = m_new
    return acc / l


INT8_MODES = ("tile", "online", "rowmax")


def _int8_block(qi, ki, vi, sq, sk, sv, N, block, i, kept, mode, quantize_p, p_levels):
    lo, hi = i * block, min((i + 1) * block, N)
    if mode == "tile":
        return _int8_block_tilewise(qi[lo:hi], ki, vi, sq[i], sk, sv, N, block, kept,
                                    quantize_p, p_levels)
    return _int8_query_rows(qi[lo:hi], ki, vi, sq[i], sk, sv, N, block, kept, mode, quantize_p,
                            p_levels)


def attention_int8(q8, k8, v8, sq, sk, sv, N: int, block: int, idx, counts=None,
                   mode: str = "tile", quantize_p: bool = True, p_levels: int = 127):
    """INT8 block-sparse attention in the permuted domain, one head.

    S = (Q8 K8^T exact in integers) * s_q[i] * s_k[j] / sqrt(d) per tile
    (PAROAttention review, key_machinery: block-wise INT8 Q/K with groups
    aligned to the attention block).

    P, in the default mode "tile" (PAROAttention review, key_machinery and
    core_discovery: block-wise quantisation of the post-softmax attention
    map, groups aligned to the FlashAttention block): the exactly normalised
    softmax P of each row over all its kept keys, quantised per (query
    block, key block) tile with that tile's own symmetric scale
    absmax(P_tile) / 127, codes round_half_even(P / scale); the tile
    contributes (codes V8) * scale * s_v[j].  This result does not depend
    on the order in which the kept tiles are visited.

    Two diagnostic modes replay the one-pass order of a flash kernel (SPADE
    review, key_machinery (iii): online softmax), where the normaliser is
    not known while a tile is quantised; there the un-normalised tile
    numerator P~ = exp(s - m) <= 1 is rounded with the fixed scale 1/127,
    p8 = round_half_even(127 P~), the tile contributes (p8 V8) * s_v[j] / 127
    and the normaliser sums the unrounded P~:
      "online": kept tiles in the listed (ascending) order, m the running
                row max, earlier sums rescaled by exp(m_old - m_new);
      "rowmax": m the row's final max.
    ``quantize_p=False`` skips the P rounding (P used exactly; all modes
    then agree).  ``p_levels = 7`` quantises P to 4 bits (levels +-7) in
    every mode: the INT4 PV variant, with V from quantize_int8(..., qmax=7).

    q8/k8/v8 [Np, d] int8, sq/sk/sv [NB] float32, idx [NB, k]; returns
    [Np, d] float64 (pad rows zero).
    """
    if mode not in INT8_MODES:
        raise ValueError(f"mode {mode!r}: one of {INT8_MODES}")
    Np, d = q8.shape
    nb = Np // block
    out = np.zeros((Np, v8.shape[1]), dtype=np.float64)
    qi = q8.astype(np.float64)
    ki = k8.astype(np.float64)
    vi = v8.astype(np.float64)
    for i in range(nb):
        lo, hi = i * block, min((i + 1) * block, N)
        if hi <= lo:
            continue
        c = idx.shape[1] if counts is None else int(counts[i])
        kept = [int(j) for j in idx[i, :c]]
        out[lo:hi] = _int8_block(qi, ki, vi, sq, sk, sv, N, block, i, kept, mode, quantize_p,
                                 p_levels)
    return out


def attention_int8_rows(q8, k8, v8, sq, sk, sv, N: int, block: int, idx, positions,
                        counts=None, mode: str = "tile", quantize_p: bool = True,
                        p_levels: int = 127):
    """Rows of :func:`attention_int8` at the given permuted positions only
    (one head), for full-size checks where the whole head is too costly.
    In mode "tile" each position's whole query block is evaluated (its rows
    share the tiles' P scales) and the requested row taken.
    Returns [len(positions), d] float64."""
    if mode not in INT8_MODES:
        raise ValueError(f"mode {mode!r}: one of {INT8_MODES}")
    qi = q8.astype(np.float64)
    ki = k8.astype(np.float64)
    vi = v8.astype(np.float64)
    res = np.zeros((len(positions), v8.shape[1]), dtype=np.float64)
    cache = {}
    for r, p in enumerate(positions):
        i = int(p) // block
        c = idx.shape[1] if counts is None else int(counts[i])
        kept = [int(j) for j in idx[i, :c]]
        if mode == "tile":
            if i not in cache:
                cache[i] = _int8_block(qi, ki, vi, sq, sk, sv, N, block, i, kept, mode,
                                       quantize_p, p_levels)
            res[r] = cache[i][int(p) - i * block]
        else:
            res[r] = _int8_query_rows(qi[p:p + 1], ki, vi, sq[i], sk, sv, N, block, kept, mode,
                                      quantize_p, p_levels)[0]
    return res
