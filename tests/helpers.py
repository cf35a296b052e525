"""Shared helpers of the GPU parity tests (no method arithmetic here: the
expected values always come from the oracle)."""

import numpy as np
import torch

from block_sparse_attention_34_b200 import paro
from block_sparse_attention_34_b200.configs import WORKLOADS, Workload
from block_sparse_attention_34_b200.synth import as_f64, make_inputs
from oracle import paro_ref as ref

# Output tolerances for floating point (bf16 and fp32-through-bf16 paths),
# and for the INT8 path against the oracle's quantise/dequantise semantics.
BF16_MAX_ABS = 2e-2
BF16_MEAN_ABS = 2e-3
INT8_MAX_ABS = 6e-2
# mean bound for INT8: a tenth of the max bound, the same ratio as bf16's pair
INT8_MEAN_ABS = 6e-3


def cuda_ok():
    return torch.cuda.is_available()


def custom(name, B, heads, d, grid, block, dtype, density, mask="topk", perms=None, seed=0):
    F, H, W = grid
    return Workload(name, B=B, heads=heads, d=d, F=F, H=H, W=W, block=block, dtype=dtype,
                    density=density, mask=mask, perms=perms, seed=seed)


def inputs(w: Workload, heads=None):
    q, k, v, perms = make_inputs(w, heads=heads)
    return q, k, v, perms


def to_dev(*ts):
    return [t.cuda() for t in ts]


def static_mask(w: Workload, q, k, perms):
    """The static per-head mask of a workload: the oracle's top-k of its
    pooled block scores at the workload density, as a bitmask."""
    grid = (w.F, w.H, w.W)
    _, _, s = ref.pooled_scores(as_f64(q), as_f64(k), grid, perms, w.block)
    kk = ref.k_for_density(w.NB, w.density)
    idx = ref.select_topk(s, kk)
    return ref.bitmask_from_idx(idx, w.NB), idx


def compare(out_gpu: torch.Tensor, want: np.ndarray, max_abs=BF16_MAX_ABS, mean_abs=BF16_MEAN_ABS):
    got = out_gpu.detach().float().cpu().double().numpy()
    err = np.abs(got - want)
    assert np.isfinite(got).all(), "non-finite output"
    assert err.max() <= max_abs, f"max abs err {err.max():.3e} > {max_abs}"
    if mean_abs is not None:
        assert err.mean() <= mean_abs, f"mean abs err {err.mean():.3e} > {mean_abs}"
    return float(err.max()), float(err.mean())


def oracle_topk(q, k, w: Workload, perms, density=None):
    """The oracle's kept lists: top-k of its float64 pooled block scores.
    Returns (idx [B,h,NB,k], scores [B,h,NB,NB], k)."""
    grid = (w.F, w.H, w.W)
    _, _, s = ref.pooled_scores(as_f64(q), as_f64(k), grid, perms, w.block)
    kk = ref.k_for_density(s.shape[-1], w.density if density is None else density)
    return ref.select_topk(s, kk), s, kk


def selection_agreement(idx_gpu: np.ndarray, idx_ref: np.ndarray, s_ref: np.ndarray, rel=1e-4):
    """Rows [B,h,NB] where the GPU's kept list (selected from fp32 scores)
    equals the oracle's (selected from float64 scores).  Every other row
    must still be a valid top-k: ascending, no repeats, the diagonal kept,
    and each block the two lists disagree on within ``rel`` x max|score| of
    the oracle's selection boundary (a near tie that fp32 scores may break
    either way)."""
    same = (idx_gpu == idx_ref).all(axis=-1)
    for b, h, i in zip(*np.nonzero(~same)):
        g = idx_gpu[b, h, i]
        assert (np.diff(g) > 0).all() and i in g, (b, h, i, g)
        row = s_ref[b, h, i]
        g_only = np.setdiff1d(g, idx_ref[b, h, i])
        r_only = np.setdiff1d(idx_ref[b, h, i], g)
        tol = rel * max(1.0, np.abs(row).max())
        assert row[r_only].max() - row[g_only].min() <= tol, (b, h, i, g_only, r_only)
    return same


def token_rows(grid, perm_id: int, block: int):
    """Natural token index of each permuted position of one head (length N)."""
    F, H, W = grid
    N = F * H * W
    return ref.reorder_head(np.arange(N, dtype=np.float64)[:, None], grid, perm_id,
                            block)[:N, 0].astype(np.int64)


def token_mask(block_rows: np.ndarray, grid, perms, block: int):
    """[B,h,NB] bool per query block -> [B,h,N] bool per natural token."""
    B, nh, _ = block_rows.shape
    N = grid[0] * grid[1] * grid[2]
    out = np.zeros((B, nh, N), dtype=bool)
    for h in range(nh):
        tok = token_rows(grid, perms[h], block)
        pos_block = np.arange(N) // block
        out[:, h, tok] = block_rows[:, h, pos_block]
    return out


def compare_rows(out_gpu: torch.Tensor, want: np.ndarray, rows: np.ndarray,
                 max_abs=BF16_MAX_ABS, mean_abs=BF16_MEAN_ABS):
    """compare() restricted to the rows where ``rows`` [B,h,N] is True."""
    got = out_gpu.detach().float().cpu().double().numpy()
    assert np.isfinite(got).all(), "non-finite output"
    err = np.abs(got - want)[rows]
    assert err.size > 0
    assert err.max() <= max_abs, f"max abs err {err.max():.3e} > {max_abs}"
    if mean_abs is not None:
        assert err.mean() <= mean_abs, f"mean abs err {err.mean():.3e} > {mean_abs}"
    return float(err.max()), float(err.mean())
