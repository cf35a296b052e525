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
