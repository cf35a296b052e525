"""Seeded synthetic inputs shared by the tests, the bench and the oracle runs.

This module holds no step of the attention method: it only draws numbers.
Both the CUDA path and the oracle consume exactly the arrays it returns.

Recipe (stated once, used everywhere):

* generator: ``np.random.default_rng(seed)`` (PCG64), seed 0 by default;
* draw order: per-head axis orders (only when a workload does not fix
  them), then the Q noise, the K noise, the V values, each drawn head by
  head as float32 standard normals of shape [N, d];
* q = 0.5*noise + phi_h(f, h, w), k = 0.5*noise' + phi_h(f, h, w), v = noise'';
* phi_h splits d into three contiguous chunks for the F, H and W axes of
  sizes ceil(d/3), ceil(d/3) and the rest.  Chunk a holds pairs
  (sin(p_a*w_m), cos(p_a*w_m)), w_m = 10000^(-2m/c_a), for the token's
  coordinate p_a on that axis, scaled by wt_a/sqrt(#pairs) so that the chunk
  has norm wt_a; an odd chunk leaves its last entry 0.  wt_a is 4 on the
  head's dominant axis and 1 on the other two.  The dominant axis is the
  innermost axis of the head's order: the axis along which that head
  aggregates is the one its order makes contiguous (PAROAttention, arXiv
  2506.16054, review "pith_summary" and "core_discovery": heads aggregate
  locally along one axis of the flattened volume, and the reorder makes that
  axis contiguous);
* the float32 sum is rounded to the workload dtype (bf16 round-to-nearest-
  even through torch), so every consumer sees identical values.

The pages measure on real video DiT activations (CogVideoX, Wan,
Hunyuan-Video); these seeded tensors stand in for them.
"""

from __future__ import annotations

import numpy as np
import torch

from .configs import Workload

AXES = "FHW"


def axis_order(perm_id: int) -> tuple:
    """Axis indices (0=F, 1=H, 2=W) of an order id, outermost first.  Ids
    6-11 (3D tile blockings) walk the tokens inside a tile in F, H, W order,
    so their innermost axis is W."""
    if perm_id >= 6:
        return (0, 1, 2)
    names = ("FHW", "FWH", "HFW", "HWF", "WFH", "WHF")[perm_id]
    return tuple(AXES.index(c) for c in names)


def draw_perms(rng: np.random.Generator, heads: int) -> np.ndarray:
    return rng.integers(0, 6, size=heads).astype(np.int8)


def features(F: int, H: int, W: int, d: int, weights) -> np.ndarray:
    """Sinusoidal features of the (f, h, w) grid coordinates, [N, d] float64."""
    c1 = -(-d // 3)
    sizes = (c1, c1, d - 2 * c1)
    coords = np.stack(np.meshgrid(np.arange(F), np.arange(H), np.arange(W),
                                  indexing="ij"), axis=-1).reshape(-1, 3)
    out = np.zeros((F * H * W, d), dtype=np.float64)
    col = 0
    for a in range(3):
        c = sizes[a]
        pairs = c // 2
        if pairs > 0:
            m = np.arange(pairs, dtype=np.float64)
            omega = 10000.0 ** (-2.0 * m / c)
            ang = coords[:, a:a + 1].astype(np.float64) * omega[None, :]
            amp = weights[a] / np.sqrt(pairs)
            out[:, col:col + 2 * pairs:2] = amp * np.sin(ang)
            out[:, col + 1:col + 2 * pairs:2] = amp * np.cos(ang)
        col += c
    return out


def torch_dtype(name: str):
    return {"f32": torch.float32, "bf16": torch.bfloat16}[name]


def make_inputs(w: Workload, heads: int | None = None, seed: int | None = None):
    """Q, K, V as CPU torch tensors [B, heads, N, d] in the workload dtype,
    plus the per-head order ids (int8 numpy array of length heads).

    ``heads`` may be smaller than the workload's head count to draw only the
    leading heads (the draw for head j does not depend on later heads only
    when the orders are fixed; for drawn orders the full head count is used
    for the order draw so that head j's order never changes).
    """
    seed = w.seed if seed is None else seed
    rng = np.random.default_rng(seed)
    H_all = w.heads
    if w.perms is not None:
        perms = np.asarray(w.perms, dtype=np.int8)
    else:
        perms = draw_perms(rng, H_all)
    nh = H_all if heads is None else heads
    dt = torch_dtype(w.dtype)
    N, d = w.N, w.d
    feats = {}
    for hh in range(nh):
        dom = axis_order(int(perms[hh]))[2]
        wts = [1.0, 1.0, 1.0]
        wts[dom] = 4.0
        key = tuple(wts)
        if key not in feats:
            feats[key] = features(w.F, w.H, w.W, d, wts).astype(np.float32)

    def head_feats(hh):
        dom = axis_order(int(perms[hh]))[2]
        wts = [1.0, 1.0, 1.0]
        wts[dom] = 4.0
        return feats[tuple(wts)]

    out = []
    for t in range(3):  # q noise, k noise, v
        x = torch.empty((w.B, nh, N, d), dtype=dt)
        for b in range(w.B):
            for hh in range(H_all):
                z = rng.standard_normal((N, d), dtype=np.float32)
                if hh >= nh:
                    continue
                if t < 2:
                    z = np.float32(0.5) * z + head_feats(hh)
                x[b, hh] = torch.from_numpy(z).to(dt)
        out.append(x)
    return out[0], out[1], out[2], perms[:nh].copy()


def as_f64(t: torch.Tensor) -> np.ndarray:
    """Exact float64 copy of a CPU tensor (bf16 and f32 upcast exactly)."""
    return t.detach().to("cpu").to(torch.float64).numpy()
