"""Degenerate and extreme shapes on the GPU, against the oracle: a single
token (N = 1: one block with 1 valid row and 127 pad rows, the softmax over
one key gives that key's value), one-axis grids, a grid smaller than every
3D tile, a tail-free grid, the largest supported head count (1024, orders
cycling through all 12 ids), and a call with no kept block at all (k = 0:
zeros).  Every path the shape can take is run: the tcgen05 bf16 kernel
(both input layouts), the mma.sync kernel (d = 64), INT8 in both P forms,
and the compensated kernel.  Outputs start as NaN, so every row must be
written."""

import numpy as np
import pytest
import torch

from block_sparse_attention_34_b200 import paro
from block_sparse_attention_34_b200.pipeline import Pipeline
from block_sparse_attention_34_b200.synth import as_f64
from oracle import paro_ref as ref
from oracle import pasa_ref as pasa

from helpers import INT8_MAX_ABS, INT8_MEAN_ABS, BF16_MAX_ABS, BF16_MEAN_ABS, compare, custom, \
    inputs, oracle_topk, to_dev

pytestmark = pytest.mark.gpu

SHAPES = [
    custom("one_token", 1, 2, 128, (1, 1, 1), 128, "bf16", 1.0, perms=(0, 8)),
    custom("one_token_d64", 1, 2, 64, (1, 1, 1), 64, "bf16", 1.0, perms=(5, 7)),
    custom("w_only_300", 1, 3, 128, (1, 1, 300), 128, "bf16", 0.67, perms=(0, 3, 11)),
    custom("f_only_200", 2, 2, 128, (200, 1, 1), 128, "bf16", 0.5, perms=(4, 9)),
    custom("smaller_than_tiles", 1, 6, 128, (1, 3, 5), 128, "bf16", 1.0,
           perms=(6, 7, 8, 9, 10, 11)),
    custom("no_tail_256", 1, 2, 128, (2, 8, 16), 128, "bf16", 0.5, perms=(2, 6)),
]


def problem(w, perms):
    return paro.Problem(w.B, w.heads, (w.F, w.H, w.W), w.d, w.block, perms)


def nan_out(w, dtype=torch.bfloat16):
    return torch.full((w.B, w.heads, w.N, w.d), float("nan"), dtype=dtype, device="cuda")


@pytest.mark.parametrize("w", SHAPES, ids=lambda w: w.name)
def test_bf16_shapes_both_layouts(w):
    q, k, v, perms = inputs(w)
    pr = problem(w, perms)
    idx, _, _ = oracle_topk(q, k, w, perms)
    want = ref.attention(as_f64(q), as_f64(k), as_f64(v), (w.F, w.H, w.W), perms, w.block, idx)
    qd, kd, vd = to_dev(q, k, v)
    idx_d = torch.from_numpy(np.ascontiguousarray(idx, dtype=np.int32)).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = paro.block_sparse_attn(qd, kd, vd, pr, idx_d, out=nan_out(w), status=status)
    qp, kp, vp = (paro.reorder(x, pr) for x in (qd, kd, vd))
    out_p = paro.block_sparse_attn(qp, kp, vp, pr, idx_d, out=nan_out(w), status=status,
                                   permuted=True)
    torch.cuda.synchronize()
    assert status.item() == 0
    compare(out, want)
    compare(out_p, want)
    if w.N == 1:  # one key: the output is that key's value
        assert np.abs(want[:, :, 0] - as_f64(v)[:, :, 0]).max() < 1e-12


@pytest.mark.parametrize("w", [s for s in SHAPES if s.d == 128], ids=lambda w: w.name)
def test_int8_shapes_both_p_forms(w):
    q, k, v, perms = inputs(w)
    pr = problem(w, perms)
    grid = (w.F, w.H, w.W)
    idx, _, _ = oracle_topk(q, k, w, perms)
    idx_d = torch.from_numpy(np.ascontiguousarray(idx, dtype=np.int32)).cuda()
    dev, host = [], []
    for x in (q, k, v):
        (xd,) = to_dev(x)
        dev.append(paro.quantize_int8(xd, pr))
        host.append(ref.quantize_int8(ref.reorder(x.float().numpy(), grid, perms, w.block),
                                      w.N, w.block))
    (q8, sq), (k8, sk), (v8, sv) = host
    for p_tile, mode, tol in ((False, "online", (BF16_MAX_ABS, BF16_MEAN_ABS)),
                              (True, "tile", (BF16_MAX_ABS, BF16_MEAN_ABS)),
                              (False, "tile", (INT8_MAX_ABS, INT8_MEAN_ABS))):
        status = torch.zeros(1, dtype=torch.int32, device="cuda")
        out = paro.block_sparse_attn(dev[0][0], dev[1][0], dev[2][0], pr, idx_d,
                                     scales=(dev[0][1], dev[1][1], dev[2][1]), out=nan_out(w),
                                     status=status, p_tile=p_tile)
        torch.cuda.synchronize()
        assert status.item() == 0
        outp = np.zeros((w.B, w.heads, q8.shape[2], w.d))
        for b in range(w.B):
            for h in range(w.heads):
                outp[b, h] = ref.attention_int8(q8[b, h], k8[b, h], v8[b, h], sq[b, h],
                                                sk[b, h], sv[b, h], w.N, w.block, idx[b, h],
                                                mode=mode)
        compare(out, ref.inverse_reorder(outp, grid, perms, w.block), *tol)


@pytest.mark.parametrize("w", [s for s in SHAPES if s.d == 128], ids=lambda w: w.name)
def test_compensated_shapes(w):
    q, k, v, perms = inputs(w)
    pr = problem(w, perms)
    idx, _, _ = oracle_topk(q, k, w, perms, density=0.34 if w.NB > 2 else None)
    want = pasa.attention_compensated(as_f64(q), as_f64(k), as_f64(v), (w.F, w.H, w.W), perms,
                                      w.block, idx)
    qd, kd, vd = to_dev(q, k, v)
    qp, _ = paro.reorder(qd, pr, with_pool=True)
    kp, k_pool = paro.reorder(kd, pr, with_pool=True)
    vp, v_pool = paro.reorder(vd, pr, with_pool=True)
    idx_d = torch.from_numpy(np.ascontiguousarray(idx, dtype=np.int32)).cuda()
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = paro.block_sparse_attn_compensated(qp, kp, vp, pr, idx_d, paro.round_bf16(k_pool),
                                             paro.round_bf16(v_pool), out=nan_out(w),
                                             status=status, permuted=True)
    torch.cuda.synchronize()
    assert status.item() == 0
    compare(out, want)


def test_max_heads_1024():
    """The largest head count the library takes, orders cycling through all
    12 ids, through the Pipeline (selection on the GPU, compared with the
    oracle's kept lists: with NB = 2 and density 0.5 every row keeps only
    its diagonal, so the lists are fixed)."""
    w = custom("heads_1024", 1, 1024, 128, (1, 2, 100), 128, "bf16", 0.5,
               perms=tuple(i % 12 for i in range(1024)))
    q, k, v, perms = inputs(w)
    pipe = Pipeline(w.B, w.heads, (w.F, w.H, w.W), w.d, w.block, perms, w.density)
    pipe.out.fill_(float("nan"))
    out = pipe.run(*to_dev(q, k, v))
    torch.cuda.synchronize()
    assert pipe.status.item() == 0 and pipe.k == 1
    idx = np.broadcast_to(np.arange(w.NB, dtype=np.int32)[:, None], (1, w.heads, w.NB, 1))
    assert (pipe.idx.cpu().numpy() == idx).all()
    want = ref.attention(as_f64(q), as_f64(k), as_f64(v), (w.F, w.H, w.W), perms, w.block,
                         np.ascontiguousarray(idx))
    compare(out, want)


def test_no_kept_block_gives_zeros():
    """k = 0 (an idx with no column): every output row is zero, on every
    attention entry that takes it."""
    w = SHAPES[2]
    q, k, v, perms = inputs(w)
    pr = problem(w, perms)
    qd, kd, vd = to_dev(q, k, v)
    idx = torch.zeros((w.B, w.heads, w.NB, 0), dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = paro.block_sparse_attn(qd, kd, vd, pr, idx, out=nan_out(w), status=status)
    out_m = paro.block_sparse_attn(qd, kd, vd, pr, idx, out=nan_out(w), status=status,
                                   baseline=True)
    torch.cuda.synchronize()
    assert status.item() == 0
    assert (out == 0).all() and (out_m == 0).all()
