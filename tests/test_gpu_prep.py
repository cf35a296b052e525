"""GPU parity of the HBM-bound steps against the oracle, through the C ABI:
reorder / inverse reorder (bit-exact), pooled block scores (float tolerance),
top-k selection and mask compaction (bit-exact on identical scores), INT8
quantisation (bit-exact codes and scales)."""

import numpy as np
import pytest
import torch

from block_sparse_attention_34_b200 import paro
from block_sparse_attention_34_b200.configs import WORKLOADS
from block_sparse_attention_34_b200.synth import as_f64
from oracle import paro_ref as ref

from helpers import custom, inputs, to_dev

pytestmark = pytest.mark.gpu

# small grids with ragged tails, every order (axis orders and tile
# blockings), both dtypes and head dims
CASES = [
    custom("ragged_f32", 1, 6, 64, (3, 5, 7), 64, "f32", 0.5, perms=(0, 1, 2, 3, 4, 5)),
    custom("ragged_bf16", 2, 6, 128, (5, 7, 9), 128, "bf16", 0.5, perms=(5, 4, 3, 2, 1, 0)),
    custom("ragged_bf16_b64", 1, 3, 128, (2, 9, 11), 64, "bf16", 0.5, perms=(1, 3, 5)),
    # the 3D tile blockings (ids 6-11), ragged edges, both block sizes
    custom("tiles_bf16", 1, 6, 128, (5, 18, 20), 128, "bf16", 0.5, perms=(6, 7, 8, 9, 10, 11)),
    custom("tiles_f32_b64", 2, 6, 64, (19, 6, 11), 64, "f32", 0.5, perms=(11, 10, 9, 8, 7, 6)),
    WORKLOADS["tiny_4x8x8"],
    WORKLOADS["small_8x16x16"],
]


def problem(w, perms):
    return paro.Problem(w.B, w.heads, (w.F, w.H, w.W), w.d, w.block, perms)


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_reorder_bit_exact(w):
    q, _, _, perms = inputs(w)
    pr = problem(w, perms)
    (qd,) = to_dev(q)
    xp = paro.reorder(qd, pr)
    want = ref.reorder(q.numpy() if q.dtype == torch.float32 else q.view(torch.int16).numpy(),
                       (w.F, w.H, w.W), perms, w.block)
    got = xp.cpu()
    got = got.numpy() if got.dtype == torch.float32 else got.view(torch.int16).numpy()
    assert (got == want).all()
    # the fused block means from the same read
    xp2, pool = paro.reorder(qd, pr, with_pool=True)
    assert torch.equal(xp2, xp)
    oq = ref.block_pool(ref.reorder(q.double().numpy(), (w.F, w.H, w.W), perms, w.block),
                        w.N, w.block)
    assert np.abs(pool.cpu().double().numpy() - oq).max() < 1e-5
    back = paro.inverse_reorder(xp, pr).cpu()
    assert torch.equal(back.view(torch.int16) if back.dtype == torch.bfloat16 else back,
                       q.view(torch.int16) if q.dtype == torch.bfloat16 else q)


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_block_scores(w):
    q, k, _, perms = inputs(w)
    pr = problem(w, perms)
    qd, kd = to_dev(q, k)
    qp, kp, s = paro.block_score(qd, kd, pr)
    oq, ok_, os_ = ref.pooled_scores(as_f64(q), as_f64(k), (w.F, w.H, w.W), perms, w.block)
    assert np.abs(qp.cpu().double().numpy() - oq).max() < 1e-5
    assert np.abs(kp.cpu().double().numpy() - ok_).max() < 1e-5
    # scores: cancellation-aware bound |q_bar||k_bar|/sqrt(d) * 1e-5
    scale = (np.linalg.norm(oq, axis=-1)[..., :, None] * np.linalg.norm(ok_, axis=-1)[..., None, :]
             / np.sqrt(w.d))
    assert (np.abs(s.cpu().double().numpy() - os_) <= 1e-5 * scale + 1e-6).all()
    # the standalone score entry point gives the same bits
    s2 = paro.score_pooled(qp, kp, pr)
    assert torch.equal(s, s2)


def random_scores(rng, B, heads, nb, kind):
    if kind == "normal":
        s = rng.standard_normal((B, heads, nb, nb)).astype(np.float32)
    else:  # heavy ties, signed zeros, NaN and infinities
        s = rng.integers(-3, 4, size=(B, heads, nb, nb)).astype(np.float32)
        m = rng.random(s.shape)
        s[m < 0.05] = -0.0
        s[(m >= 0.05) & (m < 0.07)] = np.nan
        s[(m >= 0.07) & (m < 0.08)] = np.inf
        s[(m >= 0.08) & (m < 0.09)] = -np.inf
    return s


@pytest.mark.parametrize("nb,k", [(1, 1), (4, 2), (33, 7), (256, 64), (591, 89), (929, 186), (100, 100)])
@pytest.mark.parametrize("kind", ["normal", "ties"])
def test_topk_bit_exact(nb, k, kind):
    rng = np.random.default_rng(nb * 7 + k)
    heads = 3 if nb < 500 else 1
    s = random_scores(rng, 1, heads, nb, kind)
    pr = paro.Problem(1, heads, (1, 1, nb * 64), 64, 64, [0] * heads)
    assert pr.NB == nb
    idx = paro.select_topk(torch.from_numpy(s).cuda(), pr, k).cpu().numpy()
    want = ref.select_topk(s.astype(np.float64), k)
    assert (idx == want).all()


@pytest.mark.parametrize("w", CASES[:3] + [WORKLOADS["480p_21x30x52"]], ids=lambda w: w.name)
def test_topk_on_pooled_scores(w):
    """Selection on realistic score structure: the oracle's pooled scores of
    the synthetic inputs, rounded to float32, given to both sides."""
    q, k, _, perms = inputs(w, heads=2 if w.heads > 2 else None)
    _, _, s = ref.pooled_scores(as_f64(q), as_f64(k), (w.F, w.H, w.W), perms, w.block)
    s32 = s.astype(np.float32)
    heads = q.shape[1]
    pr = paro.Problem(w.B, heads, (w.F, w.H, w.W), w.d, w.block, perms)
    kk = ref.k_for_density(pr.NB, w.density)
    assert paro.k_for_density(pr.NB, w.density) == kk
    idx = paro.select_topk(torch.from_numpy(s32).cuda(), pr, kk).cpu().numpy()
    want = ref.select_topk(s32.astype(np.float64), kk)
    assert (idx == want).all()


@pytest.mark.parametrize("nb", [1, 4, 31, 32, 33, 70, 591])
def test_compact_bit_exact(nb):
    rng = np.random.default_rng(nb)
    words = -(-nb // 32)
    bm = rng.integers(0, 2**32, size=(1, 2, nb, words), dtype=np.uint64).astype(np.uint32)
    bm[0, 0, 0] = 0  # an empty row
    pr = paro.Problem(1, 2, (1, 1, nb * 64), 64, 64, [0, 0])
    idx, counts = paro.compact_mask(torch.from_numpy(bm.view(np.int32)).cuda(), pr)
    want_idx, want_counts = ref.compact_mask(bm, nb)
    assert (counts.cpu().numpy() == want_counts).all()
    assert (idx.cpu().numpy() == want_idx).all()


@pytest.mark.parametrize("w", CASES + [WORKLOADS["longclip_33x45x80_int8"]], ids=lambda w: w.name)
def test_quantize_bit_exact(w):
    q, _, _, perms = inputs(w, heads=2 if w.heads > 6 else None)
    heads = q.shape[1]
    pr = paro.Problem(w.B, heads, (w.F, w.H, w.W), w.d, w.block, perms)
    (qd,) = to_dev(q)
    x8, sc, pool = paro.quantize_int8(qd, pr, with_pool=True)
    xp = ref.reorder(q.float().numpy(), (w.F, w.H, w.W), perms, w.block)
    want8, want_sc = ref.quantize_int8(xp, w.N, w.block)
    assert (sc.cpu().numpy() == want_sc).all()
    assert (x8.cpu().numpy() == want8).all()
    oq = ref.block_pool(xp.astype(np.float64), w.N, w.block)
    assert np.abs(pool.cpu().double().numpy() - oq).max() < 1e-5
