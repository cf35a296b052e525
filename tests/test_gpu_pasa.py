"""GPU parity of block-sparse attention with PASA's grouped first-order
compensation of the unselected key blocks (PASA, arXiv 2604.12219, Pith
review page, Figure 2 caption) against the float64 oracle
(oracle/pasa_ref.py), through the C ABI.

The kept lists are the oracle's own top-k (or variable-length prefixes of
it, empty rows included), so both sides compute the same definition; the
GPU's pooled keys and values are fp32 means of the bf16 rows, rounded to
bf16 in the kernel like the K and V tiles, or rounded once per call by
pa_round_bf16 and loaded like the K and V tiles (the bf16-means form, which
must give the same bits).  bf16 with d = 128 and block 128
runs on the tcgen05 kernel (pooled tiles after the kept ones), the other
shapes and fp32 on the mma.sync kernel.  Outputs start as NaN, so every row
must be written.  Tolerance: the bf16 one (2e-2 max-abs, 2e-3 mean-abs)."""

import numpy as np
import pytest
import torch

from block_sparse_attention_34_b200 import paro
from block_sparse_attention_34_b200.configs import WORKLOADS
from block_sparse_attention_34_b200.synth import as_f64
from oracle import paro_ref as ref
from oracle import pasa_ref as pasa

from helpers import BF16_MAX_ABS, BF16_MEAN_ABS, compare, compare_rows, custom, inputs, \
    oracle_topk, selection_agreement, to_dev, token_mask

pytestmark = pytest.mark.gpu

CASES = [
    custom("pasa_512", 1, 2, 128, (4, 8, 16), 128, "bf16", 0.5, perms=(0, 5)),
    custom("pasa_ragged_315", 1, 3, 128, (5, 7, 9), 128, "bf16", 0.34, perms=(1, 3, 4)),
    custom("pasa_d64_b64_240", 2, 2, 64, (4, 6, 10), 64, "bf16", 0.5, perms=(2, 0)),
    custom("pasa_f32_384", 1, 2, 128, (3, 8, 16), 128, "f32", 0.34, perms=(4, 1)),
    # more key blocks than one pooled tile holds (NB = 144 > 128, NB = 80 > 64)
    custom("pasa_nb144", 1, 1, 128, (8, 32, 72), 128, "bf16", 0.1, perms=(3,)),
    custom("pasa_b64_nb80", 1, 2, 64, (4, 32, 40), 64, "bf16", 0.15, perms=(5, 2)),
]


def problem(w, perms):
    return paro.Problem(w.B, w.heads, (w.F, w.H, w.W), w.d, w.block, perms)


def tcgen05_shape(w):
    return w.dtype == "bf16" and w.d == 128 and w.block == 128


def run_gpu(w, q, k, v, perms, idx, counts, permuted, bf16_means=False):
    pr = problem(w, perms)
    qd, kd, vd = to_dev(q, k, v)
    qp, _ = paro.reorder(qd, pr, with_pool=True)
    kp, k_pool = paro.reorder(kd, pr, with_pool=True)
    vp, v_pool = paro.reorder(vd, pr, with_pool=True)
    if bf16_means:
        k_pool, v_pool = paro.round_bf16(k_pool), paro.round_bf16(v_pool)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    idx_d = torch.from_numpy(np.ascontiguousarray(idx, dtype=np.int32)).cuda()
    cnt_d = None if counts is None else torch.from_numpy(
        np.ascontiguousarray(counts, dtype=np.int32)).cuda()
    # every output row must be written
    out = torch.full((w.B, w.heads, w.N, w.d), float("nan"), dtype=qd.dtype, device="cuda")
    if permuted:
        out = paro.block_sparse_attn_compensated(qp, kp, vp, pr, idx_d, k_pool, v_pool, cnt_d,
                                                 out=out, status=status, permuted=True)
    else:
        out = paro.block_sparse_attn_compensated(qd, kd, vd, pr, idx_d, k_pool, v_pool, cnt_d,
                                                 out=out, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    return out


@pytest.mark.parametrize("permuted", [True, False], ids=["permuted", "natural"])
@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_compensated_matches_oracle(w, permuted):
    q, k, v, perms = inputs(w)
    idx, _, _ = oracle_topk(q, k, w, perms)
    out = run_gpu(w, q, k, v, perms, idx, None, permuted)
    want = pasa.attention_compensated(as_f64(q), as_f64(k), as_f64(v), (w.F, w.H, w.W), perms,
                                      w.block, idx)
    compare(out, want)
    if tcgen05_shape(w):
        # bf16 block means loaded like K and V tiles: the same bits
        out2 = run_gpu(w, q, k, v, perms, idx, None, permuted, bf16_means=True)
        assert torch.equal(out2, out)
    # the compensation is not a no-op on these inputs (unless every block is kept)
    plain = ref.attention(as_f64(q), as_f64(k), as_f64(v), (w.F, w.H, w.W), perms, w.block, idx)
    if idx.shape[-1] < w.NB:
        assert np.abs(want - plain).max() > 1e-3


def test_variable_counts_and_empty_rows():
    w = CASES[1]
    q, k, v, perms = inputs(w)
    idx, _, kk = oracle_topk(q, k, w, perms, density=1.0)  # all NB blocks, ascending
    rng = np.random.default_rng(5)
    counts = rng.integers(0, w.NB + 1, size=idx.shape[:-1]).astype(np.int32)
    counts[0, 0, 0] = 0  # a query block with no kept block: compensation alone
    counts[0, 1, 1] = w.NB  # and one with every block kept: plain dense rows
    idx = idx.copy()
    for b in range(w.B):
        for h in range(w.heads):
            for i in range(w.NB):
                # a kept list is any ascending subset; take a seeded one
                pick = np.sort(rng.choice(w.NB, counts[b, h, i], replace=False))
                idx[b, h, i, :] = -1
                idx[b, h, i, :pick.size] = pick
    want = pasa.attention_compensated(as_f64(q), as_f64(k), as_f64(v), (w.F, w.H, w.W), perms,
                                      w.block, idx, counts)
    for permuted in (False, True):
        for bf16_means in (False, True):
            out = run_gpu(w, q, k, v, perms, idx, counts, permuted, bf16_means)
            compare(out, want)


def test_round_bf16_is_round_to_nearest_even():
    x = torch.randn(1000003, dtype=torch.float32, device="cuda") * 3.0
    x[:4] = torch.tensor([1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -0.0, 65504.0])
    y = paro.round_bf16(x)
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), x.to(torch.bfloat16).view(torch.int16))


def test_bf16_means_need_the_tcgen05_kernel():
    w = CASES[2]  # d = 64, block = 64: the mma.sync kernel
    q, k, v, perms = inputs(w)
    idx, _, _ = oracle_topk(q, k, w, perms)
    with pytest.raises(paro.ParoError, match="UNSUPPORTED"):
        run_gpu(w, q, k, v, perms, idx, None, permuted=True, bf16_means=True)


def test_api_compensate_flag():
    w = CASES[0]
    q, k, v, perms = inputs(w)
    qd, kd, vd = to_dev(q, k, v)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, idx = paro.attention(qd, kd, vd, (w.F, w.H, w.W), perms, w.block, w.density,
                              status=status, compensate=True)
    torch.cuda.synchronize()
    assert status.item() == 0
    idx_ref, s_ref, _ = oracle_topk(q, k, w, perms)
    agree = selection_agreement(idx.cpu().numpy(), idx_ref, s_ref)
    assert agree.mean() >= 0.95
    want = pasa.attention_compensated(as_f64(q), as_f64(k), as_f64(v), (w.F, w.H, w.W), perms,
                                      w.block, idx_ref)
    compare_rows(out, want, token_mask(agree, (w.F, w.H, w.W), perms, w.block))


def test_every_block_kept_equals_plain_attention():
    w = custom("pasa_dense_780", 1, 2, 128, (6, 10, 13), 128, "bf16", 1.0, perms=(4, 0))
    q, k, v, perms = inputs(w)
    idx, _, _ = oracle_topk(q, k, w, perms)
    out = run_gpu(w, q, k, v, perms, idx, None, permuted=True)
    want = ref.attention(as_f64(q), as_f64(k), as_f64(v), (w.F, w.H, w.W), perms, w.block, idx)
    compare(out, want)


def test_480p_full_size_sampled():
    """The measured PASA workload (480p layer, 12 heads, top-k at 0.25, the
    compensated kernel on permuted tiles with bf16 block means) with the oracle's kept lists of
    every head; seeded rows plus each head's last token (ragged tail) are
    compared with the oracle's row evaluator."""
    w = WORKLOADS["480p_21x30x52"]
    q, k, v, perms = inputs(w)
    grid = (w.F, w.H, w.W)
    kk = ref.k_for_density(w.NB, w.density)
    idx = np.zeros((w.B, w.heads, w.NB, kk), dtype=np.int32)
    for h in range(w.heads):
        _, _, s = ref.pooled_scores(as_f64(q[:, h:h + 1]), as_f64(k[:, h:h + 1]), grid,
                                    perms[h:h + 1], w.block)
        idx[:, h:h + 1] = ref.select_topk(s, kk)
    out = run_gpu(w, q, k, v, perms, idx, None, permuted=True, bf16_means=True)
    rng = np.random.default_rng(13)
    rows = [(0, int(rng.integers(w.heads)), int(rng.integers(w.N))) for _ in range(96)]
    rows += [(0, h, w.N - 1) for h in range(w.heads)]
    want = pasa.compensated_rows(as_f64(q), as_f64(k), as_f64(v), grid, perms, w.block, idx, rows)
    got = out[0].float().cpu().numpy()
    got = np.stack([got[h, n] for (_, h, n) in rows]).astype(np.float64)
    err = np.abs(got - want)
    assert np.isfinite(got).all()
    assert err.max() <= BF16_MAX_ABS and err.mean() <= BF16_MEAN_ABS, (err.max(), err.mean())
