"""GPU parity of PAROAttention's offline stage (row softmax and block
statistics of the dense map on the tensor cores, the permutation metric and
choice, static masks by block-sum thresholding) against the oracle
(oracle/paro_offline_ref.py), through the C ABI.

Tolerances come from fp32 arithmetic on the GPU against float64: the
probabilities carry ~1e-6 relative error, so a block's count of entries
below eps may differ only by entries within 1e-4 eps of eps; sums and
maxima agree to 1e-4 relative; the order pick and the masks agree wherever
the oracle's decision is not a near tie, and are valid choices otherwise."""

import math

import numpy as np
import pytest
import torch

from block_sparse_attention_34_b200 import paro
from block_sparse_attention_34_b200.synth import as_f64
from oracle import paro_offline_ref as off
from oracle import paro_ref as ref
from oracle import selection_ref as sel

from helpers import custom, inputs, to_dev

pytestmark = pytest.mark.gpu

CASES = [
    custom("off_512", 1, 2, 128, (4, 8, 16), 128, "bf16", 0.5, perms=(0, 0)),
    custom("off_ragged_315", 1, 3, 128, (5, 7, 9), 128, "bf16", 0.5, perms=(0, 0, 0)),
    custom("off_2048", 2, 1, 128, (8, 16, 16), 128, "bf16", 0.5, perms=(0,)),
]


def oracle_head(qh, kh, grid, block, eps=1e-3):
    p = off.attention_map(qh, kh)
    return p, [off.block_stats(p, grid, o, block, eps) for o in range(6)]


def check_counts(got, want, pmap, grid, order, block, eps):
    """count may differ only by entries within 1e-4 eps of eps."""
    near = np.abs(off.permuted_map(pmap, grid, order) - eps) <= 1e-4 * eps
    N = pmap.shape[0]
    nb = -(-N // block)
    for i in range(nb):
        for j in range(nb):
            slack = near[i * block:(i + 1) * block, j * block:(j + 1) * block].sum()
            assert abs(got[i, j] - want[i, j]) <= slack, (order, i, j, got[i, j], want[i, j])


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_row_and_block_stats(w):
    q, k, _, _ = inputs(w)
    grid = (w.F, w.H, w.W)
    qd, kd = to_dev(q, k)
    B, heads = q.shape[:2]
    eps = 1e-3
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    row_max = row_sum = None
    stats = []
    for o in range(6):
        pr = paro.Problem(B, heads, grid, w.d, w.block, [o] * heads)
        qp, kp = paro.reorder(qd, pr), paro.reorder(kd, pr)
        if row_max is None:
            row_max, row_sum = paro.map_row_stats(qp, kp, pr, o, status)
        stats.append({key: (v.cpu().double().numpy() if v is not None else None) for key, v in
                      paro.map_block_stats(qp, kp, pr, o, row_max, row_sum, eps, True,
                                           status).items()})
    torch.cuda.synchronize()
    assert status.item() == 0
    rm, rs = row_max.cpu().double().numpy(), row_sum.cpu().double().numpy()
    for b in range(B):
        for h in range(heads):
            qh, kh = as_f64(q)[b, h], as_f64(k)[b, h]
            s = qh @ kh.T / math.sqrt(w.d)
            m = s.max(axis=1)
            assert np.abs(rm[b, h] - m * math.log2(math.e)).max() < 1e-4 * max(1.0, np.abs(m).max())
            lsum = np.exp(s - m[:, None]).sum(axis=1)
            assert np.abs(rs[b, h] / lsum - 1).max() < 1e-4
            pmap, want = oracle_head(qh, kh, grid, w.block, eps)
            for o in range(6):
                got = stats[o]
                check_counts(got["count"][b, h], want[o]["count"], pmap, grid, o, w.block, eps)
                assert np.abs(got["total"][b, h] - want[o]["total"]).max() <= 1e-4 * want[o]["size"].max()
                assert np.abs(got["peak"][b, h] - want[o]["peak"]).max() <= 1e-4
                with np.errstate(divide="ignore"):
                    lt = np.log(got["total"][b, h])
                assert np.allclose(got["log_total"][b, h], lt, rtol=1e-5, atol=1e-6)


def valid_mask_rows(total_row, i, sigma, got_row, rel=1e-4):
    """A GPU mask row is valid if it is the rule's row for a prefix that
    stops where the oracle's running block sum is within rel of sigma times
    its total, under any order of blocks whose sums are within rel."""
    logs = np.log(np.maximum(total_row, 1e-300))
    want = np.unique(np.concatenate(([i], sel.topp_row(logs, sigma))))
    if got_row == want.tolist():
        return True
    g = set(got_row) - {i}
    w_ = set(want.tolist()) - {i}
    diff = g ^ w_
    tot = total_row.sum()
    # every block in the difference is at the threshold: its sum is within
    # rel of the smallest kept sum of the oracle's set
    edge = min(total_row[j] for j in w_) if w_ else 0.0
    return all(abs(total_row[j] - edge) <= rel * tot for j in diff)


def test_offline_stage_matches_oracle():
    w = CASES[0]
    q, k, _, _ = inputs(w)
    grid = (w.F, w.H, w.W)
    qd, kd = to_dev(q, k)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    res = paro.paro_offline(qd, kd, grid, w.block, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    for h in range(w.heads):
        metric, sf, inc = off.permutation_metric(as_f64(q)[0, h], as_f64(k)[0, h], grid, w.block)
        assert np.abs(res["sparse_frac"][0, h].cpu().numpy() - sf).max() <= 1.0 / (w.NB ** 2) + 1e-6
        assert np.abs(res["incoherence"][0, h].cpu().numpy() / np.maximum(inc, 1e-30) - 1).max() < 1e-3
        # the oracle's candidates: its pick and every order within 1e-3 of it
        # (orders whose blocks hold the same token sets tie exactly)
        ties = [o for o in range(6) if metric[o] - metric.min() <= 1e-3]
        assert off.choose_order(metric) in ties
        assert int(res["orders"][0, h].item()) in ties
        # the GPU's static masks are the block-sum thresholding of one of them
        pmap = off.attention_map(as_f64(q)[0, h], as_f64(k)[0, h])
        idx = res["idx"][0, h].cpu().numpy()
        cnt = res["counts"][0, h].cpu().numpy()
        rows = [idx[i, :cnt[i]].tolist() for i in range(w.NB)]
        assert any(all(valid_mask_rows(tot[i], i, 0.9, rows[i]) for i in range(w.NB))
                   for tot in (off.block_stats(pmap, grid, o, w.block)["total"] for o in ties))


def test_frame_local_map_picks_frame_order_and_diagonal_masks():
    F, H, W, d = 4, 8, 16, 128  # H*W = 128 = block: one frame per block in FHW
    rng = np.random.default_rng(9)
    dirs = np.linalg.qr(rng.standard_normal((d, d)))[0][:F] * 12.0
    x = np.repeat(dirs, H * W, axis=0)
    qk = torch.from_numpy(np.stack([x, x])[None]).to(torch.bfloat16).cuda()  # [1, 2, N, d]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    res = paro.paro_offline(qk, qk, (F, H, W), 128, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    assert res["orders"].cpu().tolist() == [[0, 0]]
    assert (res["counts"] == 1).all()
    assert (res["idx"][..., 0].cpu() == torch.arange(F)).all()
