"""GPU parity of block-sparse attention against the float64 oracle, through
the C ABI.  Small cases are compared element by element on every output;
the full-size 720p-shaped layer (the bench workload, same launch) is
compared on seeded samples of output rows, which the oracle evaluates one
by one from the same definition."""

import numpy as np
import pytest
import torch

from block_sparse_attention_34_b200 import paro
from block_sparse_attention_34_b200.configs import WORKLOADS
from block_sparse_attention_34_b200.pipeline import Pipeline
from block_sparse_attention_34_b200.synth import as_f64
from oracle import paro_ref as ref

from helpers import (BF16_MAX_ABS, BF16_MEAN_ABS, compare, compare_rows, custom, inputs,
                     oracle_topk, selection_agreement, static_mask, to_dev, token_mask)

pytestmark = pytest.mark.gpu


def problem(w, perms, heads=None):
    return paro.Problem(w.B, heads or w.heads, (w.F, w.H, w.W), w.d, w.block, perms)


@pytest.mark.parametrize("name", ["tiny_4x8x8", "small_8x16x16"])
def test_static_mask_workloads(name):
    w = WORKLOADS[name]
    q, k, v, perms = inputs(w)
    bm, idx_ref = static_mask(w, q, k, perms)
    pr = problem(w, perms)
    qd, kd, vd = to_dev(q, k, v)
    idx, counts = paro.compact_mask(torch.from_numpy(bm.view(np.int32)).cuda(), pr)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = paro.block_sparse_attn(qd, kd, vd, pr, idx, counts, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    want = ref.attention(as_f64(q), as_f64(k), as_f64(v), (w.F, w.H, w.W), perms, w.block,
                         idx_ref)
    compare(out, want)


TC_CASES = [
    custom("ragged_315", 1, 6, 128, (5, 7, 9), 128, "bf16", 0.67, perms=(0, 1, 2, 3, 4, 5)),
    custom("ragged_780", 2, 3, 128, (6, 10, 13), 128, "bf16", 0.6, perms=(5, 2, 4)),
    custom("multi_tile_2048", 1, 2, 128, (8, 16, 16), 128, "bf16", 0.75, perms=(3, 1)),
    custom("dense_780", 1, 2, 128, (6, 10, 13), 128, "bf16", 1.0, perms=(4, 0)),
]


PATHS = {"tcgen05_permuted": dict(permuted=True), "tcgen05_gather": dict(permuted=False),
         "mma_sync": dict(baseline=True)}


@pytest.mark.parametrize("path", list(PATHS))
@pytest.mark.parametrize("w", TC_CASES, ids=lambda w: w.name)
def test_topk_pipeline_small(w, path):
    q, k, v, perms = inputs(w)
    pr = problem(w, perms)
    qd, kd, vd = to_dev(q, k, v)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, idx = paro.attention(qd, kd, vd, (w.F, w.H, w.W), perms, w.block, w.density,
                              status=status, **PATHS[path])
    torch.cuda.synchronize()
    assert status.item() == 0
    check_against_oracle_selection(w, q, k, v, perms, out, idx)


def check_against_oracle_selection(w, q, k, v, perms, out, idx):
    """Kept lists equal the oracle's (near ties excepted) and the output
    equals the oracle's attention over the oracle's lists on those rows."""
    idx_ref, s_ref, _ = oracle_topk(q, k, w, perms)
    agree = selection_agreement(idx.cpu().numpy(), idx_ref, s_ref)
    assert agree.mean() >= 0.95
    want = ref.attention(as_f64(q), as_f64(k), as_f64(v), (w.F, w.H, w.W), perms, w.block, idx_ref)
    compare_rows(out, want, token_mask(agree, (w.F, w.H, w.W), perms, w.block))


@pytest.mark.parametrize("path", list(PATHS))
def test_variable_counts_and_edge_rows(path):
    """Ragged kept lists (counts), rows that skip their diagonal, an empty
    row (zeros), and the last (partial) block kept by every row."""
    w = custom("edge_1300", 1, 4, 128, (5, 10, 26), 128, "bf16", 1.0, perms=(0, 3, 5, 1))
    q, k, v, perms = inputs(w)
    nb = w.NB
    rng = np.random.default_rng(5)
    idx = np.full((1, w.heads, nb, nb), -1, dtype=np.int32)
    counts = np.zeros((1, w.heads, nb), dtype=np.int32)
    for h in range(w.heads):
        for i in range(nb):
            c = int(rng.integers(1, nb + 1))
            pick = set(rng.choice(nb, c, replace=False).tolist()) | {nb - 1}
            if (h + i) % 3 == 0:
                pick.discard(i)
                pick.add(nb - 1)
            row = sorted(pick)
            idx[0, h, i, :len(row)] = row
            counts[0, h, i] = len(row)
    counts[0, 1, 2] = 0  # empty row -> zeros
    pr = problem(w, perms)
    qd, kd, vd = to_dev(q, k, v)
    if PATHS[path].get("permuted"):
        qd, kd, vd = (paro.reorder(x, pr) for x in (qd, kd, vd))
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = paro.block_sparse_attn(qd, kd, vd, pr, torch.from_numpy(idx).cuda(),
                                 torch.from_numpy(counts).cuda(), status=status, **PATHS[path])
    torch.cuda.synchronize()
    assert status.item() == 0
    want = ref.attention(as_f64(q), as_f64(k), as_f64(v), (w.F, w.H, w.W), perms, w.block, idx,
                         counts)
    compare(out, want)


@pytest.mark.parametrize("path", list(PATHS))
def test_malformed_list_is_reported_not_fatal(path):
    w = custom("bad_list", 1, 2, 128, (4, 8, 16), 128, "bf16", 1.0, perms=(0, 5))
    q, k, v, perms = inputs(w)
    pr = problem(w, perms)
    qd, kd, vd = to_dev(q, k, v)
    if PATHS[path].get("permuted"):
        qd, kd, vd = (paro.reorder(x, pr) for x in (qd, kd, vd))
    idx = torch.tensor([[[[0, 1], [1, 1], [2, 3], [0, 9]], [[0, 1], [1, 0], [2, 3], [3, 2]]]],
                       dtype=torch.int32, device="cuda")  # repeats, out of range, descending
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = torch.full((1, 2, w.N, w.d), 7.0, dtype=torch.bfloat16, device="cuda")
    paro.block_sparse_attn(qd, kd, vd, pr, idx, out=out, status=status, **PATHS[path])
    torch.cuda.synchronize()
    assert status.item() == paro.PA_ERR_DEVICE_CHECK
    # the well-formed rows are still right
    want = ref.attention(as_f64(q), as_f64(k), as_f64(v), (w.F, w.H, w.W), perms, w.block,
                         np.array([[[[0, 1], [0, 1], [2, 3], [0, 1]], [[0, 1], [0, 1], [2, 3], [2, 3]]]]))
    got = out.float().cpu().numpy()
    blk = {}
    for h in range(2):
        x = ref.reorder_head(np.arange(w.N, dtype=np.float64)[:, None], (w.F, w.H, w.W), perms[h],
                             w.block)[:w.N, 0].astype(int)
        for i, good in enumerate([[True, False, True, False], [True, False, True, False]][h]):
            rows = x[i * w.block:(i + 1) * w.block]
            if good:
                assert np.abs(got[0, h, rows] - want[0, h, rows]).max() < BF16_MAX_ABS
            else:
                assert (got[0, h, rows] == 7.0).all()


def test_480p_two_heads_full():
    w = WORKLOADS["480p_21x30x52"]
    q, k, v, perms = inputs(w, heads=2)
    pr = problem(w, perms, heads=2)
    qd, kd, vd = to_dev(q, k, v)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, idx = paro.attention(qd, kd, vd, (w.F, w.H, w.W), perms, w.block, w.density,
                              status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    check_against_oracle_selection(w, q, k, v, perms, out, idx)


@pytest.fixture(scope="module")
def c720():
    w = WORKLOADS["720p_21x45x80"]
    q, k, v, perms = inputs(w)
    return w, q, k, v, perms


def sampled_rows(w, n, seed):
    rng = np.random.default_rng(seed)
    rows = [(0, int(rng.integers(w.heads)), int(rng.integers(w.N))) for _ in range(n)]
    # always include the last token of every head (ragged tail block)
    rows += [(0, h, w.N - 1) for h in range(0, w.heads, 7)]
    return rows


@pytest.mark.parametrize("density", [0.15, 1.0])
def test_720p_full_size_sampled(c720, density):
    """The bench's launch sequence (Pipeline) on the full 720p-shaped layer."""
    w, q, k, v, perms = c720
    pipe = Pipeline(w.B, w.heads, (w.F, w.H, w.W), w.d, w.block, perms, density)
    assert pipe.k == ref.k_for_density(w.NB, density)
    qkv = to_dev(q, k, v)
    out = pipe.run(*qkv)
    torch.cuda.synchronize()
    assert pipe.status.item() == 0
    idx_h = pipe.idx.cpu().numpy()
    rows = sampled_rows(w, 192 if density < 1.0 else 48, seed=11)
    heads = sorted({h for (_, h, _) in rows})
    idx_ref = np.zeros_like(idx_h)
    if density < 1.0:
        # the kept lists of the sampled heads are the oracle's top-k of its
        # float64 pooled scores (near ties excepted), and the scores agree
        agree = np.ones(idx_h.shape[:3], dtype=bool)
        for hh in heads:
            _, _, s_ref = ref.pooled_scores(as_f64(q[:, hh:hh + 1]), as_f64(k[:, hh:hh + 1]),
                                            (w.F, w.H, w.W), perms[hh:hh + 1], w.block)
            got_s = pipe.scores[:, hh:hh + 1].cpu().double().numpy()
            assert np.abs(got_s - s_ref).max() < 1e-4 * max(1.0, np.abs(s_ref).max())
            idx_ref[:, hh:hh + 1] = ref.select_topk(s_ref, ref.k_for_density(w.NB, density))
            agree[:, hh:hh + 1] = selection_agreement(idx_h[:, hh:hh + 1], idx_ref[:, hh:hh + 1],
                                                      s_ref)
        tok_ok = token_mask(agree, (w.F, w.H, w.W), perms, w.block)
        rows = [r for r in rows if tok_ok[r]]
        assert len(rows) >= 150
    else:
        idx_ref[:] = np.arange(w.NB, dtype=np.int32)
        assert (idx_h == idx_ref).all()
    want = ref.attention_rows(as_f64(q), as_f64(k), as_f64(v), (w.F, w.H, w.W), perms, w.block,
                              idx_ref, rows)
    got = out[0].float().cpu().numpy()
    got = np.stack([got[h, n] for (_, h, n) in rows]).astype(np.float64)
    err = np.abs(got - want)
    assert np.isfinite(got).all()
    assert err.max() <= BF16_MAX_ABS and err.mean() <= BF16_MEAN_ABS, (err.max(), err.mean())
    # every output row was written (the buffer came from torch.empty)
    assert torch.isfinite(out).all()
