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
    # 3D tile blockings (ids 6-11) on a grid no tile divides
    custom("tiles_1800", 1, 6, 128, (5, 18, 20), 128, "bf16", 0.5, perms=(6, 7, 8, 9, 10, 11)),
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


def oracle_lists(w, q, k, perms, idx_gpu, density=None):
    """Per head: the oracle's kept lists (top-k of its float64 pooled
    scores), and the [B,h,NB] rows where the GPU's lists equal them (the
    others must be valid near-tie choices)."""
    idx_ref = np.zeros_like(idx_gpu)
    agree = np.ones(idx_gpu.shape[:3], dtype=bool)
    dens = w.density if density is None else density
    for hh in range(w.heads):
        sl = slice(hh, hh + 1)
        _, _, s_ref = ref.pooled_scores(as_f64(q[:, sl]), as_f64(k[:, sl]), (w.F, w.H, w.W),
                                        perms[sl], w.block)
        idx_ref[:, sl] = ref.select_topk(s_ref, ref.k_for_density(w.NB, dens))
        agree[:, sl] = selection_agreement(idx_gpu[:, sl], idx_ref[:, sl], s_ref)
    return idx_ref, agree


def test_480p_all_heads_full():
    """The bench's launch sequence (Pipeline) on the whole 480p-shaped layer
    (21x30x52 tokens, 12 heads, density 0.25): every output row of every
    head against the oracle over the oracle's kept lists."""
    w = WORKLOADS["480p_21x30x52"]
    q, k, v, perms = inputs(w)
    pipe = Pipeline(w.B, w.heads, (w.F, w.H, w.W), w.d, w.block, perms, w.density)
    pipe.out.fill_(float("nan"))  # every row must be written
    out = pipe.run(*to_dev(q, k, v))
    torch.cuda.synchronize()
    assert pipe.status.item() == 0
    assert torch.isfinite(out).all()
    assert pipe.k == ref.k_for_density(w.NB, w.density)
    idx_ref, agree = oracle_lists(w, q, k, perms, pipe.idx.cpu().numpy())
    assert agree.mean() >= 0.95
    want = ref.attention(as_f64(q), as_f64(k), as_f64(v), (w.F, w.H, w.W), perms, w.block, idx_ref)
    compare_rows(out, want, token_mask(agree, (w.F, w.H, w.W), perms, w.block))


@pytest.fixture(scope="module")
def c720():
    w = WORKLOADS["720p_21x45x80"]
    q, k, v, perms = inputs(w)
    return w, q, k, v, perms


def sampled_rows(w, per_head, seed):
    """per_head seeded rows of every head, plus each head's last token (the
    ragged tail block)."""
    rng = np.random.default_rng(seed)
    rows = []
    for h in range(w.heads):
        rows += [(0, h, int(n)) for n in rng.integers(0, w.N, per_head)]
        rows.append((0, h, w.N - 1))
    return rows


def full_size_sampled(w, q, k, v, perms, density, per_head, seed, min_rows):
    """Pipeline at full size; sampled rows of every head against the oracle
    row evaluator over the oracle's kept lists."""
    pipe = Pipeline(w.B, w.heads, (w.F, w.H, w.W), w.d, w.block, perms, density)
    assert pipe.k == ref.k_for_density(w.NB, density)
    pipe.out.fill_(float("nan"))  # every row must be written
    out = pipe.run(*to_dev(q, k, v))
    torch.cuda.synchronize()
    assert pipe.status.item() == 0
    assert torch.isfinite(out).all()
    idx_h = pipe.idx.cpu().numpy()
    rows = sampled_rows(w, per_head, seed)
    if density < 1.0:
        idx_ref, agree = oracle_lists(w, q, k, perms, idx_h, density)
        tok_ok = token_mask(agree, (w.F, w.H, w.W), perms, w.block)
        rows = [r for r in rows if tok_ok[r]]
        assert len(rows) >= min_rows
    else:
        idx_ref = np.broadcast_to(np.arange(w.NB, dtype=np.int32), idx_h.shape).copy()
        assert (idx_h == idx_ref).all()
    want = ref.attention_rows(as_f64(q), as_f64(k), as_f64(v), (w.F, w.H, w.W), perms, w.block,
                              idx_ref, rows)
    got = out[0].float().cpu().numpy()
    got = np.stack([got[h, n] for (_, h, n) in rows]).astype(np.float64)
    err = np.abs(got - want)
    assert err.max() <= BF16_MAX_ABS and err.mean() <= BF16_MEAN_ABS, (err.max(), err.mean())
    return err


@pytest.mark.parametrize("density", [0.15, 1.0])
def test_720p_full_size_sampled(c720, density):
    """The bench's launch sequence (Pipeline) on the full 720p-shaped layer
    (21x45x80 tokens, 40 heads): 5 seeded rows of every head (1 at density
    1.0) plus every head's last token."""
    w, q, k, v, perms = c720
    full_size_sampled(w, q, k, v, perms, density, 5 if density < 1.0 else 1, 11, 200)


def test_longclip_bf16_full_size_sampled():
    """The long-clip shape (33x45x80 tokens, 24 heads, density 0.20) in bf16
    through the Pipeline: 8 seeded rows of every head plus every head's last
    token."""
    w = WORKLOADS["longclip_33x45x80_int8"]
    q, k, v, perms = inputs(w)
    full_size_sampled(w, q, k, v, perms, w.density, 8, 13, 180)
