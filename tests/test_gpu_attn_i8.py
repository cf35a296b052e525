"""GPU parity of the INT8 block-sparse attention (tcgen05 kind::i8) against
the oracle's INT8 semantics, through the C ABI.

The oracle's default reading of the pages: per-block symmetric Q/K/V codes;
the exactly normalised post-softmax P quantised per (query block, key
block) tile with the tile's own absmax / L (L = 127, or 7 for 4-bit P).
The kernel's two-pass form (PA_ATTN_P_TILE) computes that reading and is
compared with it at the bf16 tolerance (2e-2 / 2e-3).  The one-pass form
(the un-normalised tile numerator rounded with the fixed scale 1/L under a
running row max) is compared with the oracle's "online" replay of that
order at the bf16 tolerance, and at 8 bits with the tile reading at the
INT8 tolerance (6e-2 max-abs / 6e-3 mean-abs); at 4 bits the two readings
differ by more than that (measured on these cases: up to 5e-2 max, 8e-3
mean), which is why INT4 PV takes the two-pass form by default.

The codes and scales the kernel reads come from pa_quantize_int8 and are
first checked bit-exact against the oracle's quantisation; the kept lists
are the oracle's.  Small cases are compared on every output row; the
full-size long-clip layer on sampled rows."""

import numpy as np
import pytest
import torch

from block_sparse_attention_34_b200 import paro
from block_sparse_attention_34_b200.configs import WORKLOADS
from block_sparse_attention_34_b200.pipeline import Pipeline
from block_sparse_attention_34_b200.synth import as_f64
from oracle import paro_ref as ref

from helpers import (BF16_MAX_ABS, BF16_MEAN_ABS, INT8_MAX_ABS, INT8_MEAN_ABS, compare,
                     compare_rows, custom, inputs, oracle_topk, selection_agreement, to_dev,
                     token_mask, token_rows)

pytestmark = pytest.mark.gpu

CASES = [
    custom("ragged_315", 1, 6, 128, (5, 7, 9), 128, "bf16", 0.67, perms=(0, 1, 2, 3, 4, 5)),
    custom("ragged_780", 2, 3, 128, (6, 10, 13), 128, "bf16", 0.6, perms=(5, 2, 4)),
    custom("multi_tile_2048", 1, 2, 128, (8, 16, 16), 128, "bf16", 0.75, perms=(3, 1)),
    custom("dense_780", 1, 2, 128, (6, 10, 13), 128, "bf16", 1.0, perms=(4, 0)),
    custom("tiles_1800", 1, 3, 128, (5, 18, 20), 128, "bf16", 0.5, perms=(6, 8, 10)),
]


def problem(w, perms, heads=None):
    return paro.Problem(w.B, heads or w.heads, (w.F, w.H, w.W), w.d, w.block, perms)


def quantized(w, pr, perms, *xs, bits=(8, 8, 8)):
    """GPU codes/scales of each input (8-bit, or 4-bit where bits says so),
    checked bit-exact against the oracle's quantisation of the same permuted
    float32 values; returns ([(x8, scale)] on the device, [(x8, scale)] of
    the oracle)."""
    dev, host = [], []
    for x, nbits in zip(xs, bits):
        (xd,) = to_dev(x)
        x8, sc = paro.quantize_int8(xd, pr, bits=nbits)
        xp = ref.reorder(x.float().numpy(), (w.F, w.H, w.W), perms, w.block)
        want8, want_sc = ref.quantize_int8(xp, w.N, w.block, qmax=127 if nbits == 8 else 7)
        assert (x8.cpu().numpy() == want8).all() and (sc.cpu().numpy() == want_sc).all()
        dev.append((x8, sc))
        host.append((want8, want_sc))
    return dev, host


def oracle_int8(w, perms, host, idx, counts=None, p_levels=127, mode="tile"):
    """Oracle INT8 attention of every head, mapped to natural order."""
    (q8, sq), (k8, sk), (v8, sv) = host
    B, nh = q8.shape[:2]
    outp = np.zeros((B, nh, q8.shape[2], w.d))
    for b in range(B):
        for h in range(nh):
            outp[b, h] = ref.attention_int8(q8[b, h], k8[b, h], v8[b, h], sq[b, h], sk[b, h],
                                            sv[b, h], w.N, w.block, idx[b, h],
                                            None if counts is None else counts[b, h],
                                            p_levels=p_levels, mode=mode)
    return ref.inverse_reorder(outp, (w.F, w.H, w.W), perms, w.block)


def run_i8(pr, dev, idx, counts=None, out=None, p4=False, p_tile=False):
    (q8, sq), (k8, sk), (v8, sv) = dev
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    if out is None:  # every row must be written
        out = torch.full((pr.B, pr.heads, pr.N, pr.d), float("nan"), dtype=torch.bfloat16,
                         device="cuda")
    out = paro.block_sparse_attn(q8, k8, v8, pr, torch.as_tensor(idx).cuda(),
                                 None if counts is None else torch.as_tensor(counts).cuda(),
                                 scales=(sq, sk, sv), out=out, status=status, p4=p4,
                                 p_tile=p_tile)
    torch.cuda.synchronize()
    return out, status.item()


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_i8_topk_small(w):
    q, k, v, perms = inputs(w)
    pr = problem(w, perms)
    dev, host = quantized(w, pr, perms, q, k, v)
    idx_ref, _, _ = oracle_topk(q, k, w, perms)
    out, st = run_i8(pr, dev, idx_ref)
    assert st == 0 and out.dtype == torch.bfloat16
    want = oracle_int8(w, perms, host, idx_ref)
    compare(out, want, INT8_MAX_ABS, INT8_MEAN_ABS)
    # the kernel's own one-pass order, tighter
    compare(out, oracle_int8(w, perms, host, idx_ref, mode="online"), BF16_MAX_ABS,
            BF16_MEAN_ABS)
    # the two-pass form computes the tile reading itself
    out_t, st = run_i8(pr, dev, idx_ref, p_tile=True)
    assert st == 0
    compare(out_t, want, BF16_MAX_ABS, BF16_MEAN_ABS)


def test_i8_variable_counts_and_edge_rows():
    """Ragged kept lists, rows without their diagonal, an empty row (zeros)
    and the partial last block kept by every row."""
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
    counts[0, 1, 2] = 0
    pr = problem(w, perms)
    dev, host = quantized(w, pr, perms, q, k, v)
    out, st = run_i8(pr, dev, idx, counts)
    assert st == 0
    want = oracle_int8(w, perms, host, idx, counts)
    compare(out, want, INT8_MAX_ABS, INT8_MEAN_ABS)
    compare(out, oracle_int8(w, perms, host, idx, counts, mode="online"), BF16_MAX_ABS,
            BF16_MEAN_ABS)
    tok = token_rows((w.F, w.H, w.W), perms[1], w.block)[2 * w.block:3 * w.block]
    assert (out[0, 1, torch.from_numpy(tok).cuda()] == 0).all()
    for p4 in (False, True):
        dev_p, host_p = (dev, host) if not p4 else quantized(w, pr, perms, q, k, v,
                                                             bits=(8, 8, 4))
        out_t, st = run_i8(pr, dev_p, idx, counts, p4=p4, p_tile=True)
        assert st == 0
        compare(out_t, oracle_int8(w, perms, host_p, idx, counts, p_levels=7 if p4 else 127),
                BF16_MAX_ABS, BF16_MEAN_ABS)
        assert (out_t[0, 1, torch.from_numpy(tok).cuda()] == 0).all()


def test_i8_malformed_list_is_reported_not_fatal():
    w = custom("bad_list", 1, 2, 128, (4, 8, 16), 128, "bf16", 1.0, perms=(0, 5))
    q, k, v, perms = inputs(w)
    pr = problem(w, perms)
    dev, host = quantized(w, pr, perms, q, k, v)
    idx = np.array([[[[0, 1], [1, 1], [2, 3], [0, 9]], [[0, 1], [1, 0], [2, 3], [3, 2]]]],
                   dtype=np.int32)  # repeats, out of range, descending
    out = torch.full((1, 2, w.N, w.d), 7.0, dtype=torch.bfloat16, device="cuda")
    out, st = run_i8(pr, dev, idx, out=out)
    assert st == paro.PA_ERR_DEVICE_CHECK
    good = np.array([[[[0, 1], [0, 1], [2, 3], [0, 1]], [[0, 1], [0, 1], [2, 3], [2, 3]]]],
                    dtype=np.int32)
    want = oracle_int8(w, perms, host, good)
    got = out.float().cpu().numpy()
    for h in range(2):
        tok = token_rows((w.F, w.H, w.W), perms[h], w.block)
        for i, ok in enumerate([True, False, True, False]):
            rows = tok[i * w.block:(i + 1) * w.block]
            if ok:
                assert np.abs(got[0, h, rows] - want[0, h, rows]).max() < INT8_MAX_ABS
            else:
                assert (got[0, h, rows] == 7.0).all()


def test_i8_whole_path_small():
    """paro.attention(int8=True): quantise with block means -> scores ->
    top-k -> INT8 attention; kept lists agree with the oracle's."""
    w = CASES[1]
    q, k, v, perms = inputs(w)
    pr = problem(w, perms)
    qd, kd, vd = to_dev(q, k, v)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, idx = paro.attention(qd, kd, vd, (w.F, w.H, w.W), perms, w.block, w.density, int8=True,
                              status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    idx_ref, s_ref, _ = oracle_topk(q, k, w, perms)
    agree = selection_agreement(idx.cpu().numpy(), idx_ref, s_ref)
    assert agree.mean() >= 0.95
    _, host = quantized(w, pr, perms, q, k, v)
    want = oracle_int8(w, perms, host, idx_ref)
    compare_rows(out, want, token_mask(agree, (w.F, w.H, w.W), perms, w.block), INT8_MAX_ABS,
                 INT8_MEAN_ABS)


def test_i8_longclip_full_size_sampled():
    """The bench's INT8 launch sequence (Pipeline) on the full long-clip
    layer (33x45x80 tokens, 24 heads), checked on sampled rows of six heads:
    quantised codes, kept lists and outputs against the oracle's INT8
    reading (6e-2 / 6e-3; the kernel's one-pass order tighter), and the
    INT8 output's distance from the float64 attention of the unquantised
    inputs reported beside the bf16 kernel's on the same rows."""
    w = WORKLOADS["longclip_33x45x80_int8"]
    q, k, v, perms = inputs(w)
    grid = (w.F, w.H, w.W)
    qd, kd, vd = to_dev(q, k, v)
    pipe = Pipeline(w.B, w.heads, grid, w.d, w.block, perms, w.density, int8=True)
    pipe.out.fill_(float("nan"))  # every row must be written
    out = pipe.run(qd, kd, vd)
    torch.cuda.synchronize()
    assert pipe.status.item() == 0
    assert torch.isfinite(out).all()
    assert pipe.k == ref.k_for_density(w.NB, w.density)
    pipe16 = Pipeline(w.B, w.heads, grid, w.d, w.block, perms, w.density)
    out16 = pipe16.run(qd, kd, vd)
    torch.cuda.synchronize()
    assert pipe16.status.item() == 0
    # the two-pass form on the same kept lists (its own selection is the same
    # computation, so the lists are compared)
    pipe_t = Pipeline(w.B, w.heads, grid, w.d, w.block, perms, w.density, int8=True,
                      p_tile=True)
    pipe_t.out.fill_(float("nan"))
    out_t = pipe_t.run(qd, kd, vd)
    torch.cuda.synchronize()
    assert pipe_t.status.item() == 0 and torch.equal(pipe_t.idx, pipe.idx)
    assert torch.isfinite(out_t).all()
    idx_h = pipe.idx.cpu().numpy()
    rng = np.random.default_rng(21)
    errs, errs_online, errs_tile, err_f64, err16_f64 = [], [], [], [], []
    for hh in (0, 5, 9, 14, 19, w.heads - 1):
        sl = slice(hh, hh + 1)
        ph = perms[sl]
        xp = [ref.reorder(x[:, sl].float().numpy(), grid, ph, w.block) for x in (q, k, v)]
        host = [ref.quantize_int8(x, w.N, w.block) for x in xp]
        for (x8, sc), dev8, dev_sc in zip(host, pipe.xq, pipe.sc):
            assert (dev8[:, sl].cpu().numpy() == x8).all()
            assert (dev_sc[:, sl].cpu().numpy() == sc).all()
        _, _, s_ref = ref.pooled_scores(as_f64(q[:, sl]), as_f64(k[:, sl]), grid, ph, w.block)
        idx_ref = ref.select_topk(s_ref, ref.k_for_density(w.NB, w.density))
        agree = selection_agreement(idx_h[:, sl], idx_ref, s_ref)[0, 0]
        # sampled permuted positions whose query block agrees, plus the tail
        pos = [int(p) for p in rng.integers(0, w.N, 24) if agree[int(p) // w.block]]
        if agree[(w.N - 1) // w.block]:
            pos.append(w.N - 1)
        assert len(pos) >= 16
        (q8, sq), (k8, sk), (v8, sv) = host
        args = (q8[0, 0], k8[0, 0], v8[0, 0], sq[0, 0], sk[0, 0], sv[0, 0], w.N, w.block,
                idx_ref[0, 0], pos)
        want = ref.attention_int8_rows(*args)
        want_online = ref.attention_int8_rows(*args, mode="online")
        tok = token_rows(grid, perms[hh], w.block)[pos]
        tok_d = torch.from_numpy(tok).cuda()
        got = out[0, hh, tok_d].float().cpu().double().numpy()
        errs.append(np.abs(got - want))
        errs_online.append(np.abs(got - want_online))
        errs_tile.append(np.abs(out_t[0, hh, tok_d].float().cpu().double().numpy() - want))
        f64 = ref.attention_rows(as_f64(q[:, sl]), as_f64(k[:, sl]), as_f64(v[:, sl]), grid, ph,
                                 w.block, idx_ref, [(0, 0, int(n)) for n in tok])
        err_f64.append(np.abs(got - f64))
        err16_f64.append(np.abs(out16[0, hh, tok_d].float().cpu().double().numpy() - f64))
    err = np.concatenate(errs)
    assert err.max() <= INT8_MAX_ABS and err.mean() <= INT8_MEAN_ABS, (err.max(), err.mean())
    err_o = np.concatenate(errs_online)
    assert err_o.max() <= BF16_MAX_ABS and err_o.mean() <= BF16_MEAN_ABS, (err_o.max(),
                                                                           err_o.mean())
    err_t = np.concatenate(errs_tile)
    assert err_t.max() <= BF16_MAX_ABS and err_t.mean() <= BF16_MEAN_ABS, (err_t.max(),
                                                                           err_t.mean())
    e8, e16 = np.concatenate(err_f64), np.concatenate(err16_f64)
    print(f"long clip, sampled rows: INT8 vs float64 attention of the unquantised inputs "
          f"max {e8.max():.3e} mean {e8.mean():.3e}; bf16 kernel max {e16.max():.3e} "
          f"mean {e16.mean():.3e}")
    # the INT8 path stays within its own tolerance of unquantised attention
    assert e8.max() <= INT8_MAX_ABS and e8.mean() <= INT8_MEAN_ABS


@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_int4_pv_small(w):
    """INT4 PV: q, k 8-bit, v 4-bit codes (bit-exact against the oracle's
    quantiser), P to 4 bits in the kernel: the two-pass form against the
    oracle's tile reading, the one-pass form against its online replay,
    both at the bf16 tolerance."""
    q, k, v, perms = inputs(w)
    pr = problem(w, perms)
    dev, host = quantized(w, pr, perms, q, k, v, bits=(8, 8, 4))
    assert int(dev[2][0].abs().max().item()) <= 7
    idx_ref, _, _ = oracle_topk(q, k, w, perms)
    out, st = run_i8(pr, dev, idx_ref, p4=True, p_tile=True)
    assert st == 0
    compare(out, oracle_int8(w, perms, host, idx_ref, p_levels=7), BF16_MAX_ABS, BF16_MEAN_ABS)
    out1, st = run_i8(pr, dev, idx_ref, p4=True)
    assert st == 0
    compare(out1, oracle_int8(w, perms, host, idx_ref, p_levels=7, mode="online"), BF16_MAX_ABS,
            BF16_MEAN_ABS)


def test_int4_pv_whole_path():
    w = CASES[1]
    q, k, v, perms = inputs(w)
    pr = problem(w, perms)
    qd, kd, vd = to_dev(q, k, v)
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, idx = paro.attention(qd, kd, vd, (w.F, w.H, w.W), perms, w.block, w.density, int8=True,
                              int4_pv=True, status=status)
    torch.cuda.synchronize()
    assert status.item() == 0
    idx_ref, s_ref, _ = oracle_topk(q, k, w, perms)
    agree = selection_agreement(idx.cpu().numpy(), idx_ref, s_ref)
    _, host = quantized(w, pr, perms, q, k, v, bits=(8, 8, 4))
    # INT4 PV takes the pages' tile reading by default
    want = oracle_int8(w, perms, host, idx_ref, p_levels=7)
    compare_rows(out, want, token_mask(agree, (w.F, w.H, w.W), perms, w.block), BF16_MAX_ABS,
                 BF16_MEAN_ABS)
