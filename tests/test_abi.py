"""The C ABI library on the CPU: it loads, exports every function that
include/paro.h declares, and rejects malformed arguments on the host before
any CUDA call (so these run without a GPU)."""

import ctypes
import os
import re

import numpy as np
import pytest

from block_sparse_attention_34_b200 import paro
from oracle import paro_ref as ref

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(paro.LIB_PATH):
        from block_sparse_attention_34_b200 import build
        build.build()
    return paro.load()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "paro.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_[a-z0-9_]+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), n
    assert lib.pa_abi_version() == paro.ABI_VERSION == 8


def test_k_for_density_matches_oracle(lib):
    rng = np.random.default_rng(0)
    for nb in [1, 2, 4, 10, 32, 256, 591, 929, 1000]:
        for dens in [0.0, 1e-9, 0.1, 0.15, 0.2, 0.25, 0.3, 0.5, 0.7, 1.0, 2.0,
                     *rng.random(20).tolist()]:
            assert lib.pa_k_for_density(nb, dens) == ref.k_for_density(nb, dens), (nb, dens)
    assert lib.pa_k_for_density(0, 0.5) == 0


def test_num_blocks(lib):
    assert lib.pa_num_blocks(paro.PaShape(1, 40, 21, 45, 80, 128, 128)) == 591
    assert lib.pa_num_blocks(paro.PaShape(1, 24, 33, 45, 80, 128, 128)) == 929
    assert lib.pa_num_blocks(paro.PaShape(1, 1, 0, 4, 4, 64, 64)) == -1


FAKE = ctypes.c_void_p(4096)  # never dereferenced: every case fails validation first


def perms_of(*ids):
    a = np.array(ids, dtype=np.int8)
    return a, a.ctypes.data_as(ctypes.c_void_p)


def test_host_validation(lib):
    good = paro.PaShape(1, 2, 4, 8, 8, 64, 64)
    keep, pp = perms_of(0, 5)
    # unsupported head dim and block
    assert lib.pa_reorder(FAKE, FAKE, paro.PA_BF16, paro.PaShape(1, 2, 4, 8, 8, 96, 64), pp, None, None) == paro.PA_ERR_UNSUPPORTED
    assert lib.pa_reorder(FAKE, FAKE, paro.PA_BF16, paro.PaShape(1, 2, 4, 8, 8, 64, 32), pp, None, None) == paro.PA_ERR_UNSUPPORTED
    assert b"block=32" in lib.pa_last_error()
    # malformed shape
    assert lib.pa_reorder(FAKE, FAKE, paro.PA_BF16, paro.PaShape(1, 0, 4, 8, 8, 64, 64), pp, None, None) == paro.PA_ERR_INVALID_ARG
    # wrong dtype for reorder
    assert lib.pa_reorder(FAKE, FAKE, paro.PA_I8, good, pp, None, None) == paro.PA_ERR_INVALID_ARG
    # bad order id
    keep2, bad = perms_of(0, 12)  # ids 0-11 are valid (axis orders, tile blockings)
    assert lib.pa_reorder(FAKE, FAKE, paro.PA_BF16, good, bad, None, None) == paro.PA_ERR_INVALID_ARG
    assert b"perms[1]=12" in lib.pa_last_error()
    keep3, neg = perms_of(-1, 0)
    assert lib.pa_reorder(FAKE, FAKE, paro.PA_BF16, good, neg, None, None) == paro.PA_ERR_INVALID_ARG
    # NULL perms / pointers / misaligned pointers
    assert lib.pa_reorder(FAKE, FAKE, paro.PA_BF16, good, None, None, None) == paro.PA_ERR_INVALID_ARG
    assert lib.pa_reorder(None, FAKE, paro.PA_BF16, good, pp, None, None) == paro.PA_ERR_INVALID_ARG
    assert lib.pa_reorder(ctypes.c_void_p(4100), FAKE, paro.PA_BF16, good, pp, None, None) == paro.PA_ERR_INVALID_ARG
    # top-k: k out of range
    assert lib.pa_select_topk(FAKE, good, 0, FAKE, None) == paro.PA_ERR_INVALID_ARG
    assert lib.pa_select_topk(FAKE, good, 5, FAKE, None) == paro.PA_ERR_INVALID_ARG  # NB = 4
    # attention: INT8 without scales; k_max above NB
    assert lib.pa_block_sparse_attn(FAKE, FAKE, FAKE, paro.PA_I8, 0, paro.PaShape(1, 2, 4, 8, 8, 128, 128),
                                    pp, FAKE, None, 1, None, None, None, FAKE, None, None) == paro.PA_ERR_INVALID_ARG
    assert lib.pa_block_sparse_attn(FAKE, FAKE, FAKE, paro.PA_BF16, 0, good, pp, FAKE, None, 9,
                                    None, None, None, FAKE, None, None) == paro.PA_ERR_INVALID_ARG
    # INT8 needs the tcgen05 shape
    assert lib.pa_block_sparse_attn(FAKE, FAKE, FAKE, paro.PA_I8, 0, good, pp, FAKE, None, 2,
                                    FAKE, FAKE, FAKE, FAKE, None, None) == paro.PA_ERR_UNSUPPORTED
    # baseline refuses INT8
    assert lib.pa_block_sparse_attn_mma(FAKE, FAKE, FAKE, paro.PA_I8, 0, good, pp, FAKE, None, 2,
                                        FAKE, None, None) == paro.PA_ERR_INVALID_ARG
    # unknown flag bits
    assert lib.pa_block_sparse_attn(FAKE, FAKE, FAKE, paro.PA_BF16, 6, good, pp, FAKE, None, 2,
                                    None, None, None, FAKE, None, None) == paro.PA_ERR_INVALID_ARG
    # too many heads
    many = np.zeros(2000, dtype=np.int8)
    assert lib.pa_reorder(FAKE, FAKE, paro.PA_BF16, paro.PaShape(1, 2000, 4, 8, 8, 64, 64),
                          many.ctypes.data_as(ctypes.c_void_p), None, None) == paro.PA_ERR_UNSUPPORTED


def test_binding_refuses_cpu_tensors(lib):
    import torch
    pr = paro.Problem(1, 2, (4, 8, 8), 64, 64, [0, 5])
    x = torch.zeros(1, 2, 256, 64)
    with pytest.raises(ValueError):
        paro.reorder(x, pr)


def test_selection_variant_validation(lib):
    good = paro.PaShape(1, 2, 4, 8, 8, 64, 64)  # NB = 4
    # hybrid: k range, finite top_p, null outputs, NB limit
    assert lib.pa_select_hybrid(FAKE, good, -1, 0.5, 1, FAKE, FAKE, None) == paro.PA_ERR_INVALID_ARG
    assert lib.pa_select_hybrid(FAKE, good, 5, 0.5, 1, FAKE, FAKE, None) == paro.PA_ERR_INVALID_ARG
    assert lib.pa_select_hybrid(FAKE, good, 2, float("nan"), 1, FAKE, FAKE, None) == paro.PA_ERR_INVALID_ARG
    assert b"top_p" in lib.pa_last_error()
    assert lib.pa_select_hybrid(FAKE, good, 2, 0.5, 1, FAKE, None, None) == paro.PA_ERR_INVALID_ARG
    big = paro.PaShape(1, 1, 1, 1, 4097 * 64, 64, 64)  # NB = 4097
    assert lib.pa_select_hybrid(FAKE, big, 2, 0.5, 1, FAKE, FAKE, None) == paro.PA_ERR_UNSUPPORTED
    # SICS: float inputs only, non-null buffers
    assert lib.pa_sics_scores(FAKE, FAKE, paro.PA_I8, good, FAKE, None, None) == paro.PA_ERR_INVALID_ARG
    assert lib.pa_sics_scores(FAKE, None, paro.PA_BF16, good, FAKE, None, None) == paro.PA_ERR_INVALID_ARG


def test_p4_flag_validation(lib):
    good = paro.PaShape(1, 2, 4, 8, 8, 64, 64)
    keep, pp = perms_of(0, 5)
    # PA_ATTN_P4 needs int8 inputs; unknown bits are refused
    assert lib.pa_block_sparse_attn(FAKE, FAKE, FAKE, paro.PA_BF16, paro.PA_ATTN_P4, good, pp, FAKE,
                                    None, 1, None, None, None, FAKE, None, None) == paro.PA_ERR_INVALID_ARG
    assert b"P4" in lib.pa_last_error()
    # PA_ATTN_P_TILE (4) needs int8 inputs too; bit 8 is unknown
    assert lib.pa_block_sparse_attn(FAKE, FAKE, FAKE, paro.PA_BF16, paro.PA_ATTN_P_TILE, good, pp,
                                    FAKE, None, 1, None, None, None, FAKE, None, None) == paro.PA_ERR_INVALID_ARG
    assert b"P_TILE" in lib.pa_last_error()
    assert lib.pa_block_sparse_attn(FAKE, FAKE, FAKE, paro.PA_BF16, 8, good, pp, FAKE,
                                    None, 1, None, None, None, FAKE, None, None) == paro.PA_ERR_INVALID_ARG
    assert b"unknown flags" in lib.pa_last_error()
    assert lib.pa_quantize_int4(FAKE, paro.PA_I8, good, pp, FAKE, FAKE, None, None) == paro.PA_ERR_INVALID_ARG


def test_offline_stage_validation(lib):
    good = paro.PaShape(1, 2, 4, 8, 8, 128, 128)
    small = paro.PaShape(1, 2, 4, 8, 8, 64, 64)
    assert lib.pa_map_row_stats(FAKE, FAKE, good, 6, FAKE, FAKE, None, None) == paro.PA_ERR_INVALID_ARG
    assert lib.pa_map_row_stats(FAKE, FAKE, small, 0, FAKE, FAKE, None, None) == paro.PA_ERR_UNSUPPORTED
    assert lib.pa_map_row_stats(FAKE, None, good, 0, FAKE, FAKE, None, None) == paro.PA_ERR_INVALID_ARG
    assert lib.pa_map_block_stats(FAKE, FAKE, good, 0, FAKE, FAKE, float("nan"), FAKE, FAKE, FAKE,
                                  None, None, None) == paro.PA_ERR_INVALID_ARG
    assert lib.pa_paro_metric(FAKE, FAKE, FAKE, good, -1, 0.9, FAKE, FAKE, None) == paro.PA_ERR_INVALID_ARG
    assert lib.pa_paro_choose(FAKE, FAKE, good, float("inf"), FAKE, FAKE, None) == paro.PA_ERR_INVALID_ARG


def test_empty_kept_lists_need_no_idx(lib):
    """k_max = 0: idx is never read, so NULL passes the idx check; the call
    here still fails validation, later, on a misaligned out (so no CUDA call
    is made), and its message names the alignment, not idx.  k_max > 0 with
    NULL idx is refused."""
    good = paro.PaShape(1, 2, 4, 8, 8, 64, 64)
    keep, pp = perms_of(0, 5)
    bad_out = ctypes.c_void_p(4100)
    st = lib.pa_block_sparse_attn(FAKE, FAKE, FAKE, paro.PA_BF16, 0, good, pp, None, None, 0,
                                  None, None, None, bad_out, None, None)
    assert st == paro.PA_ERR_INVALID_ARG and b"aligned" in lib.pa_last_error()
    st = lib.pa_block_sparse_attn(FAKE, FAKE, FAKE, paro.PA_BF16, 0, good, pp, None, None, 1,
                                  None, None, None, FAKE, None, None)
    assert st == paro.PA_ERR_INVALID_ARG and b"idx" in lib.pa_last_error()
    fn = lib.pa_block_sparse_attn_compensated
    assert fn(FAKE, FAKE, FAKE, paro.PA_BF16, 0, good, pp, None, None, 0, FAKE, FAKE,
              paro.PA_F32, bad_out, None, None) == paro.PA_ERR_INVALID_ARG
    assert b"aligned" in lib.pa_last_error()
    assert fn(FAKE, FAKE, FAKE, paro.PA_BF16, 0, good, pp, None, None, 2, FAKE, FAKE,
              paro.PA_F32, FAKE, None, None) == paro.PA_ERR_INVALID_ARG
    assert b"idx" in lib.pa_last_error()


def test_compensated_attention_validation(lib):
    good = paro.PaShape(1, 2, 4, 8, 8, 64, 64)  # NB = 4
    keep, pp = perms_of(0, 5)
    fn = lib.pa_block_sparse_attn_compensated
    # the pooled summaries are required and 16-byte aligned
    assert fn(FAKE, FAKE, FAKE, paro.PA_BF16, 0, good, pp, FAKE, None, 2, None, FAKE, paro.PA_F32, FAKE, None,
              None) == paro.PA_ERR_INVALID_ARG
    assert b"k_pool" in lib.pa_last_error()
    assert fn(FAKE, FAKE, FAKE, paro.PA_BF16, 0, good, pp, FAKE, None, 2, FAKE,
              ctypes.c_void_p(4100), paro.PA_F32, FAKE, None, None) == paro.PA_ERR_INVALID_ARG
    # bf16 / fp32 only, no INT4 flag, k_max within [0, NB]
    assert fn(FAKE, FAKE, FAKE, paro.PA_I8, 0, good, pp, FAKE, None, 2, FAKE, FAKE, paro.PA_F32, FAKE, None,
              None) == paro.PA_ERR_INVALID_ARG
    assert fn(FAKE, FAKE, FAKE, paro.PA_BF16, paro.PA_ATTN_P4, good, pp, FAKE, None, 2, FAKE, FAKE, paro.PA_F32,
              FAKE, None, None) == paro.PA_ERR_INVALID_ARG
    assert fn(FAKE, FAKE, FAKE, paro.PA_BF16, 0, good, pp, FAKE, None, 5, FAKE, FAKE, paro.PA_F32, FAKE, None,
              None) == paro.PA_ERR_INVALID_ARG
    # one bit per key block in shared memory: NB <= 4096
    big = paro.PaShape(1, 2, 65, 64, 64, 64, 64)  # NB = 4160
    assert fn(FAKE, FAKE, FAKE, paro.PA_BF16, 0, big, pp, FAKE, None, 2, FAKE, FAKE, paro.PA_F32, FAKE, None,
              None) == paro.PA_ERR_UNSUPPORTED
    assert b"4096" in lib.pa_last_error()
    # the means are float or bf16; bf16 means need the tcgen05 kernel (d = 128,
    # block = 128, PA_BF16), so this d = 64 shape is unsupported
    assert fn(FAKE, FAKE, FAKE, paro.PA_BF16, 0, good, pp, FAKE, None, 2, FAKE, FAKE, paro.PA_I8,
              FAKE, None, None) == paro.PA_ERR_INVALID_ARG
    assert fn(FAKE, FAKE, FAKE, paro.PA_BF16, 0, good, pp, FAKE, None, 2, FAKE, FAKE,
              paro.PA_BF16, FAKE, None, None) == paro.PA_ERR_UNSUPPORTED
    assert b"tcgen05" in lib.pa_last_error()
    wide = paro.PaShape(1, 2, 4, 8, 16, 128, 128)
    assert fn(FAKE, FAKE, FAKE, paro.PA_F32, 0, wide, pp, FAKE, None, 2, FAKE, FAKE,
              paro.PA_BF16, FAKE, None, None) == paro.PA_ERR_UNSUPPORTED


def test_round_bf16_validation(lib):
    fn = lib.pa_round_bf16
    assert fn(None, None, 0, None) == paro.PA_OK  # nothing to do
    assert fn(FAKE, FAKE, -1, None) == paro.PA_ERR_INVALID_ARG
    assert fn(None, FAKE, 8, None) == paro.PA_ERR_INVALID_ARG
    assert fn(FAKE, ctypes.c_void_p(4100), 8, None) == paro.PA_ERR_INVALID_ARG
    assert b"aligned" in lib.pa_last_error()


def test_topk_nb_limit_is_reported(lib):
    """NB above the shared-memory bound of the top-k kernel is refused as
    unsupported before any launch (14528 = 232448 B / (4 rows x 4 B))."""
    idx = ctypes.c_void_p(4096)
    # 1 x 1 x 14529 tokens, block 1 is not a supported block; use block 64:
    # N = 64 * 14529 gives NB = 14529
    st = lib.pa_select_topk(FAKE, paro.PaShape(1, 1, 1, 1, 64 * 14529, 64, 64), 1, idx, None)
    assert st == paro.PA_ERR_UNSUPPORTED
    assert b"14528" in lib.pa_last_error()


def test_clear_status_rejects_null(lib):
    assert lib.pa_clear_status(None, None) == paro.PA_ERR_INVALID_ARG


# --- the Python binding refuses mismatched tensors before any library call ---

@pytest.fixture()
def host_binding(monkeypatch):
    """The binding with its CUDA-device check disabled and a library that
    fails the test if it is ever called: every case below must be refused
    by the binding's own shape and dtype checks."""
    import torch

    class NoLib:
        def __getattr__(self, name):
            raise AssertionError(f"library call {name} reached with a bad argument")

    monkeypatch.setattr(paro, "_need_cuda", lambda *ts: None)
    monkeypatch.setattr(paro, "load", lambda: NoLib())
    return torch


def test_binding_rejects_bad_shapes(host_binding):
    torch = host_binding
    pr = paro.Problem(1, 2, (4, 8, 16), 128, 128, [0, 5])  # N 512, NB 4, N_p 512
    pr_r = paro.Problem(1, 2, (3, 5, 9), 128, 128, [0, 5])  # N 135, NB 2, N_p 256
    nat = torch.zeros(pr_r.natural, dtype=torch.bfloat16)
    perm = torch.zeros(pr_r.permuted, dtype=torch.bfloat16)
    idx = torch.zeros(pr_r.per_block + (2,), dtype=torch.int32)
    bad = [
        # permuted=True with natural-order tensors: a tiled load would read
        # past the allocation
        lambda: paro.block_sparse_attn(nat, nat, nat, pr_r, idx, permuted=True),
        # natural-order call with permuted tensors
        lambda: paro.block_sparse_attn(perm, perm, perm, pr_r, idx),
        # k and v of another dtype than q
        lambda: paro.block_sparse_attn(nat, nat.float(), nat, pr_r, idx),
        # kept lists wider than NB, or of another row count
        lambda: paro.block_sparse_attn(nat, nat, nat, pr_r,
                                       torch.zeros(pr_r.per_block + (3,), dtype=torch.int32)),
        lambda: paro.block_sparse_attn(nat, nat, nat, pr_r,
                                       torch.zeros((1, 2, 3, 2), dtype=torch.int32)),
        lambda: paro.block_sparse_attn(nat, nat, nat, pr_r, idx.long()),
        # counts of the wrong length, output of the wrong shape or dtype
        lambda: paro.block_sparse_attn(nat, nat, nat, pr_r, idx,
                                       torch.zeros((1, 2, 3), dtype=torch.int32)),
        lambda: paro.block_sparse_attn(nat, nat, nat, pr_r, idx, out=torch.zeros(pr_r.permuted)),
        lambda: paro.block_sparse_attn(nat, nat, nat, pr_r, idx,
                                       out=torch.zeros(pr_r.natural, dtype=torch.float32)),
        # int8 without scales, or with scales of the wrong length
        lambda: paro.block_sparse_attn(*(torch.zeros(pr_r.permuted, dtype=torch.int8),) * 3,
                                       pr_r, idx),
        lambda: paro.block_sparse_attn(*(torch.zeros(pr_r.permuted, dtype=torch.int8),) * 3,
                                       pr_r, idx, scales=(torch.zeros(3),) * 3),
        # top-k output narrower than k
        lambda: paro.select_topk(torch.zeros(pr.square), pr, 3,
                                 torch.zeros(pr.per_block + (2,), dtype=torch.int32)),
        lambda: paro.select_topk(torch.zeros(pr.square, dtype=torch.float64), pr, 2),
        # reorder into a buffer without the tail padding
        lambda: paro.reorder(nat, pr_r, out=torch.zeros(pr_r.natural, dtype=torch.bfloat16)),
        lambda: paro.reorder(nat, pr_r, pool=torch.zeros((1, 2, 2, 64))),
        lambda: paro.inverse_reorder(nat, pr_r),
        lambda: paro.quantize_int8(nat, pr_r, x_q=torch.zeros(pr_r.natural, dtype=torch.int8)),
        lambda: paro.score_pooled(torch.zeros(pr.pooled), torch.zeros(pr.pooled), pr,
                                  torch.zeros((1, 2, 4, 5))),
        lambda: paro.compact_mask(torch.zeros((1, 2, 4, 2), dtype=torch.int32), pr),
        lambda: paro.block_score(nat, nat.float(), pr_r),
        lambda: paro.block_sparse_attn_compensated(nat, nat, nat, pr_r, idx,
                                                   torch.zeros((1, 2, 2, 64)),
                                                   torch.zeros(pr_r.pooled)),
        # k_pool and v_pool of different dtypes, or an integer dtype
        lambda: paro.block_sparse_attn_compensated(nat, nat, nat, pr_r, idx,
                                                   torch.zeros(pr_r.pooled, dtype=torch.bfloat16),
                                                   torch.zeros(pr_r.pooled)),
        lambda: paro.block_sparse_attn_compensated(nat, nat, nat, pr_r, idx,
                                                   torch.zeros(pr_r.pooled, dtype=torch.int32),
                                                   torch.zeros(pr_r.pooled, dtype=torch.int32)),
        lambda: paro.round_bf16(torch.zeros(8, dtype=torch.bfloat16)),
        lambda: paro.round_bf16(torch.zeros(8), out=torch.zeros(8, dtype=torch.bfloat16)[:4]),
    ]
    for i, call in enumerate(bad):
        with pytest.raises(ValueError):
            call()


def test_binding_passes_good_shapes_to_the_library(host_binding):
    """The same calls with well-formed tensors get past the checks (they
    reach the stand-in library, which raises AssertionError)."""
    torch = host_binding
    pr_r = paro.Problem(1, 2, (3, 5, 9), 128, 128, [0, 5])
    nat = torch.zeros(pr_r.natural, dtype=torch.bfloat16)
    perm = torch.zeros(pr_r.permuted, dtype=torch.bfloat16)
    i8 = torch.zeros(pr_r.permuted, dtype=torch.int8)
    idx = torch.zeros(pr_r.per_block + (2,), dtype=torch.int32)
    sc = torch.zeros(pr_r.per_block)
    good = [
        lambda: paro.block_sparse_attn(nat, nat, nat, pr_r, idx),
        lambda: paro.block_sparse_attn(perm, perm, perm, pr_r, idx, permuted=True),
        lambda: paro.block_sparse_attn(i8, i8, i8, pr_r, idx, scales=(sc, sc, sc)),
        lambda: paro.reorder(nat, pr_r, with_pool=True),
        lambda: paro.select_topk(torch.zeros(pr_r.square), pr_r, 2),
        lambda: paro.block_sparse_attn_compensated(perm, perm, perm, pr_r, idx,
                                                   torch.zeros(pr_r.pooled),
                                                   torch.zeros(pr_r.pooled), permuted=True),
        lambda: paro.block_sparse_attn_compensated(
            perm, perm, perm, pr_r, idx, torch.zeros(pr_r.pooled, dtype=torch.bfloat16),
            torch.zeros(pr_r.pooled, dtype=torch.bfloat16), permuted=True),
        lambda: paro.round_bf16(torch.zeros(8)),
    ]
    for call in good:
        with pytest.raises(AssertionError, match="library call"):
            call()


def test_stall_hook_arguments_are_checked(lib):
    """The failure-path test hook validates its arguments on the host."""
    assert lib.pa_test_inject_v_stall(0, 0, 1, 10) == paro.PA_ERR_INVALID_ARG  # below 1 us
    assert lib.pa_test_inject_v_stall(-1, 0, 1, 1_000_000) == paro.PA_ERR_INVALID_ARG
    assert lib.pa_test_inject_v_stall(0, 0, 1, 2_000_000_000) == paro.PA_ERR_INVALID_ARG
    assert lib.pa_test_inject_v_stall(-1, -1, -1, 0) == paro.PA_OK  # off


def test_binding_chooses_the_p_reading_flags(monkeypatch):
    """The flags the binding hands pa_block_sparse_attn for the INT8 and
    INT4 paths: INT4 PV takes the per-tile reading (PA_ATTN_P_TILE) by
    default, INT8 the one-pass form unless p_tile is asked for (a recording
    stand-in for the library; CPU tensors, nothing dereferenced)."""
    import torch

    calls = []

    class Recorder:
        def pa_k_for_density(self, nb, density):
            return ref.k_for_density(nb, density)

        def pa_block_sparse_attn(self, *args):
            calls.append(int(args[4]))  # flags
            return paro.PA_OK

        def __getattr__(self, name):
            return lambda *args: paro.PA_OK

    monkeypatch.setattr(paro, "_need_cuda", lambda *ts: None)
    monkeypatch.setattr(paro, "_stream", lambda: None)
    monkeypatch.setattr(paro, "load", lambda: Recorder())
    q = torch.zeros((1, 2, 4 * 8 * 16, 128), dtype=torch.bfloat16)
    for kw, want in [({"int8": True}, 0),
                     ({"int8": True, "p_tile": True}, paro.PA_ATTN_P_TILE),
                     ({"int8": True, "int4_pv": True}, paro.PA_ATTN_P4 | paro.PA_ATTN_P_TILE),
                     ({"int8": True, "int4_pv": True, "p_tile": False}, paro.PA_ATTN_P4)]:
        calls.clear()
        paro.attention(q, q, q, (4, 8, 16), [0, 5], 128, 0.5, **kw)
        assert calls == [want], (kw, calls)
