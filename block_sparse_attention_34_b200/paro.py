"""Thin Python binding of libparo (include/paro.h).

Argument marshalling only: every step runs in the library's CUDA kernels on
the caller's current torch stream.  Torch supplies device memory and
streams.  There is no CPU fallback: if the library is missing or a call
fails, an exception is raised.
"""

from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libparo.so")

PA_OK, PA_ERR_INVALID_ARG, PA_ERR_UNSUPPORTED, PA_ERR_CUDA, PA_ERR_TIMEOUT, PA_ERR_DEVICE_CHECK = range(6)
ABI_VERSION = 8  # the pa_abi_version() these signatures describe
PA_F32, PA_BF16, PA_I8 = 0, 1, 2
PA_ATTN_PERMUTED = 1
PA_ATTN_P4 = 2  # with int8 inputs: 4-bit P codes (INT4 PV)
PA_ATTN_P_TILE = 4  # with int8 inputs: normalised P, one scale per tile (two passes)
STATUS_NAMES = {0: "PA_OK", 1: "PA_ERR_INVALID_ARG", 2: "PA_ERR_UNSUPPORTED", 3: "PA_ERR_CUDA",
                4: "PA_ERR_TIMEOUT", 5: "PA_ERR_DEVICE_CHECK"}
ORDER_IDS = {"FHW": 0, "FWH": 1, "HFW": 2, "HWF": 3, "WFH": 4, "WHF": 5}
# ids 6-11: 3D tile blockings (tf, th, tw) of the block size (include/paro.h)
TILE_IDS = {128: {"T1x8x16": 6, "T1x16x8": 7, "T2x8x8": 8, "T4x4x8": 9, "T8x4x4": 10,
                  "T16x2x4": 11},
            64: {"T1x8x8": 6, "T1x4x16": 7, "T2x4x8": 8, "T4x4x4": 9, "T8x2x4": 10,
                 "T16x2x2": 11}}
N_ORDERS = 12


class PaShape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("B", "heads", "F", "H", "W", "d", "block")]


class ParoError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


_lib = None
_P = ctypes.c_void_p
_I = ctypes.c_int32


def load():
    """Load libparo.so (built by ``python -m block_sparse_attention_34_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m block_sparse_attention_34_b200.build` (needs nvcc)")
    lib = ctypes.CDLL(LIB_PATH)
    sig = {
        "pa_abi_version": ([], _I),
        "pa_last_error": ([], ctypes.c_char_p),
        "pa_clear_status": ([_P, _P], _I),
        "pa_test_inject_v_stall": ([_I, _I, _I, ctypes.c_uint64], _I),
        "pa_num_blocks": ([PaShape], _I),
        "pa_k_for_density": ([_I, ctypes.c_double], _I),
        "pa_reorder": ([_P, _P, _I, PaShape, _P, _P, _P], _I),
        "pa_inverse_reorder": ([_P, _P, _I, PaShape, _P, _P], _I),
        "pa_block_score": ([_P, _P, _I, PaShape, _P, _P, _P, _P, _P], _I),
        "pa_score_pooled": ([_P, _P, PaShape, _P, _P], _I),
        "pa_select_topk": ([_P, PaShape, _I, _P, _P], _I),
        "pa_compact_mask": ([_P, PaShape, _P, _P, _P], _I),
        "pa_select_hybrid": ([_P, PaShape, _I, ctypes.c_double, _I, _P, _P, _P], _I),
        "pa_sics_scores": ([_P, _P, _I, PaShape, _P, _P, _P], _I),
        "pa_map_row_stats": ([_P, _P, PaShape, _I, _P, _P, _P, _P], _I),
        "pa_map_block_stats": ([_P, _P, PaShape, _I, _P, _P, ctypes.c_float, _P, _P, _P, _P, _P,
                                _P], _I),
        "pa_paro_metric": ([_P, _P, _P, PaShape, _I, ctypes.c_float, _P, _P, _P], _I),
        "pa_paro_choose": ([_P, _P, PaShape, ctypes.c_float, _P, _P, _P], _I),
        "pa_quantize_int8": ([_P, _I, PaShape, _P, _P, _P, _P, _P], _I),
        "pa_quantize_int4": ([_P, _I, PaShape, _P, _P, _P, _P, _P], _I),
        "pa_block_sparse_attn": ([_P, _P, _P, _I, ctypes.c_uint32, PaShape, _P, _P, _P, _I, _P, _P, _P,
                                  _P, _P, _P], _I),
        "pa_block_sparse_attn_mma": ([_P, _P, _P, _I, ctypes.c_uint32, PaShape, _P, _P, _P, _I, _P, _P,
                                      _P], _I),
        "pa_block_sparse_attn_compensated": ([_P, _P, _P, _I, ctypes.c_uint32, PaShape, _P, _P, _P, _I,
                                              _P, _P, _I, _P, _P, _P], _I),
        "pa_round_bf16": ([_P, _P, ctypes.c_int64, _P], _I),
    }
    lib.pa_abi_version.restype = _I
    if lib.pa_abi_version() != ABI_VERSION:
        raise RuntimeError(f"{LIB_PATH} has ABI version {lib.pa_abi_version()}, this binding "
                           f"needs {ABI_VERSION}: rebuild it with "
                           "`python -m block_sparse_attention_34_b200.build`")
    for name, (args, res) in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = res
    _lib = lib
    return lib


def _check(status: int):
    if status != PA_OK:
        raise ParoError(status, load().pa_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return PA_F32
    if t.dtype == torch.bfloat16:
        return PA_BF16
    if t.dtype == torch.int8:
        return PA_I8
    raise TypeError(f"unsupported dtype {t.dtype}")


def _need_cuda(*ts):
    dev = None
    for t in ts:
        if t is not None:
            if not t.is_cuda:
                raise ValueError("tensors must be on a CUDA device (no CPU path)")
            if not t.is_contiguous():
                raise ValueError("tensors must be contiguous")
            if dev is None:
                dev = t.device
            elif t.device != dev:
                raise ValueError(f"tensors on different devices ({dev} and {t.device})")


_FLOAT = (torch.float32, torch.bfloat16)


def _expect(t, name, shape, dtypes):
    """Raise ValueError unless tensor ``t`` has exactly ``shape`` and one of
    ``dtypes``: the library reads and writes whole buffers of the sizes the
    shape implies, so a smaller buffer must never reach it."""
    if t is None:
        return
    if tuple(t.shape) != tuple(int(x) for x in shape):
        raise ValueError(f"{name}: shape {tuple(t.shape)}, expected {tuple(shape)}")
    if isinstance(dtypes, torch.dtype):
        dtypes = (dtypes,)
    if t.dtype not in dtypes:
        raise ValueError(f"{name}: dtype {t.dtype}, expected one of {dtypes}")


def _same_dtype(*named):
    ts = [(n, t) for n, t in named if t is not None]
    for n, t in ts[1:]:
        if t.dtype != ts[0][1].dtype:
            raise ValueError(f"{n}: dtype {t.dtype} differs from {ts[0][0]}'s {ts[0][1].dtype}")


class Problem:
    """Sizes of one attention call plus the per-head order ids."""

    def __init__(self, B, heads, grid, d, block, perms):
        self.B, self.heads, self.d, self.block = int(B), int(heads), int(d), int(block)
        self.F, self.H, self.W = (int(x) for x in grid)
        self.N = self.F * self.H * self.W
        self.NB = -(-self.N // self.block)
        self.N_p = self.NB * self.block
        p = np.asarray(perms, dtype=np.int8)
        if p.shape != (self.heads,):
            raise ValueError(f"perms must have one order id per head ({self.heads})")
        self._perms = np.ascontiguousarray(p)
        self.shape = PaShape(self.B, self.heads, self.F, self.H, self.W, self.d, self.block)

    @property
    def natural(self):
        return (self.B, self.heads, self.N, self.d)

    @property
    def permuted(self):
        return (self.B, self.heads, self.N_p, self.d)

    @property
    def pooled(self):
        return (self.B, self.heads, self.NB, self.d)

    @property
    def square(self):
        return (self.B, self.heads, self.NB, self.NB)

    @property
    def per_block(self):
        return (self.B, self.heads, self.NB)

    @property
    def perms_ptr(self):
        return self._perms.ctypes.data_as(ctypes.c_void_p)

    @classmethod
    def from_qkv(cls, q, grid, perms, block):
        B, h, N, d = q.shape
        return cls(B, h, grid, d, block, perms)


def clear_status(status):
    """Enqueue status[0] = PA_OK on the current stream (a memset)."""
    _need_cuda(status)
    _expect_status(status)
    _check(load().pa_clear_status(_ptr(status), _stream()))


def test_inject_v_stall(query_block: int, batch_head: int, tile: int, wait_limit_ns: int):
    """Failure-path test hook (pa_test_inject_v_stall): the V loader of one
    CTA of the tcgen05 bf16 kernel skips one kept tile, so a bounded wait
    runs out after ``wait_limit_ns``; ``tile < 0`` switches it off."""
    _check(load().pa_test_inject_v_stall(int(query_block), int(batch_head), int(tile),
                                         int(wait_limit_ns)))


def k_for_density(nb: int, density: float) -> int:
    return int(load().pa_k_for_density(int(nb), float(density)))


def reorder(x, pr: Problem, out=None, pool=None, with_pool=False):
    """Permuted copy [B, heads, N_p, d] of natural-order x; with
    ``with_pool`` (or a given ``pool`` buffer) also the block means, from
    the same read: returns (x_perm, pool)."""
    _need_cuda(x, out, pool)
    _expect(x, "x", pr.natural, _FLOAT)
    _expect(out, "out", pr.permuted, x.dtype)
    _expect(pool, "pool", pr.pooled, torch.float32)
    out = out if out is not None else torch.empty((pr.B, pr.heads, pr.N_p, pr.d), dtype=x.dtype,
                                                  device=x.device)
    if with_pool and pool is None:
        pool = torch.empty((pr.B, pr.heads, pr.NB, pr.d), dtype=torch.float32, device=x.device)
    _check(load().pa_reorder(_ptr(x), _ptr(out), _dtype_code(x), pr.shape, pr.perms_ptr,
                             _ptr(pool), _stream()))
    return (out, pool) if (with_pool or pool is not None) else out


def inverse_reorder(xp, pr: Problem, out=None):
    _need_cuda(xp, out)
    _expect(xp, "xp", pr.permuted, _FLOAT)
    _expect(out, "out", pr.natural, xp.dtype)
    out = out if out is not None else torch.empty((pr.B, pr.heads, pr.N, pr.d), dtype=xp.dtype,
                                                  device=xp.device)
    _check(load().pa_inverse_reorder(_ptr(xp), _ptr(out), _dtype_code(xp), pr.shape, pr.perms_ptr,
                                     _stream()))
    return out


def block_score(q, k, pr: Problem, q_pool=None, k_pool=None, scores=None):
    _need_cuda(q, k, q_pool, k_pool, scores)
    _expect(q, "q", pr.natural, _FLOAT)
    _expect(k, "k", pr.natural, q.dtype)
    _expect(q_pool, "q_pool", pr.pooled, torch.float32)
    _expect(k_pool, "k_pool", pr.pooled, torch.float32)
    _expect(scores, "scores", pr.square, torch.float32)
    dev = q.device
    q_pool = q_pool if q_pool is not None else torch.empty((pr.B, pr.heads, pr.NB, pr.d), dtype=torch.float32, device=dev)
    k_pool = k_pool if k_pool is not None else torch.empty_like(q_pool)
    scores = scores if scores is not None else torch.empty((pr.B, pr.heads, pr.NB, pr.NB), dtype=torch.float32, device=dev)
    _check(load().pa_block_score(_ptr(q), _ptr(k), _dtype_code(q), pr.shape, pr.perms_ptr,
                                 _ptr(q_pool), _ptr(k_pool), _ptr(scores), _stream()))
    return q_pool, k_pool, scores


def score_pooled(q_pool, k_pool, pr: Problem, scores=None):
    _need_cuda(q_pool, k_pool, scores)
    _expect(q_pool, "q_pool", pr.pooled, torch.float32)
    _expect(k_pool, "k_pool", pr.pooled, torch.float32)
    _expect(scores, "scores", pr.square, torch.float32)
    scores = scores if scores is not None else torch.empty((pr.B, pr.heads, pr.NB, pr.NB), dtype=torch.float32, device=q_pool.device)
    _check(load().pa_score_pooled(_ptr(q_pool), _ptr(k_pool), pr.shape, _ptr(scores), _stream()))
    return scores


def select_topk(scores, pr: Problem, k: int, idx=None):
    _need_cuda(scores, idx)
    _expect(scores, "scores", pr.square, torch.float32)
    _expect(idx, "idx", pr.per_block + (int(k),), torch.int32)
    idx = idx if idx is not None else torch.empty((pr.B, pr.heads, pr.NB, k), dtype=torch.int32, device=scores.device)
    _check(load().pa_select_topk(_ptr(scores), pr.shape, int(k), _ptr(idx), _stream()))
    return idx


def compact_mask(bitmask, pr: Problem, idx=None, counts=None):
    _need_cuda(bitmask, idx, counts)
    _expect(bitmask, "bitmask", pr.per_block + (-(-pr.NB // 32),), (torch.int32, torch.uint32))
    _expect(idx, "idx", pr.square, torch.int32)
    _expect(counts, "counts", pr.per_block, torch.int32)
    dev = bitmask.device
    idx = idx if idx is not None else torch.empty((pr.B, pr.heads, pr.NB, pr.NB), dtype=torch.int32, device=dev)
    counts = counts if counts is not None else torch.empty((pr.B, pr.heads, pr.NB), dtype=torch.int32, device=dev)
    _check(load().pa_compact_mask(_ptr(bitmask), pr.shape, _ptr(idx), _ptr(counts), _stream()))
    return idx, counts


def select_hybrid(scores, pr: Problem, k: int, top_p: float, window: int, idx=None, counts=None):
    """Union of the diagonal, a local window, Top-K and Top-P per query-block
    row -> (idx [B,h,NB,NB] ascending, -1 padded; counts [B,h,NB])."""
    _need_cuda(scores, idx, counts)
    _expect(scores, "scores", pr.square, torch.float32)
    _expect(idx, "idx", pr.square, torch.int32)
    _expect(counts, "counts", pr.per_block, torch.int32)
    dev = scores.device
    idx = idx if idx is not None else torch.empty((pr.B, pr.heads, pr.NB, pr.NB), dtype=torch.int32, device=dev)
    counts = counts if counts is not None else torch.empty((pr.B, pr.heads, pr.NB), dtype=torch.int32, device=dev)
    _check(load().pa_select_hybrid(_ptr(scores), pr.shape, int(k), float(top_p), int(window), _ptr(idx),
                                   _ptr(counts), _stream()))
    return idx, counts


def sics_scores(q, k, pr: Problem, scores=None, orders=None):
    """Blocking scores of the 12 candidates (six axis orders, six 3D tile
    blockings): SICS of q's and k's blocks -> (scores [B,h,12], orders
    [heads] int8, each head's pick by the library: the largest score summed
    over the batch, ties to the lower id)."""
    _need_cuda(q, k, scores, orders)
    _expect(q, "q", pr.natural, _FLOAT)
    _expect(k, "k", pr.natural, q.dtype)
    _expect(scores, "scores", (pr.B, pr.heads, N_ORDERS), torch.float32)
    _expect(orders, "orders", (pr.heads,), torch.int8)
    scores = scores if scores is not None else torch.empty((pr.B, pr.heads, N_ORDERS), dtype=torch.float32, device=q.device)
    orders = orders if orders is not None else torch.empty((pr.heads,), dtype=torch.int8, device=q.device)
    _check(load().pa_sics_scores(_ptr(q), _ptr(k), _dtype_code(q), pr.shape, _ptr(scores),
                                 _ptr(orders), _stream()))
    return scores, orders


def map_row_stats(q_perm, k_perm, pr: Problem, order: int, status=None):
    """Row softmax (log2 max, sum) of every token of the dense map, from
    copies of q, k permuted by ``order`` -> ([B,h,N], [B,h,N])."""
    _need_cuda(q_perm, k_perm)
    _expect(q_perm, "q_perm", pr.permuted, torch.bfloat16)
    _expect(k_perm, "k_perm", pr.permuted, torch.bfloat16)
    dev = q_perm.device
    m = torch.empty((pr.B, pr.heads, pr.N), dtype=torch.float32, device=dev)
    l = torch.empty_like(m)
    _check(load().pa_map_row_stats(_ptr(q_perm), _ptr(k_perm), pr.shape, int(order), _ptr(m),
                                   _ptr(l), _ptr(status), _stream()))
    return m, l


def map_block_stats(q_perm, k_perm, pr: Problem, order: int, row_max, row_sum, eps=1e-3,
                    with_log=True, status=None):
    """Per block of the map in ``order``: dict of [B,h,NB,NB] count / total
    / peak (and log_total)."""
    _need_cuda(q_perm, k_perm, row_max, row_sum)
    _expect(q_perm, "q_perm", pr.permuted, torch.bfloat16)
    _expect(k_perm, "k_perm", pr.permuted, torch.bfloat16)
    _expect(row_max, "row_max", (pr.B, pr.heads, pr.N), torch.float32)
    _expect(row_sum, "row_sum", (pr.B, pr.heads, pr.N), torch.float32)
    dev = q_perm.device
    out = {key: torch.empty((pr.B, pr.heads, pr.NB, pr.NB), dtype=torch.float32, device=dev)
           for key in ("count", "total", "peak")}
    out["log_total"] = torch.empty_like(out["total"]) if with_log else None
    _check(load().pa_map_block_stats(_ptr(q_perm), _ptr(k_perm), pr.shape, int(order),
                                     _ptr(row_max), _ptr(row_sum), float(eps), _ptr(out["count"]),
                                     _ptr(out["total"]), _ptr(out["peak"]),
                                     _ptr(out["log_total"]), _ptr(status), _stream()))
    return out


def paro_offline(q, k, grid, block, eps=1e-3, rho=0.9, alpha=0.5, sigma=0.9, status=None):
    """PAROAttention's offline stage for natural-order q, k (bf16, d = 128,
    block = 128): the six orders' block statistics of the dense map, the
    per-head metric and order, and the static mask of each head's chosen
    order by block-sum thresholding at ``sigma``.  Returns a dict: orders
    [B,h] int8, metric / sparse_frac / incoherence [B,h,6], idx [B,h,NB,NB]
    and counts [B,h,NB] (the chosen order's mask, per head)."""
    B, heads = q.shape[:2]
    dev = q.device
    probs = [Problem(B, heads, grid, q.shape[-1], block, [o] * heads) for o in range(6)]
    pr0 = probs[0]
    sf = torch.empty((B, heads, 6), dtype=torch.float32, device=dev)
    inc = torch.empty_like(sf)
    idx_all = torch.empty((6, B, heads, pr0.NB, pr0.NB), dtype=torch.int32, device=dev)
    cnt_all = torch.empty((6, B, heads, pr0.NB), dtype=torch.int32, device=dev)
    row_max = row_sum = None
    for o, pr in enumerate(probs):
        qp, kp = reorder(q, pr), reorder(k, pr)
        if row_max is None:
            row_max, row_sum = map_row_stats(qp, kp, pr, o, status)
        st = map_block_stats(qp, kp, pr, o, row_max, row_sum, eps, True, status)
        _check(load().pa_paro_metric(_ptr(st["count"]), _ptr(st["total"]), _ptr(st["peak"]),
                                     pr.shape, o, float(rho), _ptr(sf), _ptr(inc), _stream()))
        select_hybrid(st["log_total"], pr, 0, sigma, -1, idx_all[o], cnt_all[o])
        del qp, kp, st
    metric = torch.empty_like(sf)
    orders = torch.empty((B, heads), dtype=torch.int8, device=dev)
    _check(load().pa_paro_choose(_ptr(sf), _ptr(inc), pr0.shape, float(alpha), _ptr(metric),
                                 _ptr(orders), _stream()))
    # each head's mask in its chosen order (a gather of the six candidates)
    pick = orders.long()
    bi = torch.arange(B, device=dev)[:, None]
    hi = torch.arange(heads, device=dev)[None, :]
    return {"orders": orders, "metric": metric, "sparse_frac": sf, "incoherence": inc,
            "idx": idx_all[pick, bi, hi], "counts": cnt_all[pick, bi, hi]}


def quantize_int8(x, pr: Problem, with_pool=False, x_q=None, scales=None, pool=None, bits=8):
    """Per-block symmetric quantisation in the permuted order: 8-bit codes
    (levels +-127), or ``bits=4`` (levels +-7, one code per byte)."""
    _need_cuda(x, x_q, scales, pool)
    _expect(x, "x", pr.natural, _FLOAT)
    _expect(x_q, "x_q", pr.permuted, torch.int8)
    _expect(scales, "scales", pr.per_block, torch.float32)
    _expect(pool, "pool", pr.pooled, torch.float32)
    dev = x.device
    x_q = x_q if x_q is not None else torch.empty((pr.B, pr.heads, pr.N_p, pr.d), dtype=torch.int8, device=dev)
    scales = scales if scales is not None else torch.empty((pr.B, pr.heads, pr.NB), dtype=torch.float32, device=dev)
    if with_pool and pool is None:
        pool = torch.empty((pr.B, pr.heads, pr.NB, pr.d), dtype=torch.float32, device=dev)
    if bits not in (4, 8):
        raise ValueError(f"bits={bits}: 4 or 8")
    fn = load().pa_quantize_int8 if bits == 8 else load().pa_quantize_int4
    _check(fn(_ptr(x), _dtype_code(x), pr.shape, pr.perms_ptr, _ptr(x_q),
                                   _ptr(scales), _ptr(pool), _stream()))
    return (x_q, scales, pool) if with_pool else (x_q, scales)


def _check_lists(idx, counts, pr: Problem):
    """idx [B,h,NB,k_max] int32 with 0 <= k_max <= NB; counts [B,h,NB] int32."""
    if idx is None:
        raise ValueError("idx is required")
    if idx.dim() != 4 or tuple(idx.shape[:3]) != pr.per_block or idx.shape[3] > pr.NB:
        raise ValueError(f"idx: shape {tuple(idx.shape)}, expected {pr.per_block + ('k<=NB',)}")
    _expect(idx, "idx", tuple(idx.shape), torch.int32)
    _expect(counts, "counts", pr.per_block, torch.int32)


def _expect_status(status):
    if status is not None and (status.dtype != torch.int32 or status.numel() < 1):
        raise ValueError("status: an int32 tensor of at least one element")


def block_sparse_attn(q, k, v, pr: Problem, idx, counts=None, scales=None, out=None,
                      status=None, baseline=False, permuted=False, p4=False, p_tile=False):
    """O = block-sparse attention over the kept tiles, natural token order.

    ``permuted``: q, k, v are [B, heads, N_p, d] from :func:`reorder`.
    ``scales`` = (q_scale, k_scale, v_scale) for int8 q/k/v from
    :func:`quantize_int8` (output bf16); with them ``p4`` quantises P to 4
    bits and ``p_tile`` quantises the normalised P with one scale per tile
    (two passes over the kept tiles) instead of the one-pass fixed scale.
    ``baseline=True`` runs the mma.sync comparison kernel instead of the
    tcgen05 one."""
    _need_cuda(q, k, v, idx, counts, out, status, *(scales or ()))
    code = _dtype_code(q)
    _same_dtype(("q", q), ("k", k), ("v", v))
    rows = pr.permuted if (permuted or code == PA_I8) else pr.natural
    for name, t in (("q", q), ("k", k), ("v", v)):
        _expect(t, name, rows, (torch.float32, torch.bfloat16, torch.int8))
    _check_lists(idx, counts, pr)
    if code == PA_I8:
        if scales is None or len(scales) != 3:
            raise ValueError("int8 q, k, v need scales=(q_scale, k_scale, v_scale)")
        for name, t in zip(("q_scale", "k_scale", "v_scale"), scales):
            _expect(t, name, pr.per_block, torch.float32)
    out_dtype = torch.bfloat16 if code == PA_I8 else q.dtype
    _expect(out, "out", pr.natural, out_dtype)
    _expect_status(status)
    out = out if out is not None else torch.empty((pr.B, pr.heads, pr.N, pr.d), dtype=out_dtype, device=q.device)
    k_max = int(idx.shape[-1])
    flags = ((PA_ATTN_PERMUTED if permuted else 0) | (PA_ATTN_P4 if p4 else 0)
             | (PA_ATTN_P_TILE if p_tile else 0))
    lib = load()
    if baseline:
        st = lib.pa_block_sparse_attn_mma(_ptr(q), _ptr(k), _ptr(v), code, flags, pr.shape,
                                          pr.perms_ptr, _ptr(idx), _ptr(counts), k_max, _ptr(out),
                                          _ptr(status), _stream())
    else:
        qs, ks, vs = scales if scales is not None else (None, None, None)
        st = lib.pa_block_sparse_attn(_ptr(q), _ptr(k), _ptr(v), code, flags, pr.shape,
                                      pr.perms_ptr, _ptr(idx), _ptr(counts), k_max, _ptr(qs),
                                      _ptr(ks), _ptr(vs), _ptr(out), _ptr(status), _stream())
    _check(st)
    return out


def block_sparse_attn_compensated(q, k, v, pr: Problem, idx, k_pool, v_pool, counts=None,
                                  out=None, status=None, permuted=False):
    """Block-sparse attention in which every unselected key block still
    enters the softmax as one pooled key row (mean key, mean value, weight
    = its valid keys): PASA's grouped first-order compensation.  k_pool,
    v_pool [B, heads, NB, d] block means (from :func:`reorder` with
    ``with_pool`` or :func:`block_score`), both float32, or both bfloat16
    (:func:`round_bf16`; bf16 q, k, v with d = block = 128 only, the faster
    form).  bf16 or fp32 q, k, v; output natural order, q's dtype."""
    _need_cuda(q, k, v, idx, counts, k_pool, v_pool, out, status)
    _same_dtype(("q", q), ("k", k), ("v", v))
    rows = pr.permuted if permuted else pr.natural
    for name, t in (("q", q), ("k", k), ("v", v)):
        _expect(t, name, rows, _FLOAT)
    _check_lists(idx, counts, pr)
    pool_dt = k_pool.dtype if k_pool is not None else torch.float32
    if pool_dt not in (torch.float32, torch.bfloat16):
        raise ValueError(f"k_pool dtype {pool_dt}: float32 or bfloat16")
    _expect(k_pool, "k_pool", pr.pooled, pool_dt)
    _expect(v_pool, "v_pool", pr.pooled, pool_dt)
    _expect(out, "out", pr.natural, q.dtype)
    _expect_status(status)
    out = out if out is not None else torch.empty((pr.B, pr.heads, pr.N, pr.d), dtype=q.dtype,
                                                  device=q.device)
    st = load().pa_block_sparse_attn_compensated(
        _ptr(q), _ptr(k), _ptr(v), _dtype_code(q), PA_ATTN_PERMUTED if permuted else 0, pr.shape,
        pr.perms_ptr, _ptr(idx), _ptr(counts), int(idx.shape[-1]), _ptr(k_pool), _ptr(v_pool),
        _dtype_code(k_pool), _ptr(out), _ptr(status), _stream())
    _check(st)
    return out


def round_bf16(x, out=None):
    """x (float32, CUDA, contiguous) rounded to bfloat16 by the library's
    kernel: the bf16 block means :func:`block_sparse_attn_compensated`
    loads with the K and V tiles' copy engine."""
    _need_cuda(x, out)
    if x.dtype != torch.float32 or not x.is_contiguous():
        raise ValueError("x must be a contiguous float32 tensor")
    if out is None:
        out = torch.empty(x.shape, dtype=torch.bfloat16, device=x.device)
    elif out.dtype != torch.bfloat16 or out.shape != x.shape or not out.is_contiguous():
        raise ValueError(f"out must be a contiguous bfloat16 tensor of shape {tuple(x.shape)}")
    _check(load().pa_round_bf16(_ptr(x), _ptr(out), x.numel(), _stream()))
    return out


def choose_orders_sics(q, k, grid, block):
    """SPADE's blocking choice per head, made by the library: the candidate
    (axis order or 3D tile blocking) whose blocks have the largest SICS of q
    and k -> list of order ids (copied to the host: the calls that follow
    take the order ids as host data)."""
    B, heads = q.shape[:2]
    pr = Problem(B, heads, grid, q.shape[-1], block, [0] * heads)
    _, orders = sics_scores(q, k, pr)
    return [int(o) for o in orders.cpu().tolist()]


def attention(q, k, v, grid, perms, block, density, int8=False, baseline=False, status=None,
              permuted=True, int4_pv=False, selection="topk", top_p=0.0, window=-1,
              compensate=False, p_tile=None):
    """The whole path for one call: reorder with block means (one read of
    q, k, v) -> pooled block scores -> kept blocks -> block-sparse attention
    over the permuted tiles, stored back in natural order.

    ``perms``: one axis-order id per head, or "sics" to pick each head's
    order by the SICS blocking score (SPADE).  ``selection``: "topk" (the
    diagonal plus the k-1 best blocks, k from ``density``) or "hybrid" (the
    union of that Top-K, the Top-P set at ``top_p`` and the local window
    |i - j| <= ``window``, with per-row counts).  ``int8`` runs the INT8
    kernel (``int4_pv``: 4-bit P and V; ``p_tile``: P normalised and
    quantised per tile, the pages' reading, by default with ``int4_pv``
    only, since at 8 bits the one-pass form stays within the INT8
    tolerance of it).  ``permuted=False`` skips the
    reorder pass (the kernel gathers token rows); ``baseline=True`` runs the
    mma.sync comparison kernel.  ``compensate`` adds PASA's grouped
    first-order compensation of the unselected blocks (bf16 / fp32 only;
    :func:`block_sparse_attn_compensated`).  Returns (out, idx) — with the
    hybrid filter, idx is (idx, counts)."""
    if isinstance(perms, str):
        if perms != "sics":
            raise ValueError(f"perms={perms!r}: order ids or 'sics'")
        perms = choose_orders_sics(q, k, grid, block)
    pr = Problem.from_qkv(q, grid, perms, block)
    kk = k_for_density(pr.NB, density)

    def select(scores):
        if selection == "hybrid":
            return select_hybrid(scores, pr, kk, top_p, window)
        if selection != "topk":
            raise ValueError(f"selection={selection!r}: topk or hybrid")
        return select_topk(scores, pr, kk), None

    if compensate:
        if int8:
            raise ValueError("compensate runs on bf16 / fp32 inputs")
        qp, q_pool = reorder(q, pr, with_pool=True)
        kp, k_pool = reorder(k, pr, with_pool=True)
        vp, v_pool = reorder(v, pr, with_pool=True)
        idx, counts = select(score_pooled(q_pool, k_pool, pr))
        if q.dtype == torch.bfloat16 and pr.d == 128 and pr.block == 128:
            # the tcgen05 kernel loads bf16 means like K and V tiles
            k_pool, v_pool = round_bf16(k_pool), round_bf16(v_pool)
        out = block_sparse_attn_compensated(qp, kp, vp, pr, idx, k_pool, v_pool, counts,
                                            status=status, permuted=True)
    elif int8:
        q8, qs, qp = quantize_int8(q, pr, with_pool=True)
        k8, ks, kp = quantize_int8(k, pr, with_pool=True)
        v8, vs = quantize_int8(v, pr, bits=4 if int4_pv else 8)
        idx, counts = select(score_pooled(qp, kp, pr))
        out = block_sparse_attn(q8, k8, v8, pr, idx, counts, scales=(qs, ks, vs), status=status,
                                p4=int4_pv, p_tile=int4_pv if p_tile is None else p_tile)
    elif permuted and not baseline:
        qp, q_pool = reorder(q, pr, with_pool=True)
        kp, k_pool = reorder(k, pr, with_pool=True)
        vp = reorder(v, pr)
        idx, counts = select(score_pooled(q_pool, k_pool, pr))
        out = block_sparse_attn(qp, kp, vp, pr, idx, counts, status=status, permuted=True)
    else:
        _, _, scores = block_score(q, k, pr)
        idx, counts = select(scores)
        out = block_sparse_attn(q, k, v, pr, idx, counts, baseline=baseline, status=status)
    return out, (idx if counts is None else (idx, counts))
