"""One attention call of the path with its device buffers preallocated, so
that repeated calls (a DiT's layers and denoising steps) launch kernels only.

Launch sequence of :meth:`Pipeline.run` (every step through the C ABI, on the
current torch stream; the status word is cleared first, by a memset):

  bf16:  reorder+pool(q), reorder+pool(k), reorder(v)  -- one HBM pass each
         score_pooled -> select_topk (or select_hybrid: diagonal, window,
         Top-K and Top-P with per-row counts) -> block_sparse_attn(permuted tiles)
  int8:  quantize+pool(q), quantize+pool(k), quantize(v)  (v to 4 bits with int4_pv)
         score_pooled -> select_topk -> block_sparse_attn(int8; 4-bit P with int4_pv;
         P normalised and quantised per tile with p_tile, by default with int4_pv)

The output is written in natural token order; the inverse reorder is the
attention kernel's store.
"""

from __future__ import annotations

import torch

from . import paro


class Pipeline:
    def __init__(self, B, heads, grid, d, block, perms, density, dtype=torch.bfloat16,
                 device="cuda", int8=False, baseline=False, selection="topk", top_p=0.0,
                 window=-1, int4_pv=False, p_tile=None):
        self.pr = paro.Problem(B, heads, grid, d, block, perms)
        pr = self.pr
        self.k = paro.k_for_density(pr.NB, density)
        self.int8 = int8 or int4_pv
        self.int4_pv = int4_pv
        self.p_tile = int4_pv if p_tile is None else bool(p_tile)
        self.baseline = baseline
        if selection not in ("topk", "hybrid"):
            raise ValueError(f"selection {selection!r}: topk or hybrid")
        self.selection = selection
        self.top_p = float(top_p)
        self.window = int(window)
        dev = torch.device(device)
        if self.int8:
            self.xq = [torch.empty((B, heads, pr.N_p, d), dtype=torch.int8, device=dev) for _ in range(3)]
            self.sc = [torch.empty((B, heads, pr.NB), dtype=torch.float32, device=dev) for _ in range(3)]
        elif not baseline:
            self.xp = [torch.empty((B, heads, pr.N_p, d), dtype=dtype, device=dev) for _ in range(3)]
        self.q_pool = torch.empty((B, heads, pr.NB, d), dtype=torch.float32, device=dev)
        self.k_pool = torch.empty_like(self.q_pool)
        self.scores = torch.empty((B, heads, pr.NB, pr.NB), dtype=torch.float32, device=dev)
        if selection == "hybrid":  # variable counts: rows padded to NB
            self.idx = torch.empty((B, heads, pr.NB, pr.NB), dtype=torch.int32, device=dev)
            self.counts = torch.empty((B, heads, pr.NB), dtype=torch.int32, device=dev)
        else:
            self.idx = torch.empty((B, heads, pr.NB, self.k), dtype=torch.int32, device=dev)
            self.counts = None
        out_dtype = torch.bfloat16 if self.int8 else dtype
        self.out = torch.empty((B, heads, pr.N, d), dtype=out_dtype, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)

    @property
    def launches(self) -> int:
        """Kernel launches of one :meth:`run` (all of them this library's)."""
        return 5 if self.baseline else 6

    def select(self, q, k, v):
        pr = self.pr
        if self.int8:
            paro.quantize_int8(q, pr, x_q=self.xq[0], scales=self.sc[0], pool=self.q_pool)
            paro.quantize_int8(k, pr, x_q=self.xq[1], scales=self.sc[1], pool=self.k_pool)
            paro.quantize_int8(v, pr, x_q=self.xq[2], scales=self.sc[2],
                               bits=4 if self.int4_pv else 8)
            paro.score_pooled(self.q_pool, self.k_pool, pr, scores=self.scores)
        elif self.baseline:
            paro.block_score(q, k, pr, self.q_pool, self.k_pool, self.scores)
        else:
            paro.reorder(q, pr, out=self.xp[0], pool=self.q_pool)
            paro.reorder(k, pr, out=self.xp[1], pool=self.k_pool)
            paro.reorder(v, pr, out=self.xp[2])
            paro.score_pooled(self.q_pool, self.k_pool, pr, scores=self.scores)
        if self.selection == "hybrid":
            paro.select_hybrid(self.scores, pr, self.k, self.top_p, self.window, self.idx,
                               self.counts)
        else:
            paro.select_topk(self.scores, pr, self.k, self.idx)

    def attend(self, q, k, v):
        pr = self.pr
        if self.int8:
            paro.block_sparse_attn(*self.xq, pr, self.idx, self.counts, scales=tuple(self.sc),
                                   out=self.out, status=self.status, p4=self.int4_pv,
                                   p_tile=self.p_tile)
        elif self.baseline:
            paro.block_sparse_attn(q, k, v, pr, self.idx, self.counts, out=self.out,
                                   status=self.status, baseline=True)
        else:
            paro.block_sparse_attn(*self.xp, pr, self.idx, self.counts, out=self.out,
                                   status=self.status, permuted=True)

    def kept_tiles(self) -> int:
        """Kept (query block, key block) tiles of the last selection (reads
        the per-row counts back for the hybrid filter)."""
        pr = self.pr
        if self.counts is not None:
            return int(self.counts.sum().item())
        return pr.B * pr.heads * pr.NB * self.k

    def run(self, q, k, v):
        # one status word for the whole call sequence, cleared per call (a
        # kernel that finds a timeout recorded there skips its work)
        paro.clear_status(self.status)
        self.select(q, k, v)
        self.attend(q, k, v)
        return self.out


def chunk_ranges(B: int, heads: int, chunks: int):
    """Split a [B, heads, ...] call into at most ``chunks`` pieces, each
    contiguous in memory: head ranges of the one batch element when B = 1,
    else ranges of whole batch elements.  Returns [(b0, b1, h0, h1)]."""
    if B == 1:
        n = max(1, min(chunks, heads))
        cuts = [round(i * heads / n) for i in range(n + 1)]
        return [(0, 1, cuts[i], cuts[i + 1]) for i in range(n) if cuts[i + 1] > cuts[i]]
    n = max(1, min(chunks, B))
    cuts = [round(i * B / n) for i in range(n + 1)]
    return [(cuts[i], cuts[i + 1], 0, heads) for i in range(n) if cuts[i + 1] > cuts[i]]


class StreamedPipeline:
    """The same call on inputs in pinned host memory, with the copies
    overlapped with the work: the layer is split into contiguous chunks of
    heads (or batch elements), each with its own preallocated
    :class:`Pipeline`; chunk c's host -> device copies run on a copy stream,
    its selection and attention on a compute stream once they landed, and
    its output's device -> host copy on a third stream once the attention
    finished, so chunk c's work overlaps chunk c+1's upload and chunk c-1's
    download.  Every step of the path is per head, so the result equals the
    one-shot :class:`Pipeline`'s bit for bit."""

    def __init__(self, B, heads, grid, d, block, perms, density, chunks=8, device="cuda",
                 **kw):
        dev = torch.device(device)
        perms = list(perms)
        self.ranges = chunk_ranges(B, heads, chunks)
        self.pipes = [Pipeline(b1 - b0, h1 - h0, grid, d, block, perms[h0:h1], density,
                               device=dev, **kw) for (b0, b1, h0, h1) in self.ranges]
        p0 = self.pipes[0]
        shape = (B, heads, p0.pr.N, d)
        dtype = kw.get("dtype", torch.bfloat16)
        self.dev_in = [[torch.empty((b1 - b0, h1 - h0) + shape[2:], dtype=dtype, device=dev)
                        for _ in range(3)] for (b0, b1, h0, h1) in self.ranges]
        self.streams = [torch.cuda.Stream(device=dev) for _ in range(3)]  # h2d, compute, d2h
        self.k = p0.k

    def run(self, host_q, host_k, host_v, host_out):
        """host_q/k/v [B, heads, N, d] and host_out [B, heads, N, d] pinned
        host tensors; returns host_out once its copies are enqueued (on the
        caller's stream order: the caller's current stream waits for them)."""
        cur = torch.cuda.current_stream()
        h2d, comp, d2h = self.streams
        for s in self.streams:
            s.wait_stream(cur)  # nothing starts before the caller's prior work
        for (b0, b1, h0, h1), pipe, dev in zip(self.ranges, self.pipes, self.dev_in):
            with torch.cuda.stream(h2d):
                for t, h in zip(dev, (host_q, host_k, host_v)):
                    t.copy_(h[b0:b1, h0:h1], non_blocking=True)
                landed = torch.cuda.Event()
                landed.record(h2d)
            with torch.cuda.stream(comp):
                comp.wait_event(landed)
                pipe.run(*dev)
                done = torch.cuda.Event()
                done.record(comp)
            with torch.cuda.stream(d2h):
                d2h.wait_event(done)
                host_out[b0:b1, h0:h1].copy_(pipe.out, non_blocking=True)
        for s in self.streams:
            cur.wait_stream(s)
        return host_out

    def status(self) -> int:
        """The first nonzero device status of the chunks (reads it back)."""
        for pipe in self.pipes:
            st = int(pipe.status.item())
            if st != 0:
                return st
        return 0
