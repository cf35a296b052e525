/*
 * paro.h -- C ABI of libparo: per-head block-sparse attention over the
 * F x H x W token grid of a video diffusion transformer, on NVIDIA B200
 * (sm_100a).
 *
 * The path, one attention call:
 *   1. per-head reorder of the flattened tokens to one of the six axis orders
 *      of [F, H, W] (or one of SPADE's six 3D tile blockings)
 *                                    (PAROAttention, arXiv 2506.16054, Pith
 *                                     verdict page, key_machinery);
 *   2. mean-pooled Q/K block summaries and block scores
 *                                    (SPADE, arXiv 2608.03335, Pith verdict
 *                                     page, key_machinery (iii) and the
 *                                     referee's note on the MEAN summariser);
 *   3. top-k key blocks per query block, or a static bitmask
 *                                    (PASA, arXiv 2604.12219, Figure 2;
 *                                     PAROAttention review: bitmask masks);
 *   4. online-softmax attention over the kept (query block, key block) tiles
 *      only, optionally with INT8 Q/K/V and INT8 P
 *                                    (SPADE review, key_machinery (iii);
 *                                     PAROAttention review, key_machinery);
 *   5. inverse reorder of the output (fused into step 4's store).
 *
 * Around it: SPADE's selection variants (pa_sics_scores, pa_select_hybrid),
 * INT4 P V (pa_quantize_int4 with PA_ATTN_P4), the per-tile reading of the
 * INT8/INT4 post-softmax map (PA_ATTN_P_TILE), PAROAttention's offline stage
 * (pa_map_row_stats, pa_map_block_stats, pa_paro_metric, pa_paro_choose) and
 * PASA's compensation of the unselected blocks
 * (pa_block_sparse_attn_compensated, with pa_round_bf16 for bf16 block
 * means); pa_clear_status resets the device status word, and
 * pa_test_inject_v_stall is the host-set hook of the bounded-wait test.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - N = F*H*W tokens per head; NB = ceil(N / block) blocks; N_p = NB*block.
 * - Order ids (one int8 per head, HOST memory, length shape.heads, the same
 *   for every batch index): 0 FHW, 1 FWH, 2 HFW, 3 HWF, 4 WFH, 5 WHF, the
 *   letters listing the axes outermost -> innermost.  FHW is the natural
 *   flattening n = f*H*W + h*W + w.  Ids 6-11 are SPADE's 3D tile blockings
 *   (SPADE review, key_machinery (i)): tiles of tf x th x tw tokens, tiles
 *   in (f, h, w) order of their tile coordinates, tokens inside a tile in
 *   (f, h, w) order, partial tiles at the far edges; (tf, th, tw) for
 *   block 128: 6 (1,8,16), 7 (1,16,8), 8 (2,8,8), 9 (4,4,8), 10 (8,4,4),
 *   11 (16,2,4); for block 64: 6 (1,8,8), 7 (1,4,16), 8 (2,4,8), 9 (4,4,4),
 *   10 (8,2,4), 11 (16,2,2).  Token n of a head sits at position pos(n) of
 *   that head's order; block i holds positions [i*block, (i+1)*block);
 *   positions >= N are zero padding.
 * - Q, K, V and the attention output are [B, heads, N, d] row-major in the
 *   natural order, contiguous, device memory, base 16-byte aligned.
 *   INT8 tensors and pooled summaries are in the permuted order.
 * - Every pointer argument except `perms` is DEVICE memory owned by the
 *   caller; the library allocates no device memory and keeps no pointer
 *   after a call returns.
 * - `stream` is a cudaStream_t (NULL = legacy default stream).  Every call
 *   only enqueues work on it and returns; nothing synchronises.
 * - Supported: d in {64, 128}; block in {64, 128}; 1 <= heads <= 1024;
 *   B >= 1; F, H, W >= 1; B*heads*N_p*d < 2^40.
 * - Errors: argument errors return PA_ERR_INVALID_ARG (or
 *   PA_ERR_UNSUPPORTED for valid but unsupported sizes) before any launch;
 *   a failed launch returns PA_ERR_CUDA.  pa_last_error() then gives a
 *   message (thread-local, valid until the next call on the thread).
 *   Device-side checks (malformed index lists, a bounded wait that ran
 *   out) write a nonzero pa_status code into *dev_status when dev_status is
 *   not NULL (first error wins) and skip the offending work; they never
 *   trap.  Read it after synchronising the stream.  A kernel that finds
 *   PA_ERR_TIMEOUT already recorded there skips its work, so one expired
 *   wait ends the launch quickly: reset the word to 0 before reusing it.
 */
#ifndef PARO_H
#define PARO_H

#include <stdint.h>

#if defined(__GNUC__)
#define PA_API __attribute__((visibility("default")))
#else
#define PA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID_ARG = 1,
  PA_ERR_UNSUPPORTED = 2,
  PA_ERR_CUDA = 3,
  PA_ERR_TIMEOUT = 4,
  PA_ERR_DEVICE_CHECK = 5
} pa_status;

typedef enum { PA_F32 = 0, PA_BF16 = 1, PA_I8 = 2 } pa_dtype;

typedef struct {
  int32_t B, heads, F, H, W, d, block;
} pa_shape;

/* Version of this ABI (bumped on any signature change): 8. */
PA_API int32_t pa_abi_version(void);

/* Message of the last failed call on this thread ("" if none). */
PA_API const char* pa_last_error(void);

/* Enqueue a reset of the device status word *dev_status (one int32, device
 * memory) to PA_OK on `stream` (a memset; no kernel).  A kernel that finds
 * PA_ERR_TIMEOUT recorded skips its work, so a caller reusing one status
 * word across calls clears it before each call sequence.  Not part of the
 * pages' method: bookkeeping of this library's error reporting. */
PA_API pa_status pa_clear_status(int32_t* dev_status, void* stream);

/* Test hook of the failure path (not part of the pages' method).  For the
 * pa_block_sparse_attn launches on the tcgen05 bf16 kernel that follow
 * (d = 128, block = 128, PA_BF16), the V-tile loader of the CTA of query
 * block `query_block` and batch-head `batch_head` (b * heads + h) skips kept
 * tile number `tile` of its list (issues no copy and no arrival), so the
 * MMA issuer's bounded wait for that tile runs out; every bounded wait of
 * the kernel then gives up after `wait_limit_ns` (1 us .. 1 s) instead of
 * 1 s.  The CTA records PA_ERR_TIMEOUT on dev_status, every role leaves its
 * loop, copies and MMAs in flight are drained and tensor memory is
 * released; CTAs that start later find the status and skip their work.  No
 * trap, no fault, nothing left waiting.  tile < 0 switches the hook off
 * (the default).  Process-wide setting, read at launch; not for concurrent
 * use. */
PA_API pa_status pa_test_inject_v_stall(int32_t query_block, int32_t batch_head, int32_t tile,
                                        uint64_t wait_limit_ns);

/* NB = ceil(F*H*W / block), or -1 for a malformed shape. */
PA_API int32_t pa_num_blocks(pa_shape shape);

/* Kept key blocks per query block for a density:
 * ceil(density * nb) clamped to [1, nb], with density*nb rounded to 9
 * decimals first (so 0.3 * 10 keeps 3, not 4).  Returns 0 for nb <= 0.
 * (The pages give the density; the rounding rule is this library's.) */
PA_API int32_t pa_k_for_density(int32_t nb, double density);

/* Step 1 (PAROAttention review, key_machinery: per-head permutation among
 * the six axis orders).  x [B,heads,N,d] natural -> x_perm [B,heads,N_p,d]
 * permuted, pad rows written as zeros.  dtype PA_F32 or PA_BF16 (same for
 * both buffers).  pool, if not NULL, [B,heads,NB,d] float, receives the
 * mean of each permuted block's valid rows (step 2's summary, as
 * pa_block_score's q_pool) from the same read of x. */
PA_API pa_status pa_reorder(const void* x, void* x_perm, pa_dtype dtype, pa_shape shape,
                            const int8_t* perms, float* pool, void* stream);

/* Step 5 standalone: x_perm [B,heads,N_p,d] permuted -> x [B,heads,N,d]
 * natural; pad rows are dropped. */
PA_API pa_status pa_inverse_reorder(const void* x_perm, void* x, pa_dtype dtype, pa_shape shape,
                             const int8_t* perms, void* stream);

/* Step 2 (SPADE review: MEAN summariser; intra-estimation).  From
 * natural-order q, k (PA_F32 or PA_BF16):
 *   q_pool[b,h,i,:] = mean of the valid rows of permuted block i of q (fp32),
 *   k_pool likewise,
 *   scores[b,h,i,j] = dot(q_pool[b,h,i,:], k_pool[b,h,j,:]) / sqrt(d) (fp32).
 * q_pool, k_pool [B,heads,NB,d] float and scores [B,heads,NB,NB] float are
 * all outputs and required. */
PA_API pa_status pa_block_score(const void* q, const void* k, pa_dtype dtype, pa_shape shape,
                         const int8_t* perms, float* q_pool, float* k_pool, float* scores,
                         void* stream);

/* The score half of pa_block_score alone, from pooled summaries already in
 * memory (e.g. the `pool` outputs of pa_quantize_int8):
 *   scores[b,h,i,j] = dot(q_pool[b,h,i,:], k_pool[b,h,j,:]) / sqrt(d). */
PA_API pa_status pa_score_pooled(const float* q_pool, const float* k_pool, pa_shape shape,
                          float* scores, void* stream);

/* Step 3, online (PASA review, Figure 2: at most k key blocks per query
 * block; SPADE review: Top-K filter).  Row (b,h,i) of scores
 * [B,heads,NB,NB] -> idx[b,h,i,0..k-1] (int32, ascending): block i itself,
 * then the k-1 largest other scores, ties to the lower block index, NaN
 * read as -inf, -0.0 equal to +0.0.  1 <= k <= NB; NB <= 14528
 * (PA_ERR_UNSUPPORTED above: four rows of NB keys share a CTA's shared
 * memory). */
PA_API pa_status pa_select_topk(const float* scores, pa_shape shape, int32_t k, int32_t* idx,
                         void* stream);

/* Step 3, hybrid filter (SPADE review, core_discovery: head-wise Top-K /
 * Top-P and local-window filters).  Row (b,h,i) of scores [B,heads,NB,NB]
 * keeps the union of
 *   - block i itself,
 *   - the local window {j : |i - j| <= window} (window < 0: none),
 *   - the Top-K set of pa_select_topk (k >= 1; k = 0: none),
 *   - the Top-P set: blocks in decreasing score order (ties to the lower
 *     index, NaN read as -inf), the shortest run whose softmax weights
 *     exp(s_j - max_j s_j) (summed in fp64; NaN weighs 0; a row whose max
 *     is +inf weighs its +inf entries 1 and the rest 0) reach
 *     top_p * (their row total); all blocks if none does; none if
 *     top_p <= 0 or the row is all -inf / NaN.
 * Output idx [B,heads,NB,NB] int32 (kept indices ascending, the rest -1)
 * and counts [B,heads,NB] int32, the format pa_block_sparse_attn takes with
 * k_max = NB.  0 <= k <= NB, top_p finite, NB <= 4096 (PA_ERR_UNSUPPORTED
 * above: a row is sorted in shared memory). */
PA_API pa_status pa_select_hybrid(const float* scores, pa_shape shape, int32_t k, double top_p,
                           int32_t window, int32_t* idx, int32_t* counts, void* stream);

/* Blocking-scheme score (SPADE review, key_machinery (ii): the Sum of
 * Intra-block Cosine Similarities, one pass per block by the identity
 * sum_{s != t} cos(x_s, x_t) = |sum_t xh_t|^2 - sum_t |xh_t|^2, xh = x/|x|,
 * zero rows adding nothing) of every candidate blocking (key_machinery
 * (i): spatial, temporal and mixed 3D blockings; the ids of the order table
 * above, 0-11: the six axis orders and the six tile blockings).  For every
 * candidate o and every (b,h):
 *   scores[b,h,o] = sum over the blocks of candidate o (runs of `block`
 *                   positions of its token order) of SICS(q's rows) +
 *                   SICS(k's rows).
 * q, k natural order [B,heads,N,d] (PA_F32 or PA_BF16), 16-byte aligned;
 * scores [B,heads,12] float, overwritten (accumulated in fp32 with atomics,
 * so the last bits vary between runs).  orders, if not NULL, [heads] int8
 * device memory, receives each head's pick: the candidate with the largest
 * score summed over the batch (a head has one blocking), ties to the lower
 * id -- SPADE's choice, to pass as the head's order id. */
PA_API pa_status pa_sics_scores(const void* q, const void* k, pa_dtype dtype, pa_shape shape,
                         float* scores, int8_t* orders, void* stream);

/* PAROAttention's offline stage (PAROAttention review, key_machinery: the
 * per-head order is chosen offline by a metric balancing block
 * sparsifiability against block incoherence; static masks by block-sum
 * thresholding; referee note on Eq. (1): n^{<eps}_{ij}).  Every entry walks
 * all NB x NB tiles of the dense map P = softmax(q k^T / sqrt(d)) of one
 * head on the tensor cores.  q_perm, k_perm: [B,heads,N_p,d] bf16 copies
 * permuted by one order for every head (pa_reorder with perms all = order);
 * d = 128, block = 128.  dev_status as for pa_block_sparse_attn.
 *
 * Row softmax of every token (no order changes it): with
 * s_c = q.k_c log2(e) / sqrt(d), row_max[b,h,n] = max_c s_c and
 * row_sum[b,h,n] = sum_c 2^(s_c - row_max), indexed by natural token n;
 * [B,heads,N] float outputs. */
PA_API pa_status pa_map_row_stats(const void* q_perm, const void* k_perm, pa_shape shape,
                           int32_t order, float* row_max, float* row_sum, int32_t* dev_status,
                           void* stream);

/* Block statistics of the map in one order, from the row softmax above:
 * for block (i, j) of the permuted map (its valid rows and columns), with
 * p = 2^(s - row_max) / row_sum,
 *   count[b,h,i,j] = #{p < eps},  total[...] = sum p,  peak[...] = max p
 * ([B,heads,NB,NB] float, overwritten), and when log_total is not NULL,
 * log_total = log(total) (-inf for 0): the scores whose pa_select_hybrid
 * Top-P set (k = 0, top_p = sigma, window = -1) is the static mask by
 * block-sum thresholding at sigma.  total and count are summed with
 * atomics, so their last bits vary between runs. */
PA_API pa_status pa_map_block_stats(const void* q_perm, const void* k_perm, pa_shape shape,
                             int32_t order, const float* row_max, const float* row_sum,
                             float eps, float* count, float* total, float* peak,
                             float* log_total, int32_t* dev_status, void* stream);

/* Per (b,h), for the statistics of one order:
 *   sparse_frac[b,h,order] = fraction of blocks with count >= rho * size,
 *   incoherence[b,h,order] = mean over blocks of positive mean of
 *                            peak / (total / size)
 * (size = valid rows x valid columns of the block); [B,heads,6] float,
 * only slot `order` written. */
PA_API pa_status pa_paro_metric(const float* count, const float* total, const float* peak,
                         pa_shape shape, int32_t order, float rho, float* sparse_frac,
                         float* incoherence, void* stream);

/* Per (b,h) from all six orders' slots: metric[o] = alpha (1 - sf[o]) /
 * max_o (1 - sf) + (1 - alpha) inc[o] / max_o inc (a term that is 0 for
 * every order adds 0); orders[b,h] = argmin, ties to the lower id (int8).
 * metric [B,heads,6] float, orders [B,heads] int8. */
PA_API pa_status pa_paro_choose(const float* sparse_frac, const float* incoherence, pa_shape shape,
                         float alpha, float* metric, int8_t* orders, void* stream);

/* Step 3, static (PAROAttention review, key_machinery: static masks stored
 * as bitmasks).  bitmask [B,heads,NB,ceil(NB/32)] uint32, bit (j % 32) of
 * word (j / 32) set when key block j is kept for query block i ->
 * idx [B,heads,NB,NB] int32 (kept indices ascending, the rest -1) and
 * counts [B,heads,NB] int32.  Bits at j >= NB are ignored. */
PA_API pa_status pa_compact_mask(const uint32_t* bitmask, pa_shape shape, int32_t* idx,
                          int32_t* counts, void* stream);

/* Per-block symmetric INT8 quantisation in the permuted order
 * (PAROAttention review, key_machinery: block-wise INT8 aligned to the
 * attention block).  For permuted block i of x (PA_F32 or PA_BF16,
 * natural order in):
 *   absmax = max |x| over the block's valid rows,
 *   x_q    = clamp(round_half_even(x * fl32(127/absmax)), -127, 127),
 *   scale  = fl32(absmax / 127)   (0 and all-zero codes when absmax = 0),
 * all in float32 round-to-nearest.  x_q [B,heads,N_p,d] int8 (pad rows 0),
 * scales [B,heads,NB] float.  pool, if not NULL, [B,heads,NB,d] float,
 * receives the block mean of x (as pa_block_score's q_pool) from the same
 * read. */
PA_API pa_status pa_quantize_int8(const void* x, pa_dtype dtype, pa_shape shape, const int8_t* perms,
                           int8_t* x_q, float* scales, float* pool, void* stream);

/* The same quantisation with 4-bit levels (the INT4 PV variant): 7 in place
 * of 127 everywhere above, codes in [-7, 7], one per int8 byte (the tensor
 * cores take them as int8 operands, so the products stay exact). */
PA_API pa_status pa_quantize_int4(const void* x, pa_dtype dtype, pa_shape shape, const int8_t* perms,
                           int8_t* x_q, float* scales, float* pool, void* stream);

/* Step 4 + fused step 5 (SPADE review, key_machinery (iii): flash
 * block-sparse attention with an online softmax; the inverse reorder is
 * the output store).  For every valid query token n of head (b,h), with
 * i = pos(n) / block:
 *   out[b,h,n,:] = sum_c softmax_c(q_n . k_c / sqrt(d)) v_c
 * over the tokens c whose block is listed in idx row (b,h,i) (the first
 * counts[b,h,i] entries, or all k when counts is NULL).
 *
 * idx [B,heads,NB,k] int32; each used entry in [0, NB), ascending, no
 * repeats (a malformed row is skipped with PA_ERR_DEVICE_CHECK on
 * dev_status; its rows of out are left unwritten).  A row whose count is
 * 0 produces zeros; with k_max = 0 every row does, and idx may be NULL.
 *
 * dtype PA_BF16: q, k, v, out bf16, natural order; P rounded to bf16 for
 *   the P V product, fp32 accumulation.
 * dtype PA_F32: q, k, v, out float, natural order; the products run in
 *   bf16 (inputs rounded to bf16 on load), fp32 accumulation.
 * dtype PA_I8: q, k, v are int8 [B,heads,N_p,d] from pa_quantize_int8
 *   (permuted) with scales q_scale, k_scale, v_scale [B,heads,NB]; out is
 *   bf16 natural order.  S = (Q8 K8^T in int32) * q_scale * k_scale /
 *   sqrt(d); per tile P~ = exp(s - running row max) is quantised to
 *   round_half_even(127 P~) and P V runs in int8 with int32
 *   accumulation, scaled by v_scale / 127; the normaliser sums the
 *   unrounded P~.
 * q_scale/k_scale/v_scale are ignored (may be NULL) unless dtype is PA_I8.
 *
 * flags: PA_ATTN_PERMUTED when q, k, v are [B,heads,N_p,d] in the permuted
 * order (pa_reorder's output) instead of [B,heads,N,d] natural.  Then every
 * tile of a head is 128 contiguous rows and the sm_100a kernel loads it with
 * TMA tiled boxes; with natural-order inputs the kernel gathers token rows
 * itself (no extra pass, but gathers feed the tensor cores more slowly).
 * PA_I8 inputs are always permuted (the flag is implied).  The output is
 * always natural order. */
#define PA_ATTN_PERMUTED 1u
/* With PA_I8: P is quantised to 4 bits, p4 = round_half_even(7 P~), and the
 * tile contributes (p4 V) * v_scale / 7 — the INT4 PV variant
 * (PAROAttention review: block-wise INT8/INT4 quantisation of the
 * post-softmax map and PV), with v (and its scales) from pa_quantize_int4;
 * q and k stay INT8. */
#define PA_ATTN_P4 2u
/* With PA_I8 (alone or with PA_ATTN_P4): the post-softmax map is quantised
 * after it is normalised, one symmetric scale per (query block, key block)
 * tile (PAROAttention review, key_machinery and core_discovery: block-wise
 * quantisation of the attention map, groups aligned to the attention
 * block).  Per tile: P = exp(s - m) / l with the row's exact max m and sum
 * l over all its kept keys, a = max of P over the tile's valid rows and
 * keys, codes round_half_even(L P / a) (L = 127, or 7 with PA_ATTN_P4),
 * and the tile contributes (codes V) * (a / L) * v_scale.  The kernel takes
 * two passes over the kept tiles (Q K^T twice), so it is slower than the
 * one-pass form above, whose per-tile scale is fixed at 1/L. */
#define PA_ATTN_P_TILE 4u

PA_API pa_status pa_block_sparse_attn(const void* q, const void* k, const void* v, pa_dtype dtype,
                               uint32_t flags, pa_shape shape, const int8_t* perms, const int32_t* idx,
                               const int32_t* counts, int32_t k_max, const float* q_scale,
                               const float* k_scale, const float* v_scale, void* out,
                               int32_t* dev_status, void* stream);

/* The same computation as pa_block_sparse_attn for dtype PA_F32 or PA_BF16,
 * on the legacy warp-level tensor-core path (mma.sync m16n8k16, one CTA per
 * query block, K/V tiles gathered into padded shared memory).  It is the
 * comparison baseline for the tcgen05 kernel, and it is also what
 * pa_block_sparse_attn itself runs for the shapes the tcgen05 kernel does
 * not take (d = 64, block = 64, or PA_F32).  Same arguments, layouts,
 * ownership and errors as pa_block_sparse_attn, without the INT8 scales. */
PA_API pa_status pa_block_sparse_attn_mma(const void* q, const void* k, const void* v, pa_dtype dtype,
                                   uint32_t flags, pa_shape shape, const int8_t* perms, const int32_t* idx,
                                   const int32_t* counts, int32_t k_max, void* out,
                                   int32_t* dev_status, void* stream);

/* Block-sparse attention with PASA's grouped first-order compensation of
 * the unselected key blocks (PASA review, Figure 2 caption: the key blocks
 * outside a query's kept set get a grouped first-order compensation instead
 * of being dropped; section 3.3: a Taylor expansion approximation).  The
 * page prints no formula; the reading implemented: exp(q.k_c / sqrt(d)) is
 * expanded to first order about the block's mean score q.kbar_j / sqrt(d),
 * whose linear term sums to zero over the block, and the block's values are
 * grouped the same way, so for every valid query token n (query block i):
 *   out[n] = (sum_{c kept} e^{s_c} v_c + sum_{j in U_i} n_j e^{sbar_j} vbar_j)
 *          / (sum_{c kept} e^{s_c} + sum_{j in U_i} n_j e^{sbar_j}),
 *   s_c = q_n.k_c / sqrt(d),  sbar_j = q_n.kbar_j / sqrt(d),
 * where U_i = the key blocks with at least one valid key that are not in
 * idx row (b,h,i), n_j = the valid keys of block j, and kbar_j, vbar_j are
 * the means of those keys and values.
 *
 * Arguments, layouts, ownership and errors as pa_block_sparse_attn_mma
 * (dtype PA_F32 or PA_BF16, flags 0 or PA_ATTN_PERMUTED; k_max = 0 is
 * allowed, with idx NULL or not, and gives the compensation alone), plus:
 *   k_pool, v_pool  [B,heads,NB,d], 16-byte aligned, read only: the
 *                   means of the valid rows of each permuted block of k and
 *                   v (the pool output of pa_reorder or pa_block_score),
 *                   element type pool_dtype.
 *   pool_dtype      PA_F32, or PA_BF16 for the same means rounded to bf16
 *                   (pa_round_bf16); PA_BF16 needs the tcgen05 kernel
 *                   (PA_ERR_UNSUPPORTED otherwise).
 * PA_BF16 with d = 128 and block = 128 runs on the tcgen05 kernel: after a
 * row's kept tiles come ceil(NB/128) tiles of pooled key rows (128 blocks'
 * means each), in the same online softmax; float means are rounded to bf16
 * by the kernel's loader warps, bf16 means are loaded like the K and V
 * tiles (the faster form).  Other shapes and PA_F32 run on the mma.sync
 * kernel, which rounds pooled blocks to bf16 like the K and V tiles.
 * NB <= 4096 (PA_ERR_UNSUPPORTED above: the kept list is held as one bit
 * per block in shared memory). */
PA_API pa_status pa_block_sparse_attn_compensated(const void* q, const void* k, const void* v,
                                           pa_dtype dtype, uint32_t flags, pa_shape shape,
                                           const int8_t* perms, const int32_t* idx,
                                           const int32_t* counts, int32_t k_max,
                                           const void* k_pool, const void* v_pool,
                                           pa_dtype pool_dtype, void* out,
                                           int32_t* dev_status, void* stream);

/* y[i] = x[i] rounded to bf16 (round to nearest even) for i < n: the bf16
 * block means that pa_block_sparse_attn_compensated takes with pool_dtype
 * PA_BF16.  x: n floats, y: n bf16, device memory, 16-byte aligned, not
 * overlapping; n = 0 does nothing.  Not an operation of the pages: a
 * storage conversion, so that the attention kernel moves 2-byte means. */
PA_API pa_status pa_round_bf16(const float* x, void* y, int64_t n, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* PARO_H */
