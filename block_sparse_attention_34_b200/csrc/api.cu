// The C ABI of libparo (declared in include/paro.h): argument validation,
// the per-call Grid description, and dispatch to the kernels.  Nothing here
// allocates device memory or synchronises.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>

#include "common.cuh"

namespace paro {
cudaError_t launch_attn_sm100(const void* q, const void* k, const void* v, pa_dtype dt,
                              const Grid& g, const int32_t* idx, const int32_t* counts,
                              int k_max, const float* qs, const float* ks, const float* vs,
                              float p_levels, void* out, int32_t* status, bool permuted,
                              cudaStream_t s, const void* k_pool = nullptr,
                              const void* v_pool = nullptr, pa_dtype pool_dtype = PA_F32);
bool attn_sm100_supports(pa_dtype dt, const Grid& g);
}  // namespace paro

namespace paro {
namespace {
StallTest g_stall{-1, -1, -1, 0, 1000000000ull};
}  // namespace
StallTest stall_test() { return g_stall; }
}  // namespace paro

namespace {

thread_local std::string g_error;

pa_status fail(pa_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_error = buf;
  return st;
}

pa_status ok() {
  g_error.clear();
  return PA_OK;
}

pa_status cuda_status(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return ok();
  return fail(PA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Validates the sizes and fills the grid description (order tables included).
pa_status make_grid(const pa_shape& s, const int8_t* perms, bool need_perms, paro::Grid* g) {
  if (s.B < 1 || s.heads < 1 || s.F < 1 || s.H < 1 || s.W < 1 || s.d < 1 || s.block < 1)
    return fail(PA_ERR_INVALID_ARG, "shape fields must be >= 1 (B=%d heads=%d F=%d H=%d W=%d d=%d block=%d)",
                s.B, s.heads, s.F, s.H, s.W, s.d, s.block);
  if (s.heads > paro::kMaxHeads)
    return fail(PA_ERR_UNSUPPORTED, "heads=%d exceeds the supported maximum %d", s.heads, paro::kMaxHeads);
  if (s.d != 64 && s.d != 128)
    return fail(PA_ERR_UNSUPPORTED, "head dim d=%d unsupported (64 or 128)", s.d);
  if (s.block != 64 && s.block != 128)
    return fail(PA_ERR_UNSUPPORTED, "block=%d unsupported (64 or 128)", s.block);
  const int64_t N = (int64_t)s.F * s.H * s.W;
  const int64_t NB = (N + s.block - 1) / s.block;
  const int64_t Np = NB * s.block;
  if (Np > (int64_t)1 << 30)
    return fail(PA_ERR_UNSUPPORTED, "N=%lld tokens per head exceeds 2^30", (long long)N);
  if ((int64_t)s.B * s.heads * Np * s.d >= ((int64_t)1 << 40))
    return fail(PA_ERR_UNSUPPORTED, "tensor of B*heads*N_p*d elements too large");
  std::memset(g, 0, sizeof(*g));
  g->B = s.B;
  g->heads = s.heads;
  g->F = s.F;
  g->H = s.H;
  g->W = s.W;
  g->d = s.d;
  g->block = s.block;
  g->N = (int32_t)N;
  g->NB = (int32_t)NB;
  g->Np = (int32_t)Np;
  const int size[3] = {s.F, s.H, s.W};
  const int stride[3] = {s.H * s.W, s.W, 1};
  // axes of each order id, outermost first: FHW FWH HFW HWF WFH WHF
  static const int axes[6][3] = {{0, 1, 2}, {0, 2, 1}, {1, 0, 2}, {1, 2, 0}, {2, 0, 1}, {2, 1, 0}};
  for (int o = 0; o < 6; ++o) {
    g->mid[o] = size[axes[o][1]];
    g->inn[o] = size[axes[o][2]];
    g->so[o] = stride[axes[o][0]];
    g->sm[o] = stride[axes[o][1]];
    g->si[o] = stride[axes[o][2]];
  }
  // the 3D tile blockings of ids 6-11 (tf, th, tw; volume = block): two
  // spatial (tf = 1), two mixed, two temporal
  static const int tiles128[6][3] = {{1, 8, 16}, {1, 16, 8}, {2, 8, 8},
                                     {4, 4, 8},  {8, 4, 4},  {16, 2, 4}};
  static const int tiles64[6][3] = {{1, 8, 8}, {1, 4, 16}, {2, 4, 8},
                                    {4, 4, 4}, {8, 2, 4},  {16, 2, 2}};
  for (int t = 0; t < 6; ++t) {
    const int* sh = s.block == 128 ? tiles128[t] : tiles64[t];
    g->tf[t] = sh[0];
    g->th[t] = sh[1];
    g->tw[t] = sh[2];
  }
  if (need_perms) {
    if (perms == nullptr) return fail(PA_ERR_INVALID_ARG, "perms is NULL");
    for (int h = 0; h < s.heads; ++h) {
      if (perms[h] < 0 || perms[h] >= paro::kOrders)
        return fail(PA_ERR_INVALID_ARG, "perms[%d]=%d is not an order id 0..%d", h,
                    (int)perms[h], paro::kOrders - 1);
      g->perm[h] = perms[h];
    }
  }
  return PA_OK;
}

#define PA_REQUIRE(cond, ...)                                   \
  do {                                                          \
    if (!(cond)) return fail(PA_ERR_INVALID_ARG, __VA_ARGS__); \
  } while (0)

pa_status check_float_dtype(pa_dtype dt) {
  if (dt != PA_F32 && dt != PA_BF16)
    return fail(PA_ERR_INVALID_ARG, "dtype %d: expected PA_F32 or PA_BF16", (int)dt);
  return PA_OK;
}

}  // namespace

extern "C" {

int32_t pa_abi_version(void) { return 8; }

pa_status pa_clear_status(int32_t* dev_status, void* stream) {
  PA_REQUIRE(dev_status != nullptr, "dev_status must be non-NULL");
  return cuda_status(cudaMemsetAsync(dev_status, 0, sizeof(int32_t), (cudaStream_t)stream),
                     "pa_clear_status memset");
}

const char* pa_last_error(void) { return g_error.c_str(); }

pa_status pa_test_inject_v_stall(int32_t query_block, int32_t batch_head, int32_t tile,
                                 uint64_t wait_limit_ns) {
  if (tile < 0) {
    paro::g_stall = paro::StallTest{-1, -1, -1, 0, 1000000000ull};
    return ok();
  }
  PA_REQUIRE(query_block >= 0 && batch_head >= 0, "query_block and batch_head must be >= 0");
  PA_REQUIRE(wait_limit_ns >= 1000 && wait_limit_ns <= 1000000000ull,
             "wait_limit_ns=%llu must be in [1 us, 1 s]", (unsigned long long)wait_limit_ns);
  paro::g_stall = paro::StallTest{query_block, batch_head, tile, 0, wait_limit_ns};
  return ok();
}

int32_t pa_num_blocks(pa_shape s) {
  if (s.F < 1 || s.H < 1 || s.W < 1 || s.block < 1) return -1;
  const int64_t N = (int64_t)s.F * s.H * s.W;
  const int64_t nb = (N + s.block - 1) / s.block;
  return nb > INT32_MAX ? -1 : (int32_t)nb;
}

int32_t pa_k_for_density(int32_t nb, double density) {
  if (nb <= 0) return 0;
  double x = density * (double)nb;
  if (!(x == x)) return 1;  // NaN density keeps the diagonal only
  x = std::nearbyint(x * 1e9) / 1e9;  // round to 9 decimals
  double c = std::ceil(x);
  if (c < 1.0) c = 1.0;
  if (c > (double)nb) c = (double)nb;
  return (int32_t)c;
}

pa_status pa_reorder(const void* x, void* x_perm, pa_dtype dtype, pa_shape shape,
                     const int8_t* perms, float* pool, void* stream) {
  paro::Grid g;
  pa_status st = check_float_dtype(dtype);
  if (st != PA_OK) return st;
  if ((st = make_grid(shape, perms, true, &g)) != PA_OK) return st;
  PA_REQUIRE(x && x_perm, "x and x_perm must be non-NULL");
  PA_REQUIRE(aligned16(x) && aligned16(x_perm), "x and x_perm must be 16-byte aligned");
  return cuda_status(paro::launch_reorder_pool(x, x_perm, dtype, g, pool, (cudaStream_t)stream),
                     "pa_reorder launch");
}

pa_status pa_inverse_reorder(const void* x_perm, void* x, pa_dtype dtype, pa_shape shape,
                             const int8_t* perms, void* stream) {
  paro::Grid g;
  pa_status st = check_float_dtype(dtype);
  if (st != PA_OK) return st;
  if ((st = make_grid(shape, perms, true, &g)) != PA_OK) return st;
  PA_REQUIRE(x && x_perm, "x and x_perm must be non-NULL");
  PA_REQUIRE(aligned16(x) && aligned16(x_perm), "x and x_perm must be 16-byte aligned");
  return cuda_status(paro::launch_reorder(x_perm, x, dtype, g, true, (cudaStream_t)stream),
                     "pa_inverse_reorder launch");
}

pa_status pa_block_score(const void* q, const void* k, pa_dtype dtype, pa_shape shape,
                         const int8_t* perms, float* q_pool, float* k_pool, float* scores,
                         void* stream) {
  paro::Grid g;
  pa_status st = check_float_dtype(dtype);
  if (st != PA_OK) return st;
  if ((st = make_grid(shape, perms, true, &g)) != PA_OK) return st;
  PA_REQUIRE(q && k && q_pool && k_pool && scores,
             "q, k, q_pool, k_pool and scores must be non-NULL");
  PA_REQUIRE(aligned16(q) && aligned16(k), "q and k must be 16-byte aligned");
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = paro::launch_pool(q, dtype, g, q_pool, s);
  if (e == cudaSuccess) e = paro::launch_pool(k, dtype, g, k_pool, s);
  if (e == cudaSuccess) e = paro::launch_score(q_pool, k_pool, g, scores, s);
  return cuda_status(e, "pa_block_score launch");
}

pa_status pa_score_pooled(const float* q_pool, const float* k_pool, pa_shape shape,
                          float* scores, void* stream) {
  paro::Grid g;
  pa_status st = make_grid(shape, nullptr, false, &g);
  if (st != PA_OK) return st;
  PA_REQUIRE(q_pool && k_pool && scores, "q_pool, k_pool and scores must be non-NULL");
  return cuda_status(paro::launch_score(q_pool, k_pool, g, scores, (cudaStream_t)stream),
                     "pa_score_pooled launch");
}

pa_status pa_select_topk(const float* scores, pa_shape shape, int32_t k, int32_t* idx,
                         void* stream) {
  paro::Grid g;
  pa_status st = make_grid(shape, nullptr, false, &g);
  if (st != PA_OK) return st;
  PA_REQUIRE(scores && idx, "scores and idx must be non-NULL");
  PA_REQUIRE(k >= 1 && k <= g.NB, "k=%d must be in [1, NB=%d]", k, g.NB);
  if (g.NB > paro::kTopkMaxNB)
    return fail(PA_ERR_UNSUPPORTED, "NB=%d exceeds %d (a row's keys must fit in shared memory)",
                g.NB, paro::kTopkMaxNB);
  return cuda_status(paro::launch_topk(scores, g, k, idx, (cudaStream_t)stream),
                     "pa_select_topk launch");
}

pa_status pa_select_hybrid(const float* scores, pa_shape shape, int32_t k, double top_p,
                           int32_t window, int32_t* idx, int32_t* counts, void* stream) {
  paro::Grid g;
  pa_status st = make_grid(shape, nullptr, false, &g);
  if (st != PA_OK) return st;
  PA_REQUIRE(scores && idx && counts, "scores, idx and counts must be non-NULL");
  PA_REQUIRE(k >= 0 && k <= g.NB, "k=%d must be in [0, NB=%d]", k, g.NB);
  PA_REQUIRE(std::isfinite(top_p), "top_p must be finite");
  if (g.NB > 4096) return fail(PA_ERR_UNSUPPORTED, "NB=%d exceeds 4096 for pa_select_hybrid", g.NB);
  return cuda_status(
      paro::launch_hybrid(scores, g, k, top_p, window, idx, counts, (cudaStream_t)stream),
      "pa_select_hybrid launch");
}

pa_status pa_sics_scores(const void* q, const void* k, pa_dtype dtype, pa_shape shape,
                         float* scores, int8_t* orders, void* stream) {
  paro::Grid g;
  pa_status st = make_grid(shape, nullptr, false, &g);
  if (st != PA_OK) return st;
  PA_REQUIRE(dtype == PA_F32 || dtype == PA_BF16, "dtype %d: pa_sics_scores takes F32 or BF16",
             (int)dtype);
  PA_REQUIRE(q && k && scores, "q, k and scores must be non-NULL");
  PA_REQUIRE(aligned16(q) && aligned16(k), "q and k must be 16-byte aligned");
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e =
      cudaMemsetAsync(scores, 0, (size_t)g.B * g.heads * paro::kOrders * sizeof(float), s);
  if (e == cudaSuccess) e = paro::launch_sics(q, dtype, g, scores, s);
  if (e == cudaSuccess) e = paro::launch_sics(k, dtype, g, scores, s);
  if (e == cudaSuccess && orders != nullptr) e = paro::launch_sics_pick(scores, g, orders, s);
  return cuda_status(e, "pa_sics_scores launch");
}

static pa_status map_common(const void* qp, const void* kp, pa_shape shape, int32_t order,
                            paro::Grid* g) {
  pa_status st = make_grid(shape, nullptr, false, g);
  if (st != PA_OK) return st;
  PA_REQUIRE(qp && kp, "q_perm and k_perm must be non-NULL");
  PA_REQUIRE(aligned16(qp) && aligned16(kp), "q_perm and k_perm must be 16-byte aligned");
  PA_REQUIRE(order >= 0 && order < 6, "order=%d must be in [0, 6)", order);
  if (g->d != 128 || g->block != 128)
    return fail(PA_ERR_UNSUPPORTED, "the map statistics need d=128, block=128 (tcgen05 kernel)");
  if ((int64_t)g->B * g->heads * g->Np >= ((int64_t)1 << 31))
    return fail(PA_ERR_UNSUPPORTED, "B*heads*N_p exceeds 2^31 rows");
  return PA_OK;
}

pa_status pa_map_row_stats(const void* q_perm, const void* k_perm, pa_shape shape, int32_t order,
                           float* row_max, float* row_sum, int32_t* dev_status, void* stream) {
  paro::Grid g;
  pa_status st = map_common(q_perm, k_perm, shape, order, &g);
  if (st != PA_OK) return st;
  PA_REQUIRE(row_max && row_sum, "row_max and row_sum must be non-NULL");
  return cuda_status(paro::launch_map_stats(q_perm, k_perm, g, order, false, row_max, row_sum,
                                            0.f, nullptr, nullptr, nullptr, dev_status,
                                            (cudaStream_t)stream),
                     "pa_map_row_stats launch");
}

pa_status pa_map_block_stats(const void* q_perm, const void* k_perm, pa_shape shape,
                             int32_t order, const float* row_max, const float* row_sum, float eps,
                             float* count, float* total, float* peak, float* log_total,
                             int32_t* dev_status, void* stream) {
  paro::Grid g;
  pa_status st = map_common(q_perm, k_perm, shape, order, &g);
  if (st != PA_OK) return st;
  PA_REQUIRE(row_max && row_sum && count && total && peak,
             "row_max, row_sum, count, total and peak must be non-NULL");
  PA_REQUIRE(std::isfinite(eps), "eps must be finite");
  cudaStream_t s = (cudaStream_t)stream;
  const size_t n = (size_t)g.B * g.heads * g.NB * g.NB;
  cudaError_t e = cudaMemsetAsync(count, 0, n * sizeof(float), s);
  if (e == cudaSuccess) e = cudaMemsetAsync(total, 0, n * sizeof(float), s);
  if (e == cudaSuccess) e = cudaMemsetAsync(peak, 0, n * sizeof(float), s);
  if (e == cudaSuccess)
    e = paro::launch_map_stats(q_perm, k_perm, g, order, true, const_cast<float*>(row_max),
                               const_cast<float*>(row_sum), eps, count, total, peak, dev_status,
                               s);
  if (e == cudaSuccess && log_total != nullptr)
    e = paro::launch_log_total(total, log_total, (int64_t)n, s);
  return cuda_status(e, "pa_map_block_stats launch");
}

pa_status pa_paro_metric(const float* count, const float* total, const float* peak,
                         pa_shape shape, int32_t order, float rho, float* sparse_frac,
                         float* incoherence, void* stream) {
  paro::Grid g;
  pa_status st = make_grid(shape, nullptr, false, &g);
  if (st != PA_OK) return st;
  PA_REQUIRE(count && total && peak && sparse_frac && incoherence, "NULL argument");
  PA_REQUIRE(order >= 0 && order < 6, "order=%d must be in [0, 6)", order);
  PA_REQUIRE(std::isfinite(rho), "rho must be finite");
  return cuda_status(paro::launch_paro_metric(count, total, peak, g, order, rho, sparse_frac,
                                              incoherence, (cudaStream_t)stream),
                     "pa_paro_metric launch");
}

pa_status pa_paro_choose(const float* sparse_frac, const float* incoherence, pa_shape shape,
                         float alpha, float* metric, int8_t* orders, void* stream) {
  paro::Grid g;
  pa_status st = make_grid(shape, nullptr, false, &g);
  if (st != PA_OK) return st;
  PA_REQUIRE(sparse_frac && incoherence && metric && orders, "NULL argument");
  PA_REQUIRE(std::isfinite(alpha), "alpha must be finite");
  return cuda_status(paro::launch_paro_choose(sparse_frac, incoherence, (int64_t)g.B * g.heads,
                                              alpha, metric, orders, (cudaStream_t)stream),
                     "pa_paro_choose launch");
}

pa_status pa_compact_mask(const uint32_t* bitmask, pa_shape shape, int32_t* idx, int32_t* counts,
                          void* stream) {
  paro::Grid g;
  pa_status st = make_grid(shape, nullptr, false, &g);
  if (st != PA_OK) return st;
  PA_REQUIRE(bitmask && idx && counts, "bitmask, idx and counts must be non-NULL");
  return cuda_status(paro::launch_compact(bitmask, g, idx, counts, (cudaStream_t)stream),
                     "pa_compact_mask launch");
}

static pa_status quantize_common(const void* x, pa_dtype dtype, pa_shape shape,
                                 const int8_t* perms, int8_t* x_q, float* scales, float* pool,
                                 int qmax, void* stream) {
  paro::Grid g;
  pa_status st = check_float_dtype(dtype);
  if (st != PA_OK) return st;
  if ((st = make_grid(shape, perms, true, &g)) != PA_OK) return st;
  PA_REQUIRE(x && x_q && scales, "x, x_q and scales must be non-NULL");
  PA_REQUIRE(aligned16(x) && aligned16(x_q), "x and x_q must be 16-byte aligned");
  return cuda_status(
      paro::launch_quantize(x, dtype, g, x_q, scales, pool, qmax, (cudaStream_t)stream),
      "pa_quantize launch");
}

pa_status pa_quantize_int8(const void* x, pa_dtype dtype, pa_shape shape, const int8_t* perms,
                           int8_t* x_q, float* scales, float* pool, void* stream) {
  return quantize_common(x, dtype, shape, perms, x_q, scales, pool, 127, stream);
}

pa_status pa_quantize_int4(const void* x, pa_dtype dtype, pa_shape shape, const int8_t* perms,
                           int8_t* x_q, float* scales, float* pool, void* stream) {
  return quantize_common(x, dtype, shape, perms, x_q, scales, pool, 7, stream);
}

static pa_status attn_common(const void* q, const void* k, const void* v, pa_dtype dtype,
                             uint32_t flags, pa_shape shape, const int8_t* perms, const int32_t* idx,
                             const int32_t* counts, int32_t k_max, const float* q_scale,
                             const float* k_scale, const float* v_scale, void* out,
                             int32_t* dev_status, void* stream, bool force_mma) {
  paro::Grid g;
  pa_status st = make_grid(shape, perms, true, &g);
  if (st != PA_OK) return st;
  PA_REQUIRE(dtype == PA_F32 || dtype == PA_BF16 || dtype == PA_I8, "dtype %d unknown", (int)dtype);
  PA_REQUIRE(q && k && v && out, "q, k, v and out must be non-NULL");
  PA_REQUIRE(idx || k_max == 0, "idx must be non-NULL when k_max > 0");
  PA_REQUIRE(aligned16(q) && aligned16(k) && aligned16(v) && aligned16(out),
             "q, k, v and out must be 16-byte aligned");
  PA_REQUIRE(k_max >= 0 && k_max <= g.NB, "k_max=%d must be in [0, NB=%d]", k_max, g.NB);
  if (dtype == PA_I8) {
    PA_REQUIRE(q_scale && k_scale && v_scale, "INT8 attention needs q_scale, k_scale, v_scale");
  }
  PA_REQUIRE((flags & ~(PA_ATTN_PERMUTED | PA_ATTN_P4 | PA_ATTN_P_TILE)) == 0,
             "unknown flags 0x%x", flags);
  PA_REQUIRE(!(flags & PA_ATTN_P4) || dtype == PA_I8, "PA_ATTN_P4 needs dtype PA_I8");
  PA_REQUIRE(!(flags & PA_ATTN_P_TILE) || dtype == PA_I8, "PA_ATTN_P_TILE needs dtype PA_I8");
  const float p_levels = (flags & PA_ATTN_P4) ? 7.f : 127.f;
  const bool permuted = dtype == PA_I8 || (flags & PA_ATTN_PERMUTED) != 0;
  cudaStream_t s = (cudaStream_t)stream;
  const bool sm100 = !force_mma && paro::attn_sm100_supports(dtype, g);
  if (dtype == PA_I8 && !sm100)
    return fail(PA_ERR_UNSUPPORTED, "INT8 attention needs d=128, block=128 (tcgen05 kernel)");
  if (k_max == 0) {
    // every row has no kept block: the output is all zeros
    const size_t es = dtype == PA_F32 ? 4 : 2;
    return cuda_status(cudaMemsetAsync(out, 0, (size_t)g.B * g.heads * g.N * g.d * es, s),
                       "pa_block_sparse_attn memset");
  }
  cudaError_t e;
  if (dtype == PA_I8)
    e = paro::launch_attn_i8(q, k, v, g, idx, counts, k_max, q_scale, k_scale, v_scale, p_levels,
                             (flags & PA_ATTN_P_TILE) != 0, out, dev_status, s);
  else if (sm100)
    e = paro::launch_attn_sm100(q, k, v, dtype, g, idx, counts, k_max, q_scale, k_scale, v_scale,
                                p_levels, out, dev_status, permuted, s);
  else
    e = paro::launch_attn_mma(q, k, v, dtype, g, idx, counts, k_max, out, dev_status, permuted, s);
  return cuda_status(e, "pa_block_sparse_attn launch");
}

pa_status pa_block_sparse_attn(const void* q, const void* k, const void* v, pa_dtype dtype,
                               uint32_t flags, pa_shape shape, const int8_t* perms,
                               const int32_t* idx, const int32_t* counts, int32_t k_max,
                               const float* q_scale, const float* k_scale, const float* v_scale,
                               void* out, int32_t* dev_status, void* stream) {
  return attn_common(q, k, v, dtype, flags, shape, perms, idx, counts, k_max, q_scale, k_scale,
                     v_scale, out, dev_status, stream, false);
}

pa_status pa_block_sparse_attn_mma(const void* q, const void* k, const void* v, pa_dtype dtype,
                                   uint32_t flags, pa_shape shape, const int8_t* perms,
                                   const int32_t* idx, const int32_t* counts, int32_t k_max,
                                   void* out, int32_t* dev_status, void* stream) {
  PA_REQUIRE(dtype != PA_I8, "the mma.sync baseline takes PA_F32 or PA_BF16");
  return attn_common(q, k, v, dtype, flags, shape, perms, idx, counts, k_max, nullptr, nullptr,
                     nullptr, out, dev_status, stream, true);
}

pa_status pa_block_sparse_attn_compensated(const void* q, const void* k, const void* v,
                                           pa_dtype dtype, uint32_t flags, pa_shape shape,
                                           const int8_t* perms, const int32_t* idx,
                                           const int32_t* counts, int32_t k_max,
                                           const void* k_pool, const void* v_pool,
                                           pa_dtype pool_dtype, void* out, int32_t* dev_status,
                                           void* stream) {
  paro::Grid g;
  pa_status st = make_grid(shape, perms, true, &g);
  if (st != PA_OK) return st;
  PA_REQUIRE(dtype == PA_F32 || dtype == PA_BF16,
             "dtype %d: pa_block_sparse_attn_compensated takes PA_F32 or PA_BF16", (int)dtype);
  PA_REQUIRE(q && k && v && out && k_pool && v_pool,
             "q, k, v, k_pool, v_pool and out must be non-NULL");
  PA_REQUIRE(idx || k_max == 0, "idx must be non-NULL when k_max > 0");
  PA_REQUIRE(aligned16(q) && aligned16(k) && aligned16(v) && aligned16(out) &&
                 aligned16(k_pool) && aligned16(v_pool),
             "q, k, v, k_pool, v_pool and out must be 16-byte aligned");
  PA_REQUIRE(k_max >= 0 && k_max <= g.NB, "k_max=%d must be in [0, NB=%d]", k_max, g.NB);
  PA_REQUIRE((flags & ~PA_ATTN_PERMUTED) == 0, "unknown flags 0x%x", flags);
  PA_REQUIRE(pool_dtype == PA_F32 || pool_dtype == PA_BF16,
             "pool_dtype %d: the block means are PA_F32 or PA_BF16", (int)pool_dtype);
  const bool sm100 = dtype == PA_BF16 && paro::attn_sm100_supports(dtype, g);
  if (pool_dtype == PA_BF16 && !sm100)
    return fail(PA_ERR_UNSUPPORTED,
                "bf16 block means need the tcgen05 kernel (PA_BF16, d=128, block=128)");
  if (g.NB > 4096) return fail(PA_ERR_UNSUPPORTED, "NB=%d above 4096 (one bit per block in shared memory)", g.NB);
  const bool permuted = (flags & PA_ATTN_PERMUTED) != 0;
  cudaStream_t s = (cudaStream_t)stream;
  // the tcgen05 kernel for bf16, d = 128, block = 128; the mma.sync one otherwise
  if (sm100)
    return cuda_status(paro::launch_attn_sm100(q, k, v, dtype, g, idx, counts, k_max, nullptr,
                                               nullptr, nullptr, 127.f, out, dev_status, permuted,
                                               s, k_pool, v_pool, pool_dtype),
                       "pa_block_sparse_attn_compensated launch");
  return cuda_status(paro::launch_attn_mma(q, k, v, dtype, g, idx, counts, k_max, out, dev_status,
                                           permuted, s, static_cast<const float*>(k_pool),
                                           static_cast<const float*>(v_pool)),
                     "pa_block_sparse_attn_compensated launch");
}

pa_status pa_round_bf16(const float* x, void* y, int64_t n, void* stream) {
  PA_REQUIRE(n >= 0, "n=%lld must be >= 0", (long long)n);
  if (n == 0) return PA_OK;
  PA_REQUIRE(x && y, "x and y must be non-NULL");
  PA_REQUIRE(aligned16(x) && aligned16(y), "x and y must be 16-byte aligned");
  PA_REQUIRE(n <= ((int64_t)1 << 40), "n=%lld too large", (long long)n);
  return cuda_status(paro::launch_round_bf16(x, y, n, (cudaStream_t)stream), "pa_round_bf16 launch");
}

}  // extern "C"
