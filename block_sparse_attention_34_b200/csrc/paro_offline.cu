// PAROAttention's offline stage on the tensor cores (PAROAttention, arXiv
// 2506.16054, Pith verdict page, key_machinery: per-head order chosen by a
// metric that balances block sparsifiability against block incoherence,
// static masks by block-sum thresholding; referee note on Eq. (1): the count
// n^{<eps}_{ij} of entries of block (i, j) below eps).
//
// Both passes walk every (query block, key block) tile of the dense map
// P = softmax(Q K^T / sqrt(d)) of one axis order, from the order's permuted
// copies of q and k (pa_reorder; bf16, d = 128, block = 128):
//   pass 1 (row_stats):   per token, m = max_c s_c and l = sum_c 2^(s_c - m)
//                         with s = q.k log2(e) / sqrt(d): the softmax of
//                         every row, which no order changes;
//   pass 2 (block_stats): per tile, with p = 2^(s - m_row) / l_row, the
//                         count of p < eps, the sum and the max of p over the
//                         tile's valid rows and columns.
// One CTA per (query block, head): 10 warps.  Warps 0-7 read S, two per TMEM
// lane quarter (columns 64 (w >> 2) .. +63), one row per thread: in pass 1
// each half keeps its own running max and sum and the two are merged once
// at the end (exact: l = l0 2^(m0 - m) + l1 2^(m1 - m)); in pass 2 each
// warp reduces its 32 x 64 partial statistics and adds them to the tile's
// counters with global atomics (the counters start at zero; the max is
// taken on the float bits, all p >= 0).  Warp 8 allocates TMEM and issues
// QK^T into a double-buffered S (two 128-column buffers), so the MMA of
// tile j+1 runs while tile j is read; warp 9 streams Q once and the K tiles
// through a two-stage ring with TMA (two CTAs per SM share the tensor
// core and hide each other's waits).  Every wait is bounded as in the
// attention kernels (PA_ERR_TIMEOUT).
#include "sm100.cuh"
#include "tmem.cuh"

namespace paro {
namespace {

using namespace sm100;

constexpr int kBlock = 128;
constexpr int kD = 128;
constexpr int kStages = 2;  // two CTAs per SM (shared memory, TMEM 2 x 256 columns)
constexpr int kMmaWarp = 8;
constexpr int kLoadWarp = 9;
constexpr int kThreads = 10 * 32;
constexpr int kRowThreads = 256;
constexpr uint32_t kTile = kBlock * kD * 2;  // 32 KB: two 64-column panels
constexpr uint32_t kHalf = kBlock * 128;     // 16 KB
constexpr uint32_t kOffBar = 0;
constexpr uint32_t kOffSlot = 256;
constexpr uint32_t kOffMerge = 512;  // pass-1 merge: [2 halves][2][128] f32 = 2 KB
constexpr uint32_t kOffQ = 3072;
constexpr uint32_t kOffK = kOffQ + kTile;
constexpr uint32_t kSmemBytes = kOffK + kStages * kTile;  // 101,376 B
static_assert(2 * (kSmemBytes + 1024) <= 232448, "two CTAs per SM");
static_assert(kOffQ % 1024 == 0, "swizzled tiles need 1024-byte alignment");
constexpr uint32_t kTmemCols = 256;

enum : uint32_t {
  BQ = 0,
  BK0 = 1,               // K stage full (kStages)
  BKF0 = BK0 + kStages,  // K stage free
  BS0 = BKF0 + kStages,  // S buffer b holds tile j (2)
  BSF0 = BS0 + 2,        // S buffer b read (2)
  BM = BSF0 + 2,         // pass-1 halves written
  BDRAIN,
  NBAR
};
static_assert(NBAR * 8 <= kOffSlot, "barrier region");

template <bool kBlockStats>
__global__ void __launch_bounds__(kThreads, 2)
    map_stats_kernel(const __grid_constant__ CUtensorMap map_q,
                     const __grid_constant__ CUtensorMap map_k, const __grid_constant__ Grid g,
                     int order, float scale_log2, float* __restrict__ row_max,
                     float* __restrict__ row_sum, float eps, float* __restrict__ count,
                     float* __restrict__ total, float* __restrict__ peak,
                     int32_t* __restrict__ status) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t base = smem_u32(smem_raw);
  if ((base & 1023u) != 0) {
    if (threadIdx.x == 0) report(status, PA_ERR_UNSUPPORTED);
    return;
  }
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem_raw + kOffSlot);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  float* merge = reinterpret_cast<float*>(smem_raw + kOffMerge);
  auto bar = [&](uint32_t slot) { return base + kOffBar + slot * 8u; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x;
  const int64_t bh = blockIdx.y;
  const int nb = g.NB;
  Ctl ctl{abort_flag, status};
  const bool expired =
      status != nullptr && *reinterpret_cast<volatile int32_t*>(status) == PA_ERR_TIMEOUT;

  if (threadIdx.x == 0) {
    mbar_init(bar(BQ), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(BK0 + s), 1);
      mbar_init(bar(BKF0 + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(BS0 + b), 1);
      mbar_init(bar(BSF0 + b), kRowThreads);
    }
    mbar_init(bar(BM), kRowThreads);
    mbar_init(bar(BDRAIN), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == kMmaWarp) tmem_alloc(smem_u32(tmem_slot), kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int n_tiles = expired ? 0 : nb;
  const int row0 = (int)(bh * g.Np);

  if (warp == kLoadWarp) {
    // ------------------------------------------------------ loads ------
    if (lane == 0 && n_tiles > 0) {
      mbar_arrive_tx(bar(BQ), kTile);
      tma_load_2d(base + kOffQ, &map_q, 0, row0 + i * kBlock, bar(BQ));
      tma_load_2d(base + kOffQ + kHalf, &map_q, 64, row0 + i * kBlock, bar(BQ));
      int issued = 0;
      for (int j = 0; j < n_tiles; ++j) {
        const int s = j % kStages;
        if (j >= kStages && !wait_phase(bar(BKF0 + s), ((j / kStages) - 1) & 1, ctl)) break;
        mbar_arrive_tx(bar(BK0 + s), kTile);
        tma_load_2d(base + kOffK + s * kTile, &map_k, 0, row0 + j * kBlock, bar(BK0 + s));
        tma_load_2d(base + kOffK + s * kTile + kHalf, &map_k, 64, row0 + j * kBlock, bar(BK0 + s));
        issued = j + 1;
      }
      drain_phase(bar(BQ), 0);
      for (int j = issued > kStages ? issued - kStages : 0; j < issued; ++j)
        drain_phase(bar(BK0 + j % kStages), (j / kStages) & 1);
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ---------------------------------------------------------- MMA ----
    if (lane == 0 && n_tiles > 0) {
      constexpr uint32_t id_qk = idesc_bf16(kBlock, kBlock, false);
      bool ok = wait_phase(bar(BQ), 0, ctl);
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int s = j % kStages, b = j & 1;
        if (!wait_phase(bar(BK0 + s), (j / kStages) & 1, ctl)) break;
        if (j >= 2 && !wait_phase(bar(BSF0 + b), ((j >> 1) - 1) & 1, ctl)) break;
        tc_fence_after();
        const uint32_t ka = base + kOffK + s * kTile;
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
          mma_f16_ss(tmem + b * 128, sw128_desc(base + kOffQ + off, 16, 1024),
                     sw128_desc(ka + off, 16, 1024), id_qk, kk > 0 ? 1u : 0u);
        }
        mma_commit(bar(BS0 + b));
        mma_commit(bar(BKF0 + s));
      }
      mma_commit(bar(BDRAIN));
      drain_phase(bar(BDRAIN), 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ row statistics ----
    const int quarter = warp & 3, hc = warp >> 2;
    const int r = quarter * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    const int p = i * kBlock + r;
    const bool row_ok = p < g.N;
    const int64_t tok = row_ok ? bh * (int64_t)g.N + natural_index(g, order, p) : 0;
    float m = -INFINITY, l = 0.f;  // pass 1: this half's running max and sum
    float m_row = 0.f, inv_l = 0.f;  // pass 2: the row's softmax
    if (kBlockStats && row_ok) {
      m_row = __ldg(row_max + tok);
      inv_l = 1.f / __ldg(row_sum + tok);
    }
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      const int b = j & 1;
      if (!warp_wait(bar(BS0 + b), (j >> 1) & 1, ctl)) { ok = false; break; }
      tc_fence_after();
      uint32_t sr[64];
      tmem_ld64(lane_addr + b * 128 + hc * 64, sr);
      tc_fence_before();
      mbar_arrive(bar(BSF0 + b));
      const int valid = min(64, g.N - j * kBlock - hc * 64);  // may be <= 0
      // full 64-column halves take an unpredicated loop with four partial
      // accumulators (short dependency chains); only the tail tile masks
      if (!kBlockStats) {
        float mt = -INFINITY;
        if (valid >= 64) {
          float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int c = 0; c < 64; ++c) m4[c & 3] = fmaxf(m4[c & 3], __uint_as_float(sr[c]));
          mt = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * scale_log2;
        } else {
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (c < valid) mt = fmaxf(mt, __uint_as_float(sr[c]) * scale_log2);
        }
        const float m_new = fmaxf(m, mt);
        if (m_new != -INFINITY) {
          float acc = 0.f;
          if (valid >= 64) {
            // two columns per paired f32x2 FMA and add
            const float2 sc2 = make_float2(scale_log2, scale_log2), nm2 = make_float2(-m_new, -m_new);
            float2 a2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
            for (int c = 0; c < 64; c += 2) {
              const float2 t = ffma2(make_float2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])),
                                     sc2, nm2);
              a2[(c >> 1) & 1] = fadd2(a2[(c >> 1) & 1], make_float2(ex2(t.x), ex2(t.y)));
            }
            acc = (a2[0].x + a2[0].y) + (a2[1].x + a2[1].y);
          } else {
#pragma unroll
            for (int c = 0; c < 64; ++c)
              if (c < valid) acc += ex2(fmaf(__uint_as_float(sr[c]), scale_log2, -m_new));
          }
          l = (m == -INFINITY ? 0.f : l * ex2(m - m_new)) + acc;
          m = m_new;
        }
      } else {
        float cnt = 0.f, sum = 0.f, mx = 0.f;
        if (row_ok && valid >= 64) {
          // two columns per paired f32x2 FMA, multiply and add
          const float2 sc2 = make_float2(scale_log2, scale_log2), nm2 = make_float2(-m_row, -m_row);
          const float2 il2 = make_float2(inv_l, inv_l);
          float2 c2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
          float2 s2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
          float x4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int c = 0; c < 64; c += 2) {
            const float2 t = ffma2(make_float2(__uint_as_float(sr[c]), __uint_as_float(sr[c + 1])),
                                   sc2, nm2);
            const float2 pv = fmul2(make_float2(ex2(t.x), ex2(t.y)), il2);
            const int u = (c >> 1) & 1;
            c2[u] = fadd2(c2[u], make_float2(pv.x < eps ? 1.f : 0.f, pv.y < eps ? 1.f : 0.f));
            s2[u] = fadd2(s2[u], pv);
            x4[2 * u] = fmaxf(x4[2 * u], pv.x);
            x4[2 * u + 1] = fmaxf(x4[2 * u + 1], pv.y);
          }
          cnt = (c2[0].x + c2[0].y) + (c2[1].x + c2[1].y);
          sum = (s2[0].x + s2[0].y) + (s2[1].x + s2[1].y);
          mx = fmaxf(fmaxf(x4[0], x4[1]), fmaxf(x4[2], x4[3]));
        } else if (row_ok) {
#pragma unroll
          for (int c = 0; c < 64; ++c) {
            if (c < valid) {
              const float pv = ex2(fmaf(__uint_as_float(sr[c]), scale_log2, -m_row)) * inv_l;
              cnt += pv < eps ? 1.f : 0.f;
              sum += pv;
              mx = fmaxf(mx, pv);
            }
          }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
          sum += __shfl_xor_sync(0xffffffffu, sum, o);
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        }
        if (lane == 0) {
          const int64_t t = (bh * nb + i) * (int64_t)nb + j;
          atomicAdd(count + t, cnt);
          atomicAdd(total + t, sum);
          atomicMax(reinterpret_cast<unsigned int*>(peak + t), __float_as_uint(mx));
        }
      }
    }
    if (!kBlockStats && ok && n_tiles > 0) {
      // merge the two halves of the row: l = l0 2^(m0 - m) + l1 2^(m1 - m)
      merge[(hc * 2 + 0) * 128 + r] = m;
      merge[(hc * 2 + 1) * 128 + r] = l;
      mbar_arrive(bar(BM));
      if (all_wait(bar(BM), 0, ctl) && hc == 0 && row_ok) {
        const float m1 = merge[(2 + 0) * 128 + r], l1 = merge[(2 + 1) * 128 + r];
        const float mm = fmaxf(m, m1);
        const float lt = (m == -INFINITY ? 0.f : l * ex2(m - mm)) +
                         (m1 == -INFINITY ? 0.f : l1 * ex2(m1 - mm));
        row_max[tok] = mm;
        row_sum[tok] = lt;
      }
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// log of the block sums (-inf for an empty block): the scores whose Top-P
// set is the block-sum thresholding of the static mask
__global__ void log_kernel(const float* __restrict__ total, float* __restrict__ log_total,
                           int64_t n) {
  for (int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; t < n;
       t += (int64_t)gridDim.x * blockDim.x)
    log_total[t] = logf(total[t]);
}

// Per (b, h): the fraction of blocks with count >= rho * size and the mean
// over blocks of positive mean of max / mean, for one order.
__global__ void metric_kernel(const float* __restrict__ count, const float* __restrict__ total,
                              const float* __restrict__ peak, const __grid_constant__ Grid g,
                              int order, float rho, float* __restrict__ sparse_frac,
                              float* __restrict__ incoh) {
  const int64_t bh = blockIdx.x;
  const int nb = g.NB;
  float sp = 0.f, inc = 0.f, pos = 0.f;
  for (int64_t t = threadIdx.x; t < (int64_t)nb * nb; t += blockDim.x) {
    const int i = (int)(t / nb), j = (int)(t % nb);
    const float rows = (float)min(g.block, g.N - i * g.block);
    const float cols = (float)min(g.block, g.N - j * g.block);
    const float size = rows * cols;
    const int64_t a = bh * (int64_t)nb * nb + t;
    sp += count[a] >= rho * size ? 1.f : 0.f;
    const float mean = total[a] / size;
    if (mean > 0.f) {
      inc += peak[a] / mean;
      pos += 1.f;
    }
  }
  __shared__ float red[3][32];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    sp += __shfl_xor_sync(0xffffffffu, sp, o);
    inc += __shfl_xor_sync(0xffffffffu, inc, o);
    pos += __shfl_xor_sync(0xffffffffu, pos, o);
  }
  if (lane == 0) {
    red[0][w] = sp;
    red[1][w] = inc;
    red[2][w] = pos;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float a = 0.f, b = 0.f, c = 0.f;
    for (int u = 0; u < (int)(blockDim.x >> 5); ++u) {
      a += red[0][u];
      b += red[1][u];
      c += red[2][u];
    }
    sparse_frac[bh * 6 + order] = a / ((float)nb * nb);
    incoh[bh * 6 + order] = c > 0.f ? b / c : 0.f;
  }
}

// Per (b, h): M[o] = alpha (1 - sf[o]) / max_o(1 - sf) + (1 - alpha) inc[o] /
// max_o inc (a term that is 0 for every order adds 0); the order is the
// argmin, ties to the lower id.
__global__ void choose_kernel(const float* __restrict__ sparse_frac,
                              const float* __restrict__ incoh, int64_t rows, float alpha,
                              float* __restrict__ metric, int8_t* __restrict__ orders) {
  const int64_t bh = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (bh >= rows) return;
  float dmax = 0.f, imax = 0.f;
  for (int o = 0; o < 6; ++o) {
    dmax = fmaxf(dmax, 1.f - sparse_frac[bh * 6 + o]);
    imax = fmaxf(imax, incoh[bh * 6 + o]);
  }
  int best = 0;
  float best_m = INFINITY;
  for (int o = 0; o < 6; ++o) {
    const float dn = dmax > 0.f ? (1.f - sparse_frac[bh * 6 + o]) / dmax : 0.f;
    const float in = imax > 0.f ? incoh[bh * 6 + o] / imax : 0.f;
    const float mo = alpha * dn + (1.f - alpha) * in;
    metric[bh * 6 + o] = mo;
    if (mo < best_m) {
      best_m = mo;
      best = o;
    }
  }
  orders[bh] = (int8_t)best;
}

}  // namespace

cudaError_t launch_map_stats(const void* qp, const void* kp, const Grid& g, int order,
                             bool block_stats, float* row_max, float* row_sum, float eps,
                             float* count, float* total, float* peak, int32_t* status,
                             cudaStream_t s) {
  if (g.d != kD || g.block != kBlock) return cudaErrorInvalidValue;
  const uint64_t rows = (uint64_t)g.B * g.heads * g.Np;
  CUtensorMap mq{}, mk{};
  if (!encode_tile_map(&mq, qp, rows, kD, 2, 64, kBlock) ||
      !encode_tile_map(&mk, kp, rows, kD, 2, 64, kBlock))
    return cudaErrorInvalidValue;
  const float c = (float)(1.4426950408889634 / sqrt((double)kD));
  dim3 grid(g.NB, g.B * g.heads);
  cudaError_t e;
  if (block_stats) {
    e = cudaFuncSetAttribute(map_stats_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    map_stats_kernel<true><<<grid, kThreads, kSmemBytes, s>>>(mq, mk, g, order, c, row_max,
                                                              row_sum, eps, count, total, peak,
                                                              status);
  } else {
    e = cudaFuncSetAttribute(map_stats_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    map_stats_kernel<false><<<grid, kThreads, kSmemBytes, s>>>(mq, mk, g, order, c, row_max,
                                                               row_sum, eps, count, total, peak,
                                                               status);
  }
  return cudaGetLastError();
}

cudaError_t launch_log_total(const float* total, float* log_total, int64_t n, cudaStream_t s) {
  const int64_t blocks = (n + 255) / 256;
  log_kernel<<<(unsigned)(blocks < 148 * 8 ? blocks : 148 * 8), 256, 0, s>>>(total, log_total, n);
  return cudaGetLastError();
}

cudaError_t launch_paro_metric(const float* count, const float* total, const float* peak,
                               const Grid& g, int order, float rho, float* sparse_frac,
                               float* incoh, cudaStream_t s) {
  metric_kernel<<<g.B * g.heads, 256, 0, s>>>(count, total, peak, g, order, rho, sparse_frac,
                                              incoh);
  return cudaGetLastError();
}

cudaError_t launch_paro_choose(const float* sparse_frac, const float* incoh, int64_t rows,
                               float alpha, float* metric, int8_t* orders, cudaStream_t s) {
  choose_kernel<<<(unsigned)((rows + 127) / 128), 128, 0, s>>>(sparse_frac, incoh, rows, alpha,
                                                               metric, orders);
  return cudaGetLastError();
}

}  // namespace paro
