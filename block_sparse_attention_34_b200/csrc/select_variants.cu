// Selection variants of SPADE (arXiv 2608.03335, Pith verdict page):
//
// * sics_kernel — the Sum of Intra-block Cosine Similarities of a blocking
//   (key_machinery (ii); the one-pass form of Eq. (5)): for a block of rows
//   x_t, sum over ordered pairs s != t of cos(x_s, x_t) =
//   |sum_t xh_t|^2 - sum_t |xh_t|^2 with xh = x / |x| (zero rows add nothing).
//   The candidate blockings are the six axis orders of [F, H, W] with the
//   call's block size; one CTA reduces one block of one order of one
//   (batch, head) and adds its value to scores[b, h, order].  Rows are read
//   at their natural positions (no permuted copy), 16 bytes per lane.
//
// * hybrid_kernel — the union of the diagonal block, a local window
//   |i - j| <= w, the Top-K set (diagonal + k-1 largest others, ties to the
//   lower index, NaN as -inf) and the Top-P set (the shortest run of blocks,
//   in decreasing score order, whose softmax weight reaches p of the row's
//   total) for one query-block row (core_discovery: Top-K / Top-P and
//   local-window filters).  One CTA per row: the (score, index) keys are
//   bitonic-sorted in shared memory, the softmax weights exp(s - max) are
//   summed in fp64 in that order, the kept blocks are marked in a bitmask
//   and written out ascending, padded with -1, with the row's count.
#include "common.cuh"

namespace paro {
namespace {

constexpr int kSicsThreads = 128;
static_assert(kSicsThreads >= 128, "one thread per row of a block (block <= 128)");

// Rows are read 16 bytes per lane: a row of d elements takes L = d *
// sizeof(T) / 16 lanes (8 for d=64 bf16, 16 for d=128 bf16, 32 for d=128
// f32), so a warp reads 32 / L rows per load, two loads in flight.  Each
// lane keeps the running sum of its 16-byte slice of xh; |xh|^2 of a row is
// ss / ss (one value per row, no second pass).
template <typename T>
__global__ void __launch_bounds__(kSicsThreads)
    sics_kernel(const T* __restrict__ x, const __grid_constant__ Grid g,
                float* __restrict__ scores) {
  constexpr int kE = 16 / sizeof(T);  // elements per 16-byte slice
  __shared__ float part[kSicsThreads / 32][256];
  __shared__ float diag_part[kSicsThreads / 32];
  __shared__ int nat[kSicsThreads];  // natural row of each of the block's rows, -1 past N
  const int i = blockIdx.x, order = blockIdx.y;
  const int64_t bh = blockIdx.z;
  // one index computation per row (block <= 128 rows), not one per lane
  if ((int)threadIdx.x < g.block) {
    const int p = i * g.block + (int)threadIdx.x;
    nat[threadIdx.x] = p < g.N ? natural_index(g, order, p) : -1;
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int L = g.d * (int)sizeof(T) / 16;  // lanes per row: 4, 8, 16 or 32
  const int rows_per_load = 32 / L;
  const int slot = lane % L, sub = lane / L;  // slice within the row, row within the load
  float acc[kE], dsum = 0.f;
#pragma unroll
  for (int e = 0; e < kE; ++e) acc[e] = 0.f;
  const T* head = x + bh * (int64_t)g.N * g.d;
  const int step = rows_per_load * (kSicsThreads / 32);
  for (int r0 = warp * rows_per_load; r0 < g.block; r0 += 2 * step) {
    uint4 raw[2];
    bool have[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int r = r0 + u * step + sub;
      const int n = r < g.block ? nat[r] : -1;
      have[u] = n >= 0;
      raw[u] = have[u] ? __ldg(reinterpret_cast<const uint4*>(head + (int64_t)n * g.d) + slot)
                       : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      float v[kE];
      Chunk<T>::unpack(raw[u], v);
      float ss = 0.f;
#pragma unroll
      for (int e = 0; e < kE; ++e) ss = fmaf(v[e], v[e], ss);
      for (int o = L >> 1; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      if (have[u] && ss > 0.f) {
        const float inv = rsqrtf(ss);
#pragma unroll
        for (int e = 0; e < kE; ++e) acc[e] = fmaf(v[e], inv, acc[e]);
        if (slot == 0) dsum += ss * inv * inv;
      }
    }
  }
  // fold the rows-per-load groups of the warp (lanes with the same slot)
  for (int o = L; o < 32; o <<= 1) {
#pragma unroll
    for (int e = 0; e < kE; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], o);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) dsum += __shfl_xor_sync(0xffffffffu, dsum, o);
  if (lane < L) {
#pragma unroll
    for (int e = 0; e < kE; ++e) part[warp][slot * kE + e] = acc[e];
  }
  if (lane == 0) diag_part[warp] = dsum;
  __syncthreads();
  if (warp == 0) {
    float sq = 0.f;
    for (int c = lane; c < g.d; c += 32) {
      float t = 0.f;
#pragma unroll
      for (int w = 0; w < kSicsThreads / 32; ++w) t += part[w][c];
      sq = fmaf(t, t, sq);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, o);
    if (lane == 0) {
      float dg = 0.f;
#pragma unroll
      for (int w = 0; w < kSicsThreads / 32; ++w) dg += diag_part[w];
      atomicAdd(scores + bh * kOrders + order, sq - dg);
    }
  }
}

constexpr int kHybThreads = 256;
constexpr int kHybMaxNB = 4096;

// Order-preserving 32-bit key of a score: NaN -> -inf, -0 -> +0.
__device__ __forceinline__ uint32_t sort_key(float f) {
  uint32_t b = __float_as_uint(f);
  if (f != f) b = 0xFF800000u;
  if (b == 0x80000000u) b = 0u;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__global__ void __launch_bounds__(kHybThreads)
    hybrid_kernel(const float* __restrict__ scores, const __grid_constant__ Grid g, int k,
                  double p, int w, int32_t* __restrict__ idx, int32_t* __restrict__ counts) {
  extern __shared__ __align__(16) unsigned char smem[];
  const int nb = g.NB;
  int m = 1;
  while (m < nb) m <<= 1;
  uint64_t* key = reinterpret_cast<uint64_t*>(smem);            // [m]
  double* cum = reinterpret_cast<double*>(key + m);             // [m]
  uint32_t* bits = reinterpret_cast<uint32_t*>(cum + m);        // [ceil(nb/32)]
  __shared__ double chunk_off[kHybThreads];
  __shared__ int s_diag_pos, s_len, s_count;
  const int64_t row = blockIdx.x;
  const int i = (int)(row % nb);
  const float* s = scores + row * nb;
  const int t = threadIdx.x, lane = t & 31, warp = t >> 5;
  const int words = (nb + 31) / 32;

  // (score desc, index asc) as one 64-bit key sorted descending; pads last
  for (int j = t; j < m; j += kHybThreads)
    key[j] = j < nb ? ((uint64_t)sort_key(__ldg(s + j)) << 32) | (uint64_t)(0xFFFFFFFFu - j) : 0ull;
  for (int j = t; j < words; j += kHybThreads) bits[j] = 0u;
  __syncthreads();
  for (int size = 2; size <= m; size <<= 1) {
    for (int stride = size >> 1; stride > 0; stride >>= 1) {
      for (int a = t; a < m; a += kHybThreads) {
        const int b = a ^ stride;
        if (b > a) {
          const bool desc = (a & size) == 0;
          const uint64_t ka = key[a], kb = key[b];
          if (desc ? ka < kb : ka > kb) {
            key[a] = kb;
            key[b] = ka;
          }
        }
      }
      __syncthreads();
    }
  }
  // softmax weights in sorted order (fp64), and their inclusive prefix sum
  const float top = __ldg(s + (0xFFFFFFFFu - (uint32_t)key[0]));
  const bool top_nan = top != top;
  const float mx = top_nan ? -INFINITY : top;
  const int chunk = (m + kHybThreads - 1) / kHybThreads;
  const int lo = t * chunk, hi = min(m, lo + chunk);
  double run = 0.0;
  for (int a = lo; a < hi; ++a) {
    double wgt = 0.0;
    if (a < nb) {
      const int j = (int)(0xFFFFFFFFu - (uint32_t)key[a]);
      const float v = __ldg(s + j);
      if (j == i) s_diag_pos = a;
      if (v == v && mx != -INFINITY)
        wgt = mx == INFINITY ? (v == INFINITY ? 1.0 : 0.0) : exp((double)v - (double)mx);
    }
    run += wgt;
    cum[a] = run;
  }
  // offsets of the threads' runs, chained left to right by one thread, so
  // that cum is non-decreasing and constant across zero weights (the offset
  // of run t+1 is exactly the last prefix value of run t)
  chunk_off[t] = run;
  __syncthreads();
  if (t == 0) {
    double acc = 0.0;
    for (int u = 0; u < kHybThreads; ++u) {
      const double r = chunk_off[u];
      chunk_off[u] = acc;
      acc += r;
    }
  }
  __syncthreads();
  const double off = chunk_off[t];
  for (int a = lo; a < hi; ++a) cum[a] = off + cum[a];
  if (t == 0) {
    s_len = nb;  // first sorted position reaching p * total (nb: none)
    s_count = 0;
  }
  __syncthreads();
  // Top-P length: the first sorted position whose prefix reaches p * total
  const double total = cum[nb - 1];
  const bool use_p = p > 0.0 && mx != -INFINITY;  // the same for every thread
  if (use_p) {
    const double target = p * total;
    int first = nb;
    for (int a = t; a < nb; a += kHybThreads)
      if (cum[a] >= target) first = min(first, a);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) first = min(first, __shfl_xor_sync(0xffffffffu, first, o));
    if (lane == 0) atomicMin(&s_len, first);
  }
  __syncthreads();
  const int len = !use_p ? 0 : (s_len < nb ? s_len + 1 : nb);
  const int dpos = s_diag_pos;
  // mark: diagonal, window, Top-K (diagonal + k-1 best others), Top-P prefix
  for (int a = t; a < nb; a += kHybThreads) {
    const int j = (int)(0xFFFFFFFFu - (uint32_t)key[a]);
    const int rank_other = a - (dpos < a ? 1 : 0);  // rank among non-diagonal blocks
    bool keep = a < len;
    if (k >= 1 && j != i && rank_other < k - 1) keep = true;
    if (w >= 0 && abs(j - i) <= w) keep = true;
    if (j == i) keep = true;
    if (keep) atomicOr(bits + (j >> 5), 1u << (j & 31));
  }
  __syncthreads();
  // ascending compaction: warp 0 walks the words with a running count
  int32_t* out = idx + row * nb;
  if (warp == 0) {
    int base = 0;
    for (int w0 = 0; w0 < words; w0 += 32) {
      const int wi = w0 + lane;
      const uint32_t bw = wi < words ? bits[wi] : 0u;
      const int c = __popc(bw);
      int incl_c = c;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, incl_c, o);
        if (lane >= o) incl_c += y;
      }
      int pos = base + incl_c - c;
      uint32_t rest = bw;
      while (rest) {
        const int bit = __ffs(rest) - 1;
        rest &= rest - 1;
        out[pos++] = wi * 32 + bit;
      }
      base += __shfl_sync(0xffffffffu, incl_c, 31);
    }
    if (lane == 0) s_count = base;
  }
  __syncthreads();
  const int cnt = s_count;
  for (int a = cnt + t; a < nb; a += kHybThreads) out[a] = -1;
  if (t == 0) counts[row] = cnt;
}

// One thread per head: the argmax over the candidates of the head's score
// summed over the batch (a head has one blocking), ties to the lower id.
__global__ void sics_pick_kernel(const float* __restrict__ scores, const __grid_constant__ Grid g,
                                 int8_t* __restrict__ orders) {
  const int h = blockIdx.x * blockDim.x + threadIdx.x;
  if (h >= g.heads) return;
  int best = 0;
  float best_v = -INFINITY;
  for (int o = 0; o < kOrders; ++o) {
    float v = 0.f;
    for (int b = 0; b < g.B; ++b) v += scores[((int64_t)b * g.heads + h) * kOrders + o];
    if (v > best_v) {
      best_v = v;
      best = o;
    }
  }
  orders[h] = (int8_t)best;
}

}  // namespace

cudaError_t launch_sics_pick(const float* scores, const Grid& g, int8_t* orders, cudaStream_t s) {
  sics_pick_kernel<<<(g.heads + 127) / 128, 128, 0, s>>>(scores, g, orders);
  return cudaGetLastError();
}

size_t hybrid_smem_bytes(int nb) {
  int m = 1;
  while (m < nb) m <<= 1;
  return (size_t)m * (sizeof(uint64_t) + sizeof(double)) + (size_t)((nb + 31) / 32) * 4;
}

cudaError_t launch_sics(const void* x, pa_dtype dt, const Grid& g, float* scores,
                        cudaStream_t s) {
  dim3 grid(g.NB, kOrders, g.B * g.heads);
  if (dt == PA_BF16)
    sics_kernel<__nv_bfloat16><<<grid, kSicsThreads, 0, s>>>(
        static_cast<const __nv_bfloat16*>(x), g, scores);
  else
    sics_kernel<float><<<grid, kSicsThreads, 0, s>>>(static_cast<const float*>(x), g, scores);
  return cudaGetLastError();
}

cudaError_t launch_hybrid(const float* scores, const Grid& g, int k, double p, int w,
                          int32_t* idx, int32_t* counts, cudaStream_t s) {
  if (g.NB > kHybMaxNB) return cudaErrorInvalidValue;
  const size_t smem = hybrid_smem_bytes(g.NB);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(hybrid_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
  }
  const int64_t rows = (int64_t)g.B * g.heads * g.NB;
  hybrid_kernel<<<(unsigned)rows, kHybThreads, smem, s>>>(scores, g, k, p, w, idx, counts);
  return cudaGetLastError();
}

}  // namespace paro
