// HBM-bound kernels of the path: the standalone reorder and inverse reorder,
// block mean-pooling, pooled block scores, top-k block selection, bitmask
// compaction and per-block INT8 quantisation.
//
// Every token row is d * sizeof(T) contiguous bytes (128 or 256 here), so
// any per-head axis order is read and written with whole 16-byte vectors:
// a row is moved by d*sizeof(T)/16 consecutive lanes, fully coalesced at row
// granularity whatever the order.
#include "common.cuh"

namespace paro {
namespace {

constexpr int kThreads = 256;

// ------------------------------------------------------------ reorder ----
// Forward: one thread per 16-byte chunk of an output row of the permuted
// sequence [B*heads, Np, d] (pad rows -> zeros).  Inverse: one thread per
// chunk of an output row of the natural sequence [B*heads, N, d], gathering
// from the permuted row at pos(n) -- equivalently scattering; we walk the
// permuted positions p < N so both directions share the index map, and
// write to the natural row.
__global__ void __launch_bounds__(kThreads) reorder_kernel(const uint4* __restrict__ src,
                                                           uint4* __restrict__ dst, const __grid_constant__ Grid g,
                                                           int vpr, int inverse) {
  const int64_t rows = (int64_t)g.B * g.heads * (inverse ? g.N : g.Np);
  const int64_t total = rows * vpr;
  for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < total;
       t += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = t / vpr;
    const int c = (int)(t - row * vpr);
    const int per = inverse ? g.N : g.Np;
    const int64_t bh = row / per;
    const int p = (int)(row - bh * per);
    const int h = (int)(bh % g.heads);
    if (!inverse) {
      uint4 v = make_uint4(0, 0, 0, 0);
      if (p < g.N) {
        const int n = natural_index(g, g.perm[h], p);
        v = __ldg(src + ((bh * g.N + n) * vpr + c));
      }
      dst[(bh * g.Np + p) * vpr + c] = v;
    } else {
      const int n = natural_index(g, g.perm[h], p);
      dst[(bh * g.N + n) * vpr + c] = __ldg(src + ((bh * g.Np + p) * vpr + c));
    }
  }
}

// ------------------------------------------------- pooling and reorder ---
// One CTA per (permuted block i, head bh).  Reads the block's token rows
// once (natural positions from the head's order); optionally writes them
// contiguously to the permuted tensor xp (pad rows as zeros) and/or the
// fp32 mean of the block's valid rows to pool.  Thread t owns chunk
// (t % vpr) of rows t / vpr, + kThreads/vpr, ...
template <typename T>
__global__ void __launch_bounds__(kThreads) pool_kernel(const T* __restrict__ x, const __grid_constant__ Grid g,
                                                        float* __restrict__ pool,
                                                        T* __restrict__ xp) {
  constexpr int E = Chunk<T>::n;
  extern __shared__ float red[];  // [groups][d]
  const int vpr = g.d / E;
  const int groups = kThreads / vpr;
  const int i = blockIdx.x;
  const int64_t bh = blockIdx.y;
  const int h = (int)(bh % g.heads);
  const int order = g.perm[h];
  const int c = threadIdx.x % vpr;
  const int rg = threadIdx.x / vpr;
  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
  const int p0 = i * g.block;
  const int valid = min(g.block, g.N - p0);
  const uint4* base = reinterpret_cast<const uint4*>(x + bh * (int64_t)g.N * g.d);
  uint4* dst = xp != nullptr
                   ? reinterpret_cast<uint4*>(xp + (bh * (int64_t)g.Np + p0) * g.d)
                   : nullptr;
  const int rows = dst != nullptr ? g.block : valid;
  for (int r = rg; r < rows; r += groups) {
    uint4 u = make_uint4(0, 0, 0, 0);
    if (r < valid) u = __ldg(base + (int64_t)natural_index(g, order, p0 + r) * vpr + c);
    if (dst != nullptr) dst[(int64_t)r * vpr + c] = u;
    if (pool != nullptr) {
      float f[E];
      Chunk<T>::unpack(u, f);
#pragma unroll
      for (int e = 0; e < E; ++e) acc[e] += f[e];
    }
  }
  if (pool == nullptr) return;  // uniform across the CTA
#pragma unroll
  for (int e = 0; e < E; ++e) red[rg * g.d + c * E + e] = acc[e];
  __syncthreads();
  for (int col = threadIdx.x; col < g.d; col += kThreads) {
    float s = 0.f;
    for (int r = 0; r < groups; ++r) s += red[r * g.d + col];
    pool[(bh * g.NB + i) * g.d + col] = s / (float)valid;
  }
}

// The same for sizes fixed at compile time (bf16, d = 128, block = 128, the
// tcgen05 path's shape): each thread issues all its rows' loads before the
// first store, so the CTA keeps its whole block in flight; the sums and the
// outputs are the same, bit for bit (rows accumulated in the same order).
template <typename T, int D, int BLOCK>
__global__ void __launch_bounds__(kThreads) pool_kernel_fixed(const T* __restrict__ x,
                                                              const __grid_constant__ Grid g,
                                                              float* __restrict__ pool,
                                                              T* __restrict__ xp) {
  constexpr int E = Chunk<T>::n;
  constexpr int VPR = D / E;
  constexpr int GROUPS = kThreads / VPR;
  constexpr int RPT = BLOCK / GROUPS;
  __shared__ float red[GROUPS][D];
  const int i = blockIdx.x;
  const int64_t bh = blockIdx.y;
  const int h = (int)(bh % g.heads);
  const int order = g.perm[h];
  const int c = threadIdx.x % VPR;
  const int rg = threadIdx.x / VPR;
  const int p0 = i * BLOCK;
  const int valid = min(BLOCK, g.N - p0);
  const uint4* base = reinterpret_cast<const uint4*>(x + bh * (int64_t)g.N * D);
  uint4 u[RPT];
#pragma unroll
  for (int k = 0; k < RPT; ++k) {
    const int r = rg + k * GROUPS;
    u[k] = r < valid ? __ldg(base + (int64_t)natural_index(g, order, p0 + r) * VPR + c)
                     : make_uint4(0, 0, 0, 0);
  }
  if (xp != nullptr) {
    uint4* dst = reinterpret_cast<uint4*>(xp + (bh * (int64_t)g.Np + p0) * D);
#pragma unroll
    for (int k = 0; k < RPT; ++k) dst[(int64_t)(rg + k * GROUPS) * VPR + c] = u[k];
  }
  if (pool == nullptr) return;  // uniform across the CTA
  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
#pragma unroll
  for (int k = 0; k < RPT; ++k) {
    if (xp == nullptr && rg + k * GROUPS >= valid) break;  // as the generic loop's bound
    float f[E];
    Chunk<T>::unpack(u[k], f);
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] += f[e];
  }
#pragma unroll
  for (int e = 0; e < E; ++e) red[rg][c * E + e] = acc[e];
  __syncthreads();
  for (int col = threadIdx.x; col < D; col += kThreads) {
    float sum = 0.f;
    for (int r = 0; r < GROUPS; ++r) sum += red[r][col];
    pool[(bh * g.NB + i) * D + col] = sum / (float)valid;
  }
}

// --------------------------------------------------------------- scores ---
// S[bh, i, j] = dot(qp[bh, i], kp[bh, j]) * inv_sqrt_d, fp32 SIMT tiles of
// 64 x 64 (the whole matrix is < 0.1% of the attention FLOPs).
constexpr int ST = 64, SK = 32;
__global__ void __launch_bounds__(kThreads) score_kernel(const float* __restrict__ qp,
                                                         const float* __restrict__ kp, const __grid_constant__ Grid g,
                                                         float inv_sqrt_d,
                                                         float* __restrict__ out) {
  __shared__ float As[SK][ST + 4];
  __shared__ float Bs[SK][ST + 4];
  const int64_t bh = blockIdx.z;
  const int i0 = blockIdx.y * ST, j0 = blockIdx.x * ST;
  const float* A = qp + bh * (int64_t)g.NB * g.d;
  const float* Bm = kp + bh * (int64_t)g.NB * g.d;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < g.d; k0 += SK) {
    for (int e = threadIdx.x; e < ST * SK; e += kThreads) {
      const int r = e / SK, kk = e % SK;
      As[kk][r] = (i0 + r < g.NB) ? A[(int64_t)(i0 + r) * g.d + k0 + kk] : 0.f;
      Bs[kk][r] = (j0 + r < g.NB) ? Bm[(int64_t)(j0 + r) * g.d + k0 + kk] : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < SK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        a[u] = As[kk][ty * 4 + u];
        b[u] = Bs[kk][tx * 4 + u];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int w = 0; w < 4; ++w) acc[u][w] = fmaf(a[u], b[w], acc[u][w]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int i = i0 + ty * 4 + u;
    if (i >= g.NB) continue;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const int j = j0 + tx * 4 + w;
      if (j < g.NB) out[(bh * g.NB + i) * g.NB + j] = acc[u][w] * inv_sqrt_d;
    }
  }
}

// ----------------------------------------------------------------- top-k --
// Order-preserving map of a score to 32 bits: NaN -> -inf, -0 -> +0, the
// diagonal -> above every finite or infinite score.  With the block index as
// the tie-break (lower index first) every key of a row is distinct, so the
// selection is exact and unique.
__device__ __forceinline__ uint32_t score_key(float f, bool diag) {
  if (diag) return 0xFFFFFFFFu;
  uint32_t b = __float_as_uint(f);
  if (f != f) b = 0xFF800000u;  // NaN -> -inf
  if (b == 0x80000000u) b = 0u;  // -0 -> +0
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}


// One warp per row (bh, i).  Phase 1 finds, bit by bit from the top, the
// 32-bit key t of the k-th largest key (counting multiplicity).  Every key
// above t is kept; of the keys equal to t the r = k - #{key > t} lowest
// indices are kept.  Phase 2 walks the row in ascending index order and
// writes the kept indices with ballots, so the output is ascending.
__global__ void __launch_bounds__(kTopkWarps * 32) topk_kernel(const float* __restrict__ scores,
                                                               const __grid_constant__ Grid g, int k,
                                                               int32_t* __restrict__ idx) {
  extern __shared__ uint32_t keys[];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t row = (int64_t)blockIdx.x * kTopkWarps + warp;
  const int64_t rows = (int64_t)g.B * g.heads * g.NB;
  if (row >= rows) return;
  const int nb = g.NB;
  const int i = (int)(row % nb);
  uint32_t* key = keys + warp * nb;
  const float* s = scores + row * nb;
  for (int j = lane; j < nb; j += 32) key[j] = score_key(__ldg(s + j), j == i);
  __syncwarp();
  uint32_t t = 0;
  for (int bit = 31; bit >= 0; --bit) {
    const uint32_t cand = t | (1u << bit);
    int cnt = 0;
    for (int j = lane; j < nb; j += 32) cnt += key[j] >= cand;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) cnt += __shfl_xor_sync(0xffffffffu, cnt, o);
    if (cnt >= k) t = cand;
  }
  int above = 0;
  for (int j = lane; j < nb; j += 32) above += key[j] > t;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) above += __shfl_xor_sync(0xffffffffu, above, o);
  const int r = k - above;  // ties at t still to take, lowest index first
  int written = 0, ties = 0;
  int32_t* out = idx + row * k;
  for (int j0 = 0; j0 < nb; j0 += 32) {
    const int j = j0 + lane;
    const uint32_t kj = j < nb ? key[j] : 0u;
    const bool tie = j < nb && kj == t;
    const unsigned tmask = __ballot_sync(0xffffffffu, tie);
    const int tie_rank = ties + __popc(tmask & ((1u << lane) - 1u));
    const bool sel = j < nb && (kj > t || (tie && tie_rank < r));
    const unsigned smask = __ballot_sync(0xffffffffu, sel);
    if (sel) out[written + __popc(smask & ((1u << lane) - 1u))] = j;
    written += __popc(smask);
    ties += __popc(tmask);
  }
}

// ------------------------------------------------------ mask compaction ---
__global__ void __launch_bounds__(kTopkWarps * 32) compact_kernel(const uint32_t* __restrict__ bm,
                                                                  const __grid_constant__ Grid g,
                                                                  int32_t* __restrict__ idx,
                                                                  int32_t* __restrict__ counts) {
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t row = (int64_t)blockIdx.x * kTopkWarps + warp;
  const int64_t rows = (int64_t)g.B * g.heads * g.NB;
  if (row >= rows) return;
  const int nb = g.NB, words = (nb + 31) / 32;
  const uint32_t* w = bm + row * words;
  int32_t* out = idx + row * nb;
  int written = 0;
  for (int c = 0; c < words; ++c) {
    const int j = c * 32 + lane;
    const bool sel = j < nb && ((__ldg(w + c) >> lane) & 1u);
    const unsigned m = __ballot_sync(0xffffffffu, sel);
    if (sel) out[written + __popc(m & ((1u << lane) - 1u))] = j;
    written += __popc(m);
  }
  for (int j = written + lane; j < nb; j += 32) out[j] = -1;
  if (lane == 0) counts[row] = written;
}

// ---------------------------------------------------- INT8 quantisation ---
// One CTA per (permuted block i, head bh).  The block stays in registers
// between the absmax pass and the code pass, so x is read once; the block
// mean (for the pooled scores) comes from the same registers.
template <typename T, int D, int BLOCK>
__global__ void __launch_bounds__(kThreads) quant_kernel(const T* __restrict__ x, const __grid_constant__ Grid g,
                                                         int8_t* __restrict__ xq,
                                                         float* __restrict__ scales,
                                                         float* __restrict__ pool, int qmax) {
  constexpr int E = Chunk<T>::n;
  constexpr int VPR = D / E;
  constexpr int GROUPS = kThreads / VPR;
  constexpr int RPT = BLOCK / GROUPS;  // rows per thread
  __shared__ float red[kThreads / 32];
  __shared__ float psum[GROUPS][D];
  const int i = blockIdx.x;
  const int64_t bh = blockIdx.y;
  const int h = (int)(bh % g.heads);
  const int order = g.perm[h];
  const int c = threadIdx.x % VPR;
  const int rg = threadIdx.x / VPR;
  const int p0 = i * BLOCK;
  const int valid = min(BLOCK, g.N - p0);
  const uint4* base = reinterpret_cast<const uint4*>(x + bh * (int64_t)g.N * g.d);
  // the block's rows stay in registers as loaded (packed: half the
  // registers for bf16, so more CTAs keep loads in flight), unpacked at
  // each use
  uint4 raw[RPT];
#pragma unroll
  for (int u = 0; u < RPT; ++u) {
    const int r = rg + u * GROUPS;
    raw[u] = r < valid ? __ldg(base + (int64_t)natural_index(g, order, p0 + r) * VPR + c)
                       : make_uint4(0, 0, 0, 0);
  }
  float amax = 0.f;
  float acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) acc[e] = 0.f;
#pragma unroll
  for (int u = 0; u < RPT; ++u) {
    float f[E];
    Chunk<T>::unpack(raw[u], f);
#pragma unroll
    for (int e = 0; e < E; ++e) {
      amax = fmaxf(amax, fabsf(f[e]));
      acc[e] += f[e];
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if (threadIdx.x % 32 == 0) red[threadIdx.x / 32] = amax;
  if (pool != nullptr) {
#pragma unroll
    for (int e = 0; e < E; ++e) psum[rg][c * E + e] = acc[e];
  }
  __syncthreads();
  // only the packed rows stay live across the reduction (the compiler may
  // not keep the unpacked values from the first pass)
#pragma unroll
  for (int u = 0; u < RPT; ++u)
    asm volatile("" : "+r"(raw[u].x), "+r"(raw[u].y), "+r"(raw[u].z), "+r"(raw[u].w));
  amax = 0.f;
#pragma unroll
  for (int w = 0; w < kThreads / 32; ++w) amax = fmaxf(amax, red[w]);
  const float qf = (float)qmax;
  const float inv = amax > 0.f ? __fdiv_rn(qf, amax) : 0.f;
  // code = rint_half_even(fl32(x * inv)): the product rounded to fp32 first
  // (the reading), then added to 1.5 * 2^23, which rounds it to the nearest
  // integer, ties to even (|x * inv| <= qmax < 2^22), held in the low bits
  constexpr float kMagic = 12582912.0f;
  constexpr int32_t kMagicBits = 0x4B400000;
  int8_t* outb = xq + (bh * (int64_t)g.Np + p0) * D;
#pragma unroll
  for (int u = 0; u < RPT; ++u) {
    const int r = rg + u * GROUPS;
    float f[E];
    Chunk<T>::unpack(raw[u], f);
    uint32_t packed[E / 4];
#pragma unroll
    for (int e4 = 0; e4 < E / 4; ++e4) {
      uint32_t wv = 0;
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const float t = __fmul_rn(f[e4 * 4 + b], inv);
        int qv = (int32_t)__float_as_uint(__fadd_rn(t, kMagic)) - kMagicBits;
        qv = max(-qmax, min(qmax, qv));
        wv |= (uint32_t)(qv & 0xFF) << (8 * b);
      }
      packed[e4] = wv;
    }
    int8_t* dst = outb + (int64_t)r * D + c * E;
    if constexpr (E == 8) {
      *reinterpret_cast<uint2*>(dst) = make_uint2(packed[0], packed[1]);
    } else {
      *reinterpret_cast<uint32_t*>(dst) = packed[0];
    }
  }
  if (threadIdx.x == 0) scales[bh * g.NB + i] = amax > 0.f ? __fdiv_rn(amax, qf) : 0.f;
  if (pool != nullptr) {
    for (int col = threadIdx.x; col < D; col += kThreads) {
      float s = 0.f;
      for (int r = 0; r < GROUPS; ++r) s += psum[r][col];
      pool[(bh * g.NB + i) * D + col] = s / (float)valid;
    }
  }
}

int grid_for(int64_t work, int threads) {
  const int64_t b = (work + threads - 1) / threads;
  return (int)(b < 148 * 64 ? (b < 1 ? 1 : b) : 148 * 64);
}

}  // namespace

cudaError_t launch_reorder(const void* x, void* xp, pa_dtype dt, const Grid& g, bool inverse,
                           cudaStream_t s) {
  const int es = dt == PA_F32 ? 4 : 2;
  const int vpr = g.d * es / 16;
  const int64_t rows = (int64_t)g.B * g.heads * (inverse ? g.N : g.Np);
  reorder_kernel<<<grid_for(rows * vpr, kThreads), kThreads, 0, s>>>(
      reinterpret_cast<const uint4*>(x), reinterpret_cast<uint4*>(xp), g, vpr, inverse ? 1 : 0);
  return cudaGetLastError();
}

cudaError_t launch_reorder_pool(const void* x, void* xp, pa_dtype dt, const Grid& g, float* pool,
                                cudaStream_t s) {
  const int E = dt == PA_F32 ? 4 : 8;
  const int groups = kThreads / (g.d / E);
  const size_t smem = (size_t)groups * g.d * sizeof(float);
  dim3 grid(g.NB, g.B * g.heads);
  if (dt == PA_BF16 && g.d == 128 && g.block == 128)
    pool_kernel_fixed<__nv_bfloat16, 128, 128><<<grid, kThreads, 0, s>>>(
        static_cast<const __nv_bfloat16*>(x), g, pool, static_cast<__nv_bfloat16*>(xp));
  else if (dt == PA_F32)
    pool_kernel<float><<<grid, kThreads, smem, s>>>(static_cast<const float*>(x), g, pool,
                                                    static_cast<float*>(xp));
  else
    pool_kernel<__nv_bfloat16><<<grid, kThreads, smem, s>>>(
        static_cast<const __nv_bfloat16*>(x), g, pool, static_cast<__nv_bfloat16*>(xp));
  return cudaGetLastError();
}

cudaError_t launch_pool(const void* x, pa_dtype dt, const Grid& g, float* pool, cudaStream_t s) {
  return launch_reorder_pool(x, nullptr, dt, g, pool, s);
}

cudaError_t launch_score(const float* qp, const float* kp, const Grid& g, float* scores,
                         cudaStream_t s) {
  dim3 grid((g.NB + ST - 1) / ST, (g.NB + ST - 1) / ST, g.B * g.heads);
  const float inv_sqrt_d = (float)(1.0 / sqrt((double)g.d));
  score_kernel<<<grid, kThreads, 0, s>>>(qp, kp, g, inv_sqrt_d, scores);
  return cudaGetLastError();
}

cudaError_t launch_topk(const float* scores, const Grid& g, int k, int32_t* idx, cudaStream_t s) {
  const int64_t rows = (int64_t)g.B * g.heads * g.NB;
  const size_t smem = (size_t)kTopkWarps * g.NB * sizeof(uint32_t);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
  }
  topk_kernel<<<(unsigned)((rows + kTopkWarps - 1) / kTopkWarps), kTopkWarps * 32, smem, s>>>(
      scores, g, k, idx);
  return cudaGetLastError();
}

cudaError_t launch_compact(const uint32_t* bm, const Grid& g, int32_t* idx, int32_t* counts,
                           cudaStream_t s) {
  const int64_t rows = (int64_t)g.B * g.heads * g.NB;
  compact_kernel<<<(unsigned)((rows + kTopkWarps - 1) / kTopkWarps), kTopkWarps * 32, 0, s>>>(
      bm, g, idx, counts);
  return cudaGetLastError();
}

template <typename T, int D, int BLOCK>
static void quant_launch(const void* x, const Grid& g, int8_t* xq, float* sc, float* pool,
                         int qmax, cudaStream_t s) {
  dim3 grid(g.NB, g.B * g.heads);
  quant_kernel<T, D, BLOCK><<<grid, kThreads, 0, s>>>(static_cast<const T*>(x), g, xq, sc, pool,
                                                      qmax);
}

cudaError_t launch_quantize(const void* x, pa_dtype dt, const Grid& g, int8_t* xq, float* scales,
                            float* pool, int qmax, cudaStream_t s) {
  const bool bf = dt == PA_BF16;
#define PARO_Q(D, BL)                                                        \
  if (g.d == D && g.block == BL) {                                           \
    if (bf)                                                                  \
      quant_launch<__nv_bfloat16, D, BL>(x, g, xq, scales, pool, qmax, s);   \
    else                                                                     \
      quant_launch<float, D, BL>(x, g, xq, scales, pool, qmax, s);           \
    return cudaGetLastError();                                               \
  }
  PARO_Q(64, 64)
  PARO_Q(64, 128)
  PARO_Q(128, 64)
  PARO_Q(128, 128)
#undef PARO_Q
  return cudaErrorInvalidValue;
}

namespace {
// y[i] = x[i] rounded to bf16 (round-to-nearest-even), 8 elements per thread.
__global__ void round_bf16_kernel(const float* __restrict__ x, __nv_bfloat16* __restrict__ y,
                                  int64_t n) {
  const int64_t i0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) * 8;
  if (i0 + 8 <= n) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(x + i0));
    const float4 b = __ldg(reinterpret_cast<const float4*>(x + i0) + 1);
    uint4 w;
    __nv_bfloat162 t;
    t = __floats2bfloat162_rn(a.x, a.y); w.x = *reinterpret_cast<uint32_t*>(&t);
    t = __floats2bfloat162_rn(a.z, a.w); w.y = *reinterpret_cast<uint32_t*>(&t);
    t = __floats2bfloat162_rn(b.x, b.y); w.z = *reinterpret_cast<uint32_t*>(&t);
    t = __floats2bfloat162_rn(b.z, b.w); w.w = *reinterpret_cast<uint32_t*>(&t);
    *reinterpret_cast<uint4*>(y + i0) = w;
  } else {
    for (int64_t i = i0; i < n; ++i) y[i] = __float2bfloat16_rn(x[i]);
  }
}
}  // namespace

cudaError_t launch_round_bf16(const float* x, void* y, int64_t n, cudaStream_t s) {
  const int64_t threads = (n + 7) / 8;
  const unsigned blocks = (unsigned)((threads + 255) / 256);
  round_bf16_kernel<<<blocks, 256, 0, s>>>(x, static_cast<__nv_bfloat16*>(y), n);
  return cudaGetLastError();
}

}  // namespace paro
