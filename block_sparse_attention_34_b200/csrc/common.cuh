// Shared device-side definitions of libparo: the grid/order description every
// kernel receives by value, the position -> natural-token map of a head's
// axis order, and the device status word.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "paro.h"

namespace paro {

constexpr int kMaxHeads = 1024;

// Top-k selection: warps per CTA, each holding one row of NB 32-bit keys in
// shared memory, so NB is bounded by the opt-in shared memory per CTA.
constexpr int kTopkWarps = 4;
constexpr int kSmemOptIn = 232448;  // bytes of shared memory a CTA may opt into
constexpr int kTopkMaxNB = kSmemOptIn / (kTopkWarps * 4);  // 14528

// Token orders: ids 0-5 are the six axis orders of [F, H, W] (PAROAttention
// review), ids 6-11 SPADE's 3D tile blockings (SPADE review,
// key_machinery (i): spatial, temporal and mixed blocking candidates): tiles
// of tf x th x tw tokens (tf*th*tw = the block size), tiles in (f, h, w)
// order, tokens inside a tile in (f, h, w) order, partial tiles at the far
// edges of a grid the tile does not divide.
constexpr int kAxisOrders = 6;
constexpr int kOrders = 12;

// Sizes of one call plus the per-order index tables.  For an axis order o
// (letters outer -> inner) a permuted position p decomposes as p = (c_out *
// mid[o] + c_mid) * inn[o] + c_in, and the token's natural index is
// c_out*so[o] + c_mid*sm[o] + c_in*si[o] (natural strides: F -> H*W, H -> W,
// W -> 1).  Tile order 6 + t has the tile shape (tf[t], th[t], tw[t]).
struct Grid {
  int32_t B, heads, F, H, W, d, block;
  int32_t N, NB, Np;
  int32_t mid[6], inn[6], so[6], sm[6], si[6];
  int32_t tf[6], th[6], tw[6];
  int8_t perm[kMaxHeads];
};

// Test hook of the bounded waits (pa_test_inject_v_stall): the V-tile
// loader of CTA (cta_x, cta_y) of the tcgen05 bf16 attention kernel skips
// kept tile `tile` (no copy, no arrival), and every bounded wait of that
// kernel gives up after limit_ns.  tile < 0: off (limit 1 s).
struct StallTest {
  int32_t cta_x, cta_y, tile, pad;
  uint64_t limit_ns;
};
StallTest stall_test();  // host: the current setting

__device__ __forceinline__ int natural_index(const Grid& g, int order, int p) {
  if (order < kAxisOrders) {
    const int inn = g.inn[order], mid = g.mid[order];
    const int ci = p % inn;
    const int t = p / inn;
    const int cm = t % mid;
    const int co = t / mid;
    return co * g.so[order] + cm * g.sm[order] + ci * g.si[order];
  }
  // tile-major order: the slab of tile rows a (frames a*tf ..), the row of
  // tiles b (heights b*th ..) inside it, the tile c (widths c*tw ..), then
  // the token inside the (possibly partial) tile
  const int t = order - kAxisOrders;
  const int tf = g.tf[t], th = g.th[t], tw = g.tw[t];
  const int HW = g.H * g.W;
  const int a = p / (tf * HW);
  int rem = p - a * tf * HW;
  const int sf = min(tf, g.F - a * tf);
  const int b = rem / (sf * th * g.W);
  rem -= b * sf * th * g.W;
  const int sh = min(th, g.H - b * th);
  const int c = rem / (sf * sh * tw);
  rem -= c * sf * sh * tw;
  const int sw = min(tw, g.W - c * tw);
  const int f1 = rem / (sh * sw);
  rem -= f1 * sh * sw;
  const int h1 = rem / sw;
  const int w1 = rem - h1 * sw;
  return (a * tf + f1) * HW + (b * th + h1) * g.W + c * tw + w1;
}

// First error wins; never traps.
__device__ __forceinline__ void report(int32_t* status, int code) {
  if (status != nullptr) atomicCAS(status, 0, code);
}

__device__ __forceinline__ float to_float(float x) { return x; }
__device__ __forceinline__ float to_float(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T>
__device__ __forceinline__ T from_float(float x);
template <>
__device__ __forceinline__ float from_float<float>(float x) { return x; }
template <>
__device__ __forceinline__ __nv_bfloat16 from_float<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

// Unpack a 16-byte chunk of T into floats (8 bf16 or 4 f32).
template <typename T>
struct Chunk;
template <>
struct Chunk<__nv_bfloat16> {
  static constexpr int n = 8;
  __device__ static void unpack(const uint4& u, float* f) {
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 t = __bfloat1622float2(h[i]);
      f[2 * i] = t.x;
      f[2 * i + 1] = t.y;
    }
  }
};
template <>
struct Chunk<float> {
  static constexpr int n = 4;
  __device__ static void unpack(const uint4& u, float* f) {
    f[0] = __uint_as_float(u.x);
    f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z);
    f[3] = __uint_as_float(u.w);
  }
};

}  // namespace paro

// Launchers implemented in the kernel files, called by the C ABI layer.
// Each returns cudaGetLastError() of its launch.
namespace paro {
cudaError_t launch_reorder(const void* x, void* xp, pa_dtype dt, const Grid& g, bool inverse,
                           cudaStream_t s);
cudaError_t launch_reorder_pool(const void* x, void* xp, pa_dtype dt, const Grid& g, float* pool,
                                cudaStream_t s);
cudaError_t launch_pool(const void* x, pa_dtype dt, const Grid& g, float* pool, cudaStream_t s);
cudaError_t launch_score(const float* qp, const float* kp, const Grid& g, float* scores,
                         cudaStream_t s);
cudaError_t launch_topk(const float* scores, const Grid& g, int k, int32_t* idx, cudaStream_t s);
cudaError_t launch_compact(const uint32_t* bm, const Grid& g, int32_t* idx, int32_t* counts,
                           cudaStream_t s);
// qmax: 127 for INT8 codes, 7 for 4-bit codes (one per byte)
cudaError_t launch_quantize(const void* x, pa_dtype dt, const Grid& g, int8_t* xq, float* scales,
                            float* pool, int qmax, cudaStream_t s);
// k_pool, v_pool [B*heads, NB, d] float (both or neither): the block means of
// k and v; with them every unselected key block enters as one pooled key
// row of weight n_j (PASA's grouped first-order compensation), NB <= 4096.
cudaError_t launch_attn_mma(const void* q, const void* k, const void* v, pa_dtype dt,
                            const Grid& g, const int32_t* idx, const int32_t* counts, int k_max,
                            void* out, int32_t* status, bool permuted, cudaStream_t s,
                            const float* k_pool = nullptr, const float* v_pool = nullptr);
// Selection variants (select_variants.cu)
cudaError_t launch_sics(const void* x, pa_dtype dt, const Grid& g, float* scores, cudaStream_t s);
cudaError_t launch_sics_pick(const float* scores, const Grid& g, int8_t* orders, cudaStream_t s);
// y[i] = bf16(x[i]) for n floats (x, y 16-byte aligned)
cudaError_t launch_round_bf16(const float* x, void* y, int64_t n, cudaStream_t s);
cudaError_t launch_hybrid(const float* scores, const Grid& g, int k, double p, int w,
                          int32_t* idx, int32_t* counts, cudaStream_t s);
// PAROAttention offline stage (paro_offline.cu)
cudaError_t launch_map_stats(const void* qp, const void* kp, const Grid& g, int order,
                             bool block_stats, float* row_max, float* row_sum, float eps,
                             float* count, float* total, float* peak, int32_t* status,
                             cudaStream_t s);
cudaError_t launch_log_total(const float* total, float* log_total, int64_t n, cudaStream_t s);
cudaError_t launch_paro_metric(const float* count, const float* total, const float* peak,
                               const Grid& g, int order, float rho, float* sparse_frac,
                               float* incoh, cudaStream_t s);
cudaError_t launch_paro_choose(const float* sparse_frac, const float* incoh, int64_t rows,
                               float alpha, float* metric, int8_t* orders, cudaStream_t s);
// INT8 tcgen05 attention (d = 128, block = 128, permuted int8 inputs)
// p_levels: P code levels, 127 (INT8) or 7 (4-bit); p_tile: the two-pass
// form (normalised P, one scale per tile) instead of rne(p_levels * P~)
cudaError_t launch_attn_i8(const void* q, const void* k, const void* v, const Grid& g,
                           const int32_t* idx, const int32_t* counts, int k_max, const float* qs,
                           const float* ks, const float* vs, float p_levels, bool p_tile,
                           void* out, int32_t* status, cudaStream_t s);
}  // namespace paro
