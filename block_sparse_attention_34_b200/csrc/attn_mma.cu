// Block-sparse flash attention on the legacy warp-level tensor-core path
// (mma.sync m16n8k16 bf16 -> fp32).  This is the comparison baseline for the
// tcgen05 kernel and the path for the shapes that kernel does not take
// (block 64, d 64, fp32 inputs).
//
// One CTA per (query block i, head bh), BLOCK/16 warps, 16 query rows per
// warp.  For each kept key block j (ascending, from the compacted index
// list) the K and V tiles are gathered row by row from their natural
// positions -- the head's axis order is applied in the load, so no reordered
// copy of K or V ever exists -- then S = Q K^T, an online softmax in base 2
// with a running row max and sum, and O += P V with P rounded to bf16.  The
// epilogue divides by the row sum and stores each row at its natural
// position (the inverse reorder).
//
// Algorithm: SPADE, arXiv 2608.03335, Pith verdict page, key_machinery
// (iii) (flash block-sparse attention with an online softmax); the mask is
// the additive 0/-inf block mask of its section 2.2, Eq. (2).
//
// With kComp (PASA, arXiv 2604.12219, Pith review page, Figure 2 caption:
// grouped first-order compensation of the unselected key blocks), the same
// online softmax then runs over the head's pooled key blocks as extra key
// rows: key block j enters as its mean key kbar_j with value vbar_j and
// weight n_j (its valid keys), i.e. score q.kbar_j/sqrt(d) + log(n_j) --
// the first-order expansion of exp about the block's mean score, whose
// linear term sums to zero over the block -- for every j that is not in
// the query block's kept list; kept blocks and pad columns get -inf.
#include "common.cuh"

namespace paro {
namespace {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void mma_bf16(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 t = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&t);
}

// Gather `rows` token rows starting at permuted position p0 of one head into
// a bf16 smem tile with row stride LD elements; rows past N become zeros.
template <typename TIn, int D, int LD>
__device__ __forceinline__ void gather_tile(__nv_bfloat16* dst, const TIn* __restrict__ head,
                                            const Grid& g, int order, int p0, int rows,
                                            bool permuted) {
  constexpr int E = 16 / sizeof(TIn);
  constexpr int VPR = D / E;
  for (int e = threadIdx.x; e < rows * VPR; e += blockDim.x) {
    const int r = e / VPR, c = e % VPR;
    const int p = p0 + r;
    __nv_bfloat16* d = dst + r * LD + c * E;
    if (p < g.N) {
      const int n = permuted ? p : natural_index(g, order, p);
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(head + (int64_t)n * D) + c);
      if constexpr (E == 8) {
        *reinterpret_cast<uint4*>(d) = u;
      } else {
        uint2 w;
        w.x = pack_bf16(__uint_as_float(u.x), __uint_as_float(u.y));
        w.y = pack_bf16(__uint_as_float(u.z), __uint_as_float(u.w));
        *reinterpret_cast<uint2*>(d) = w;
      }
    } else {
      if constexpr (E == 8) {
        *reinterpret_cast<uint4*>(d) = make_uint4(0, 0, 0, 0);
      } else {
        *reinterpret_cast<uint2*>(d) = make_uint2(0, 0);
      }
    }
  }
}

// Rows t0 .. t0+BLOCK-1 of a [nb, D] float summary into a bf16 smem tile
// (row stride LD); rows past nb become zeros.
template <int D, int LD, int BLOCK>
__device__ __forceinline__ void gather_pool_tile(__nv_bfloat16* dst, const float* __restrict__ src,
                                                 int t0, int nb) {
  constexpr int V4 = D / 4;
  for (int e = threadIdx.x; e < BLOCK * V4; e += blockDim.x) {
    const int r = e / V4, c = e % V4;
    uint2 w = make_uint2(0, 0);
    if (t0 + r < nb) {
      const float4 f = __ldg(reinterpret_cast<const float4*>(src + (int64_t)(t0 + r) * D) + c);
      w.x = pack_bf16(f.x, f.y);
      w.y = pack_bf16(f.z, f.w);
    }
    *reinterpret_cast<uint2*>(dst + r * LD + c * 4) = w;
  }
}

// S = Q K^T of one warp's 16 query rows against the BLOCK key rows in Ks.
template <int D, int LD, int NT>
__device__ __forceinline__ void qk_tile(const uint32_t (&qf)[D / 16][4],
                                        const __nv_bfloat16* Ks, int lane, float (&s)[NT][4]) {
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; kk += 2) {
      uint32_t b0, b1, b2, b3;
      const int r = nt * 8 + (lane % 8);
      const int c = kk * 16 + (lane / 8) * 8;
      ldsm_x4(smem_u32(Ks + r * LD + c), b0, b1, b2, b3);
      mma_bf16(s[nt], qf[kk], b0, b1);
      mma_bf16(s[nt], qf[kk + 1], b2, b3);
    }
  }
}

// Online-softmax update with a tile of base-2 scores s (masked entries
// -inf; rows 0 and 1 of the thread's fragment), then O += P V with P
// rounded to bf16.
template <int D, int LD, int NT, int DT, int BLOCK>
__device__ __forceinline__ void softmax_pv(float (&s)[NT][4], const __nv_bfloat16* Vs, int lane,
                                           float (&o)[DT][4], float& m0, float& m1, float& l0,
                                           float& l1) {
  float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    mx0 = fmaxf(mx0, fmaxf(s[nt][0], s[nt][1]));
    mx1 = fmaxf(mx1, fmaxf(s[nt][2], s[nt][3]));
  }
#pragma unroll
  for (int off = 1; off < 4; off <<= 1) {
    mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
    mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
  }
  const float n0 = fmaxf(m0, mx0), n1 = fmaxf(m1, mx1);
  const float u0 = n0 == -INFINITY ? 0.f : n0, u1 = n1 == -INFINITY ? 0.f : n1;
  const float a0 = exp2f(m0 - u0), a1 = exp2f(m1 - u1);
  m0 = n0;
  m1 = n1;
  float rs0 = 0.f, rs1 = 0.f;
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    s[nt][0] = exp2f(s[nt][0] - u0);
    s[nt][1] = exp2f(s[nt][1] - u0);
    s[nt][2] = exp2f(s[nt][2] - u1);
    s[nt][3] = exp2f(s[nt][3] - u1);
    rs0 += s[nt][0] + s[nt][1];
    rs1 += s[nt][2] + s[nt][3];
  }
  l0 = l0 * a0 + rs0;
  l1 = l1 * a1 + rs1;
#pragma unroll
  for (int t = 0; t < DT; ++t) {
    o[t][0] *= a0;
    o[t][1] *= a0;
    o[t][2] *= a1;
    o[t][3] *= a1;
  }
  // P from the S accumulators re-packed as A fragments
#pragma unroll
  for (int kk = 0; kk < BLOCK / 16; ++kk) {
    uint32_t a[4];
    a[0] = pack_bf16(s[2 * kk][0], s[2 * kk][1]);
    a[1] = pack_bf16(s[2 * kk][2], s[2 * kk][3]);
    a[2] = pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]);
    a[3] = pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
    for (int t = 0; t < DT; t += 2) {
      uint32_t b0, b1, b2, b3;
      const int r = kk * 16 + (lane % 8) + ((lane / 8) % 2) * 8;
      const int c = t * 8 + (lane / 16) * 8;
      ldsm_x4_t(smem_u32(Vs + r * LD + c), b0, b1, b2, b3);
      mma_bf16(o[t], a, b0, b1);
      mma_bf16(o[t + 1], a, b2, b3);
    }
  }
}

// Compensation needs one bit per key block of the query block's kept list.
constexpr int kCompMaxNB = 4096;

template <typename TIn, int D, int BLOCK, bool kComp>
__global__ void __launch_bounds__(BLOCK * 2)
    attn_mma_kernel(const TIn* __restrict__ q, const TIn* __restrict__ k,
                    const TIn* __restrict__ v, const __grid_constant__ Grid g,
                    const int32_t* __restrict__ idx, const int32_t* __restrict__ counts,
                    int k_max, float scale_log2, TIn* __restrict__ out,
                    int32_t* __restrict__ status, int permuted,
                    const float* __restrict__ k_pool, const float* __restrict__ v_pool) {
  constexpr int LD = D + 8;  // padded row: conflict-free ldmatrix
  constexpr int NT = BLOCK / 8;  // n-tiles of S
  constexpr int DT = D / 8;  // n-tiles of O
  extern __shared__ __align__(16) unsigned char smem_raw[];
  __nv_bfloat16* Qs = reinterpret_cast<__nv_bfloat16*>(smem_raw);
  __nv_bfloat16* Ks = Qs + BLOCK * LD;
  __nv_bfloat16* Vs = Ks + BLOCK * LD;

  const int i = blockIdx.x;
  const int64_t bh = blockIdx.y;
  const int h = (int)(bh % g.heads);
  const int order = g.perm[h];
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const int64_t row = bh * g.NB + i;
  const int64_t rows_per_head = permuted ? g.Np : g.N;
  const TIn* qh = q + bh * rows_per_head * D;
  const TIn* kh = k + bh * rows_per_head * D;
  const TIn* vh = v + bh * rows_per_head * D;

  int cnt = counts != nullptr ? __ldg(counts + row) : k_max;
  if (cnt < 0 || cnt > k_max) {
    if (threadIdx.x == 0) report(status, PA_ERR_DEVICE_CHECK);
    return;
  }
  const int32_t* ids = idx + row * k_max;

  gather_tile<TIn, D, LD>(Qs, qh, g, order, i * BLOCK, BLOCK, permuted != 0);
  __syncthreads();
  uint32_t qf[D / 16][4];
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    const int r = warp * 16 + (lane % 16);
    const int c = kk * 16 + (lane / 16) * 8;
    ldsm_x4(smem_u32(Qs + r * LD + c), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
  }

  float o[DT][4];
#pragma unroll
  for (int t = 0; t < DT; ++t) o[t][0] = o[t][1] = o[t][2] = o[t][3] = 0.f;
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  int prev = -1;

  for (int jj = 0; jj < cnt; ++jj) {
    const int j = __ldg(ids + jj);
    if (j <= prev || j >= g.NB) {  // uniform across the CTA
      if (threadIdx.x == 0) report(status, PA_ERR_DEVICE_CHECK);
      return;
    }
    prev = j;
    __syncthreads();  // previous tiles fully consumed
    gather_tile<TIn, D, LD>(Ks, kh, g, order, j * BLOCK, BLOCK, permuted != 0);
    gather_tile<TIn, D, LD>(Vs, vh, g, order, j * BLOCK, BLOCK, permuted != 0);
    __syncthreads();

    float s[NT][4];
    qk_tile<D, LD, NT>(qf, Ks, lane, s);
    // scale to base 2, mask pad keys
    const int c0 = j * BLOCK + 2 * (lane % 4);
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const bool ok = c0 + nt * 8 + e < g.N;
        s[nt][e] = ok ? s[nt][e] * scale_log2 : -INFINITY;
        s[nt][2 + e] = ok ? s[nt][2 + e] * scale_log2 : -INFINITY;
      }
    }
    softmax_pv<D, LD, NT, DT, BLOCK>(s, Vs, lane, o, m0, m1, l0, l1);
  }

  if constexpr (kComp) {
    // unselected key blocks as pooled key rows (weight n_j): one bit per
    // kept block first (the list was validated above)
    uint32_t* kept_bits = reinterpret_cast<uint32_t*>(Vs + BLOCK * LD);
    const int words = (g.NB + 31) >> 5;
    __syncthreads();  // last kept tile consumed
    for (int w = threadIdx.x; w < words; w += blockDim.x) kept_bits[w] = 0u;
    __syncthreads();
    for (int jj = threadIdx.x; jj < cnt; jj += blockDim.x) {
      const int j = __ldg(ids + jj);
      atomicOr(kept_bits + (j >> 5), 1u << (j & 31));
    }
    const float* kp = k_pool + bh * (int64_t)g.NB * D;
    const float* vp = v_pool + bh * (int64_t)g.NB * D;
    for (int t0 = 0; t0 < g.NB; t0 += BLOCK) {
      __syncthreads();  // bits written / previous tiles consumed
      gather_pool_tile<D, LD, BLOCK>(Ks, kp, t0, g.NB);
      gather_pool_tile<D, LD, BLOCK>(Vs, vp, t0, g.NB);
      __syncthreads();
      float s[NT][4];
      qk_tile<D, LD, NT>(qf, Ks, lane, s);
      const int c0 = t0 + 2 * (lane % 4);
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int c = c0 + nt * 8 + e;  // key block index
          const int n_c = c < g.NB ? min(BLOCK, g.N - c * BLOCK) : 0;
          const bool ok = n_c > 0 && ((kept_bits[c >> 5] >> (c & 31)) & 1u) == 0u;
          const float bias = ok ? log2f((float)n_c) : 0.f;
          s[nt][e] = ok ? fmaf(s[nt][e], scale_log2, bias) : -INFINITY;
          s[nt][2 + e] = ok ? fmaf(s[nt][2 + e], scale_log2, bias) : -INFINITY;
        }
      }
      softmax_pv<D, LD, NT, DT, BLOCK>(s, Vs, lane, o, m0, m1, l0, l1);
    }
  }

  // epilogue: normalise, stage through smem, store rows at natural positions
#pragma unroll
  for (int off = 1; off < 4; off <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, off);
    l1 += __shfl_xor_sync(0xffffffffu, l1, off);
  }
  const float i0 = l0 > 0.f ? 1.f / l0 : 0.f;
  const float i1 = l1 > 0.f ? 1.f / l1 : 0.f;
  __syncthreads();
  TIn* stage = reinterpret_cast<TIn*>(Ks);  // [BLOCK][D], fits in Ks+Vs
  const int r0 = warp * 16 + lane / 4;
#pragma unroll
  for (int t = 0; t < DT; ++t) {
    const int c = t * 8 + 2 * (lane % 4);
    stage[r0 * D + c] = from_float<TIn>(o[t][0] * i0);
    stage[r0 * D + c + 1] = from_float<TIn>(o[t][1] * i0);
    stage[(r0 + 8) * D + c] = from_float<TIn>(o[t][2] * i1);
    stage[(r0 + 8) * D + c + 1] = from_float<TIn>(o[t][3] * i1);
  }
  __syncthreads();
  constexpr int E = 16 / sizeof(TIn);
  constexpr int VPR = D / E;
  TIn* oh = out + bh * (int64_t)g.N * D;
  for (int e = threadIdx.x; e < BLOCK * VPR; e += blockDim.x) {
    const int r = e / VPR, c = e % VPR;
    const int p = i * BLOCK + r;
    if (p >= g.N) continue;
    const int n = natural_index(g, order, p);
    reinterpret_cast<uint4*>(oh + (int64_t)n * D)[c] =
        reinterpret_cast<const uint4*>(stage + r * D)[c];
  }
}

template <typename TIn, int D, int BLOCK, bool kComp>
cudaError_t launch_typed(const void* q, const void* k, const void* v, const Grid& g,
                         const int32_t* idx, const int32_t* counts, int k_max, void* out,
                         int32_t* status, bool permuted, const float* k_pool,
                         const float* v_pool, cudaStream_t s) {
  constexpr int LD = D + 8;
  const size_t smem = (size_t)3 * BLOCK * LD * sizeof(__nv_bfloat16) +
                      (kComp ? (size_t)kCompMaxNB / 8 : 0);
  static_assert((size_t)BLOCK * D * sizeof(TIn) <= (size_t)2 * BLOCK * LD * 2,
                "staging area must fit in the K and V tiles");
  if (kComp && g.NB > kCompMaxNB) return cudaErrorInvalidValue;
  auto kern = attn_mma_kernel<TIn, D, BLOCK, kComp>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const float scale_log2 = (float)(1.4426950408889634 / sqrt((double)D));
  dim3 grid(g.NB, g.B * g.heads);
  kern<<<grid, BLOCK * 2, smem, s>>>(static_cast<const TIn*>(q), static_cast<const TIn*>(k),
                                     static_cast<const TIn*>(v), g, idx, counts, k_max,
                                     scale_log2, static_cast<TIn*>(out), status,
                                     permuted ? 1 : 0, k_pool, v_pool);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_mma(const void* q, const void* k, const void* v, pa_dtype dt,
                            const Grid& g, const int32_t* idx, const int32_t* counts, int k_max,
                            void* out, int32_t* status, bool permuted, cudaStream_t s,
                            const float* k_pool, const float* v_pool) {
  const bool comp = k_pool != nullptr && v_pool != nullptr;
#define PARO_A(T, D, BL)                                                                       \
  if (g.d == D && g.block == BL)                                                               \
    return comp ? launch_typed<T, D, BL, true>(q, k, v, g, idx, counts, k_max, out, status,    \
                                               permuted, k_pool, v_pool, s)                    \
                : launch_typed<T, D, BL, false>(q, k, v, g, idx, counts, k_max, out, status,   \
                                                permuted, nullptr, nullptr, s);
  if (dt == PA_BF16) {
    PARO_A(__nv_bfloat16, 64, 64)
    PARO_A(__nv_bfloat16, 64, 128)
    PARO_A(__nv_bfloat16, 128, 64)
    PARO_A(__nv_bfloat16, 128, 128)
  } else if (dt == PA_F32) {
    PARO_A(float, 64, 64)
    PARO_A(float, 64, 128)
    PARO_A(float, 128, 64)
    PARO_A(float, 128, 128)
  }
#undef PARO_A
  return cudaErrorInvalidValue;
}

}  // namespace paro
