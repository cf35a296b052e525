// INT8 block-sparse attention on the sm_100a tensor cores (tcgen05.mma
// kind::i8, int32 accumulation in tensor memory), d = 128, block = 128.
//
// What it computes (PAROAttention, arXiv 2506.16054, Pith verdict page,
// key_machinery and core_discovery: block-wise INT8 quantisation with groups
// aligned to the attention block, for Q K^T and for the post-softmax map P;
// SPADE, arXiv 2608.03335, verdict page key_machinery (iii): online softmax
// over the kept tiles).  Inputs are the permuted int8 codes and per-block
// scales of pa_quantize_int8.  For query block i and each kept key block j,
// in ascending order:
//   S      = (Q8_i K8_j^T, exact int32) * s_q[i] s_k[j] / sqrt(d)
//   m      = running row max (exact), P~ = 2^(S log2 e - m) <= 1
//   P8     = round_half_even(127 P~)           (the tile's symmetric scale 1/127)
//   l      = l 2^(m_old - m) + sum P~
//   O      = O 2^(m_old - m) + (P8 V8_j, exact int32) * s_v[j] / 127
// and O / l is stored at the natural positions of the block's tokens.
//
// One CTA per (query block, head); 8 warps:
//   warps 0-3  softmax + correction: thread t owns row t (TMEM lane t); it
//              turns S(j) into P8(j) (packed 4 per 32-bit TMEM column, the
//              A operand of the P V MMA), then folds the int32 P V result of
//              the previous tile into the fp32 O accumulator in TMEM;
//   warp 4     allocates TMEM; one lane issues every tcgen05.mma and commit;
//   warp 5     loads Q, then K tiles; warp 6 loads V tiles: one lane issues
//              one TMA tiled box (128 rows x 128 bytes) per tile;
//   warp 7     validates the kept list, then idles.
// Tensor memory (512 columns): S int32 at 0, P8 double buffer (32 columns
// each) at 128 and 160, the P V int32 result at 192, O fp32 at 320.
// Shared memory: Q (16 KB) and four-stage K and V rings, each tile one
// 128-byte-swizzled panel.
//
// MMA order QK(0), QK(1), PV(0), QK(2), PV(1), ...; S(j) ready implies
// P V(j-2) completed (in-order tcgen05 completion), so P8 buffer j & 1 is
// free.  Every mbarrier wait is bounded as in the bf16 kernel; on expiry the
// kernel records PA_ERR_TIMEOUT and unwinds.
#include "sm100.cuh"

namespace paro {
namespace {

using namespace sm100;

constexpr int kBlock = 128;
constexpr int kD = 128;
constexpr int kStages = 4;
constexpr int kMmaWarp = 4;
constexpr int kKWarp = 5;
constexpr int kVWarp = 6;
constexpr int kCheckWarp = 7;
constexpr int kThreads = 8 * 32;
constexpr int kSoftThreads = 128;
constexpr uint32_t kTile = kBlock * kD;  // 16 KB: one 128-byte-swizzled panel
constexpr uint32_t kOffBar = 0;
constexpr uint32_t kOffSlot = 256;
constexpr uint32_t kSmall = 1024;
constexpr uint32_t kOffQ = kSmall;
constexpr uint32_t kOffK = kOffQ + kTile;
constexpr uint32_t kOffV = kOffK + kStages * kTile;
constexpr uint32_t kSmemBytes = kOffV + kStages * kTile;  // 148,480 B
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColP = 128, kColR = 192, kColO = 320;

enum : uint32_t {
  BQ = 0,
  BK0 = 1,    // K stage full (4)
  BV0 = 5,    // V stage full (4)
  BKF0 = 9,   // K stage free (4)
  BVF0 = 13,  // V stage free (4)
  BS = 17,    // S(j) ready
  BSF = 18,   // S(j) read
  BP0 = 19,   // P8(j) written (2)
  BPV = 21,   // P V(j) result ready
  BPVF = 22,  // P V(j) result folded into O (result columns free)
  BDRAIN = 23,
  NBAR = 24
};
static_assert(NBAR * 8 <= kOffSlot, "barrier region");

// int32 -> float exactly for |x| < 2^22 without the conversion unit:
// 1.5 * 2^23 + x lies in [2^23, 2^24), where floats are spaced by 1.
__device__ __forceinline__ float i2f_small(int32_t x) {
  return __int_as_float(x + 0x4B400000) - 12582912.0f;
}
// round-half-even of 0 <= y < 2^22 with one float add (the add rounds to
// the nearest representable value, spacing 1, ties to even)
__device__ __forceinline__ uint32_t rne_small(float y) {
  return (uint32_t)(__float_as_int(y + 12582912.0f) - 0x4B400000);
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_i8_kernel(const __grid_constant__ CUtensorMap map_q,
                   const __grid_constant__ CUtensorMap map_k,
                   const __grid_constant__ CUtensorMap map_v, const __grid_constant__ Grid g,
                   const int32_t* __restrict__ idx, const int32_t* __restrict__ counts, int k_max,
                   const float* __restrict__ q_scale, const float* __restrict__ k_scale,
                   const float* __restrict__ v_scale, float log2e_over_sqrt_d,
                   __nv_bfloat16* __restrict__ out, int32_t* __restrict__ status) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t base = smem_u32(smem_raw);
  if ((base & 1023u) != 0) {
    if (threadIdx.x == 0) report(status, PA_ERR_UNSUPPORTED);
    return;
  }
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem_raw + kOffSlot);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  volatile uint32_t* bad_flag = tmem_slot + 2;
  auto bar = [&](uint32_t slot) { return base + kOffBar + slot * 8u; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int i = blockIdx.x;
  const int64_t bh = blockIdx.y;
  const int h = (int)(bh % g.heads);
  const int order = g.perm[h];
  const int64_t row = bh * g.NB + i;
  const int32_t* ids = idx + row * k_max;
  const int cnt = counts != nullptr ? __ldg(counts + row) : k_max;
  Ctl ctl{abort_flag, status};
  const bool expired =
      status != nullptr && *reinterpret_cast<volatile int32_t*>(status) == PA_ERR_TIMEOUT;

  if (threadIdx.x == 0) {
    mbar_init(bar(BQ), 1);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(BK0 + s), 1);
      mbar_init(bar(BV0 + s), 1);
      mbar_init(bar(BKF0 + s), 1);
      mbar_init(bar(BVF0 + s), 1);
    }
    mbar_init(bar(BS), 1);
    mbar_init(bar(BSF), kSoftThreads);
    mbar_init(bar(BP0), kSoftThreads);
    mbar_init(bar(BP0 + 1), kSoftThreads);
    mbar_init(bar(BPV), 1);
    mbar_init(bar(BPVF), kSoftThreads);
    mbar_init(bar(BDRAIN), 1);
    *abort_flag = 0;
    *bad_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == kMmaWarp) tmem_alloc(smem_u32(tmem_slot), kTmemCols);
  if (warp == kCheckWarp) {
    bool bad = cnt < 0 || cnt > k_max;
    if (!bad) {
      for (int e = lane; e < cnt; e += 32) {
        const int j = __ldg(ids + e);
        const int prev = e > 0 ? __ldg(ids + e - 1) : -1;
        bad |= (j <= prev) || (j >= g.NB);
      }
    }
    if (__any_sync(0xffffffffu, bad) && lane == 0) {
      *bad_flag = 1;
      report(status, PA_ERR_DEVICE_CHECK);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const bool run = *bad_flag == 0 && !expired;
  const int n_tiles = run ? cnt : 0;
  const int row0 = (int)(bh * g.Np);

  if (warp == kKWarp || warp == kVWarp) {
    // ------------------------------------------------------ loads ------
    const bool is_k = warp == kKWarp;
    const CUtensorMap* map = is_k ? &map_k : &map_v;
    const uint32_t ring = base + (is_k ? kOffK : kOffV);
    int issued = 0;
    if (n_tiles > 0 && lane == 0) {
      if (is_k) {
        mbar_arrive_tx(bar(BQ), kTile);
        tma_load_2d(base + kOffQ, &map_q, 0, row0 + i * kBlock, bar(BQ));
      }
      for (int j = 0; j < n_tiles; ++j) {
        const int s = j % kStages;
        if (j >= kStages &&
            !wait_phase(bar((is_k ? BKF0 : BVF0) + s), ((j / kStages) - 1) & 1, ctl))
          break;
        const uint32_t full = bar((is_k ? BK0 : BV0) + s);
        mbar_arrive_tx(full, kTile);
        tma_load_2d(ring + s * kTile, map, 0, row0 + __ldg(ids + j) * kBlock, full);
        issued = j + 1;
      }
      if (is_k) drain_phase(bar(BQ), 0);
      for (int j = issued > kStages ? issued - kStages : 0; j < issued; ++j)
        drain_phase(bar((is_k ? BK0 : BV0) + j % kStages), (j / kStages) & 1);
    }
    __syncwarp();
  } else if (warp == kMmaWarp) {
    // ---------------------------------------------------------- MMA ----
    if (lane == 0 && n_tiles > 0) {
      constexpr uint32_t id_qk = idesc_s8(kBlock, kBlock, false);
      constexpr uint32_t id_pv = idesc_s8(kBlock, kD, true);
      bool ok = wait_phase(bar(BQ), 0, ctl);
      auto issue_qk = [&](int j) -> bool {
        const int s = j % kStages;
        if (!wait_phase(bar(BK0 + s), (j / kStages) & 1, ctl)) return false;
        if (j >= 1 && !wait_phase(bar(BSF), (j - 1) & 1, ctl)) return false;
        tc_fence_after();
        const uint32_t ka = base + kOffK + s * kTile;
#pragma unroll
        for (int kk = 0; kk < kD / 32; ++kk)
          mma_i8_ss(tmem + kColS, sw128_desc(base + kOffQ + kk * 32, 16, 1024),
                    sw128_desc(ka + kk * 32, 16, 1024), id_qk, kk > 0 ? 1u : 0u);
        mma_commit(bar(BS));
        mma_commit(bar(BKF0 + s));
        return true;
      };
      auto issue_pv = [&](int j) -> bool {
        const int b = j & 1, s = j % kStages;
        if (!wait_phase(bar(BP0 + b), (j >> 1) & 1, ctl)) return false;
        if (!wait_phase(bar(BV0 + s), (j / kStages) & 1, ctl)) return false;
        if (j >= 1 && !wait_phase(bar(BPVF), (j - 1) & 1, ctl)) return false;
        tc_fence_after();
        const uint32_t va = base + kOffV + s * kTile;
#pragma unroll
        for (int kk = 0; kk < kBlock / 32; ++kk) {
          asm volatile(
              "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
              "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n}\n" ::"r"(tmem + kColR),
              "r"(tmem + kColP + b * 32 + kk * 8), "l"(sw128_desc(va + kk * 32 * 128, kTile, 1024)),
              "r"(id_pv), "r"(kk > 0 ? 1u : 0u)
              : "memory");
        }
        mma_commit(bar(BPV));
        mma_commit(bar(BVF0 + s));
        return true;
      };
      ok = ok && issue_qk(0);
      for (int j = 0; ok && j < n_tiles; ++j) {
        if (j + 1 < n_tiles && !issue_qk(j + 1)) { ok = false; break; }
        if (!issue_pv(j)) { ok = false; break; }
      }
      mma_commit(bar(BDRAIN));
      drain_phase(bar(BDRAIN), 0);
    }
    __syncwarp();
  } else if (warp < 4) {
    // -------------------------------------------- softmax + correction --
    const int r = threadIdx.x;  // tile row == TMEM lane
    const uint32_t lane_addr = tmem + ((uint32_t)(warp * 32) << 16);
    const float sq = __ldg(q_scale + row) * log2e_over_sqrt_d;
    float m_run = -INFINITY, l = 0.f;
    float fold_alpha = 0.f, fold_c = 0.f;  // pending fold of the previous tile
    bool ok = true;
    // O = O * alpha + c * (P V result): the previous tile's contribution
    auto fold = [&](int jp, float alpha, float c) -> bool {
      if (!warp_wait(bar(BPV), jp & 1, ctl)) return false;
      tc_fence_after();
#pragma unroll 1
      for (int c0 = 0; c0 < 128; c0 += 32) {
        uint32_t pv[32], o[32];
        tmem_ld32(lane_addr + kColR + c0, pv);
        if (jp > 0) tmem_ld32(lane_addr + kColO + c0, o);
#pragma unroll
        for (int u = 0; u < 32; ++u) {
          const float add = (float)(int32_t)pv[u] * c;
          o[u] = __float_as_uint(jp > 0 ? fmaf(__uint_as_float(o[u]), alpha, add) : add);
        }
        tmem_st32(lane_addr + kColO + c0, o);
      }
      tc_fence_before();
      mbar_arrive(bar(BPVF));
      return true;
    };
    for (int j = 0; j < n_tiles; ++j) {
      if (!warp_wait(bar(BS), j & 1, ctl)) { ok = false; break; }
      tc_fence_after();
      uint32_t sr[128];
      tmem_ld128(lane_addr + kColS, sr);
      tc_fence_before();
      mbar_arrive(bar(BSF));  // S may take QK^T(j+1)
      const int kb = __ldg(ids + j);
      const int valid = g.N - kb * kBlock;
      const float cq = sq * __ldg(k_scale + bh * g.NB + kb);
      float mp[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) mp[u] = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; ++c) {
        float s = i2f_small((int32_t)sr[c]) * cq;
        if (valid < kBlock && c >= valid) s = -INFINITY;
        sr[c] = __float_as_uint(s);
        mp[c & 7] = fmaxf(mp[c & 7], s);
      }
      const float mt = fmaxf(fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3])),
                             fmaxf(fmaxf(mp[4], mp[5]), fmaxf(mp[6], mp[7])));
      const float m_new = fmaxf(m_run, mt);
      const float alpha = m_run == -INFINITY ? 0.f : ex2(m_run - m_new);
      // P~ = 2^(s - m) <= 1, P8 = rne(127 P~), packed 4 per column
      float rs[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) rs[u] = 0.f;
      uint32_t pk[32];
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        uint32_t w = 0;
#pragma unroll
        for (int b = 0; b < 4; ++b) {
          const float e = ex2(__uint_as_float(sr[4 * c + b]) - m_new);
          rs[b] += e;
          w |= rne_small(127.f * e) << (8 * b);
        }
        pk[c] = w;
      }
      l = l * alpha + (((rs[0] + rs[1]) + (rs[2] + rs[3])) + ((rs[4] + rs[5]) + (rs[6] + rs[7])));
      tmem_st32(lane_addr + kColP + (j & 1) * 32, pk);
      tc_fence_before();
      mbar_arrive(bar(BP0 + (j & 1)));
      // fold the previous tile's P V (its P used reference m_run)
      if (j >= 1 && !fold(j - 1, fold_alpha, fold_c)) { ok = false; break; }
      fold_alpha = alpha;  // O (ref m_run) -> ref m_new when tile j is folded
      fold_c = __ldg(v_scale + bh * g.NB + kb) * (1.f / 127.f);
      m_run = m_new;
    }
    if (ok && n_tiles > 0) ok = fold(n_tiles - 1, fold_alpha, fold_c);
    // epilogue: O / l at the natural position of the row's token
    const int p = i * kBlock + r;
    __nv_bfloat16* orow = p < g.N ? out + (bh * (int64_t)g.N + natural_index(g, order, p)) * kD
                                  : nullptr;
    if (run && cnt == 0) {
      if (orow != nullptr)
        for (int c = 0; c < 16; ++c) reinterpret_cast<uint4*>(orow)[c] = make_uint4(0, 0, 0, 0);
    } else if (ok && n_tiles > 0) {
      tc_fence_after();
      const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll 1
      for (int c0 = 0; c0 < 128; c0 += 32) {
        uint32_t o[32];
        tmem_ld32(lane_addr + kColO + c0, o);
        if (orow != nullptr) {
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const float* f = reinterpret_cast<const float*>(o) + c * 8;
            uint4 w;
            w.x = pack_bf16(f[0] * inv, f[1] * inv);
            w.y = pack_bf16(f[2] * inv, f[3] * inv);
            w.z = pack_bf16(f[4] * inv, f[5] * inv);
            w.w = pack_bf16(f[6] * inv, f[7] * inv);
            reinterpret_cast<uint4*>(orow + c0)[c] = w;
          }
        }
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

}  // namespace

cudaError_t launch_attn_i8(const void* q, const void* k, const void* v, const Grid& g,
                           const int32_t* idx, const int32_t* counts, int k_max, const float* qs,
                           const float* ks, const float* vs, void* out, int32_t* status,
                           cudaStream_t s) {
  if (g.d != kD || g.block != kBlock) return cudaErrorInvalidValue;
  const uint64_t rows = (uint64_t)g.B * g.heads * g.Np;
  CUtensorMap mq{}, mk{}, mv{};
  if (!encode_tile_map(&mq, q, rows, kD, 1, 128, kBlock) ||
      !encode_tile_map(&mk, k, rows, kD, 1, 128, kBlock) ||
      !encode_tile_map(&mv, v, rows, kD, 1, 128, kBlock))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(attn_i8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  const float c = (float)(1.4426950408889634 / sqrt((double)kD));
  dim3 grid(g.NB, g.B * g.heads);
  attn_i8_kernel<<<grid, kThreads, kSmemBytes, s>>>(mq, mk, mv, g, idx, counts, k_max, qs, ks, vs,
                                                    c, static_cast<__nv_bfloat16*>(out), status);
  return cudaGetLastError();
}

}  // namespace paro
