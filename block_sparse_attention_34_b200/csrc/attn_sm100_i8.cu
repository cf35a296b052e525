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
// (with 4-bit P, the INT4 PV variant: 7 in place of 127, and V codes in
// [-7, 7] from pa_quantize_int4; the integer MMAs are unchanged)
// and O / l is stored at the natural positions of the block's tokens.
//
// kTwoPass: the post-softmax map is quantised per tile after it
// is normalised, each tile with its own scale.  Pass 1 runs Q K^T over the
// kept tiles for the exact row max m and sum l (each 64-column half keeps
// its own pair, merged once); pass 2 runs Q K^T again and, per tile,
//   P      = 2^(S log2 e - m) / l             (the normalised map)
//   a      = max of P over the tile's valid rows and keys (shared by the
//            eight softmax warps through shared memory)
//   P8     = round_half_even(L P / a)           (L = 127, or 7 for 4 bits)
//   O      = O + (P8 V8_j, exact int32) * (a / L) s_v[j]
// so O needs no rescale and no final division.
//
// One CTA per (query block, head); 14 warps in four roles:
//   warps 0-7   softmax: warp w serves tile rows 32 (w & 3) .. +31 (its
//               TMEM lane quarter) and S columns 64 (w >> 2) .. +63.  Per
//               tile: row max of its half, traded with the partner warp of
//               the other half through shared memory (a bounded mbarrier
//               exchange: the running max stays exact), P8 of its half into
//               a 128-byte-swizzled shared-memory tile (the A operand of
//               P V), the row sum, and the tile's rescale factors;
//   warps 8-11  correction: warp w folds the int32 P V result of its 32
//               rows into the fp32 O accumulator in TMEM,
//               O = O alpha + (s_v / 127) (P8 V8), and stores O / l at the end;
//   warp 12     allocates TMEM; one lane issues every tcgen05.mma and commit;
//   warp 13     validates the kept list; one lane then issues the TMA loads
//               (Q once, then K and V tiles of 128 rows x 128 bytes).
// Tensor memory (512 columns): S int32 at 0, O fp32 at 128, the P V int32
// result double buffer at 256 and 384.
// Shared memory: Q (16 KB), five-stage K and V rings and a P8 double buffer
// (16 KB per tile, each one 128-byte-swizzled panel).
//
// int32 -> float conversions avoid the conversion unit: |S|, |P V| <=
// 128 * 127 * 127 < 2^22, so adding the bits of 1.5 * 2^23 gives a float
// equal to 1.5 * 2^23 + x exactly, and subtracting 1.5 * 2^23 recovers x.
//
// MMA order QK(0), QK(1), PV(0), QK(2), PV(1), ...  S(j) ready implies
// P V(j-2) completed (tcgen05 operations complete in issue order), so P8
// buffer j & 1 is free when the softmax writes P8(j); P V(j) waits for the
// correction of tile j-2 to free result buffer j & 1.  The softmax reads the
// kept index and block scales of tile j+1 while it works on tile j.  Every mbarrier wait
// is bounded as in the bf16 kernel; on expiry the kernel records
// PA_ERR_TIMEOUT and unwinds.
#include "sm100.cuh"
#include "tmem.cuh"

namespace paro {

#ifdef PARO_TRACE
// Phase trace (debug builds only): clock64() of each role's key events for
// one CTA, event e of tile j at g_paro_trace_i8[e * 128 + j].
__device__ long long* g_paro_trace_i8 = nullptr;
__device__ int g_paro_trace_i8_cta = 7;
#define PARO_T8(ev, j)                                                                      \
  do {                                                                                      \
    if (g_paro_trace_i8 != nullptr && blockIdx.x == g_paro_trace_i8_cta && blockIdx.y == 0 && \
        (j) < 128)                                                                          \
      g_paro_trace_i8[(ev) * 128 + (j)] = clock64();                                        \
  } while (0)
#else
#define PARO_T8(ev, j) \
  do {                 \
  } while (0)
#endif

namespace {

using namespace sm100;

constexpr int kBlock = 128;
constexpr int kD = 128;
constexpr int kStages = 5;
constexpr int kSoftWarps = 8;
constexpr int kCorrWarp0 = 8;  // warps 8..11
constexpr int kMmaWarp = 12;
constexpr int kLoadWarp = 13;
constexpr int kThreads = 14 * 32;
constexpr int kSoftThreads = kSoftWarps * 32;
constexpr int kCorrThreads = 4 * 32;
constexpr int kScaleSlots = 4;
constexpr uint32_t kTile = kBlock * kD;  // 16 KB: one 128-byte-swizzled panel
constexpr uint32_t kOffBar = 0;
constexpr uint32_t kOffAmx = 384;  // kTwoPass: per-warp tile maxima [2 parity][8 warps] f32
constexpr uint32_t kOffSlot = 512;
constexpr uint32_t kOffX = 1024;   // row-max exchange [2 parity][2 half][128] f32
constexpr uint32_t kOffA = 3072;   // rescale factor alpha [4 slots][128] f32
constexpr uint32_t kOffC = 5120;   // P V scale s_v / 127 [4 slots][128] f32
constexpr uint32_t kOffL = 7168;   // final row sums [2 half][128] f32
constexpr uint32_t kOffQ = 8192;
constexpr uint32_t kOffK = kOffQ + kTile;
constexpr uint32_t kOffV = kOffK + kStages * kTile;
constexpr uint32_t kOffP = kOffV + kStages * kTile;
constexpr uint32_t kSmemBytes = kOffP + 2 * kTile;  // 221,184 B
static_assert(kSmemBytes <= 227 * 1024, "shared memory");
static_assert(kOffQ % 1024 == 0, "swizzled tiles need 1024-byte alignment");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 128, kColR = 256;
constexpr int32_t kMagicBits = 0x4B400000;  // bits of 1.5 * 2^23
constexpr float kMagic = 12582912.0f;       // 1.5 * 2^23

enum : uint32_t {
  BQ = 0,
  BK0 = 1,                // K stage full (kStages)
  BV0 = BK0 + kStages,    // V stage full
  BKF0 = BV0 + kStages,   // K stage free
  BVF0 = BKF0 + kStages,  // V stage free
  BS = BVF0 + kStages,    // S(j) ready
  BSF,                    // S(j) read by the softmax
  BP0,                    // P8(j) written (2)
  BSC0 = BP0 + 2,         // rescale factors of tile j written in slot j % 4 (4)
  BPV0 = BSC0 + kScaleSlots,  // P V(j) ready in result buffer j & 1 (2)
  BPVF0 = BPV0 + 2,       // result buffer folded into O, free (2)
  BX0 = BPVF0 + 2,        // row-max exchange of lane quarter q (4)
  BL = BX0 + 4,           // final row sums written
  BDRAIN,
  BMG,                    // kTwoPass: pass-1 half statistics written
  BAM0,                   // kTwoPass: warp maxima of tile j written, slot j & 1 (2)
  NBAR = BAM0 + 2
};
static_assert(NBAR * 8 <= kOffAmx, "barrier region");
static_assert(kOffAmx + 16 * 4 <= kOffSlot, "tile maxima region");

// float of an int32 |x| < 2^22 held in the bits of a 32-bit register (two
// such values at once: the subtraction is one paired instruction)
__device__ __forceinline__ float2 exact_float2(uint32_t a, uint32_t b) {
  return fadd2(make_float2(__int_as_float((int32_t)a + kMagicBits),
                           __int_as_float((int32_t)b + kMagicBits)),
               make_float2(-kMagic, -kMagic));
}

// P~ = 2^(s - m) <= 1 for 64 columns of one row, P codes = rne(L P~) (L =
// levels: 127, or 7 for 4-bit P) as the low byte of the float L P~ + 1.5 *
// 2^23 (one rounding to the nearest integer, ties to even), packed 4 per
// 32-bit word; row sums of P~ in rs.
template <bool kRagged>
__device__ __forceinline__ void tile_exp(const uint32_t (&sr)[64], float2 cq2, float2 nm2,
                                         int valid, float2& rs0, float2& rs1,
                                         uint32_t (&pk)[16], float levels) {
  const float2 k127 = make_float2(levels, levels), mg2 = make_float2(kMagic, kMagic);
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    const float2 t0 = ffma2(exact_float2(sr[4 * c], sr[4 * c + 1]), cq2, nm2);
    const float2 t1 = ffma2(exact_float2(sr[4 * c + 2], sr[4 * c + 3]), cq2, nm2);
    float2 e0 = make_float2(ex2(t0.x), ex2(t0.y));
    float2 e1 = make_float2(ex2(t1.x), ex2(t1.y));
    if (kRagged) {
      if (4 * c >= valid) e0.x = 0.f;
      if (4 * c + 1 >= valid) e0.y = 0.f;
      if (4 * c + 2 >= valid) e1.x = 0.f;
      if (4 * c + 3 >= valid) e1.y = 0.f;
    }
    rs0 = fadd2(rs0, e0);
    rs1 = fadd2(rs1, e1);
    const float2 b0 = ffma2(e0, k127, mg2);
    const float2 b1 = ffma2(e1, k127, mg2);
    pk[c] = __byte_perm(__byte_perm(__float_as_uint(b0.x), __float_as_uint(b0.y), 0x0040),
                        __byte_perm(__float_as_uint(b1.x), __float_as_uint(b1.y), 0x0040), 0x5410);
  }
}

// Largest int32 score among the first `valid` of 64 columns (INT32_MIN if
// none): the order of S, since its scale is positive.
__device__ __forceinline__ int32_t half_max(const uint32_t (&sr)[64], int valid) {
  int32_t mi = INT32_MIN;
  if (valid >= 64) {
    int32_t mp[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) mp[u] = INT32_MIN;
#pragma unroll
    for (int c = 0; c < 64; ++c) mp[c & 7] = max(mp[c & 7], (int32_t)sr[c]);
    mi = max(max(max(mp[0], mp[1]), max(mp[2], mp[3])), max(max(mp[4], mp[5]), max(mp[6], mp[7])));
  } else {
#pragma unroll
    for (int c = 0; c < 64; ++c)
      if (c < valid) mi = max(mi, (int32_t)sr[c]);
  }
  return mi;
}

template <bool kTwoPass>
__global__ void __launch_bounds__(kThreads, 1)
    attn_i8_kernel(const __grid_constant__ CUtensorMap map_q,
                   const __grid_constant__ CUtensorMap map_k,
                   const __grid_constant__ CUtensorMap map_v, const __grid_constant__ Grid g,
                   const int32_t* __restrict__ idx, const int32_t* __restrict__ counts, int k_max,
                   const float* __restrict__ q_scale, const float* __restrict__ k_scale,
                   const float* __restrict__ v_scale, float log2e_over_sqrt_d, float p_levels,
                   __nv_bfloat16* __restrict__ out, int32_t* __restrict__ status) {
  static_assert(kTile == kBlock * kD, "kTile names the tile's byte size here");
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t base = smem_u32(smem_raw);
  if ((base & 1023u) != 0) {
    if (threadIdx.x == 0) report(status, PA_ERR_UNSUPPORTED);
    return;
  }
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem_raw + kOffSlot);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  volatile uint32_t* bad_flag = tmem_slot + 2;
  float* xch = reinterpret_cast<float*>(smem_raw + kOffX);
  float* s_alpha = reinterpret_cast<float*>(smem_raw + kOffA);
  float* s_cv = reinterpret_cast<float*>(smem_raw + kOffC);
  float* s_l = reinterpret_cast<float*>(smem_raw + kOffL);
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
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(BP0 + b), kSoftThreads);
      mbar_init(bar(BPV0 + b), 1);
      mbar_init(bar(BPVF0 + b), kCorrThreads);
    }
    for (int b = 0; b < kScaleSlots; ++b) mbar_init(bar(BSC0 + b), kSoftThreads / 2);
    for (int q = 0; q < 4; ++q) mbar_init(bar(BX0 + q), 64);
    mbar_init(bar(BL), kSoftThreads);
    mbar_init(bar(BDRAIN), 1);
    mbar_init(bar(BMG), kSoftThreads);
    for (int b = 0; b < 2; ++b) mbar_init(bar(BAM0 + b), kSoftWarps);
    *abort_flag = 0;
    *bad_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == kMmaWarp) tmem_alloc(smem_u32(tmem_slot), kTmemCols);
  if (warp == kLoadWarp) {
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

  if (warp == kLoadWarp) {
    // ------------------------------------------------------ loads ------
    if (n_tiles > 0 && lane == 0) {
      mbar_arrive_tx(bar(BQ), kTile);
      tma_load_2d(base + kOffQ, &map_q, 0, row0 + i * kBlock, bar(BQ));
      // K tile t of the kept entry j (kTwoPass: t < n_tiles is pass 1, K only;
      // pass 2 loads K again with V); the K ring counts t, the V ring j
      int nk = 0, nv = 0;  // K and V tiles issued
      const int n_k = kTwoPass ? 2 * n_tiles : n_tiles;
      for (int t = 0; t < n_k; ++t) {
        const bool pass1 = kTwoPass && t < n_tiles;
        const int j = kTwoPass && !pass1 ? t - n_tiles : t;
        const int s = t % kStages;
        const int y = row0 + __ldg(ids + j) * kBlock;
        if (t >= kStages && !wait_phase(bar(BKF0 + s), ((t / kStages) - 1) & 1, ctl)) break;
        PARO_T8(0, t);
        mbar_arrive_tx(bar(BK0 + s), kTile);
        tma_load_2d(base + kOffK + s * kTile, &map_k, 0, y, bar(BK0 + s));
        nk = t + 1;
        if (pass1) continue;
        const int sv = j % kStages;
        if (j >= kStages && !wait_phase(bar(BVF0 + sv), ((j / kStages) - 1) & 1, ctl)) break;
        PARO_T8(11, j);
        mbar_arrive_tx(bar(BV0 + sv), kTile);
        tma_load_2d(base + kOffV + sv * kTile, &map_v, 0, y, bar(BV0 + sv));
        nv = j + 1;
      }
      // copies still in flight land before the CTA exits
      drain_phase(bar(BQ), 0);
      for (int j = nk > kStages ? nk - kStages : 0; j < nk; ++j)
        drain_phase(bar(BK0 + j % kStages), (j / kStages) & 1);
      for (int j = nv > kStages ? nv - kStages : 0; j < nv; ++j)
        drain_phase(bar(BV0 + j % kStages), (j / kStages) & 1);
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
        PARO_T8(1, j);
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
        if (j >= 2 && !wait_phase(bar(BPVF0 + b), ((j >> 1) - 1) & 1, ctl)) return false;
        PARO_T8(2, j);
        tc_fence_after();
        const uint32_t va = base + kOffV + s * kTile, pa = base + kOffP + b * kTile;
#pragma unroll
        for (int kk = 0; kk < kBlock / 32; ++kk)
          mma_i8_ss(tmem + kColR + b * 128, sw128_desc(pa + kk * 32, 16, 1024),
                    sw128_desc(va + kk * 32 * 128, kTile, 1024), id_pv, kk > 0 ? 1u : 0u);
        mma_commit(bar(BPV0 + b));
        mma_commit(bar(BVF0 + s));
        return true;
      };
      // kTwoPass: pass 1 is Q K^T alone over the kept tiles; pass 2's Q K^T
      // count on from n_tiles (the K ring and S handshakes continue)
      const int t0 = kTwoPass ? n_tiles : 0;
      for (int t = 0; ok && t < t0; ++t) ok = issue_qk(t);
      ok = ok && issue_qk(t0);
      for (int j = 0; ok && j < n_tiles; ++j) {
        if (j + 1 < n_tiles && !issue_qk(t0 + j + 1)) break;
        if (!issue_pv(j)) break;
      }
      mma_commit(bar(BDRAIN));
      drain_phase(bar(BDRAIN), 0);
    }
    __syncwarp();
  } else if (warp >= kCorrWarp0) {
    // -------------------------------------------------- correction ----
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      const int sl = j & (kScaleSlots - 1), b = j & 1;
      if (!all_wait(bar(BSC0 + sl), (j / kScaleSlots) & 1, ctl)) { ok = false; break; }
      const float alpha = s_alpha[sl * 128 + r];
      const float2 cv2 = make_float2(s_cv[sl * 128 + r], s_cv[sl * 128 + r]);
      const float2 al2 = make_float2(alpha, alpha);
      if (lane == 0 && quarter == 0) PARO_T8(9, j);
      if (!warp_wait(bar(BPV0 + b), (j >> 1) & 1, ctl)) { ok = false; break; }
      if (lane == 0 && quarter == 0) PARO_T8(10, j);
      tc_fence_after();
      // alpha is 1 while the row max holds
      const bool keep = __all_sync(0xffffffffu, alpha == 1.f);
      const uint32_t ra = lane_addr + kColR + b * 128;
#pragma unroll 1
      for (int c0 = 0; c0 < kD; c0 += 32) {
        uint32_t pv[32], o[32];
        if (j == 0) {
          tmem_ld32(ra + c0, pv);
#pragma unroll
          for (int u = 0; u < 32; u += 2) {
            const float2 f = fmul2(exact_float2(pv[u], pv[u + 1]), cv2);
            o[u] = __float_as_uint(f.x);
            o[u + 1] = __float_as_uint(f.y);
          }
        } else {
          tmem_ld32x2(ra + c0, pv, lane_addr + kColO + c0, o);
          if (keep) {
#pragma unroll
            for (int u = 0; u < 32; u += 2) {
              const float2 f = ffma2(exact_float2(pv[u], pv[u + 1]), cv2,
                                     make_float2(__uint_as_float(o[u]), __uint_as_float(o[u + 1])));
              o[u] = __float_as_uint(f.x);
              o[u + 1] = __float_as_uint(f.y);
            }
          } else {
#pragma unroll
            for (int u = 0; u < 32; u += 2) {
              const float2 oa =
                  fmul2(make_float2(__uint_as_float(o[u]), __uint_as_float(o[u + 1])), al2);
              const float2 f = ffma2(exact_float2(pv[u], pv[u + 1]), cv2, oa);
              o[u] = __float_as_uint(f.x);
              o[u + 1] = __float_as_uint(f.y);
            }
          }
        }
        tmem_st32_async(lane_addr + kColO + c0, o);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(bar(BPVF0 + b));
      if (lane == 0 && quarter == 0) PARO_T8(12, j);
    }
    // epilogue: O / l at the natural position of the row's token
    const int p = i * kBlock + r;
    __nv_bfloat16* orow =
        p < g.N ? out + (bh * (int64_t)g.N + natural_index(g, order, p)) * kD : nullptr;
    if (run && cnt == 0) {
      if (orow != nullptr)
        for (int c = 0; c < 16; ++c) reinterpret_cast<uint4*>(orow)[c] = make_uint4(0, 0, 0, 0);
    } else if (ok && n_tiles > 0 && all_wait(bar(BL), 0, ctl)) {
      const float lt = s_l[r] + s_l[128 + r];
      const float inv = lt > 0.f ? 1.f / lt : 0.f;
      tc_fence_after();
#pragma unroll 1
      for (int c0 = 0; c0 < kD; c0 += 32) {
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
  } else {
    // ----------------------------------------------------- softmax ----
    const int quarter = warp & 3, hc = warp >> 2;
    const int r = quarter * 32 + lane;  // tile row == TMEM lane
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    const uint32_t xbar = bar(BX0 + quarter);
    const float sq = __ldg(q_scale + row) * log2e_over_sqrt_d;
    float m_run = -INFINITY;
    float2 l2 = make_float2(0.f, 0.f);
    bool ok = true;
    if constexpr (kTwoPass) {
      // ---- pass 1: exact row max and sum of this half (S read only)
      float m_h = -INFINITY, l_h = 0.f;
      for (int t = 0; t < n_tiles; ++t) {
        const int kb = __ldg(ids + t);
        const float cq = sq * __ldg(k_scale + bh * g.NB + kb);
        if (!warp_wait(bar(BS), t & 1, ctl)) { ok = false; break; }
        tc_fence_after();
        uint32_t sr[64];
        tmem_ld64(lane_addr + kColS + hc * 64, sr);
        tc_fence_before();
        mbar_arrive(bar(BSF));  // S may take the next Q K^T
        const int valid = g.N - kb * kBlock - hc * 64;
        const int32_t mi = half_max(sr, valid);
        if (mi == INT32_MIN) continue;  // no valid key in this half
        const float m_new = fmaxf(m_h, (__int_as_float(mi + kMagicBits) - kMagic) * cq);
        const float alpha = m_h == -INFINITY ? 0.f : ex2(m_h - m_new);
        float2 rs0 = make_float2(0.f, 0.f), rs1 = make_float2(0.f, 0.f);
        uint32_t pk[16];
        const float2 cq2 = make_float2(cq, cq), nm2 = make_float2(-m_new, -m_new);
        if (valid >= 64)
          tile_exp<false>(sr, cq2, nm2, valid, rs0, rs1, pk, 1.f);
        else
          tile_exp<true>(sr, cq2, nm2, valid, rs0, rs1, pk, 1.f);
        const float2 rs = fadd2(rs0, rs1);
        l_h = l_h * alpha + (rs.x + rs.y);
        m_h = m_new;
      }
      // ---- merge the two halves' (m, l): both partner warps form the same
      // row statistics
      float m = -INFINITY, inv_l = 0.f;
      if (ok && n_tiles > 0) {
        xch[hc * 128 + r] = m_h;
        xch[256 + hc * 128 + r] = l_h;
        mbar_arrive(bar(BMG));
        if (!all_wait(bar(BMG), 0, ctl)) ok = false;
        if (ok) {
          const float m_o = xch[(1 - hc) * 128 + r], l_o = xch[256 + (1 - hc) * 128 + r];
          m = fmaxf(m_h, m_o);
          const float l = (m_h == -INFINITY ? 0.f : l_h * ex2(m_h - m)) +
                          (m_o == -INFINITY ? 0.f : l_o * ex2(m_o - m));
          inv_l = l > 0.f ? 1.f / l : 0.f;
        }
      }
      // pad query rows (past N) take no part in a tile's maximum
      const bool row_valid = i * kBlock + r < g.N;
      float* amx = reinterpret_cast<float*>(smem_raw + kOffAmx);
      // ---- pass 2: normalised P, its per-tile maximum, codes, P V
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int t = n_tiles + j;
        const int kb = __ldg(ids + j);
        const float cq = sq * __ldg(k_scale + bh * g.NB + kb);
        const float vsc = __ldg(v_scale + bh * g.NB + kb);
        if (!warp_wait(bar(BS), t & 1, ctl)) { ok = false; break; }
        tc_fence_after();
        uint32_t sr[64];
        tmem_ld64(lane_addr + kColS + hc * 64, sr);
        tc_fence_before();
        mbar_arrive(bar(BSF));
        const int valid = g.N - kb * kBlock - hc * 64;
        const int32_t mi = half_max(sr, valid);
        // this row's largest P in the half: the same arithmetic as its
        // element's (below), so no code exceeds L
        float pmax = 0.f;
        if (row_valid && mi != INT32_MIN)
          pmax = ex2(fmaf(__int_as_float(mi + kMagicBits) - kMagic, cq, -m)) * inv_l;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) pmax = fmaxf(pmax, __shfl_xor_sync(0xffffffffu, pmax, o));
        if (lane == 0) {
          amx[(j & 1) * 8 + warp] = pmax;
          mbar_arrive(bar(BAM0 + (j & 1)));
        }
        // slot j & 1 is rewritten for tile j + 2 only after every warp
        // arrived for tile j + 1, i.e. after it read tile j's values
        if (!all_wait(bar(BAM0 + (j & 1)), (j >> 1) & 1, ctl)) { ok = false; break; }
        float a = amx[(j & 1) * 8];
#pragma unroll
        for (int w = 1; w < kSoftWarps; ++w) a = fmaxf(a, amx[(j & 1) * 8 + w]);
        if (hc == 0) {
          // O = O + (a / L) s_v (P8 V8): no rescale in this mode
          const int sl = j & (kScaleSlots - 1);
          s_alpha[sl * 128 + r] = 1.f;
          s_cv[sl * 128 + r] = __fdiv_rn(a, p_levels) * vsc;
          mbar_arrive(bar(BSC0 + sl));
        }
        // codes rne(L P / a) = rne(2^(s - m) * (L / (a l))); pad rows 0
        const float kq = a > 0.f && row_valid ? inv_l * __fdiv_rn(p_levels, a) : 0.f;
        const float2 cq2 = make_float2(cq, cq), nm2 = make_float2(-m, -m);
        float2 rs0 = make_float2(0.f, 0.f), rs1 = make_float2(0.f, 0.f);
        uint32_t pk[16];
        if (valid >= 64)
          tile_exp<false>(sr, cq2, nm2, valid, rs0, rs1, pk, kq);
        else
          tile_exp<true>(sr, cq2, nm2, valid, rs0, rs1, pk, kq);
        unsigned char* prow = smem_raw + kOffP + (j & 1) * kTile + r * 128;
#pragma unroll
        for (int u = 0; u < 4; ++u)
          *reinterpret_cast<uint4*>(prow + (((hc * 4 + u) ^ (r & 7)) << 4)) =
              make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
        fence_async_smem();
        mbar_arrive(bar(BP0 + (j & 1)));
      }
      if (ok && n_tiles > 0) {
        // O is already normalised: the epilogue divides by 1 + 0
        s_l[hc * 128 + r] = hc == 0 ? 1.f : 0.f;
        mbar_arrive(bar(BL));
      }
    } else {
      // kept index and block scales of the current tile, read a tile ahead
      int kb_next = 0;
      float ks_next = 0.f, vs_next = 0.f;
      if (n_tiles > 0) {
        kb_next = __ldg(ids);
        ks_next = __ldg(k_scale + bh * g.NB + kb_next);
        vs_next = __ldg(v_scale + bh * g.NB + kb_next);
      }
      for (int j = 0; j < n_tiles; ++j) {
        const int kb = kb_next;
        const float ksc = ks_next, vsc = vs_next;
        if (j + 1 < n_tiles) {
          kb_next = __ldg(ids + j + 1);
          ks_next = __ldg(k_scale + bh * g.NB + kb_next);
          vs_next = __ldg(v_scale + bh * g.NB + kb_next);
        }
        if (!warp_wait(bar(BS), j & 1, ctl)) { ok = false; break; }
        if (lane == 0 && quarter == 0) PARO_T8(3 + 3 * hc, j);
        tc_fence_after();
        uint32_t sr[64];
        tmem_ld64(lane_addr + kColS + hc * 64, sr);
        tc_fence_before();
        mbar_arrive(bar(BSF));  // S may take QK^T(j+1)
        const int valid = g.N - kb * kBlock - hc * 64;  // valid columns of this half
        const float cq = sq * ksc;
        // row max of this half in integers (cq >= 0 keeps the order)
        const int32_t mi = half_max(sr, valid);
        const float m_half =
            mi == INT32_MIN ? -INFINITY : (__int_as_float(mi + kMagicBits) - kMagic) * cq;
        // trade the half maxima with the partner warp (same rows, other half)
        float* xs = xch + (j & 1) * 256;
        xs[hc * 128 + r] = m_half;
        mbar_arrive(xbar);
        if (!all_wait(xbar, j & 1, ctl)) { ok = false; break; }
        if (lane == 0 && quarter == 0) PARO_T8(4 + 3 * hc, j);
        const float m_new = fmaxf(m_run, fmaxf(m_half, xs[(1 - hc) * 128 + r]));
        const float alpha = m_run == -INFINITY ? 0.f : ex2(m_run - m_new);
        if (hc == 0) {
          // slot j % 4 was last read by the correction of tile j - 4, which
          // completed before P V(j - 2) was issued, and so before QK(j)
          const int sl = j & (kScaleSlots - 1);
          s_alpha[sl * 128 + r] = alpha;
          s_cv[sl * 128 + r] = __fdiv_rn(vsc, p_levels);
          mbar_arrive(bar(BSC0 + sl));
        }
        // P~ = 2^(s - m) <= 1, P8 = rne(127 P~): the low byte of the float
        // 127 P~ + 1.5 * 2^23 (one rounding, to the nearest integer, ties even)
        const float2 cq2 = make_float2(cq, cq), nm2 = make_float2(-m_new, -m_new);
        float2 rs0 = make_float2(0.f, 0.f), rs1 = make_float2(0.f, 0.f);
        uint32_t pk[16];
        if (valid >= 64)
          tile_exp<false>(sr, cq2, nm2, valid, rs0, rs1, pk, p_levels);
        else
          tile_exp<true>(sr, cq2, nm2, valid, rs0, rs1, pk, p_levels);
        const float2 rs = fadd2(rs0, rs1);
        l2 = ffma2(l2, make_float2(alpha, alpha), rs);
        // this half row of P8 (64 bytes = 4 chunks of 16) into the swizzled
        // tile; the async proxy (the MMA) reads it after the fence
        unsigned char* prow = smem_raw + kOffP + (j & 1) * kTile + r * 128;
#pragma unroll
        for (int t = 0; t < 4; ++t)
          *reinterpret_cast<uint4*>(prow + (((hc * 4 + t) ^ (r & 7)) << 4)) =
              make_uint4(pk[4 * t], pk[4 * t + 1], pk[4 * t + 2], pk[4 * t + 3]);
        fence_async_smem();
        mbar_arrive(bar(BP0 + (j & 1)));
        if (lane == 0 && quarter == 0) PARO_T8(5 + 3 * hc, j);
        m_run = m_new;
      }
      if (ok && n_tiles > 0) {
        s_l[hc * 128 + r] = l2.x + l2.y;
        mbar_arrive(bar(BL));
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
                           const float* ks, const float* vs, float p_levels, bool p_tile,
                           void* out, int32_t* status, cudaStream_t s) {
  if (g.d != kD || g.block != kBlock) return cudaErrorInvalidValue;
  const uint64_t rows = (uint64_t)g.B * g.heads * g.Np;
  CUtensorMap mq{}, mk{}, mv{};
  if (!encode_tile_map(&mq, q, rows, kD, 1, 128, kBlock) ||
      !encode_tile_map(&mk, k, rows, kD, 1, 128, kBlock) ||
      !encode_tile_map(&mv, v, rows, kD, 1, 128, kBlock))
    return cudaErrorInvalidValue;
  auto kernel = p_tile ? attn_i8_kernel<true> : attn_i8_kernel<false>;
  cudaError_t e =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  const float c = (float)(1.4426950408889634 / sqrt((double)kD));
  dim3 grid(g.NB, g.B * g.heads);
  kernel<<<grid, kThreads, kSmemBytes, s>>>(mq, mk, mv, g, idx, counts, k_max, qs, ks, vs, c,
                                            p_levels, static_cast<__nv_bfloat16*>(out), status);
  return cudaGetLastError();
}

}  // namespace paro
