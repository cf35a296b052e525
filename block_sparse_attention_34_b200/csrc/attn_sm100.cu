// Block-sparse flash attention on the 5th-generation tensor cores of sm_100a
// (tcgen05.mma, accumulators in tensor memory), d = 128, block = 128, bf16.
//
// What it computes (SPADE, arXiv 2608.03335, Pith verdict page,
// key_machinery (iii): a flash block-sparse attention kernel with an online
// softmax over the kept block pairs; PAROAttention, arXiv 2506.16054, review
// key_machinery: the per-head axis order of the tokens, fused into the
// kernel's loads and stores): for query block i of head (b, h) and every key
// block j of its ascending kept list, S = Q_i K_j^T / sqrt(d), softmax, and
// O = sum_j P_j V_j / l, written to the natural positions of the block's
// tokens.
//
// One CTA per (query block, head); 12 warps with fixed roles:
//   warps 0-3  softmax A: the even-numbered kept tiles (0, 2, 4, ...);
//   warps 4-7  softmax B: the odd-numbered kept tiles.  A thread owns one
//              row of the 128-row tile (TMEM lane); each group keeps its own
//              running max, row sum and O accumulator in TMEM -- an exact
//              split of the row's kept keys into two disjoint sets -- and
//              the two partial results are merged once at the end
//              (O = (O_A 2^(m_A-m) + O_B 2^(m_B-m)) / (l_A 2^(m_A-m) +
//              l_B 2^(m_B-m))).  The two groups share the SM's sub-cores,
//              so the exponentials of one overlap the TMEM reads and max of
//              the other;
//   warp 8     allocates TMEM; one lane issues every tcgen05.mma and commit;
//   warp 9     gathers Q and then K tiles, warp 10 gathers V tiles, both with
//              TMA tile::gather4: lane l computes the natural positions of
//              rows 4l..4l+3 of the tile from the head's axis order and
//              issues two 4-row gathers (one per 64-column half) straight
//              into the 128-byte-swizzled operand layout, so the reorder
//              costs no pass over HBM;
//   warp 11    validates the kept list, then idles.
// Tensor memory (512 columns): S_A, S_B at columns 0 and 128, O_A, O_B at
// 256 and 384.  Shared memory: Q (32 KB), two-stage K and V rings
// (4 x 32 KB), P_A and P_B (2 x 32 KB) in the canonical K-major / MN-major
// SWIZZLE_128B layouts the MMA descriptors name.
//
// MMA issue order: QK(0), QK(1), PV(0), QK(2), PV(1), ... -- a K stage is
// refilled once the QK^T that read it completes, a V stage once its P V
// completes.  Every mbarrier wait is bounded (about one second of
// %globaltimer); on expiry the kernel records PA_ERR_TIMEOUT in the device
// status word, each role leaves its loop, in-flight TMA loads and MMAs are
// drained and TMEM is released before the CTA exits.
#include "sm100.cuh"

namespace paro {

#ifdef PARO_TRACE
// Phase trace (debug builds only): clock64() of each role's key events for
// one CTA, event e of tile j at g_paro_trace[e * 128 + j].
__device__ long long* g_paro_trace = nullptr;
__device__ int g_paro_trace_cta = 7;
#define PARO_T(ev, j)                                                                    \
  do {                                                                                   \
    if (g_paro_trace != nullptr && blockIdx.x == g_paro_trace_cta && blockIdx.y == 0 &&  \
        (j) < 128)                                                                       \
      g_paro_trace[(ev) * 128 + (j)] = clock64();                                        \
  } while (0)
#else
#define PARO_T(ev, j) \
  do {                \
  } while (0)
#endif

namespace {

using namespace sm100;

constexpr int kBlock = 128;
constexpr int kD = 128;
constexpr int kMmaWarp = 8;
constexpr int kKWarp = 9;
constexpr int kVWarp = 10;
constexpr int kCheckWarp = 11;
constexpr int kThreads = 12 * 32;  // 384
constexpr int kGroupThreads = 128;
constexpr uint32_t kTile = kBlock * kD * 2;  // 32 KB
constexpr uint32_t kHalf = kBlock * 128;     // 16 KB: 64 columns
// small region first: mbarriers, TMEM slot and flags, merge buffers
// [m, l][group][128 rows] float; the operand tiles start 1024-aligned
constexpr uint32_t kOffBar = 0;
constexpr uint32_t kOffSlot = 192;
constexpr uint32_t kOffMerge = 256;
constexpr uint32_t kSmall = 3072;
constexpr uint32_t kOffQ = kSmall;
constexpr uint32_t kOffK = kOffQ + kTile;      // 2 stages
constexpr uint32_t kOffV = kOffK + 2 * kTile;  // 2 stages
constexpr uint32_t kOffP = kOffV + 2 * kTile;  // P_A, P_B
constexpr uint32_t kSmemBytes = kOffP + 2 * kTile;  // 232,448 B = 227 KB
constexpr float kRescaleLog2 = 8.f;  // lazy rescale threshold (factor 256)
constexpr int kRegsLaunch = 168;  // 65,536 / 384 rounded down to a multiple of 8
constexpr int kRegsSoftmax = 200, kRegsAux = 56;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsAux <= kThreads * kRegsLaunch, "register split");
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 256;

enum : uint32_t {
  BQ = 0, BK0 = 1, BV0 = 3, BS0 = 5, BSF0 = 7, BP0 = 9, BPV0 = 11, BKF0 = 13, BDRAIN = 15,
  BM = 16, NBAR = 17
};
static_assert(NBAR * 8 <= kOffSlot, "barrier region");
static_assert(kOffMerge + 2 * 2 * 128 * 4 <= kSmall, "merge region");

// Natural row (in the [B*heads*N, d] matrix) of tile row p of head bh;
// pad rows (p >= N) point at the head's first row: their keys are masked
// to -inf and their query rows are never stored.
__device__ __forceinline__ int gather_row(const Grid& g, int order, int64_t bh, int p) {
  return (int)(bh * g.N) + (p < g.N ? natural_index(g, order, p) : 0);
}

// Lane l gathers rows 4l..4l+3 of a 128 x 128 bf16 tile (both halves).
__device__ __forceinline__ void gather_tile(uint32_t tile, const CUtensorMap* map, const Grid& g,
                                            int order, int64_t bh, int p0, int lane, uint32_t bar) {
  const int r = 4 * lane;
  const int r0 = gather_row(g, order, bh, p0 + r);
  const int r1 = gather_row(g, order, bh, p0 + r + 1);
  const int r2 = gather_row(g, order, bh, p0 + r + 2);
  const int r3 = gather_row(g, order, bh, p0 + r + 3);
  tma_gather4(tile + r * 128, map, 0, r0, r1, r2, r3, bar);
  tma_gather4(tile + kHalf + r * 128, map, 64, r0, r1, r2, r3, bar);
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_sm100_kernel(const __grid_constant__ CUtensorMap map_q,
                      const __grid_constant__ CUtensorMap map_k,
                      const __grid_constant__ CUtensorMap map_v, const __grid_constant__ Grid g,
                      const int32_t* __restrict__ idx, const int32_t* __restrict__ counts,
                      int k_max, float scale_log2, __nv_bfloat16* __restrict__ out,
                      int32_t* __restrict__ status) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // the operand tiles need 1024-byte alignment (the swizzle pattern repeats
  // every 8 rows of 128 bytes); dynamic shared memory starts at the window
  // base when, as here, there is no static shared memory
  const uint32_t base = smem_u32(smem_raw);
  if ((base & 1023u) != 0) {
    if (threadIdx.x == 0) report(status, PA_ERR_UNSUPPORTED);
    return;
  }
  unsigned char* gbase = smem_raw;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + kOffSlot);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  volatile uint32_t* bad_flag = tmem_slot + 2;
  float* merge = reinterpret_cast<float*>(gbase + kOffMerge);  // [m|l][group][row]
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
  // a wait of an earlier CTA of this launch already expired: end quickly
  const bool expired =
      status != nullptr && *reinterpret_cast<volatile int32_t*>(status) == PA_ERR_TIMEOUT;

  if (threadIdx.x == 0) {
    mbar_init(bar(BQ), 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(BK0 + s), 1);
      mbar_init(bar(BV0 + s), 1);
      mbar_init(bar(BS0 + s), 1);
      mbar_init(bar(BSF0 + s), kGroupThreads);
      mbar_init(bar(BP0 + s), kGroupThreads);
      mbar_init(bar(BPV0 + s), 1);
      mbar_init(bar(BKF0 + s), 1);
    }
    mbar_init(bar(BDRAIN), 1);
    mbar_init(bar(BM), 2 * kGroupThreads);
    *abort_flag = 0;
    *bad_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == kMmaWarp) tmem_alloc(smem_u32(tmem_slot), kTmemCols);
  if (warp == kCheckWarp) {
    // the kept list: count in range, indices ascending in [0, NB)
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
  // registers: launched at 168 per thread (384 x 168 = 64,512); the two
  // softmax warpgroups take 200, the MMA / gather / check warpgroup 56
  // (2 x 128 x 200 + 128 x 56 = 58,368 <= 64,512), and every warpgroup
  // returns to 168 before the common exit
  if (warp >= 8) {
  regs_dec<kRegsAux>();
  if (warp == kKWarp || warp == kVWarp) {
    // ------------------------------------------------------ gathers ----
    const bool is_k = warp == kKWarp;
    const CUtensorMap* map = is_k ? &map_k : &map_v;
    const uint32_t ring = base + (is_k ? kOffK : kOffV);
    int issued = 0;
    if (n_tiles > 0) {
      if (is_k) {
        if (lane == 0) mbar_arrive_tx(bar(BQ), kTile);
        __syncwarp();
        gather_tile(base + kOffQ, &map_q, g, order, bh, i * kBlock, lane, bar(BQ));
      }
      for (int j = 0; j < n_tiles; ++j) {
        const int s = j & 1;
        // the stage is free once QK^T (K) or P V (V) of tile j-2 completed
        if (j >= 2 && !warp_wait(bar((is_k ? BKF0 : BPV0) + s), ((j - 2) >> 1) & 1, ctl)) break;
        PARO_T(is_k ? 0 : 2, j);
        const int kb = __ldg(ids + j);
        if (lane == 0) mbar_arrive_tx(bar((is_k ? BK0 : BV0) + s), kTile);
        __syncwarp();
        gather_tile(ring + s * kTile, map, g, order, bh, kb * kBlock, lane,
                    bar((is_k ? BK0 : BV0) + s));
        issued = j + 1;
      }
      // on the way out make sure this warp's last loads have landed
      if (lane == 0) {
        if (is_k) drain_phase(bar(BQ), 0);
        for (int j = issued - 2 < 0 ? 0 : issued - 2; j < issued; ++j)
          drain_phase(bar((is_k ? BK0 : BV0) + (j & 1)), (j >> 1) & 1);
      }
    }
  } else if (warp == kMmaWarp) {
    // ---------------------------------------------------------- MMA ----
    if (lane == 0 && n_tiles > 0) {
      constexpr uint32_t id_qk = idesc_bf16(kBlock, kBlock, false);
      constexpr uint32_t id_pv = idesc_bf16(kBlock, kD, true);
      bool ok = wait_phase(bar(BQ), 0, ctl);
      auto issue_pv = [&](int jp) -> bool {
        const int b = jp & 1;
        if (!wait_phase(bar(BP0 + b), (jp >> 1) & 1, ctl)) return false;
        if (!wait_phase(bar(BV0 + b), (jp >> 1) & 1, ctl)) return false;
        tc_fence_after();
        const uint32_t pa = base + kOffP + b * kTile;
        const uint32_t va = base + kOffV + b * kTile;
#pragma unroll
        for (int kk = 0; kk < kBlock / 16; ++kk) {
          const uint64_t ad = sw128_desc(pa + (kk >> 2) * kHalf + (kk & 3) * 32, 16, 1024);
          const uint64_t bd = sw128_desc(va + kk * 16 * 128, kHalf, 1024);
          mma_f16_ss(tmem + kColO + b * 128, ad, bd, id_pv, (jp >= 2 || kk > 0) ? 1u : 0u);
        }
        mma_commit(bar(BPV0 + b));
        PARO_T(5, jp);
        return true;
      };
      for (int j = 0; ok && j < n_tiles; ++j) {
        const int b = j & 1;
        if (!wait_phase(bar(BK0 + b), (j >> 1) & 1, ctl)) { ok = false; break; }
        if (j >= 2 && !wait_phase(bar(BSF0 + b), ((j - 2) >> 1) & 1, ctl)) { ok = false; break; }
        tc_fence_after();
        const uint32_t ka = base + kOffK + b * kTile;
#pragma unroll
        for (int kk = 0; kk < kD / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
          mma_f16_ss(tmem + kColS + b * 128, sw128_desc(base + kOffQ + off, 16, 1024),
                     sw128_desc(ka + off, 16, 1024), id_qk, kk > 0 ? 1u : 0u);
        }
        mma_commit(bar(BS0 + b));
        mma_commit(bar(BKF0 + b));
        PARO_T(4, j);
        if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
      }
      if (ok) issue_pv(n_tiles - 1);
      // drain: every MMA issued above has completed once this commit fires
      mma_commit(bar(BDRAIN));
      drain_phase(bar(BDRAIN), 0);
    }
  }
  __syncwarp();  // setmaxnreg is warp-aligned: reconverge after the lane-0 roles
  regs_inc<kRegsLaunch>();
  } else {
    regs_inc<kRegsSoftmax>();
    // ------------------------------------------------------ softmax ----
    const int grp = warp >> 2;  // 0: even tiles, 1: odd tiles
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // tile row == TMEM lane
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    const uint32_t s_col = kColS + grp * 128, o_col = kColO + grp * 128;
    unsigned char* pt = gbase + kOffP + grp * kTile;
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    int t = 0;  // this group's tile counter
    for (int j = grp; j < n_tiles; j += 2, ++t) {
      if (!warp_wait(bar(BS0 + grp), t & 1, ctl)) { ok = false; break; }
      if (lane == 0 && quarter == 0) PARO_T(6 + 4 * grp, j);
      tc_fence_after();
      uint32_t sr[128];
      tmem_ld128(lane_addr + s_col, sr);
      tc_fence_before();
      mbar_arrive(bar(BSF0 + grp));
      if (lane == 0 && quarter == 0) PARO_T(7 + 4 * grp, j);
      const int kb = __ldg(ids + j);
      const int valid = g.N - kb * kBlock;  // keys of this block that exist
      if (valid < kBlock) {  // only the ragged last block (warp-uniform)
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c >= valid) sr[c] = __float_as_uint(-INFINITY);
      }
      float mp[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) mp[u] = __uint_as_float(sr[u]);
#pragma unroll
      for (int c = 8; c < 128; ++c) mp[c & 7] = fmaxf(mp[c & 7], __uint_as_float(sr[c]));
      const float mx = fmaxf(fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3])),
                             fmaxf(fmaxf(mp[4], mp[5]), fmaxf(mp[6], mp[7]))) *
                       scale_log2;
      if (lane == 0 && quarter == 0) PARO_T(8 + 4 * grp, j);
      // lazy rescale: keep the reference max unless the row max grew by
      // more than 2^8 (exact either way: O and l share the reference)
      const bool need = t == 0 ? false : (mx > m_used + kRescaleLog2);
      if (t == 0) m_used = mx == -INFINITY ? 0.f : mx;
      if (t >= 1) {
        // O_grp and P_grp are free once P V of this group's previous tile
        // (tile j-2) completed
        if (!warp_wait(bar(BPV0 + grp), (t - 1) & 1, ctl)) { ok = false; break; }
        if (__any_sync(0xffffffffu, need)) {
          tc_fence_after();
          const float alpha = need ? ex2(m_used - mx) : 1.f;
#pragma unroll 1
          for (int c0 = 0; c0 < 128; c0 += 32) {
            uint32_t orr[32];
            tmem_ld32(lane_addr + o_col + c0, orr);
#pragma unroll
            for (int c = 0; c < 32; ++c) orr[c] = __float_as_uint(__uint_as_float(orr[c]) * alpha);
            tmem_st32(lane_addr + o_col + c0, orr);
          }
          l *= alpha;
          if (need) m_used = mx;
        }
      }
      // P = 2^(s*scale - m) in bf16 into the swizzled K-major P tile; row
      // sum in 8 independent chains
      const float neg_m = -m_used;
      float rs[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) rs[u] = 0.f;
#pragma unroll
      for (int c = 0; c < 16; ++c) {
        float e[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          e[u] = ex2(fmaf(__uint_as_float(sr[c * 8 + u]), scale_log2, neg_m));
          rs[u] += e[u];
        }
        uint4 w;
        w.x = pack_bf16(e[0], e[1]);
        w.y = pack_bf16(e[2], e[3]);
        w.z = pack_bf16(e[4], e[5]);
        w.w = pack_bf16(e[6], e[7]);
        *reinterpret_cast<uint4*>(pt + (c >> 3) * kHalf + sw128_off(r, c & 7)) = w;
      }
      l += ((rs[0] + rs[1]) + (rs[2] + rs[3])) + ((rs[4] + rs[5]) + (rs[6] + rs[7]));
      if (lane == 0 && quarter == 0) PARO_T(9 + 4 * grp, j);
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(bar(BP0 + grp));
    }
    // ---- merge the two groups and store (group g writes columns 64g..)
    const int p = i * kBlock + r;
    __nv_bfloat16* orow = p < g.N ? out + (bh * (int64_t)g.N + natural_index(g, order, p)) * kD
                                  : nullptr;
    if (run && cnt == 0) {
      if (orow != nullptr)
        for (int c = 0; c < 8; ++c)
          reinterpret_cast<uint4*>(orow + grp * 64)[c] = make_uint4(0, 0, 0, 0);
    } else if (ok && n_tiles > 0) {
      const bool has_b = n_tiles >= 2;
      merge[(0 * 2 + grp) * 128 + r] = m_used;
      merge[(1 * 2 + grp) * 128 + r] = l;
      mbar_arrive(bar(BM));
      bool okm = all_wait(bar(BM), 0, ctl);
      float fa = 0.f, fb = 0.f, lt = 0.f;
      if (okm) {
        const float ma = merge[r], mb = has_b ? merge[128 + r] : -INFINITY;
        const float m = fmaxf(ma, mb);
        fa = ex2(ma - m);
        fb = has_b ? ex2(mb - m) : 0.f;
        lt = merge[256 + r] * fa + (has_b ? merge[384 + r] * fb : 0.f);
      }
      // both groups' last P V must be complete
      for (int gg = 0; okm && gg < 2; ++gg) {
        if (gg == 1 && !has_b) continue;
        const int jl = ((n_tiles - 1) & 1) == gg ? n_tiles - 1 : n_tiles - 2;
        okm = warp_wait(bar(BPV0 + gg), (jl >> 1) & 1, ctl);
      }
      if (okm) {
        tc_fence_after();
        const float inv = lt > 0.f ? 1.f / lt : 0.f;
        fa *= inv;
        fb *= inv;
#pragma unroll 1
        for (int c0 = 0; c0 < 64; c0 += 32) {
          const int col = grp * 64 + c0;
          uint32_t oa[32], ob[32];
          tmem_ld32(lane_addr + kColO + col, oa);
          if (has_b) {
            tmem_ld32(lane_addr + kColO + 128 + col, ob);
          } else {
#pragma unroll
            for (int c = 0; c < 32; ++c) ob[c] = 0u;
          }
          if (orow != nullptr) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              float v[8];
#pragma unroll
              for (int u = 0; u < 8; ++u)
                v[u] = __uint_as_float(oa[c * 8 + u]) * fa + __uint_as_float(ob[c * 8 + u]) * fb;
              uint4 w;
              w.x = pack_bf16(v[0], v[1]);
              w.y = pack_bf16(v[2], v[3]);
              w.z = pack_bf16(v[4], v[5]);
              w.w = pack_bf16(v[6], v[7]);
              reinterpret_cast<uint4*>(orow + col)[c] = w;
            }
          }
        }
      }
    }
    __syncwarp();
    regs_dec<kRegsLaunch>();
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

bool attn_sm100_supports(pa_dtype dt, const Grid& g) {
  return dt == PA_BF16 && g.d == kD && g.block == kBlock &&
         (int64_t)g.B * g.heads * g.N < ((int64_t)1 << 31);
}

cudaError_t launch_attn_sm100(const void* q, const void* k, const void* v, pa_dtype dt,
                              const Grid& g, const int32_t* idx, const int32_t* counts,
                              int k_max, const float* qs, const float* ks, const float* vs,
                              void* out, int32_t* status, cudaStream_t s) {
  (void)qs;
  (void)ks;
  (void)vs;
  if (!attn_sm100_supports(dt, g)) return cudaErrorInvalidValue;
  const uint64_t rows = (uint64_t)g.B * g.heads * g.N;
  CUtensorMap mq, mk, mv;
  if (!encode_gather_map(&mq, q, rows, kD, 2, 64) || !encode_gather_map(&mk, k, rows, kD, 2, 64) ||
      !encode_gather_map(&mv, v, rows, kD, 2, 64))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(attn_sm100_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  const float scale_log2 = (float)(1.4426950408889634 / sqrt((double)kD));
  dim3 grid(g.NB, g.B * g.heads);
  attn_sm100_kernel<<<grid, kThreads, kSmemBytes, s>>>(mq, mk, mv, g, idx, counts, k_max,
                                                       scale_log2,
                                                       static_cast<__nv_bfloat16*>(out), status);
  return cudaGetLastError();
}

}  // namespace paro
