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
//   warps 0-3  softmax group 0: the even-numbered kept tiles (0, 2, 4, ...);
//   warps 4-7  softmax group 1: the odd-numbered kept tiles.
//              Warp w of a group owns rows 32*(w%4) .. +31 (its tensor
//              memory lane quarter), one row per thread, all 128 keys of
//              the tile.  Each group keeps its own running max, row sum and
//              O accumulator: the even and the odd tiles are an exact split
//              of the row's keys, merged once at the end,
//              O = (O_0 2^(m_0-m) + O_1 2^(m_1-m)) / (l_0 2^(m_0-m) +
//              l_1 2^(m_1-m)).  The two groups work on consecutive tiles at
//              the same time, so one group's exponentials overlap the other
//              group's S read and the tensor cores' QK^T and P V of both.
//              A thread reads its row of S (128 fp32) from tensor memory,
//              writes its 128 probabilities as bf16 pairs over the first 64
//              columns of the same S buffer (the P V MMA's A operand), and
//              when its max grows by more than 2^8 rescales its O row;
//   warp 8     allocates tensor memory; one lane issues every tcgen05.mma
//              and commit;
//   warp 9     loads Q, then K tiles; warp 10 loads V tiles.  With inputs in
//              the permuted order (pa_reorder) every tile is 128 contiguous
//              rows: one lane issues two TMA tiled boxes (one per 64-column
//              half) into the 128-byte-swizzled operand layout.  With
//              natural-order inputs the warp gathers the token rows itself
//              (16-byte cp.async, 16 lanes per 256-byte row, natural
//              positions from the head's axis order) and each lane's arrival
//              on the stage's mbarrier fires when its copies land;
//   warp 11    validates the kept list, then idles.
// Tensor memory (512 columns): S/P of the even tiles at 0, of the odd tiles
// at 128; O_0 at 256, O_1 at 384.  Shared memory: Q (32 KB) and three-stage
// K and V rings (6 x 32 KB) in the canonical K-major / MN-major
// SWIZZLE_128B layouts the MMA descriptors name.
//
// MMA issue order QK(0), QK(1), PV(0), QK(2), PV(1), QK(3), ...: QK^T of
// tile j+2 reuses the S buffer whose P(j) the P V(j) just issued reads; the
// tcgen05.mma operations of one thread execute in issue order, so the
// overwrite follows the read.  A K stage is refilled once its QK^T
// completes, a V stage once its P V completes.  Every mbarrier wait is
// bounded (about one second of %globaltimer); on expiry the kernel records
// PA_ERR_TIMEOUT in the device status word, each role leaves its loop,
// in-flight copies and MMAs are drained and tensor memory is released
// before the CTA exits.
#include "sm100.cuh"

namespace paro {

namespace {

using namespace sm100;

constexpr int kBlock = 128;
constexpr int kD = 128;
constexpr int kStages = 3;
constexpr int kMmaWarp = 8;
constexpr int kKWarp = 9;
constexpr int kVWarp = 10;
constexpr int kCheckWarp = 11;
constexpr int kThreads = 12 * 32;  // 384
constexpr int kGroupThreads = 128;  // one softmax group
constexpr uint32_t kTile = kBlock * kD * 2;  // 32 KB
constexpr uint32_t kHalf = kBlock * 128;     // 16 KB: 64 columns
// small region first: mbarriers, TMEM slot and flags, the final merge
// buffer [m, l][2 groups][128 rows] float; the operand tiles start
// 1024-aligned
constexpr uint32_t kOffBar = 0;
constexpr uint32_t kOffSlot = 256;
constexpr uint32_t kOffMerge = 512;
constexpr uint32_t kSmall = 3072;
constexpr uint32_t kOffQ = kSmall;
constexpr uint32_t kOffK = kOffQ + kTile;            // kStages stages
constexpr uint32_t kOffV = kOffK + kStages * kTile;  // kStages stages
constexpr uint32_t kSmemBytes = kOffV + kStages * kTile;  // 232,448 B = 227 KB
constexpr float kRescaleLog2 = 8.f;  // lazy rescale threshold (factor 256)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 256;  // + 128 * group

enum : uint32_t {
  BQ = 0,
  BK0 = 1,    // K stage full (3)
  BV0 = 4,    // V stage full (3)
  BKF0 = 7,   // K stage free (3)
  BVF0 = 10,  // V stage free (3)
  BS0 = 13,   // S of the group's next tile ready (2, by group)
  BP0 = 15,   // P written by every thread of the group (2)
  BPV0 = 17,  // P V of the group's tile complete (2)
  BDRAIN = 19,
  BM = 20,    // final merge exchange
  NBAR = 21
};
static_assert(NBAR * 8 <= kOffSlot, "barrier region");
static_assert(kOffMerge + 2 * 2 * 128 * 4 <= kSmall, "merge region");

// One warp copies a 128 x 128 bf16 tile whose row r is the token at
// permuted position p0 + r of head `head` (rows past N zero-filled).  Lane l
// first finds the natural positions of rows l, l+32, l+64, l+96; copy m
// moves row 2m (lanes 0-15) and row 2m+1 (lanes 16-31), 16 bytes per lane.
__device__ __forceinline__ void copy_tile(uint32_t tile, const __nv_bfloat16* __restrict__ head,
                                          const Grid& g, int order, int p0, int lane) {
  int nat[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int p = p0 + 32 * q + lane;
    nat[q] = p < g.N ? natural_index(g, order, p) : -1;
  }
  const int c16 = lane & 15, half = c16 >> 3, c = c16 & 7;
  const char* src0 = reinterpret_cast<const char*>(head) + c16 * 16;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
#pragma unroll 8
    for (int m = 0; m < 16; ++m) {
      const int rr = 2 * m + (lane >> 4);  // row within this 32-row group
      const int n = __shfl_sync(0xffffffffu, nat[q], rr);
      const int r = 32 * q + rr;
      cp_async16(tile + half * kHalf + sw128_off(r, c),
                 src0 + (n >= 0 ? (int64_t)n * (kD * 2) : 0), n >= 0 ? 16u : 0u);
    }
  }
}

// kTma: q, k, v are in the permuted order ([B*heads*N_p, d], as written by
// pa_reorder): every tile is 128 contiguous rows, loaded with two TMA tiled
// boxes (one per 64-column half) by one lane.  Otherwise q, k, v are in the
// natural order and the copy warps gather the rows with cp.async.
template <bool kTma>
__global__ void __launch_bounds__(kThreads, 1)
    attn_sm100_kernel(const __grid_constant__ CUtensorMap map_q,
                      const __grid_constant__ CUtensorMap map_k,
                      const __grid_constant__ CUtensorMap map_v,
                      const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                      const __nv_bfloat16* __restrict__ v, const __grid_constant__ Grid g,
                      const int32_t* __restrict__ idx, const int32_t* __restrict__ counts,
                      int k_max, float scale_log2, __nv_bfloat16* __restrict__ out,
                      int32_t* __restrict__ status, const StallTest st) {
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
  const Ctl ctl{abort_flag, status, st.limit_ns};
  // a wait of an earlier CTA of this launch already expired: end quickly
  const bool expired =
      status != nullptr && *reinterpret_cast<volatile int32_t*>(status) == PA_ERR_TIMEOUT;

  if (threadIdx.x == 0) {
    constexpr uint32_t kLoadArrivals = kTma ? 1 : 32;  // one expect-tx, or one per lane
    mbar_init(bar(BQ), kLoadArrivals);
    for (int s = 0; s < kStages; ++s) {
      mbar_init(bar(BK0 + s), kLoadArrivals);
      mbar_init(bar(BV0 + s), kLoadArrivals);
      mbar_init(bar(BKF0 + s), 1);
      mbar_init(bar(BVF0 + s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(BS0 + b), 1);
      mbar_init(bar(BP0 + b), kGroupThreads);
      mbar_init(bar(BPV0 + b), 1);
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
  const __nv_bfloat16* qh = q + bh * (int64_t)g.N * kD;
  const __nv_bfloat16* kh = k + bh * (int64_t)g.N * kD;
  const __nv_bfloat16* vh = v + bh * (int64_t)g.N * kD;

  if (warp >= 8) {
    if (warp == kKWarp || warp == kVWarp) {
      // ---------------------------------------------------- copies ----
      const bool is_k = warp == kKWarp;
      const __nv_bfloat16* src = is_k ? kh : vh;
      const CUtensorMap* map = is_k ? &map_k : &map_v;
      const uint32_t ring = base + (is_k ? kOffK : kOffV);
      const int row0 = (int)(bh * g.Np);  // first row of this head (permuted order)
      int issued = 0;
      if (n_tiles > 0) {
        if (is_k) {
          if constexpr (kTma) {
            if (lane == 0) {
              mbar_arrive_tx(bar(BQ), kTile);
              tma_load_2d(base + kOffQ, &map_q, 0, row0 + i * kBlock, bar(BQ));
              tma_load_2d(base + kOffQ + kHalf, &map_q, 64, row0 + i * kBlock, bar(BQ));
            }
          } else {
            copy_tile(base + kOffQ, qh, g, order, i * kBlock, lane);
            cp_async_arrive(bar(BQ));
          }
        }
        for (int j = 0; j < n_tiles; ++j) {
          const int s = j % kStages;
          // the stage is free once QK^T (K) or P V (V) of tile j-3 completed
          if (j >= kStages &&
              !warp_wait(bar((is_k ? BKF0 : BVF0) + s), ((j / kStages) - 1) & 1, ctl))
            break;
          const int kb = __ldg(ids + j);
          const uint32_t full = bar((is_k ? BK0 : BV0) + s);
          if (!is_k && j == st.tile && i == st.cta_x && bh == st.cta_y) {
            issued = j + 1;  // test hook: this tile never arrives
            continue;
          }
          if constexpr (kTma) {
            if (lane == 0) {
              mbar_arrive_tx(full, kTile);
              tma_load_2d(ring + s * kTile, map, 0, row0 + kb * kBlock, full);
              tma_load_2d(ring + s * kTile + kHalf, map, 64, row0 + kb * kBlock, full);
            }
          } else {
            copy_tile(ring + s * kTile, src, g, order, kb * kBlock, lane);
            cp_async_arrive(full);
          }
          issued = j + 1;
        }
        // on every path this warp's copies have landed before it leaves
        if constexpr (kTma) {
          if (lane == 0) {
            if (is_k) drain_phase(bar(BQ), 0, ctl.limit_ns);
            for (int j = issued > kStages ? issued - kStages : 0; j < issued; ++j)
              drain_phase(bar((is_k ? BK0 : BV0) + j % kStages), (j / kStages) & 1,
                          ctl.limit_ns);
          }
        } else {
          cp_async_wait_all();
        }
      }
    } else if (warp == kMmaWarp) {
      // -------------------------------------------------------- MMA ----
      if (lane == 0 && n_tiles > 0) {
        constexpr uint32_t id_qk = idesc_bf16(kBlock, kBlock, false);
        constexpr uint32_t id_pv = idesc_bf16(kBlock, kD, true);
        bool ok = wait_phase(bar(BQ), 0, ctl);
        fence_async_smem();  // cp.async (generic proxy) writes -> MMA operand reads
        // QK^T of tile j into S buffer j & 1: needs K(j); the buffer's
        // previous contents, P(j-2), are read by P V(j-2), issued before
        auto issue_qk = [&](int j) -> bool {
          const int s = j % kStages, b = j & 1;
          if (!wait_phase(bar(BK0 + s), (j / kStages) & 1, ctl)) return false;
          fence_async_smem();
          tc_fence_after();
          const uint32_t ka = base + kOffK + s * kTile;
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk) {
            const uint32_t off = (kk >> 2) * kHalf + (kk & 3) * 32;
            mma_f16_ss(tmem + kColS + b * 128, sw128_desc(base + kOffQ + off, 16, 1024),
                       sw128_desc(ka + off, 16, 1024), id_qk, kk > 0 ? 1u : 0u);
          }
          mma_commit(bar(BS0 + b));
          mma_commit(bar(BKF0 + s));
          return true;
        };
        // O_b += P(j) V(j), b = j & 1: P (bf16 pairs) from the first 64
        // columns of S buffer b, V from the ring
        auto issue_pv = [&](int j) -> bool {
          const int b = j & 1, s = j % kStages;
          if (!wait_phase(bar(BP0 + b), (j >> 1) & 1, ctl)) return false;
          if (!wait_phase(bar(BV0 + s), (j / kStages) & 1, ctl)) return false;
          fence_async_smem();
          tc_fence_after();
          const uint32_t va = base + kOffV + s * kTile;
#pragma unroll
          for (int kk = 0; kk < kBlock / 16; ++kk)
            mma_f16_ts(tmem + kColO + b * 128, tmem + kColS + b * 128 + kk * 8,
                       sw128_desc(va + kk * 16 * 128, kHalf, 1024), id_pv,
                       (j >= 2 || kk > 0) ? 1u : 0u);
          mma_commit(bar(BPV0 + b));
          mma_commit(bar(BVF0 + s));
          return true;
        };
        ok = ok && issue_qk(0);
        if (ok && n_tiles > 1) ok = issue_qk(1);
        for (int j = 0; ok && j < n_tiles; ++j) {
          if (!issue_pv(j)) { ok = false; break; }
          if (j + 2 < n_tiles && !issue_qk(j + 2)) { ok = false; break; }
        }
        // drain: every MMA issued above has completed once this commit fires
        mma_commit(bar(BDRAIN));
        drain_phase(bar(BDRAIN), 0, ctl.limit_ns);
      }
    }
    __syncwarp();  // reconverge after the lane-0 roles
  } else {
    // ------------------------------------------------------ softmax ----
    const int grp = warp >> 2;  // 0: even tiles, 1: odd tiles
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;  // tile row == TMEM lane
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    const uint32_t s_col = kColS + grp * 128;
    const uint32_t o_col = kColO + grp * 128;
    float m_used = -INFINITY, l = 0.f;  // this group's reference max and row sum
    bool ok = true;
    for (int t = 0;; ++t) {
      const int j = 2 * t + grp;
      if (j >= n_tiles) break;
      if (!warp_wait(bar(BS0 + grp), t & 1, ctl)) { ok = false; break; }
      tc_fence_after();
      uint32_t sr[128];
      tmem_ld128(lane_addr + s_col, sr);
      const int valid = g.N - __ldg(ids + j) * kBlock;  // existing keys of the tile
      if (valid < kBlock) {  // only the ragged last block (warp-uniform)
#pragma unroll
        for (int c = 0; c < kBlock; ++c)
          if (c >= valid) sr[c] = __float_as_uint(-INFINITY);
      }
      float mp[8];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        mp[u] = fmax3(__uint_as_float(sr[u]), __uint_as_float(sr[u + 8]),
                      __uint_as_float(sr[u + 16]));
      // columns 24..127 in steps of 16 (the last step takes 120..127 alone)
#pragma unroll
      for (int c = 24; c < kBlock; c += 16)
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (c + u + 8 < kBlock)
            mp[u] = fmax3(mp[u], __uint_as_float(sr[c + u]), __uint_as_float(sr[c + u + 8]));
          else if (c + u < kBlock)
            mp[u] = fmaxf(mp[u], __uint_as_float(sr[c + u]));
      const float mx = fmax3(fmax3(mp[0], mp[1], mp[2]), fmax3(mp[3], mp[4], mp[5]),
                             fmaxf(mp[6], mp[7])) *
                       scale_log2;
      // lazy rescale: keep the reference max unless this row's max grew by
      // more than 2^8 (exact either way: O and l share the reference)
      const bool first = m_used == -INFINITY;
      const bool need = !first && mx > m_used + kRescaleLog2;
      const float alpha = need ? ex2(m_used - mx) : 1.f;
      if (first || need) m_used = mx;  // a tile has at least one existing key
      // P = 2^(s*scale - m) as bf16 pairs over the first 64 columns of the S
      // buffer (its fp32 values are all in registers); row sum in 8 chains
      const float neg_m = -m_used;
      float rs[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) rs[u] = 0.f;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const int e = 32 * cc + 2 * c;
          const float e0 = ex2(fmaf(__uint_as_float(sr[e]), scale_log2, neg_m));
          const float e1 = ex2(fmaf(__uint_as_float(sr[e + 1]), scale_log2, neg_m));
          rs[e & 7] += e0;
          rs[(e + 1) & 7] += e1;
          pk[c] = pack_bf16(e0, e1);
        }
        tmem_st16_async(lane_addr + s_col + 16 * cc, pk);
      }
      tmem_wait_st();
      l = l * alpha + (((rs[0] + rs[1]) + (rs[2] + rs[3])) + ((rs[4] + rs[5]) + (rs[6] + rs[7])));
      if (__any_sync(0xffffffffu, need)) {
        // O holds P V up to this group's previous tile once that MMA
        // completed; P V of this tile is issued after the arrival below
        if (!warp_wait(bar(BPV0 + grp), (t - 1) & 1, ctl)) { ok = false; break; }
        tc_fence_after();
#pragma unroll 1
        for (int c0 = 0; c0 < 128; c0 += 32) {
          uint32_t orr[32];
          tmem_ld32(lane_addr + o_col + c0, orr);
#pragma unroll
          for (int c = 0; c < 32; ++c) orr[c] = __float_as_uint(__uint_as_float(orr[c]) * alpha);
          tmem_st32(lane_addr + o_col + c0, orr);
        }
      }
      tc_fence_before();
      mbar_arrive(bar(BP0 + grp));
    }
    // ---- epilogue: merge the groups, then group g writes output columns
    // 64g .. 64g+63 of the row at the natural position of its token
    const int p = i * kBlock + r;
    __nv_bfloat16* orow = p < g.N ? out + (bh * (int64_t)g.N + natural_index(g, order, p)) * kD
                                  : nullptr;
    if (run && cnt == 0) {
      if (orow != nullptr)
        for (int c = 0; c < 8; ++c)
          reinterpret_cast<uint4*>(orow + grp * 64)[c] = make_uint4(0, 0, 0, 0);
    } else if (ok && n_tiles > 0) {
      merge[(0 * 2 + grp) * 128 + r] = m_used;
      merge[(1 * 2 + grp) * 128 + r] = l;
      mbar_arrive(bar(BM));
      bool okm = all_wait(bar(BM), 0, ctl);
      float f0 = 0.f, f1 = 0.f, lt = 0.f;
      if (okm) {
        const float m0 = merge[r], m1 = merge[128 + r];
        const float m = fmaxf(m0, m1);
        // a group that saw no tile (a one-tile list) has l = 0 and an
        // unwritten O: weight 0
        f0 = m0 == -INFINITY ? 0.f : ex2(m0 - m);
        f1 = m1 == -INFINITY ? 0.f : ex2(m1 - m);
        lt = merge[256 + r] * f0 + merge[384 + r] * f1;
      }
      // every P V has completed once the MMA lane's drain commit fired
      if (okm) okm = warp_wait(bar(BDRAIN), 0, ctl);
      if (okm) {
        tc_fence_after();
        const float inv = lt > 0.f ? 1.f / lt : 0.f;
        f0 *= inv;
        f1 *= inv;
#pragma unroll 1
        for (int c0 = 0; c0 < 64; c0 += 32) {
          const int col = grp * 64 + c0;
          uint32_t oa[32], ob[32];
          tmem_ld32x2(lane_addr + kColO + col, oa, lane_addr + kColO + 128 + col, ob);
          if (orow != nullptr) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              float vv[8];
#pragma unroll
              for (int u = 0; u < 8; ++u) {
                const float a0 = f0 != 0.f ? __uint_as_float(oa[c * 8 + u]) * f0 : 0.f;
                const float a1 = f1 != 0.f ? __uint_as_float(ob[c * 8 + u]) * f1 : 0.f;
                vv[u] = a0 + a1;
              }
              uint4 w;
              w.x = pack_bf16(vv[0], vv[1]);
              w.y = pack_bf16(vv[2], vv[3]);
              w.z = pack_bf16(vv[4], vv[5]);
              w.w = pack_bf16(vv[6], vv[7]);
              reinterpret_cast<uint4*>(orow + col)[c] = w;
            }
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

template <bool kTma>
cudaError_t launch_typed(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                         const void* q, const void* k, const void* v, const Grid& g,
                         const int32_t* idx, const int32_t* counts, int k_max, void* out,
                         int32_t* status, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(attn_sm100_kernel<kTma>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  const float scale_log2 = (float)(1.4426950408889634 / sqrt((double)kD));
  dim3 grid(g.NB, g.B * g.heads);
  attn_sm100_kernel<kTma><<<grid, kThreads, kSmemBytes, s>>>(
      mq, mk, mv, static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
      static_cast<const __nv_bfloat16*>(v), g, idx, counts, k_max, scale_log2,
      static_cast<__nv_bfloat16*>(out), status, stall_test());
  return cudaGetLastError();
}

}  // namespace

bool attn_sm100_supports(pa_dtype dt, const Grid& g) {
  return (dt == PA_BF16 || dt == PA_I8) && g.d == kD && g.block == kBlock &&
         (int64_t)g.B * g.heads * g.Np < ((int64_t)1 << 31);
}

cudaError_t launch_attn_sm100(const void* q, const void* k, const void* v, pa_dtype dt,
                              const Grid& g, const int32_t* idx, const int32_t* counts,
                              int k_max, const float* qs, const float* ks, const float* vs,
                              float p_levels, void* out, int32_t* status, bool permuted,
                              cudaStream_t s) {
  if (!attn_sm100_supports(dt, g)) return cudaErrorInvalidValue;
  if (dt == PA_I8)
    return launch_attn_i8(q, k, v, g, idx, counts, k_max, qs, ks, vs, p_levels, out, status, s);
  CUtensorMap mq{}, mk{}, mv{};
  if (permuted) {
    const uint64_t rows = (uint64_t)g.B * g.heads * g.Np;
    if (!encode_tile_map(&mq, q, rows, kD, 2, 64, kBlock) ||
        !encode_tile_map(&mk, k, rows, kD, 2, 64, kBlock) ||
        !encode_tile_map(&mv, v, rows, kD, 2, 64, kBlock))
      return cudaErrorInvalidValue;
    return launch_typed<true>(mq, mk, mv, q, k, v, g, idx, counts, k_max, out, status, s);
  }
  return launch_typed<false>(mq, mk, mv, q, k, v, g, idx, counts, k_max, out, status, s);
}

}  // namespace paro
