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
//              the tile.  A thread copies its row of S (128 fp32) from the
//              group's S buffer into registers and releases the buffer, so
//              QK^T two tiles ahead can start at once; it then computes
//              its 128 probabilities as bf16 pairs in registers (scale,
//              subtract and row sums as paired f32x2 instructions) and
//              writes them into the group's P buffer (the P V MMA's A
//              operand) once P V of the group's previous tile completed.  Both groups accumulate into one
//              O, so every row has one reference max m_j, passed along the
//              tile order through shared memory: m_j = m_{j-1} unless tile
//              j's max exceeds it by more than 2^8 (then m_j is that max and
//              the group rescales O after P V(j-1) and before P V(j): the
//              rescale is lazy and exact).  Each group keeps its own row
//              sum relative to the latest reference it used; the two are
//              added at the end;
//   warp 8     allocates tensor memory; one lane issues every tcgen05.mma
//              and commit, in the order QK(0), QK(1), then QK(j+2), PV(j)
//              for j = 0, 1, ...;
//   warp 9     loads Q, then K tiles; warp 10 loads V tiles.  With inputs in
//              the permuted order (pa_reorder) every tile is 128 contiguous
//              rows: one lane issues two TMA tiled boxes (one per 64-column
//              half) into the 128-byte-swizzled operand layout.  With
//              natural-order inputs the warp gathers the token rows itself
//              (16-byte cp.async, 16 lanes per 256-byte row, natural
//              positions from the head's axis order) and each lane's arrival
//              on the stage's mbarrier fires when its copies land.  The kept
//              block indices are read 32 at a time and passed by shuffle;
//   warp 11    validates the kept list, then idles.
// Tensor memory (512 columns): S_0 at 0 and S_1 at 128 (128 columns each),
// P_0 at 256 and P_1 at 320 (64 columns each), O at 384.  Shared memory: Q
// (32 KB) and three-stage K and V rings (6 x 32 KB) in the canonical
// K-major / MN-major SWIZZLE_128B layouts the MMA descriptors name.
//
// With PASA's compensation (kComp; PASA, arXiv 2604.12219, Figure 2 caption
// and section 3.3: the key blocks outside a query block's kept set enter
// through a grouped first-order term), ceil(NB/128) pooled tiles follow the
// kept tiles of every row: row c of pooled tile p is block b = 128p + c's
// mean key and mean value (bf16 block means loaded with TMA like the K and
// V tiles, or fp32 ones rounded to bf16 by the loader warps into the same
// swizzled stage layout).  The softmax masks kept blocks and columns past
// NB (per-tile use words from a bitset of the kept list), adds log2 of a
// full block's key count, 7, to the exponent of every used column, and
// gives the ragged last block its own count on its score.  So block b adds
// n_b e^{q.kbar_b/sqrt(d)} to the normaliser and that times vbar_b to the
// numerator, in the same online softmax.
//
// A K stage is refilled once its QK^T completes, a V stage once its P V
// completes; each MMA group signals its completion with one commit.  Every mbarrier wait is bounded (about one second of
// %globaltimer, or the limit the launch sets); on expiry the kernel records
// PA_ERR_TIMEOUT in the device status word, each role leaves its loop,
// in-flight copies and MMAs are drained and tensor memory is released
// before the CTA exits.
#include <type_traits>

#include "sm100.cuh"

namespace paro {

namespace {

using namespace sm100;

constexpr int kBlock = 128;
constexpr int kD = 128;
constexpr int kStages = 3;
constexpr int kMmaWarp = 8;   // QK^T issuer, tensor memory owner
constexpr int kKWarp = 9;
constexpr int kVWarp = 10;
constexpr int kPvWarp = 11;   // kept-list check
constexpr int kThreads = 12 * 32;  // 384
constexpr int kGroupThreads = 128;  // one softmax group
constexpr uint32_t kTile = kBlock * kD * 2;  // 32 KB
constexpr uint32_t kHalf = kBlock * 128;     // 16 KB: 64 columns
// small region first: mbarriers, TMEM slot and flags, the row sums of the
// two groups [2][128] float for the final sum, and the reference max of
// each row after each group's latest tile [2][128] float; the operand
// tiles start 1024-aligned
constexpr uint32_t kOffBar = 0;
constexpr uint32_t kOffSlot = 256;
constexpr uint32_t kOffMerge = 512;
constexpr uint32_t kOffRef = kOffMerge + 2 * 128 * 4;
constexpr uint32_t kOffBits = kOffRef + 2 * 128 * 4;  // kComp: the kept list as NB bits
constexpr int kCompMaxNB = 4096;
constexpr uint32_t kSmall = 3072;
constexpr uint32_t kOffQ = kSmall;
constexpr uint32_t kOffK = kOffQ + kTile;            // kStages stages
constexpr uint32_t kOffV = kOffK + kStages * kTile;  // kStages stages
constexpr uint32_t kSmemBytes = kOffV + kStages * kTile;  // 232,448 B = 227 KB
constexpr float kRescaleLog2 = 8.f;  // lazy rescale threshold (factor 256)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColP = 256, kColO = 384;  // S, P: + 128 / 64 * group

// QK^T(j) and P V(j) each end with one commit, into a ring of 6 barriers
// (slot j % 6, phase j / 6) that every consumer of that event waits on: the
// tile's softmax group (S ready; its P buffer free), the loaders (K or V
// stage free), the O rescale and the epilogue.  No waiter can fall 6 tiles
// behind, so a slot's phases never alias.
constexpr int kRing = 6;
enum : uint32_t {
  BQ = 0,
  BK0 = 1,    // K stage full (3)
  BV0 = 4,    // V stage full (3)
  BQK0 = 7,   // QK^T(j) complete (6)
  BPV0 = 13,  // P V(j) complete (6)
  BSF0 = 19,  // S copied out by every thread of the group (2)
  BP0 = 21,   // P written by every thread of the group (2)
  BMX0 = 23,  // the group's reference max of its tile published (2)
  BDRAIN = 25,
  BM = 26,    // final sum exchange
  NBAR = 27
};
static_assert(NBAR * 8 <= kOffSlot, "barrier region");
static_assert(kOffBits + kCompMaxNB / 8 <= kSmall, "row sum, reference and bitset regions");

// Rows t0 .. t0+127 of a [nb, 128] float block-mean array, rounded to bf16,
// into a stage in the SWIZZLE_128B layout of copy_tile (rows >= nb zero),
// by one warp with generic-proxy stores.  Lane l converts the 16-byte
// chunks e = l + 32m (row e / 16, chunk e % 16), m = 0..63, in four batches
// of 16 whose 32 global loads are all issued before any is used (the
// block means sit in L2; the batches hide its latency).
__device__ __forceinline__ void pool_tile(unsigned char* stage, const float* __restrict__ src,
                                          int t0, int nb, int lane) {
  constexpr int kBatch = 16;
#pragma unroll 1
  for (int m0 = 0; m0 < kBlock * 16 / 32; m0 += kBatch) {
    float4 a[kBatch], b[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int e = lane + 32 * (m0 + u);
      const int r = e >> 4, c16 = e & 15;
      if (t0 + r < nb) {
        const float4* f = reinterpret_cast<const float4*>(src + (int64_t)(t0 + r) * kD + c16 * 8);
        a[u] = __ldg(f);
        b[u] = __ldg(f + 1);
      } else {
        a[u] = b[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int e = lane + 32 * (m0 + u);
      const int r = e >> 4, c16 = e & 15, half = c16 >> 3, c = c16 & 7;
      uint4 w;
      w.x = pack_bf16(a[u].x, a[u].y);
      w.y = pack_bf16(a[u].z, a[u].w);
      w.z = pack_bf16(b[u].x, b[u].y);
      w.w = pack_bf16(b[u].z, b[u].w);
      *reinterpret_cast<uint4*>(stage + half * kHalf + sw128_off(r, c)) = w;
    }
  }
}

// One warp copies rows r0 .. r0+127 of a [rows, 128] bf16 array into a
// stage in the SWIZZLE_128B layout (16-byte cp.async, 16 lanes per row);
// rows at or past `valid` (relative to r0) are zero-filled.
__device__ __forceinline__ void copy_rows(uint32_t tile, const __nv_bfloat16* __restrict__ src,
                                          int64_t r0, int valid, int lane) {
  const int c16 = lane & 15, half = c16 >> 3, c = c16 & 7;
  const char* src0 = reinterpret_cast<const char*>(src + r0 * kD) + c16 * 16;
#pragma unroll 8
  for (int m = 0; m < kBlock / 2; ++m) {
    const int r = 2 * m + (lane >> 4);
    const bool ok = r < valid;
    cp_async16(tile + half * kHalf + sw128_off(r, c), src0 + (ok ? (int64_t)r * (kD * 2) : 0),
               ok ? 16u : 0u);
  }
}

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
// kComp: PASA's compensation from the block means k_pool, v_pool
// ([B*heads, NB, d]): float (rounded to bf16 by the loader warps), or, with
// pool_bf16, already bf16 and loaded like the kept tiles (map_kp, map_vp
// over the [B*heads*NB, d] rows; rows past a head's NB belong to the next
// head and are masked like the blocks past NB, rows past the array's end
// read as zero).
template <bool kTma, bool kComp>
__global__ void __launch_bounds__(kThreads, 1)
    attn_sm100_kernel(const __grid_constant__ CUtensorMap map_q,
                      const __grid_constant__ CUtensorMap map_k,
                      const __grid_constant__ CUtensorMap map_v,
                      const __grid_constant__ CUtensorMap map_kp,
                      const __grid_constant__ CUtensorMap map_vp,
                      const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                      const __nv_bfloat16* __restrict__ v, const __grid_constant__ Grid g,
                      const int32_t* __restrict__ idx, const int32_t* __restrict__ counts,
                      int k_max, float scale_log2, __nv_bfloat16* __restrict__ out,
                      int32_t* __restrict__ status, const StallTest st,
                      const void* __restrict__ k_pool, const void* __restrict__ v_pool,
                      int pool_bf16) {
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
  float* lsum = reinterpret_cast<float*>(gbase + kOffMerge);  // [group][row]
  float* mref = reinterpret_cast<float*>(gbase + kOffRef);    // [group][row]
  auto bar = [&](uint32_t slot) { return base + kOffBar + slot * 8u; };
  auto qk_done = [&](int j) { return bar(BQK0 + j % kRing); };
  auto pv_done = [&](int j) { return bar(BPV0 + j % kRing); };
  auto ring_par = [](int j) { return (uint32_t)((j / kRing) & 1); };

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
    }
    for (int x = 0; x < kRing; ++x) {
      mbar_init(bar(BQK0 + x), 1);
      mbar_init(bar(BPV0 + x), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar(BSF0 + b), kGroupThreads);
      mbar_init(bar(BP0 + b), kGroupThreads);
      mbar_init(bar(BMX0 + b), kGroupThreads);
    }
    mbar_init(bar(BDRAIN), 1);
    mbar_init(bar(BM), 2 * kGroupThreads);
    *abort_flag = 0;
    *bad_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == kMmaWarp) tmem_alloc(smem_u32(tmem_slot), kTmemCols);
  if (warp == kPvWarp) {
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
    if constexpr (kComp) {
      uint32_t* bits = reinterpret_cast<uint32_t*>(gbase + kOffBits);
      for (int x = lane; x < kCompMaxNB / 32; x += 32) bits[x] = 0u;
      __syncwarp();
      if (!__any_sync(0xffffffffu, bad))  // a malformed list is never used
        for (int e = lane; e < cnt; e += 32) {
          const int jb = __ldg(ids + e);
          atomicOr(bits + (jb >> 5), 1u << (jb & 31));
        }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const bool run = *bad_flag == 0 && !expired;
  const int n_pool = kComp ? (g.NB + kBlock - 1) / kBlock : 0;  // pooled tiles
  const int n_tiles = run ? cnt + n_pool : 0;
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
        int kb_lane = 0;  // kept index j0 + lane of the current chunk of 32
        for (int j = 0; j < n_tiles; ++j) {
          const int s = j % kStages;
          if ((j & 31) == 0) kb_lane = j + lane < cnt ? __ldg(ids + j + lane) : 0;
          const int kb = __shfl_sync(0xffffffffu, kb_lane, j & 31);
          // the stage is free once QK^T (K) or P V (V) of tile j-3 completed
          if (j >= kStages && !warp_wait(is_k ? qk_done(j - kStages) : pv_done(j - kStages),
                                         ring_par(j - kStages), ctl))
            break;
          const uint32_t full = bar((is_k ? BK0 : BV0) + s);
          if (!is_k && j == st.tile && i == st.cta_x && bh == st.cta_y) {
            issued = j + 1;  // test hook: this tile never arrives
            continue;
          }
          if (kComp && j >= cnt) {
            const int p0 = (j - cnt) * kBlock;  // first pooled block of the tile
            if (pool_bf16) {
              // bf16 block means: 128 contiguous rows, like a kept tile
              if constexpr (kTma) {
                if (lane == 0) {
                  const CUtensorMap* pmap = is_k ? &map_kp : &map_vp;
                  const int prow = (int)(bh * g.NB) + p0;
                  mbar_arrive_tx(full, kTile);
                  tma_load_2d(ring + s * kTile, pmap, 0, prow, full);
                  tma_load_2d(ring + s * kTile + kHalf, pmap, 64, prow, full);
                }
              } else {
                copy_rows(ring + s * kTile,
                          static_cast<const __nv_bfloat16*>(is_k ? k_pool : v_pool),
                          bh * (int64_t)g.NB + p0, g.NB - p0, lane);
                cp_async_arrive(full);
              }
            } else {
              // float block means, converted by this warp's generic stores;
              // ordered after the stage's previous async-proxy reads and
              // before the tensor core's
              fence_async_smem();
              pool_tile(gbase + (ring - base) + s * kTile,
                        static_cast<const float*>(is_k ? k_pool : v_pool) +
                            bh * (int64_t)g.NB * kD,
                        p0, g.NB, lane);
              fence_async_smem();
              __syncwarp();
              if (kTma) {
                if (lane == 0) mbar_arrive(full);
              } else {
                mbar_arrive(full);
              }
            }
            issued = j + 1;
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
      // Issue order QK(0), QK(1), then QK(j+2), PV(j) for j = 0, 1, ...:
      // QK^T(j+2) waits only for S(j) to be copied out (early in group
      // j & 1's work), and P(j) has the time of QK^T(j+2) and PV(j-1).  The
      // tensor pipe queues few MMAs, so time this thread spends away from
      // issuing is lost: each MMA group ends with one commit, and the
      // barriers of the next group are tested (without blocking) before the
      // current group is issued, so that a blocking wait is left only when
      // that test failed.
      if (lane == 0 && n_tiles > 0) {
        constexpr uint32_t id_qk = idesc_bf16(kBlock, kBlock, false);
        constexpr uint32_t id_pv = idesc_bf16(kBlock, kD, true);
        // descriptors of stage 0 / of Q; other stages and k-steps add their
        // byte offset / 16 to the start-address field (addresses < 256 KB,
        // so the 14-bit field never carries)
        const uint64_t dq = sw128_desc(base + kOffQ, 16, 1024);
        const uint64_t dk0 = sw128_desc(base + kOffK, 16, 1024);
        const uint64_t dv0 = sw128_desc(base + kOffV, kHalf, 1024);
        auto issue_qk = [&](int j) {  // S_b = Q K(j)^T, b = j & 1
          const uint64_t dk = dk0 + (uint64_t)((j % kStages) * (kTile >> 4));
          const uint32_t d_tmem = tmem + kColS + (j & 1) * 128;
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk) {
            const uint64_t off = ((kk >> 2) * kHalf + (kk & 3) * 32) >> 4;
            mma_f16_ss(d_tmem, dq + off, dk + off, id_qk, kk > 0 ? 1u : 0u);
          }
          mma_commit(qk_done(j));
        };
        auto issue_pv = [&](int j) {  // O += P(j) V(j), P from group (j & 1)'s buffer
          const uint64_t dv = dv0 + (uint64_t)((j % kStages) * (kTile >> 4));
          const uint32_t a_tmem = tmem + kColP + (j & 1) * 64;
#pragma unroll
          for (int kk = 0; kk < kBlock / 16; ++kk)
            mma_f16_ts(tmem + kColO, a_tmem + kk * 8, dv + (uint64_t)(kk * 128), id_pv,
                       (j > 0 || kk > 0) ? 1u : 0u);
          mma_commit(pv_done(j));
        };
        // barriers of QK^T(j): S(j-2) copied out (j >= 2) and K(j) loaded
        auto qk_ready_test = [&](int j) {
          return (j < 2 || mbar_test(bar(BSF0 + (j & 1)), ((j >> 1) - 1) & 1)) &&
                 mbar_test(bar(BK0 + j % kStages), (j / kStages) & 1);
        };
        auto qk_wait = [&](int j) {
          return (j < 2 || wait_phase(bar(BSF0 + (j & 1)), ((j >> 1) - 1) & 1, ctl)) &&
                 wait_phase(bar(BK0 + j % kStages), (j / kStages) & 1, ctl);
        };
        bool ok = wait_phase(bar(BQ), 0, ctl);
        // cp.async (generic proxy) writes -> MMA operand reads; TMA writes are
        // async-proxy and ordered by the mbarrier they complete
        if constexpr (!kTma) fence_async_smem();
        for (int j = 0; ok && j < 2 && j < n_tiles; ++j) {
          ok = qk_wait(j);
          if (!ok) break;
          if constexpr (!kTma) fence_async_smem();
          tc_fence_after();
          issue_qk(j);
        }
        bool qk_ready = false;  // QK^T(j+2)'s barriers, tested one step early
        for (int j = 0; ok && j < n_tiles; ++j) {
          // P(j) and V(j): tested now, used after QK^T(j+2) is issued
          const bool p_ready = mbar_test(bar(BP0 + (j & 1)), (j >> 1) & 1);
          const bool v_ready = mbar_test(bar(BV0 + j % kStages), (j / kStages) & 1);
          if (j + 2 < n_tiles) {
            if (!qk_ready && !qk_wait(j + 2)) { ok = false; break; }
            if constexpr (!kTma) fence_async_smem();
            tc_fence_after();
            issue_qk(j + 2);
          }
          qk_ready = j + 3 < n_tiles && qk_ready_test(j + 3);
          if (!p_ready && !wait_phase(bar(BP0 + (j & 1)), (j >> 1) & 1, ctl)) { ok = false; break; }
          if (!v_ready && !wait_phase(bar(BV0 + j % kStages), (j / kStages) & 1, ctl)) {
            ok = false;
            break;
          }
          if constexpr (!kTma) fence_async_smem();
          tc_fence_after();
          issue_pv(j);
        }
        // every MMA issued above has completed once this commit fires
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
    const uint32_t p_col = kColP + grp * 64;
    // the kept list is ascending, so only its last entry can be the ragged
    // last block of the head
    const int tail_keys = g.N - (g.NB - 1) * kBlock;
    const bool ragged_last =
        run && cnt > 0 && tail_keys < kBlock && __ldg(ids + cnt - 1) == g.NB - 1;
    // pooled tiles: a full block's weight 2^7 enters as +7 in the exponent
    // (log2 units); the ragged last block's as log2(tail_keys), i.e. a raw
    // score offset d_last relative to the full blocks'
    const float lb_full = kComp ? log2f((float)kBlock) : 0.f;
    const float d_last =
        kComp ? (log2f((float)tail_keys) - log2f((float)kBlock)) / scale_log2 : 0.f;
    float m_mine = -INFINITY, l = 0.f;  // this group's row sum, relative to m_mine
    // the group's tiles: the kept ones, then (kComp) the pooled ones, in two
    // loops so that the hot one carries no pooled-tile code
    auto step = [&](int j, auto pooled) -> bool {
      if (!warp_wait(qk_done(j), ring_par(j), ctl)) return false;
      tc_fence_after();
      uint32_t sr[128];
      tmem_ld128(lane_addr + s_col, sr);
      tc_fence_before();
      mbar_arrive(bar(BSF0 + grp));  // S_grp may take QK^T two tiles ahead
      float bias = 0.f;  // added to every score of the tile in log2 units
      if constexpr (decltype(pooled)::value) {
        // pooled tile: column c is key block p0 + c, used unless it is kept
        // or past NB (p0 is a multiple of 128 and p0 + 127 < 4096: four
        // whole bitset words); every used column's weight is 2^7 (bias),
        // the ragged last block's tail_keys (d_last on its score)
        const uint32_t* bits = reinterpret_cast<const uint32_t*>(gbase + kOffBits);
        const int p0 = (j - cnt) * kBlock;
        uint32_t uw[4];
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const int n_in = g.NB - (p0 + 32 * x);  // blocks of this word below NB
          const uint32_t valid = n_in >= 32 ? ~0u : (n_in <= 0 ? 0u : (1u << n_in) - 1u);
          uw[x] = ~bits[(p0 >> 5) + x] & valid;
        }
        bias = lb_full;
        const int c_last = g.NB - 1 - p0;
        if (tail_keys < kBlock && c_last < kBlock) {  // warp-uniform
#pragma unroll
          for (int c = 0; c < kBlock; ++c) {
            const float sv = __uint_as_float(sr[c]) + (c == c_last ? d_last : 0.f);
            sr[c] = (uw[c >> 5] >> (c & 31)) & 1u ? __float_as_uint(sv)
                                                   : __float_as_uint(-INFINITY);
          }
        } else {
#pragma unroll
          for (int c = 0; c < kBlock; ++c)
            if (!((uw[c >> 5] >> (c & 31)) & 1u)) sr[c] = __float_as_uint(-INFINITY);
        }
      } else if (ragged_last && j == cnt - 1) {  // warp-uniform
#pragma unroll
        for (int c = 0; c < kBlock; ++c)
          if (c >= tail_keys) sr[c] = __float_as_uint(-INFINITY);
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
                           scale_log2 +
                       bias;
      // the reference after tile j-1 (published by the other group), then
      // this tile's: kept unless this tile's max exceeds it by more than 2^8
      float m_prev = -INFINITY;
      if (j >= 1) {
        if (!warp_wait(bar(BMX0 + (grp ^ 1)), ((j - 1) >> 1) & 1, ctl)) return false;
        m_prev = mref[(grp ^ 1) * 128 + r];
      }
      // (a pooled tile whose blocks are all kept has mx = -inf and keeps
      // the reference)
      const float m_j = (m_prev == -INFINITY || mx > m_prev + kRescaleLog2) ? mx : m_prev;
      mref[grp * 128 + r] = m_j;
      mbar_arrive(bar(BMX0 + grp));  // release: the store above is visible to the waiter
      if (m_mine != -INFINITY) l *= ex2(m_mine - m_j);  // this group's sum, to m_j
      m_mine = m_j;
      // P = 2^(s*scale - m_j) as bf16 pairs, two columns per paired f32x2
      // FMA and add (row sum in 4 paired chains), all 128 columns into
      // registers first: the group's P buffer is written only once P V of
      // its previous tile completed, and that wait now overlaps the
      // exponentials
      const float neg_m = (m_j == -INFINITY ? 0.f : -m_j) + bias;
      const float2 sc2 = make_float2(scale_log2, scale_log2), nm2 = make_float2(neg_m, neg_m);
      float2 rs2[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) rs2[u] = make_float2(0.f, 0.f);
      uint32_t pk[64];
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        const int e = 2 * c;
        const float2 t =
            ffma2(make_float2(__uint_as_float(sr[e]), __uint_as_float(sr[e + 1])), sc2, nm2);
        const float2 ex = make_float2(ex2(t.x), ex2(t.y));
        rs2[c & 3] = fadd2(rs2[c & 3], ex);
        pk[c] = pack_bf16(ex.x, ex.y);
      }
      if (j >= 2 && !warp_wait(pv_done(j - 2), ring_par(j - 2), ctl)) return false;
      tc_fence_after();
#pragma unroll
      for (int cc = 0; cc < 4; ++cc)
        tmem_st16_async(lane_addr + p_col + 16 * cc,
                        *reinterpret_cast<const uint32_t(*)[16]>(&pk[16 * cc]));
      tmem_wait_st();
      l += ((rs2[0].x + rs2[0].y) + (rs2[1].x + rs2[1].y)) +
           ((rs2[2].x + rs2[2].y) + (rs2[3].x + rs2[3].y));
      // O holds P V up to tile j-1 relative to m_prev: rescale it before
      // P V(j) once that MMA completed (rare: the reference moved)
      const bool need = m_prev != -INFINITY && m_j != m_prev;
      if (__any_sync(0xffffffffu, need)) {
        if (!warp_wait(pv_done(j - 1), ring_par(j - 1), ctl)) return false;
        tc_fence_after();
        const float alpha = need ? ex2(m_prev - m_j) : 1.f;
#pragma unroll 1
        for (int c0 = 0; c0 < 128; c0 += 32) {
          uint32_t orr[32];
          tmem_ld32(lane_addr + kColO + c0, orr);
#pragma unroll
          for (int c = 0; c < 32; ++c) orr[c] = __float_as_uint(__uint_as_float(orr[c]) * alpha);
          tmem_st32(lane_addr + kColO + c0, orr);
        }
      }
      tc_fence_before();
      mbar_arrive(bar(BP0 + grp));
      return true;
    };
    bool ok = true;
    int jg = grp;
    for (; ok && jg < n_tiles && (!kComp || jg < cnt); jg += 2) ok = step(jg, std::false_type{});
    if constexpr (kComp)
      for (; ok && jg < n_tiles; jg += 2) ok = step(jg, std::true_type{});
    // ---- epilogue: add the groups' row sums (each relative to its own
    // latest reference; O is relative to the last tile's, the larger), then
    // group g writes output columns 64g .. 64g+63 of the row at the natural
    // position of its token
    const int p = i * kBlock + r;
    __nv_bfloat16* orow = p < g.N ? out + (bh * (int64_t)g.N + natural_index(g, order, p)) * kD
                                  : nullptr;
    if (run && n_tiles == 0) {
      if (orow != nullptr)
        for (int c = 0; c < 8; ++c)
          reinterpret_cast<uint4*>(orow + grp * 64)[c] = make_uint4(0, 0, 0, 0);
    } else if (ok && n_tiles > 0) {
      lsum[grp * 128 + r] = l;
      mref[grp * 128 + r] = m_mine;  // -inf for a group that saw no tile
      mbar_arrive(bar(BM));
      bool okm = all_wait(bar(BM), 0, ctl);
      float inv = 0.f;
      if (okm) {
        const float m0 = mref[r], m1 = mref[128 + r];
        const float m = fmaxf(m0, m1);
        const float lt = (m0 == -INFINITY ? 0.f : lsum[r] * ex2(m0 - m)) +
                         (m1 == -INFINITY ? 0.f : lsum[128 + r] * ex2(m1 - m));
        inv = lt > 0.f ? 1.f / lt : 0.f;
      }
      // every P V has completed once the last one's commit fired
      if (okm) okm = warp_wait(pv_done(n_tiles - 1), ring_par(n_tiles - 1), ctl);
      if (okm) {
        tc_fence_after();
#pragma unroll 1
        for (int c0 = 0; c0 < 64; c0 += 32) {
          const int col = grp * 64 + c0;
          uint32_t oa[32];
          tmem_ld32(lane_addr + kColO + col, oa);
          if (orow != nullptr) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              uint4 w;
              w.x = pack_bf16(__uint_as_float(oa[c * 8 + 0]) * inv, __uint_as_float(oa[c * 8 + 1]) * inv);
              w.y = pack_bf16(__uint_as_float(oa[c * 8 + 2]) * inv, __uint_as_float(oa[c * 8 + 3]) * inv);
              w.z = pack_bf16(__uint_as_float(oa[c * 8 + 4]) * inv, __uint_as_float(oa[c * 8 + 5]) * inv);
              w.w = pack_bf16(__uint_as_float(oa[c * 8 + 6]) * inv, __uint_as_float(oa[c * 8 + 7]) * inv);
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

template <bool kTma, bool kComp>
cudaError_t launch_typed(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv,
                         const CUtensorMap& mkp, const CUtensorMap& mvp, const void* q,
                         const void* k, const void* v, const Grid& g, const int32_t* idx,
                         const int32_t* counts, int k_max, void* out, int32_t* status,
                         cudaStream_t s, const void* k_pool, const void* v_pool, int pool_bf16) {
  if (kComp && g.NB > kCompMaxNB) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(attn_sm100_kernel<kTma, kComp>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  const float scale_log2 = (float)(1.4426950408889634 / sqrt((double)kD));
  dim3 grid(g.NB, g.B * g.heads);
  attn_sm100_kernel<kTma, kComp><<<grid, kThreads, kSmemBytes, s>>>(
      mq, mk, mv, mkp, mvp, static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
      static_cast<const __nv_bfloat16*>(v), g, idx, counts, k_max, scale_log2,
      static_cast<__nv_bfloat16*>(out), status, stall_test(), k_pool, v_pool, pool_bf16);
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
                              cudaStream_t s, const void* k_pool, const void* v_pool,
                              pa_dtype pool_dtype) {
  if (!attn_sm100_supports(dt, g)) return cudaErrorInvalidValue;
  const bool comp = k_pool != nullptr && v_pool != nullptr;
  if (comp && dt != PA_BF16) return cudaErrorInvalidValue;
  if (dt == PA_I8) return cudaErrorInvalidValue;  // launch_attn_i8
  CUtensorMap mq{}, mk{}, mv{}, mkp{}, mvp{};
  const int pool_bf16 = comp && pool_dtype == PA_BF16 ? 1 : 0;
  if (pool_bf16 && permuted) {
    const uint64_t prow = (uint64_t)g.B * g.heads * g.NB;
    if (!encode_tile_map(&mkp, k_pool, prow, kD, 2, 64, kBlock) ||
        !encode_tile_map(&mvp, v_pool, prow, kD, 2, 64, kBlock))
      return cudaErrorInvalidValue;
  }
  if (permuted) {
    const uint64_t rows = (uint64_t)g.B * g.heads * g.Np;
    if (!encode_tile_map(&mq, q, rows, kD, 2, 64, kBlock) ||
        !encode_tile_map(&mk, k, rows, kD, 2, 64, kBlock) ||
        !encode_tile_map(&mv, v, rows, kD, 2, 64, kBlock))
      return cudaErrorInvalidValue;
    return comp ? launch_typed<true, true>(mq, mk, mv, mkp, mvp, q, k, v, g, idx, counts, k_max,
                                           out, status, s, k_pool, v_pool, pool_bf16)
                : launch_typed<true, false>(mq, mk, mv, mkp, mvp, q, k, v, g, idx, counts, k_max,
                                            out, status, s, nullptr, nullptr, 0);
  }
  return comp ? launch_typed<false, true>(mq, mk, mv, mkp, mvp, q, k, v, g, idx, counts, k_max,
                                          out, status, s, k_pool, v_pool, pool_bf16)
              : launch_typed<false, false>(mq, mk, mv, mkp, mvp, q, k, v, g, idx, counts, k_max,
                                           out, status, s, nullptr, nullptr, 0);
}

}  // namespace paro
