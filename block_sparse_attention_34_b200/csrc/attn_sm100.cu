// Block-sparse flash attention on the 5th-generation tensor cores of sm_100a
// (tcgen05.mma, accumulators in tensor memory), d = 128, block = 128, bf16.
//
// What it computes (SPADE, arXiv 2608.03335, Pith verdict page,
// key_machinery (iii): a flash block-sparse attention kernel with an online
// softmax over the kept block pairs; PAROAttention, arXiv 2506.16054, review
// key_machinery: the per-head axis order of the tokens, fused into the
// kernel's loads and stores): for query block i of head (b, h) and every key
// block j of its ascending kept list, S = Q_i K_j^T / sqrt(d), a running
// row max / row sum softmax, and O += P V_j, then O / l written to the
// natural positions of the block's tokens.
//
// One CTA per (query block, head); 13 warps with fixed roles:
//   warps 0-7  softmax, two warpgroups splitting every tile by columns:
//              warp w owns rows 32*(w%4) .. +31 (TMEM lanes; a warp may only
//              touch its lane quarter) and key columns 64*(w/4) .. +63.  Each
//              thread reads its 64 scores from TMEM, the two halves of a row
//              exchange their maxima through shared memory, then each thread
//              writes its 64 bf16 probabilities into its half of the P tile
//              and, when the row max grew by more than 2^8, rescales its 64
//              columns of O in TMEM; the epilogue is split the same way;
//   warp 8     allocates TMEM; one lane issues every tcgen05.mma and commit;
//   warps 9-12 gather loaders (Q by all four; then warps 9-10 stream K and
//              warps 11-12 stream V): each token row is 256 contiguous bytes
//              at its natural position, copied with 16-byte cp.async
//              straight into the 128-byte-swizzled operand layout -- the
//              axis order is applied in the address, so no reordered copy
//              of any tensor exists in HBM.  A K stage is refilled as soon
//              as the QK^T that read it completes, a V stage once its P V
//              completes, so neither stream waits on the other.
// Tensor memory (512 columns): S double buffer at columns 0 and 128, O at
// 256.  Shared memory: Q (32 KB), a two-stage K and V ring (4 x 32 KB), a
// double-buffered P (2 x 32 KB), all in the canonical K-major / MN-major
// SWIZZLE_128B layouts the MMA descriptors name, after a small region of
// mbarriers and the row-max exchange buffer.
//
// The MMA warp runs one step ahead: QK^T of tile j is issued before P V of
// tile j-1, so the tensor core works on S_j while the softmax warps turn
// S_{j-1} into P_{j-1}.  Every wait on an mbarrier is bounded (about one
// second of %globaltimer); on expiry the kernel records PA_ERR_TIMEOUT in the
// device status word, every role leaves its loop, in-flight copies and MMAs
// are drained and TMEM is released before the CTA exits.
#include "common.cuh"
#include "tmem.cuh"

namespace paro {
namespace {

constexpr int kBlock = 128;
constexpr int kD = 128;
constexpr int kSoftmaxWarps = 8;
constexpr int kMmaWarp = 8;
constexpr int kLoadWarp0 = 9;
constexpr int kLoadWarps = 4;
constexpr int kSoftmaxThreads = kSoftmaxWarps * 32;                // 256
constexpr int kThreads = (kSoftmaxWarps + 1 + kLoadWarps) * 32;  // 416
constexpr uint32_t kTile = kBlock * kD * 2;                       // 32 KB
constexpr uint32_t kHalf = kBlock * 128;                          // 16 KB: 64 columns
// small region first: mbarriers (19 x 8 B), TMEM slot and flags (16 B),
// row-max exchange [2 tiles][2 halves][128 rows] float (2 KB)
constexpr uint32_t kOffBar = 0;
constexpr uint32_t kOffSlot = 192;
constexpr uint32_t kOffXmax = 256;
constexpr uint32_t kSmall = 3072;  // operand tiles start 1024-aligned after it
constexpr uint32_t kOffQ = kSmall;
constexpr uint32_t kOffK = kOffQ + kTile;      // 2 stages
constexpr uint32_t kOffV = kOffK + 2 * kTile;  // 2 stages
constexpr uint32_t kOffP = kOffV + 2 * kTile;  // 2 buffers
constexpr uint32_t kSmemBytes = kOffP + 2 * kTile;  // 232,448 B = 227 KB
constexpr uint64_t kTimeoutNs = 1000000000ull;
constexpr float kRescaleLog2 = 8.f;  // lazy rescale threshold (factor 256)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 256;

// barrier slots
enum : uint32_t {
  BQ = 0, BK0 = 1, BV0 = 3, BS0 = 5, BSF0 = 7, BP0 = 9, BPV0 = 11, BKF0 = 13, BX0 = 15,
  BDRAIN = 17, BL = 18, NBAR = 19
};
static_assert(NBAR * 8 <= kOffSlot, "barrier region");

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("{\n.reg .b64 st;\nmbarrier.arrive.shared::cta.b64 st, [%0];\n}\n" ::"r"(bar)
               : "memory");
}

__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n.reg .pred p;\nmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\nselp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

struct Ctl {
  volatile uint32_t* abort;
  int32_t* status;
};

// Bounded wait on one phase of an mbarrier (one thread).
__device__ __forceinline__ bool wait_phase(uint32_t bar, uint32_t parity, Ctl c) {
  if (mbar_try(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try(bar, parity)) return true;
    if ((it & 63u) == 0) {
      if (*c.abort) return false;
      if (global_ns() - t0 > kTimeoutNs) {
        *c.abort = 1;
        report(c.status, PA_ERR_TIMEOUT);
        return false;
      }
    }
  }
}

// Warp-uniform bounded wait: lane 0 waits, the outcome is broadcast.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, Ctl c) {
  int ok = 0;
  if ((threadIdx.x & 31) == 0) ok = wait_phase(bar, parity, c) ? 1 : 0;
  return __shfl_sync(0xffffffffu, ok, 0) != 0;
}

// Bounded wait by every lane (each acquires the data published before the
// phase completed); the outcome is made warp-uniform.
__device__ __forceinline__ bool all_wait(uint32_t bar, uint32_t parity, Ctl c) {
  const bool ok = wait_phase(bar, parity, c);
  return __all_sync(0xffffffffu, ok);
}

// --- tcgen05 -------------------------------------------------------------

// Shared-memory matrix descriptor, SWIZZLE_128B, sm_100 version field.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}

// Instruction descriptor, kind::f16: D f32, A and B bf16, A K-major.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn_major ? 1u : 0u) << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_f16_ss(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
                   bar)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
}
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;\n" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 t = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&t);
}

// Byte offset of the 16-byte chunk c (0..7) of row r inside one 64-column
// half of a SWIZZLE_128B tile: rows are 128 bytes, chunks XOR-permuted by
// the row's position within its 8-row group.
__device__ __forceinline__ uint32_t sw128_off(int r, int c) {
  return (uint32_t)(r * 128 + ((c ^ (r & 7)) << 4));
}

// One loader warp copies 32 rows (row0 .. row0+31) of a [128 x 128] bf16
// tile.  nat = natural token index of this lane's row (lane l <-> row
// row0 + l), or -1 for a pad row (zero-filled).  Each 16-lane half of the
// warp reads one whole 256-byte row per instruction.
__device__ __forceinline__ void load_rows(uint32_t tile, const __nv_bfloat16* __restrict__ head,
                                          int row0, int lane, int nat) {
#pragma unroll 4
  for (int m = 0; m < 16; ++m) {
    const int src_lane = 2 * m + (lane >> 4);
    const int n = __shfl_sync(0xffffffffu, nat, src_lane);
    const int r = row0 + src_lane;
    const int cc = lane & 15;
    const int half = cc >> 3, c = cc & 7;
    const char* src = reinterpret_cast<const char*>(head) +
                      (n >= 0 ? (int64_t)n * (kD * 2) : 0) + half * 128 + c * 16;
    cp_async16(tile + half * kHalf + sw128_off(r, c), src, n >= 0 ? 16u : 0u);
  }
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_sm100_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                      const __nv_bfloat16* __restrict__ v, const __grid_constant__ Grid g,
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
  const uint32_t bars = base + kOffBar;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + kOffSlot);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  volatile uint32_t* bad_flag = tmem_slot + 2;
  float* xmax = reinterpret_cast<float*>(gbase + kOffXmax);
  auto bar = [&](uint32_t slot) { return bars + slot * 8u; };

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
    mbar_init(bar(BQ), kLoadWarps * 32);
    for (int s = 0; s < 2; ++s) {
      mbar_init(bar(BK0 + s), kLoadWarps * 16);
      mbar_init(bar(BV0 + s), kLoadWarps * 16);
      mbar_init(bar(BKF0 + s), 1);
      mbar_init(bar(BS0 + s), 1);
      mbar_init(bar(BSF0 + s), kSoftmaxThreads);
      mbar_init(bar(BP0 + s), kSoftmaxThreads);
      mbar_init(bar(BPV0 + s), 1);
      mbar_init(bar(BX0 + s), kSoftmaxThreads);
    }
    mbar_init(bar(BDRAIN), 1);
    mbar_init(bar(BL), kSoftmaxThreads);
    *abort_flag = 0;
    *bad_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  }
  if (warp == kMmaWarp) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
  }
  if (warp == kLoadWarp0) {
    // validate the kept list once: count in range, indices ascending in [0, NB)
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

  if (warp >= kLoadWarp0) {
    // ------------------------------------------------------ loaders ----
    const int lw = warp - kLoadWarp0;
    if (n_tiles > 0) {
      {
        const int p = i * kBlock + 32 * lw + lane;
        const int nat = p < g.N ? natural_index(g, order, p) : -1;
        load_rows(base + kOffQ, qh, 32 * lw, lane, nat);
        cp_async_commit();
        cp_async_wait<0>();
        fence_async_smem();
        mbar_arrive(bar(BQ));
      }
      // warps 5-6 stream K (stage free once QK^T of tile j-2 completed),
      // warps 7-8 stream V (stage free once P V of tile j-2 completed)
      const bool is_k = lw < 2;
      const int half_rows = 64 * (lw & 1);
      const __nv_bfloat16* src = is_k ? kh : vh;
      const uint32_t ring = base + (is_k ? kOffK : kOffV);
      for (int j = 0; j < n_tiles; ++j) {
        const int s = j & 1;
        if (j >= 2 && !warp_wait(bar((is_k ? BKF0 : BPV0) + s), ((j - 2) >> 1) & 1, ctl)) break;
        const int kb = __ldg(ids + j);
#pragma unroll
        for (int g2 = 0; g2 < 2; ++g2) {
          const int row0 = half_rows + 32 * g2;
          const int p = kb * kBlock + row0 + lane;
          const int nat = p < g.N ? natural_index(g, order, p) : -1;
          load_rows(ring + s * kTile, src, row0, lane, nat);
        }
        cp_async_commit();
        cp_async_wait<0>();
        fence_async_smem();
        mbar_arrive(bar((is_k ? BK0 : BV0) + s));
      }
      cp_async_wait<0>();
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
          mma_f16_ss(tmem + kColO, ad, bd, id_pv, (jp > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(bar(BPV0 + b));
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
        if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
      }
      if (ok) issue_pv(n_tiles - 1);
      // drain: every MMA issued above has completed once this commit fires
      mma_commit(bar(BDRAIN));
      wait_phase(bar(BDRAIN), 0, ctl);
    }
  } else {
    // ------------------------------------------------------ softmax ----
    const int quarter = warp & 3, hc = warp >> 2;
    const int r = quarter * 32 + lane;  // tile row == TMEM lane
    const uint32_t lane_addr = tmem + ((uint32_t)(quarter * 32) << 16);
    float m_used = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_tiles; ++j) {
      const int b = j & 1;
      if (!warp_wait(bar(BS0 + b), (j >> 1) & 1, ctl)) { ok = false; break; }
      tc_fence_after();
      uint32_t sr[64];
      tmem_ld64(lane_addr + kColS + b * 128 + hc * 64, sr);
      tc_fence_before();
      mbar_arrive(bar(BSF0 + b));
      const int kb = __ldg(ids + j);
      const int valid = g.N - kb * kBlock - hc * 64;  // existing keys in my half
      if (valid < 64) {  // only the ragged last block (warp-uniform)
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (c >= valid) sr[c] = __float_as_uint(-INFINITY);
      }
      // raw row max of my half (8 independent chains), exchanged with the
      // other half of the row
      float mp[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) mp[u] = __uint_as_float(sr[u]);
#pragma unroll
      for (int c = 8; c < 64; ++c) mp[c & 7] = fmaxf(mp[c & 7], __uint_as_float(sr[c]));
      const float mh = fmaxf(fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3])),
                             fmaxf(fmaxf(mp[4], mp[5]), fmaxf(mp[6], mp[7])));
      float* xm = xmax + b * 256;
      xm[hc * 128 + r] = mh;
      mbar_arrive(bar(BX0 + b));
      if (!all_wait(bar(BX0 + b), (j >> 1) & 1, ctl)) { ok = false; break; }
      const float mx = fmaxf(mh, xm[(hc ^ 1) * 128 + r]) * scale_log2;
      // lazy rescale: keep the reference max unless the row max grew by
      // more than 2^8 (exact either way: O and l share the reference)
      const bool need = j == 0 ? false : (mx > m_used + kRescaleLog2);
      if (j == 0) m_used = mx == -INFINITY ? 0.f : mx;
      if (__any_sync(0xffffffffu, need)) {
        if (!warp_wait(bar(BPV0 + ((j - 1) & 1)), ((j - 1) >> 1) & 1, ctl)) { ok = false; break; }
        tc_fence_after();
        const float alpha = need ? ex2(m_used - mx) : 1.f;
#pragma unroll 1
        for (int c0 = 0; c0 < 64; c0 += 32) {
          uint32_t orr[32];
          tmem_ld32(lane_addr + kColO + hc * 64 + c0, orr);
#pragma unroll
          for (int c = 0; c < 32; ++c) orr[c] = __float_as_uint(__uint_as_float(orr[c]) * alpha);
          tmem_st32(lane_addr + kColO + hc * 64 + c0, orr);
        }
        l *= alpha;
        if (need) m_used = mx;
      }
      if (j >= 2 && !warp_wait(bar(BPV0 + b), ((j - 2) >> 1) & 1, ctl)) { ok = false; break; }
      // P = 2^(s*scale - m) in bf16 into my half of the swizzled K-major P
      // tile; row sum in 8 independent chains
      unsigned char* pt = gbase + kOffP + b * kTile + hc * kHalf;
      const float neg_m = -m_used;
      float rs[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) rs[u] = 0.f;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
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
        *reinterpret_cast<uint4*>(pt + sw128_off(r, c)) = w;
      }
      l += ((rs[0] + rs[1]) + (rs[2] + rs[3])) + ((rs[4] + rs[5]) + (rs[6] + rs[7]));
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(bar(BP0 + b));
    }
    // epilogue: the two halves add their row sums, then each writes O / l
    // for its 64 columns at the natural position of the row's token
    const int p = i * kBlock + r;
    __nv_bfloat16* orow = p < g.N ? out + (bh * (int64_t)g.N + natural_index(g, order, p)) * kD
                                  : nullptr;
    if (run && cnt == 0) {
      if (orow != nullptr)
        for (int c = 0; c < 8; ++c)
          reinterpret_cast<uint4*>(orow + hc * 64)[c] = make_uint4(0, 0, 0, 0);
    } else if (ok && n_tiles > 0) {
      const int jl = n_tiles - 1;
      // the exchange buffer the last tile did not use: its previous reads
      // (tile jl-1) finished before every thread arrived for tile jl
      float* xl = xmax + ((jl & 1) ^ 1) * 256;
      xl[hc * 128 + r] = l;
      mbar_arrive(bar(BL));
      const bool okl = all_wait(bar(BL), 0, ctl);
      const float lt = okl ? l + xl[(hc ^ 1) * 128 + r] : 0.f;
      if (okl && warp_wait(bar(BPV0 + (jl & 1)), (jl >> 1) & 1, ctl)) {
        tc_fence_after();
        const float inv = lt > 0.f ? 1.f / lt : 0.f;
#pragma unroll 1
        for (int c0 = 0; c0 < 64; c0 += 32) {
          uint32_t orr[32];
          tmem_ld32(lane_addr + kColO + hc * 64 + c0, orr);
          if (orow != nullptr) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const float* f = reinterpret_cast<const float*>(orr) + c * 8;
              uint4 w;
              w.x = pack_bf16(f[0] * inv, f[1] * inv);
              w.y = pack_bf16(f[2] * inv, f[3] * inv);
              w.z = pack_bf16(f[4] * inv, f[5] * inv);
              w.w = pack_bf16(f[6] * inv, f[7] * inv);
              reinterpret_cast<uint4*>(orow + hc * 64 + c0)[c] = w;
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    __syncwarp();
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(tmem),
                 "r"(kTmemCols)
                 : "memory");
  }
}

}  // namespace

bool attn_sm100_supports(pa_dtype dt, const Grid& g) {
  return dt == PA_BF16 && g.d == kD && g.block == kBlock;
}

cudaError_t launch_attn_sm100(const void* q, const void* k, const void* v, pa_dtype dt,
                              const Grid& g, const int32_t* idx, const int32_t* counts,
                              int k_max, const float* qs, const float* ks, const float* vs,
                              void* out, int32_t* status, cudaStream_t s) {
  (void)qs;
  (void)ks;
  (void)vs;
  if (!attn_sm100_supports(dt, g)) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(attn_sm100_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
  if (e != cudaSuccess) return e;
  const float scale_log2 = (float)(1.4426950408889634 / sqrt((double)kD));
  dim3 grid(g.NB, g.B * g.heads);
  attn_sm100_kernel<<<grid, kThreads, kSmemBytes, s>>>(
      static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
      static_cast<const __nv_bfloat16*>(v), g, idx, counts, k_max, scale_log2,
      static_cast<__nv_bfloat16*>(out), status);
  return cudaGetLastError();
}

}  // namespace paro
