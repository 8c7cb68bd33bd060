// Tensor-core GEMM for sm_100a (5th-generation tensor cores) behind every dense contraction
// of the compressor that reads the cache: the feature Gram X_(D)^T X_(D), the token Gram
// X_(T) X_(T)^T (or X_(T)^T X_(T)), the FlashJoLT sketch and power-iteration products
// X_(T) F and X_(T)^T F, and the core projection X_(D) W_s, U_s^T Z.
//
//   * operands are staged in shared memory by TMA (cp.async.bulk.tensor, rank-3 tensor maps,
//     64 x 64 bf16 boxes with the 128-byte swizzle), one thread issuing the copies;
//   * one thread issues tcgen05.mma (M = 128, N = BN, K = 16, bf16 x bf16 -> fp32) with the
//     accumulator in tensor memory; tcgen05.commit releases a shared-memory stage back to the
//     copy thread through an mbarrier, so copies of later K blocks overlap the MMAs;
//   * persistent CTAs (one per SM) walk the output tiles; two TMEM accumulators alternate
//     between tiles, so four epilogue warps read one (tcgen05.ld; warp w owns TMEM lanes
//     32 (w % 4) .. +31) and store fp32 or bf16 rows while the MMAs of the next tile run.
//
// Each operand is a 128 (A) or BN (B) x 64 tile assembled from 64 x 64 boxes; the box
// coordinates come from the operand's addressing mode, so the cache is read in place:
//   UM_XT_K    X_(T) of a unit      MN = token t, K = (slice, feature)   map {D, T, slices}
//   UM_XT_MN   X_(T)^T              MN = (slice, feature), K = token     map {D, T, slices}
//   UM_ROW_K   X_(D) of a unit      MN = row (slice, token), K = feature map {D, rows, 1}
//   UM_ROW_MN  X_(D)^T              MN = feature, K = row                map {D, rows, 1}
//   UM_DENSE_K  dense [entry][MN][K]                                     map {ld, MN, entries}
//   UM_DENSE_MN dense [entry][K][MN]                                     map {ld, K, entries}
// Cache modes take map 0 / map 1 for the K / V cache of unit u = 2 g + kv (batch entry u);
// dense modes take map b for B operand b (NB = 2 sums two B operands, F = hi + lo, into one
// accumulator; NB = 4 sums two A operands against one B, which may then be a cache operand).  The K modes are K-major in shared memory, the MN modes MN-major.  D must be
// a multiple of 64 (a 64-wide box never straddles two slices) and, for the row modes, T a
// multiple of 64 (a 64-row box never straddles two units).
//
// Every mbarrier wait is bounded (about two seconds of global time); a wait that gives up
// sets DEV_ERR_TIMEOUT in the status word, every role stops, and the CTA still waits for
// its issued MMAs (through a final commit) before it frees its tensor memory.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace jolt {

enum : int { UM_XT_K = 0, UM_XT_MN = 1, UM_ROW_K = 2, UM_ROW_MN = 3, UM_DENSE_K = 4, UM_DENSE_MN = 5 };

struct UmmaOpnd {
  int mode = UM_DENSE_MN;
  int ediv = 1;         // batch entry b reads operand entry b / ediv
  int S = 0;            // slices per unit (cache modes)
  int d_shift = 0;      // log2(D) (XT modes)
  long long rows = 0;   // rows per unit, S * T (row modes)
};

struct UmmaArgs {
  int M = 0, N = 0, K = 0;    // per batch entry: C (M x N) = A (M x K) * B (K x N)
  int batch = 0;
  int splits = 1;             // split-K: split sp covers K in [sp * kchunk, (sp + 1) * kchunk)
  int kchunk = 0;             // a multiple of 64
  UmmaOpnd A, B;
  bool b_is_a = false;        // Gram of one operand: B's tile is A's tile (M = N = 128, one tile)
  void* C = nullptr;
  int c_bf16 = 0;             // 0: fp32 output, 1: bf16 (round to nearest)
  int c_split = 0;            // 1: the fp32 result as a bf16 pair: C = bf16(v), C2 = bf16(v - C)
  void* C2 = nullptr;
  int c_accum = 0;            // fp32 output only: add the product to what C holds
  int c_trans = 0;            // 1: the tile is stored transposed, C[n * ldc + m] (batch stride sC)
  int m_fast = 0;             // 1: tiles handed out M tile fastest (consecutive tiles share B's tile)
  int tri = 0;                // 1: only output tiles that reach the diagonal or above it
                              //    (n0 + BN > m0; the upper triangle of a symmetric product);
                              // 2: B upper triangular (row k of B is zero for k > every column
                              //    of the tile): the K range ends at n0 + BN
  int bn = 0;                 // N tile: 0 chooses (256 when N > 128), else 128 or 256
  long long ldc = 0, sC = 0, ssplit = 0;   // row pitch, batch stride, split stride (elements)
  uint32_t* status = nullptr;
  int* sched = nullptr;       // device int: the next output tile to hand out (zeroed before the launch)
};

namespace umma {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int BOX_BYTES = 64 * 64 * 2;  // one 64 x 64 bf16 box
constexpr uint64_t kWaitNs = 2000000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// bounded wait for the phase with the given parity to complete: false once `limit_ns` of
// global time has passed without it
__device__ __forceinline__ bool mbar_wait_for(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  if (mbar_try(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try(bar, parity)) return true;
    if ((i & 255u) == 0 && global_ns() - t0 > limit_ns) return false;
  }
}
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity) { return mbar_wait_for(bar, parity, kWaitNs); }

// Self-test of the bounded wait: thread 0 initialises an mbarrier for one arrival, arrives
// on it only if `arrive` is set, and waits for phase 0 with the given limit.  Without the
// arrival the phase never completes, the wait gives up and DEV_ERR_TIMEOUT is raised; the
// kernel then returns normally.
__global__ void wait_selftest_kernel(int arrive, uint64_t limit_ns, uint32_t* status) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x != 0) return;
  const uint32_t b = smem_u32(&bar);
  mbar_init(b, 1);
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  if (arrive) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(b) : "memory");
  if (!mbar_wait_for(b, 0, limit_ns)) atomicOr(status, DEV_ERR_TIMEOUT);
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, int c0, int c1, int c2,
                                            uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];"
      ::"r"(dst), "l"((uint64_t)map), "r"(c0), "r"(c1), "r"(c2), "r"(bar)
      : "memory");
}

// shared-memory matrix descriptor, 128-byte swizzle, version 1 (sm_100)
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((addr & 0x3FFFFu) >> 4);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= 1ull << 46;          // descriptor version for sm_100
  d |= 2ull << 61;          // SWIZZLE_128B
  return d;
}

// instruction descriptor: kind::f16, bf16 A and B, fp32 accumulator, M = 128, N = n
__host__ __device__ constexpr uint32_t instr_desc(int n, bool a_mn, bool b_mn) {
  return (1u << 4)                        // D: fp32
         | (1u << 7)                      // A: bf16
         | (1u << 10)                     // B: bf16
         | ((a_mn ? 1u : 0u) << 15)       // A major-ness (1 = MN)
         | ((b_mn ? 1u : 0u) << 16)       // B major-ness
         | ((uint32_t)(n >> 3) << 17)     // N / 8
         | ((uint32_t)(BM >> 4) << 24);   // M / 16
}

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

__device__ __forceinline__ void fence_before_sync() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after_sync() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// 32 lanes x 32 consecutive fp32 columns of the accumulator
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// NB = 1: C = A B; NB = 2: C = A (B0 + B1); NB = 3: C = A0 B0 + A0 B1 + A1 B0 (the products of
// fp32 operands split as bf16 hi + lo, without the lo * lo term); NB = 4: C = (A0 + A1) B
template <int BN, int NB>
struct Cfg {
  static constexpr int NA_OP = NB >= 3 ? 2 : 1;                  // A operands in a stage
  static constexpr int NB_OP = NB == 3 ? 2 : (NB == 4 ? 1 : NB);  // B operands in a stage
  static constexpr int A_BYTES = BM * BK * 2;          // 16 KB
  static constexpr int B_BYTES = BN * BK * 2;          // BN/64 boxes
  static constexpr int STAGE_BYTES = NA_OP * A_BYTES + NB_OP * B_BYTES;
  static constexpr int STAGES = (200 * 1024) / STAGE_BYTES > 6 ? 6 : (200 * 1024) / STAGE_BYTES;
  static constexpr int BAR_OFF = STAGES * STAGE_BYTES;
  static constexpr int SMEM = BAR_OFF + 512 + 1024;    // barriers, TMEM address, flag, tile ring + slack
  static_assert(STAGES >= 2, "pipeline needs two stages");
};

// box coordinates (c0, c1, c2) of the 64 x 64 box at (mn, k) of batch entry e
__device__ __forceinline__ void box_coords(const UmmaOpnd& o, int e, int mn, int k, int& c0, int& c1, int& c2) {
  const int dmask = (1 << o.d_shift) - 1;
  switch (o.mode) {
    case UM_XT_K:
      c0 = k & dmask;
      c1 = mn;
      c2 = (e >> 1) * o.S + (k >> o.d_shift);
      break;
    case UM_XT_MN:
      c0 = mn & dmask;
      c1 = k;
      c2 = (e >> 1) * o.S + (mn >> o.d_shift);
      break;
    case UM_ROW_K:
      c0 = k;
      c1 = (int)((long long)(e >> 1) * o.rows + mn);
      c2 = 0;
      break;
    case UM_ROW_MN:
      c0 = mn;
      c1 = (int)((long long)(e >> 1) * o.rows + k);
      c2 = 0;
      break;
    case UM_DENSE_K:
      c0 = k;
      c1 = mn;
      c2 = e;
      break;
    default:  // UM_DENSE_MN
      c0 = mn;
      c1 = k;
      c2 = e;
      break;
  }
}

__host__ __device__ __forceinline__ bool cache_mode(int mode) { return mode <= UM_ROW_MN; }

}  // namespace umma

// Persistent: grid = min(tiles, SMs).  The output tiles, in the order (batch entry and split,
// M tile, N tile), N fastest, are handed out by an atomic counter, so CTAs that start late
// (their SM busy with other work) take fewer tiles.  Tile (m0, n0) of batch entry b (split sp
// of its K range) is C = A * sum_b B_b.  Six warps: warp 0 takes tiles from the counter,
// passes their indices to the other roles through a ring in shared memory and issues the TMA
// copies of every tile's K blocks through one ring of shared-memory stages (it runs ahead
// across tile boundaries); warp 1 issues the MMAs into one of two TMEM accumulators
// (alternating by tile); warps 2-5 (one per TMEM lane quarter) drain the other accumulator:
// the epilogue of one tile overlaps the MMAs of the next.
namespace umma {
constexpr int RING = 4;   // tile indices in flight between the roles
}
template <int BN, int NB, bool A_MN, bool B_MN>
__global__ void __launch_bounds__(192, 1)
    umma_gemm_kernel(const __grid_constant__ CUtensorMap map_a0, const __grid_constant__ CUtensorMap map_a1,
                     const __grid_constant__ CUtensorMap map_b0, const __grid_constant__ CUtensorMap map_b1,
                     UmmaArgs a) {
  using C = umma::Cfg<BN, NB>;
  using umma::RING;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  // full[S] empty[S] accfull[2] accempty[2] done ringfull[RING] ringempty[RING]
  uint64_t* bars = (uint64_t*)(smem + C::BAR_OFF);
  uint32_t* tmem_slot = (uint32_t*)(bars + 2 * C::STAGES + 5 + 2 * RING);
  volatile int* abort_flag = (volatile int*)(tmem_slot + 1);
  volatile int* ring = (volatile int*)(tmem_slot + 2);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tN = (a.N + BN - 1) / BN, tM = (a.M + umma::BM - 1) / umma::BM;
  const int per = tN * tM, total = a.batch * a.splits * per;
  const uint32_t full0 = umma::smem_u32(bars), empty0 = full0 + 8 * C::STAGES;
  const uint32_t accfull0 = empty0 + 8 * C::STAGES, accempty0 = accfull0 + 16, done_bar = accempty0 + 16;
  const uint32_t ringfull0 = done_bar + 8, ringempty0 = ringfull0 + 8 * RING;
  const bool b_is_a = a.b_is_a;
  // tile t: batch entry bz, split sp, origin (m0, n0), K blocks [kb0, kb0 + nk)
  auto tile = [&](int t, int& bz, int& sp, int& m0, int& n0, int& kb0, int& nk) -> bool {
    const int zz = t / per, rem = t - zz * per;
    bz = zz / a.splits;
    sp = zz - bz * a.splits;
    const int mi = a.m_fast ? rem % tM : rem / tN, ni = a.m_fast ? rem / tM : rem % tN;
    m0 = mi * umma::BM;
    n0 = ni * BN;
    if (a.tri == 1 && n0 + BN <= m0) return false;   // wholly below the diagonal: not needed
    kb0 = sp * (a.kchunk / umma::BK);
    const int kend = min(a.tri == 2 ? min(a.K, n0 + BN) : a.K, (sp + 1) * a.kchunk);
    nk = kend > kb0 * umma::BK ? (kend - kb0 * umma::BK + umma::BK - 1) / umma::BK : 0;
    return true;
  };
  // the next tile that is needed, or -1 when none is left
  auto fetch = [&]() -> int {
    int bz, sp, m0, n0, kb0, nk;
    for (;;) {
      const int t = atomicAdd(a.sched, 1);
      if (t >= total) return -1;
      if (tile(t, bz, sp, m0, n0, kb0, nk)) return t;
    }
  };
  // the j-th tile index of the ring (all roles read the same sequence); -1: stop, -2: the wait
  // gave up.  warp_wide: every lane of the warp calls it and gets the same answer.
  auto ring_take = [&](int j, bool warp_wide) -> int {
    const int slot = j % RING;
    const bool ok = umma::mbar_wait(ringfull0 + 8 * slot, (j / RING) & 1);
    int t = ok ? ring[slot] : -2;
    if (warp_wide) {
      if (!__all_sync(0xffffffffu, ok)) t = -2;
      __syncwarp();   // every lane has read the slot before it is handed back
    }
    if (lane == 0 && ok) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(ringempty0 + 8 * slot) : "memory");
    return t;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      umma::mbar_init(full0 + 8 * s, 1);
      umma::mbar_init(empty0 + 8 * s, 1);
    }
    for (int b = 0; b < 2; ++b) {
      umma::mbar_init(accfull0 + 8 * b, 1);
      umma::mbar_init(accempty0 + 8 * b, 4);
    }
    umma::mbar_init(done_bar, 1);
    for (int r = 0; r < RING; ++r) {
      umma::mbar_init(ringfull0 + 8 * r, 1);
      umma::mbar_init(ringempty0 + 8 * r, 5);   // the MMA thread + the four epilogue warps
    }
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     umma::smem_u32(tmem_slot)),
                 "r"(2 * BN)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  umma::fence_before_sync();
  __syncthreads();
  umma::fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ---- tile fetcher and TMA producer ----
      int it = 0;
      int next = fetch();
      for (int j = 0;; ++j) {
        const int t = *abort_flag ? -1 : next;
        const int slot = j % RING;
        if (j >= RING && !umma::mbar_wait(ringempty0 + 8 * slot, ((j / RING) & 1) ^ 1)) {
          *abort_flag = 1;
          break;
        }
        ring[slot] = t;
        asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(ringfull0 + 8 * slot) : "memory");
        if (t < 0) break;
        next = fetch();   // its latency overlaps the copies below
        int bz, sp, m0, n0, kb0, nk;
        tile(t, bz, sp, m0, n0, kb0, nk);
        const int ea = bz / a.A.ediv, eb = bz / a.B.ediv;
        const CUtensorMap* ma = (umma::cache_mode(a.A.mode) && (ea & 1)) ? &map_a1 : &map_a0;
        const uint32_t bytes = b_is_a ? (uint32_t)C::A_BYTES : (uint32_t)C::STAGE_BYTES;
        for (int i = 0; i < nk; ++i, ++it) {
          const int s = it % C::STAGES;
          if (it >= C::STAGES && !umma::mbar_wait(empty0 + 8 * s, ((it / C::STAGES) & 1) ^ 1)) {
            *abort_flag = 1;
            break;
          }
          const uint32_t fb = full0 + 8 * s;
          const uint32_t sa = umma::smem_u32(smem + s * C::STAGE_BYTES);
          const int k = (kb0 + i) * umma::BK;
          umma::mbar_expect_tx(fb, bytes);
          int c0, c1, c2;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            umma::box_coords(a.A, ea, m0 + 64 * h, k, c0, c1, c2);
            umma::tma_load_3d(sa + h * umma::BOX_BYTES, ma, c0, c1, c2, fb);
            if constexpr (C::NA_OP == 2) umma::tma_load_3d(sa + C::A_BYTES + h * umma::BOX_BYTES, &map_a1, c0, c1, c2, fb);
          }
          if (!b_is_a) {
#pragma unroll
            for (int b = 0; b < C::NB_OP; ++b) {
              const CUtensorMap* mb =
                  umma::cache_mode(a.B.mode) ? ((eb & 1) ? &map_b1 : &map_b0) : (b ? &map_b1 : &map_b0);
              const uint32_t sb = sa + C::NA_OP * C::A_BYTES + b * C::B_BYTES;
#pragma unroll
              for (int jj = 0; jj < BN / 64; ++jj) {
                umma::box_coords(a.B, eb, n0 + 64 * jj, k, c0, c1, c2);
                umma::tma_load_3d(sb + jj * umma::BOX_BYTES, mb, c0, c1, c2, fb);
              }
            }
          }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---- MMA issuer ----
      constexpr uint32_t idesc = umma::instr_desc(BN, A_MN, B_MN);
      int it = 0, tc = 0;
      for (int j = 0;; ++j) {
        const int t = ring_take(j, false);
        if (t == -2) *abort_flag = 1;
        if (t < 0) break;
        int bz, sp, m0, n0, kb0, nk;
        tile(t, bz, sp, m0, n0, kb0, nk);
        const int buf = tc & 1, use = tc >> 1;
        if (use > 0 && !umma::mbar_wait(accempty0 + 8 * buf, (use - 1) & 1)) {
          *abort_flag = 1;
          break;
        }
        umma::fence_after_sync();
        const uint32_t acc = tmem + (uint32_t)(buf * BN);
        bool ok = true;
        for (int i = 0; i < nk; ++i, ++it) {
          const int s = it % C::STAGES;
          if (!umma::mbar_wait(full0 + 8 * s, (it / C::STAGES) & 1)) {
            ok = false;
            break;
          }
          umma::fence_after_sync();
          const uint32_t sa = umma::smem_u32(smem + s * C::STAGE_BYTES);
#pragma unroll
          for (int kk = 0; kk < umma::BK / 16; ++kk) {
            // K step of 16: K-major advances 32 bytes inside the swizzle row, MN-major two
            // 8-row groups (2 x 1024 bytes)
            const uint64_t ad = A_MN ? umma::smem_desc(sa + kk * 2048, umma::BOX_BYTES, 1024)
                                     : umma::smem_desc(sa + kk * 32, 16, 1024);
#pragma unroll
            for (int b = 0; b < C::NB_OP; ++b) {
              const uint32_t sb = b_is_a ? sa : sa + C::NA_OP * C::A_BYTES + b * C::B_BYTES;
              const uint64_t bd = B_MN ? umma::smem_desc(sb + kk * 2048, umma::BOX_BYTES, 1024)
                                       : umma::smem_desc(sb + kk * 32, 16, 1024);
              umma::mma_bf16(acc, ad, bd, idesc, (i | kk | b) != 0);
            }
            if constexpr (C::NA_OP == 2) {
              // A1 B0
              const uint32_t sa1 = sa + C::A_BYTES, sb0 = sa + 2 * C::A_BYTES;
              const uint64_t ad1 = A_MN ? umma::smem_desc(sa1 + kk * 2048, umma::BOX_BYTES, 1024)
                                        : umma::smem_desc(sa1 + kk * 32, 16, 1024);
              const uint64_t bd0 = B_MN ? umma::smem_desc(sb0 + kk * 2048, umma::BOX_BYTES, 1024)
                                        : umma::smem_desc(sb0 + kk * 32, 16, 1024);
              umma::mma_bf16(acc, ad1, bd0, idesc, 1u);
            }
          }
          umma::mma_commit(empty0 + 8 * s);
        }
        if (!ok) {
          *abort_flag = 1;
          break;
        }
        umma::mma_commit(accfull0 + 8 * buf);   // fires once this tile's MMAs have completed
        ++tc;
      }
      umma::mma_commit(done_bar);
    }
  } else {
    // ---- epilogue: warp w owns TMEM lanes 32 (w % 4) .. +31, i.e. output rows m0 + 32 (w % 4) + lane ----
    const int q4 = warp & 3;
    const int esz = (a.c_bf16 || a.c_split) ? 2 : 4;
    const bool vec = ((a.ldc * esz) % 16 == 0) && ((((uintptr_t)a.C) & 15) == 0) && ((a.sC * esz) % 16 == 0) &&
                     ((a.ssplit * esz) % 16 == 0) && (!a.c_split || (((uintptr_t)a.C2) & 15) == 0);
    int tc = 0;
    for (int j = 0;; ++j) {
      const int t = ring_take(j, true);
      if (t == -2) *abort_flag = 1;
      if (t < 0) break;
      int bz, sp, m0, n0, kb0, nk;
      tile(t, bz, sp, m0, n0, kb0, nk);
      const int buf = tc & 1, use = tc >> 1;
      bool ok = !*abort_flag && umma::mbar_wait(accfull0 + 8 * buf, use & 1);
      ok = __all_sync(0xffffffffu, ok);   // the TMEM loads are warp-collective
      if (!ok) {
        *abort_flag = 1;
        break;
      }
      umma::fence_after_sync();
      const int row = m0 + q4 * 32 + lane;
      const long long off = (long long)bz * a.sC + (long long)sp * a.ssplit + (long long)row * a.ldc;
#pragma unroll 1
      for (int c0 = 0; c0 < BN; c0 += 32) {
        float v[32];
        umma::tmem_ld32(tmem + (uint32_t)(buf * BN) + ((uint32_t)(q4 * 32) << 16) + (uint32_t)c0, v);
        if (c0 + 32 >= BN) {
          // the accumulator is in registers: hand it back to the MMA warp
          umma::fence_before_sync();
          __syncwarp();
          if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(accempty0 + 8 * buf) : "memory");
        }
        if (nk == 0) {  // an empty K range (a trailing split): its partial sum is zero
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = 0.f;
        }
        if (row >= a.M) continue;
        const int n = n0 + c0;
        if (a.c_trans) {
          // C[n][row]: the warp's lanes hold 32 consecutive rows, so every store of the warp
          // covers 32 consecutive elements of one output row
          const long long toff = (long long)bz * a.sC + (long long)sp * a.ssplit + row;
          if (a.c_split) {
            bf16* hc = (bf16*)a.C + toff;
            bf16* lc = (bf16*)a.C2 + toff;
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (n + j < a.N) {
                const bf16 h = __float2bfloat16_rn(v[j]);
                hc[(long long)(n + j) * a.ldc] = h;
                lc[(long long)(n + j) * a.ldc] = __float2bfloat16_rn(v[j] - __bfloat162float(h));
              }
          } else if (a.c_bf16) {
            bf16* cc = (bf16*)a.C + toff;
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (n + j < a.N) cc[(long long)(n + j) * a.ldc] = __float2bfloat16_rn(v[j]);
          } else {
            float* cc = (float*)a.C + toff;
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (n + j < a.N) {
                float* o = cc + (long long)(n + j) * a.ldc;
                *o = a.c_accum ? *o + v[j] : v[j];
              }
          }
          continue;
        }
        if (a.c_split) {
          bf16* hrow = (bf16*)a.C + off;
          bf16* lrow = (bf16*)a.C2 + off;
          if (vec && n + 32 <= a.N) {
#pragma unroll
            for (int j = 0; j < 32; j += 8) {
              uint32_t hw[4], lw[4];
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const __nv_bfloat162 h = __floats2bfloat162_rn(v[j + 2 * q], v[j + 2 * q + 1]);
                const __nv_bfloat162 l = __floats2bfloat162_rn(v[j + 2 * q] - __low2float(h),
                                                               v[j + 2 * q + 1] - __high2float(h));
                hw[q] = *(const uint32_t*)&h;
                lw[q] = *(const uint32_t*)&l;
              }
              *(uint4*)(hrow + n + j) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
              *(uint4*)(lrow + n + j) = make_uint4(lw[0], lw[1], lw[2], lw[3]);
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (n + j < a.N) {
                const bf16 h = __float2bfloat16_rn(v[j]);
                hrow[n + j] = h;
                lrow[n + j] = __float2bfloat16_rn(v[j] - __bfloat162float(h));
              }
          }
        } else if (a.c_bf16) {
          bf16* crow = (bf16*)a.C + off;
          if (vec && n + 32 <= a.N) {
#pragma unroll
            for (int j = 0; j < 32; j += 8) {
              uint4 w;
              __nv_bfloat162 h0 = __floats2bfloat162_rn(v[j], v[j + 1]), h1 = __floats2bfloat162_rn(v[j + 2], v[j + 3]);
              __nv_bfloat162 h2 = __floats2bfloat162_rn(v[j + 4], v[j + 5]), h3 = __floats2bfloat162_rn(v[j + 6], v[j + 7]);
              w.x = *(uint32_t*)&h0;
              w.y = *(uint32_t*)&h1;
              w.z = *(uint32_t*)&h2;
              w.w = *(uint32_t*)&h3;
              *(uint4*)(crow + n + j) = w;
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (n + j < a.N) crow[n + j] = __float2bfloat16_rn(v[j]);
          }
        } else {
          float* crow = (float*)a.C + off;
          if (vec && n + 32 <= a.N) {
#pragma unroll
            for (int j = 0; j < 32; j += 4) {
              float4 o = make_float4(v[j], v[j + 1], v[j + 2], v[j + 3]);
              if (a.c_accum) {
                const float4 cc = *(const float4*)(crow + n + j);
                o.x += cc.x;
                o.y += cc.y;
                o.z += cc.z;
                o.w += cc.w;
              }
              *(float4*)(crow + n + j) = o;
            }
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (n + j < a.N) crow[n + j] = a.c_accum ? crow[n + j] + v[j] : v[j];
          }
        }
      }
      ++tc;
    }
  }
  __syncwarp();
  // every issued MMA has completed before tensor memory is freed
  const bool drained = umma::mbar_wait(done_bar, 0);
  if ((*abort_flag || !drained) && threadIdx.x == 0 && a.status) atomicOr(a.status, DEV_ERR_TIMEOUT);
  umma::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    umma::fence_after_sync();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(2 * BN) : "memory");
  }
}

// ---- host side ----------------------------------------------------------------------------
typedef CUresult (*TensorMapEncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                           const cuuint64_t*, const cuuint32_t*, const cuuint32_t*,
                                           CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                           CUtensorMapFloatOOBfill);

// the driver's tensor-map encoder, fetched once through the runtime (no link against libcuda)
inline TensorMapEncodeTiledFn tensor_map_encoder() {
  static TensorMapEncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return (TensorMapEncodeTiledFn)p;
  }();
  return fn;
}

// rank-3 bf16 tensor map over a [d2][d1][d0] array (pitches in bytes), 64 x 64 x 1 boxes,
// 128-byte swizzle, zero fill outside the array.  Returns false if the encoder refuses.
inline bool make_box_map(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t pitch1,
                         uint64_t pitch2) {
  TensorMapEncodeTiledFn enc = tensor_map_encoder();
  if (!enc || ((uintptr_t)base & 15) || (pitch1 & 15) || (pitch2 & 15)) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t pitches[2] = {pitch1, pitch2};
  cuuint32_t box[3] = {64, 64, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, pitches, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// the cache [n_layers][H][T][D] as slices (XT modes) or as rows (row modes)
inline bool map_cache_xt(CUtensorMap* m, const void* x, int n_layers, int H, int T, int D) {
  return make_box_map(m, x, D, T, (uint64_t)n_layers * H, (uint64_t)D * 2, (uint64_t)T * D * 2);
}
inline bool map_cache_rows(CUtensorMap* m, const void* x, int n_layers, int H, int T, int D) {
  const uint64_t rows = (uint64_t)n_layers * H * T;
  return make_box_map(m, x, D, rows, 1, (uint64_t)D * 2, rows * D * 2);
}
// dense [entries][rows][ld] bf16
inline bool map_dense(CUtensorMap* m, const void* p, long long ld, long long rows, long long entries) {
  return make_box_map(m, p, ld, rows, entries, (uint64_t)ld * 2, (uint64_t)rows * ld * 2);
}

struct UmmaMaps {
  CUtensorMap a0, a1, b0, b1;
};

template <int BN, int NB, bool A_MN, bool B_MN>
cudaError_t launch_umma_t(const UmmaMaps& m, const UmmaArgs& a, cudaStream_t st) {
  constexpr int smem = umma::Cfg<BN, NB>::SMEM;
  cudaError_t e = cudaFuncSetAttribute(umma_gemm_kernel<BN, NB, A_MN, B_MN>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long tiles = ceil_div(a.N, BN) * ceil_div(a.M, umma::BM) * (long long)a.batch * a.splits;
  if (tiles <= 0 || !a.sched) return cudaErrorInvalidValue;
  const unsigned grid = (unsigned)(tiles < sms ? tiles : sms);
  e = cudaMemsetAsync(a.sched, 0, sizeof(int), st);
  if (e != cudaSuccess) return e;
  count_launch();
  umma_gemm_kernel<BN, NB, A_MN, B_MN><<<grid, 192, smem, st>>>(m.a0, m.a1, m.b0, m.b1, a);
  return cudaGetLastError();
}

template <int BN, int NB>
cudaError_t launch_umma_bn(const UmmaMaps& m, const UmmaArgs& a, cudaStream_t st) {
  const bool amn = a.A.mode == UM_XT_MN || a.A.mode == UM_ROW_MN || a.A.mode == UM_DENSE_MN;
  const bool bmn = a.B.mode == UM_XT_MN || a.B.mode == UM_ROW_MN || a.B.mode == UM_DENSE_MN;
  if (amn) return bmn ? launch_umma_t<BN, NB, true, true>(m, a, st) : launch_umma_t<BN, NB, true, false>(m, a, st);
  return bmn ? launch_umma_t<BN, NB, false, true>(m, a, st) : launch_umma_t<BN, NB, false, false>(m, a, st);
}

// C = A * sum_{b < nb} B_b on the tensor cores (nb = 1, 2), C = A0 B0 + A0 B1 + A1 B0
// (nb = 3; maps a0, a1, b0, b1; N tiles of 128), or C = (A0 + A1) B (nb = 4; N tiles of 256).
// nb = 2, 3 require dense B operands, nb = 3, 4 dense A operands; b_is_a requires M = N <= 128
// and identical A and B operands.
inline cudaError_t launch_umma(const UmmaMaps& m, UmmaArgs a, int nb, cudaStream_t st) {
  if (a.splits < 1 || (a.splits > 1 && (a.kchunk <= 0 || a.kchunk % umma::BK)) || a.batch < 1 || nb < 1 || nb > 4 ||
      ((nb == 2 || nb == 3) && umma::cache_mode(a.B.mode)) ||
      (nb >= 3 && (umma::cache_mode(a.A.mode) || a.b_is_a)) || (a.b_is_a && (a.M > 128 || a.N > 128 || nb != 1)))
    return cudaErrorInvalidValue;
  if (a.splits == 1) a.kchunk = (int)round_up(a.K, umma::BK);
  if (a.c_accum && a.c_bf16) return cudaErrorInvalidValue;
  if (a.c_split && (!a.C2 || a.c_bf16 || a.c_accum)) return cudaErrorInvalidValue;
  // N tiles of 256 only with one B operand: with two (hi + lo) a 256-wide stage takes 80 KB and
  // leaves room for two pipeline stages, a 128-wide one 48 KB and four
  if (nb == 3) return launch_umma_bn<128, 3>(m, a, st);   // a 64 KB stage: three stages
  if (nb == 4) return launch_umma_bn<256, 4>(m, a, st);   // 2 x 16 KB + 32 KB: three stages
  if (a.bn == 256 || (a.bn == 0 && a.N > 128 && nb == 1))
    return nb == 2 ? launch_umma_bn<256, 2>(m, a, st) : launch_umma_bn<256, 1>(m, a, st);
  return nb == 2 ? launch_umma_bn<128, 2>(m, a, st) : launch_umma_bn<128, 1>(m, a, st);
}

// X-products of every unit.
//   z_side = false : C_u (T x N) = X_(T),u   * sum_b F_b,u   with F_b,u = Fb[u] (M x ldf)
//   z_side = true  : C_u (M x N) = X_(T),u^T * sum_b F_b,u   with F_b,u = Fb[u] (T x ldf)
// xk / xv: the K and V caches [n_layers][H][T][D] bf16; F1 may be null (one B operand).
// C: fp32, or with C2 the result as a bf16 hi (C) + lo (C2) pair, pitch ldc.
// With F = F0 + F1 (an fp32 operand as bf16 hi + lo) the product runs transposed, C^T =
// (F0 + F1)^T X^T: the pair is the A operand and the cache a 256-wide B tile, so a stage holds
// one cache tile for two MMAs (a 128-wide B tile with the pair on the B side needs a third more
// shared-memory traffic per MMA, which the MMAs then wait on).  The tiles are stored
// transposed and handed out M tile fastest, so the CTAs working at one time share the cache
// tile in L2.
inline cudaError_t umma_x_product(const void* xk, const void* xv, int n_layers, int H, int T, int D, int S,
                                  int nunits, bool z_side, const bf16* F0, const bf16* F1, int ldf, int N, void* C,
                                  long long ldc, uint32_t* status, int* sched, cudaStream_t st, void* C2 = nullptr) {
  if (D % 64 || ldf % 8 || N > ldf) return cudaErrorInvalidValue;
  int dshift = 0;
  while ((1 << dshift) < D) ++dshift;
  const int M = S * D;
  const long long krows = z_side ? T : M;
  UmmaMaps m;
  UmmaArgs a;
  if (F1) {
    if (!map_dense(&m.a0, F0, ldf, krows, nunits) || !map_dense(&m.a1, F1, ldf, krows, nunits) ||
        !map_cache_xt(&m.b0, xk, n_layers, H, T, D) || !map_cache_xt(&m.b1, xv, n_layers, H, T, D))
      return cudaErrorInvalidValue;
    a.M = N;
    a.N = z_side ? M : T;
    a.K = z_side ? T : M;
    a.A.mode = UM_DENSE_MN;
    a.B.mode = z_side ? UM_XT_MN : UM_XT_K;
    a.B.S = S;
    a.B.d_shift = dshift;
    a.c_trans = 1;
    a.m_fast = 1;
  } else {
    if (!map_cache_xt(&m.a0, xk, n_layers, H, T, D) || !map_cache_xt(&m.a1, xv, n_layers, H, T, D) ||
        !map_dense(&m.b0, F0, ldf, krows, nunits))
      return cudaErrorInvalidValue;
    m.b1 = m.b0;
    a.M = z_side ? M : T;
    a.N = N;
    a.K = z_side ? T : M;
    a.A.mode = z_side ? UM_XT_MN : UM_XT_K;
    a.A.S = S;
    a.A.d_shift = dshift;
    a.B.mode = UM_DENSE_MN;
  }
  a.batch = nunits;
  a.C = C;
  a.ldc = ldc;
  a.sC = (long long)(z_side ? M : T) * ldc;
  a.status = status;
  a.sched = sched;
  if (C2) {
    a.c_split = 1;
    a.C2 = C2;
  }
  return launch_umma(m, a, F1 ? 4 : 1, st);
}

}  // namespace jolt
