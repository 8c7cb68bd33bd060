// Distortion table on the 5th-generation tensor cores (D = 128, up to 4 token-rank cuts).
//
// One CTA owns 128 consecutive tokens of one slice s of unit u (TMEM lane = token row) and
// walks every feature-rank candidate r_D.  For a candidate, the reconstruction of the tile in
// the rotated basis, U_s[:, :r_T] P'(r_D)[:r_T, :], is needed at every token-rank cut r_T.
// The token-rank axis is cut into segments [c_{i-1}, c_i) and the tensor cores accumulate
// each segment in its own TMEM accumulator (4 x 128 fp32 columns, all of tensor memory):
//   * one thread issues the TMA copies of the U tile (128 x 64 bf16, K-major) and of P'
//     (64 x 128 bf16, rows of the operator) for every 64-wide K block;
//   * one thread issues tcgen05.mma (M = 128, N = 128, K = 16) into the accumulator of the
//     segment the K step belongs to and commits an mbarrier when a segment is complete;
//   * sixteen epilogue warps (four per TMEM lane quarter, 32 columns each) read a
//     finished segment with tcgen05.ld, release it at once (the next candidate's MMAs into
//     that segment may start), add it to a running sum kept in registers, and evaluate the
//     quantiser of every bit-width on rho = x' - running sum, block by block -- the
//     arithmetic of table_kernel (kernels.cuh), which is why the two give the same entries.
// x' (the tile rotated along the features) is formed once per CTA in shared memory by the
// epilogue warps while the copy and MMA warps start on the first operands.
//
// Every mbarrier wait is bounded (umma::mbar_wait); a wait that gives up raises
// DEV_ERR_TIMEOUT and the CTA stops issuing work, keeps its named-barrier schedule, and waits
// (bounded) for its issued MMAs before it frees tensor memory.
#pragma once

#include "kernels.cuh"
#include "umma.cuh"

namespace jolt {
namespace ttc {
constexpr int ROWS = 128;                                  // tokens per CTA
constexpr int DIM = 128;                                   // features = MMA N
constexpr int BK = 64;
constexpr int STAGES = 4;
constexpr int U_BYTES = ROWS * BK * 2;                     // 16 KB
constexpr int P_BYTES = BK * DIM * 2;                      // 16 KB
constexpr int STAGE_BYTES = U_BYTES + P_BYTES;
constexpr int XS_LD = DIM + 4;                             // fp32 pitch of the rotated tile
constexpr int XS_BYTES = ROWS * XS_LD * 4;
constexpr int EPI_WARPS = 16;                             // four per TMEM lane quarter
constexpr int EPI_COLS = DIM / (EPI_WARPS / 4);            // columns per epilogue warp
constexpr int THREADS = (EPI_WARPS + 2) * 32;              // + TMA warp + MMA warp
constexpr int MAXT = 4;                                    // token-rank cuts
constexpr int BAR_OFF = STAGES * STAGE_BYTES + XS_BYTES;
constexpr int SMEM = 1024 + BAR_OFF + 512;                 // alignment slack + barriers
constexpr int TMEM_COLS = 512;
}  // namespace ttc

struct TableTcArgs {
  CacheView cv;
  int rTmax;
  Cands cand;
  uint64_t seed;
  double* partial;      // [unit][S][tiles][nD][nT][nB]
  int tiles;            // ceil(T / 128)
  uint32_t* status;
};

// the tile's rows rotated along the features into xs (fp32, pitch XS_LD): sign flip, the
// Walsh-Hadamard butterflies in the order of fwht_regs (strides 1, 2, ..., 64), 1 / sqrt(D).
// Run by the NTHREADS = 4 x ROWS epilogue threads (threads 0 .. NTHREADS-1) alone, four per
// row, 32 features each: strides 1 .. 16 in registers, strides 32 and 64 with the partner
// threads p ^ 1 and p ^ 2 (lanes of the same warp).  The operations are those of one thread
// per row, so the result is the same bit for bit.  Ends with named barrier 1 over the
// NTHREADS threads, while the copy and MMA warps start on the operands.
template <typename TX, int NTHREADS>
__device__ __forceinline__ void ttc_rotate_tile(const TX* X, int T, int t0, const float* sig, float* xs) {
  using namespace ttc;
  static_assert(NTHREADS == 4 * ROWS && DIM == 128, "four threads per row, 32 features each");
  constexpr int V = 16 / sizeof(TX);   // elements per 16-byte load
  const int r = threadIdx.x >> 2, p = threadIdx.x & 3, t = t0 + r;
  float v[32];
  if (t < T) {
    const TX* src = X + (long long)t * DIM + 32 * p;
#pragma unroll
    for (int q = 0; q < 32 / V; ++q) {
      const uint4 w = *reinterpret_cast<const uint4*>(src + q * V);
      const TX* e = reinterpret_cast<const TX*>(&w);
#pragma unroll
      for (int i = 0; i < V; ++i) v[q * V + i] = ld_as_float(e + i) * sig[32 * p + q * V + i];
    }
  } else {
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = 0.f;
  }
  fwht_regs<32>(v);
  // a pair (lower a, upper b) becomes (a + b, a - b): the upper thread of the pair forms
  // partner - own, the lower own + partner
  const bool up32 = (p & 1) != 0, up64 = (p & 2) != 0;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const float o = __shfl_xor_sync(0xffffffffu, v[i], 1);
    v[i] = up32 ? o - v[i] : v[i] + o;
  }
  const float sc = (float)(1.0 / sqrt((double)DIM));
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const float o = __shfl_xor_sync(0xffffffffu, v[i], 2);
    v[i] = (up64 ? o - v[i] : v[i] + o) * sc;
  }
  float* dst = xs + r * XS_LD + 32 * p;
#pragma unroll
  for (int i = 0; i < 32; i += 4) *reinterpret_cast<float4*>(dst + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
  asm volatile("bar.sync 1, %0;" ::"n"(NTHREADS) : "memory");
}

__device__ __forceinline__ void ttc_tmem_ld16(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// ---------------------------------------------------------------------------------------
// Quantiser error sums of one 16-wide block for the table (packed pairs throughout):
//   * block min / max by three-input min / max (exact, the same values as a two-input tree);
//   * lo and the fp16 step exactly as the encoder forms them (rd16, quant_step_cvt);
//   * code = round-half-even(d / step) through the approximate reciprocal of step, the error
//     (d - code * step)^2 summed in four packed partial sums.
// The approximate reciprocal can move a code only where d / step lies within a few ulp of a
// half-integer, where both neighbouring codes give the same squared error to that precision,
// so the table entry (a sum of squared errors) is unchanged to fp32 resolution; the stored
// codes come from the encoder, which uses the correctly rounded reciprocal.
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ float ttc_min3(float a, float b, float c) {
  float r;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ float ttc_max3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
__device__ __forceinline__ float ttc_rcp_approx(float x) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(x));
  return r;
}

// squared-error sums of one bit-width over one block, added into one packed partial sum `a`
// that runs over all blocks of the thread for the current cut (the five bit-widths give the
// scheduler independent chains); a block whose scale overflows fp16 makes the sums +inf
template <int B>
__device__ __forceinline__ void ttc_bit_error(const float2* v, const float2* d, float mx, float lo, float2& a) {
  if constexpr (B == 0) {
#pragma unroll
    for (int j = 0; j < 8; ++j) a = __ffma2_rn(v[j], v[j], a);
  } else {
    const float step = quant_step_cvt(mx, lo, B);
    const bool ok = isfinite(lo) && step <= kFp16Max;
    const float inv = step > 0.f ? ttc_rcp_approx(step) : 0.f;
    const float2 inv2 = make_float2(inv, inv), nstep2 = make_float2(-step, -step);
    const float2 sh = make_float2(kRoundShift, kRoundShift), nsh = make_float2(-kRoundShift, -kRoundShift);
    float2 b0 = a;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float2 c = __fadd2_rn(__ffma2_rn(d[j], inv2, sh), nsh);
      const float2 e = __ffma2_rn(c, nstep2, d[j]);
      b0 = __ffma2_rn(e, e, b0);
    }
    a = ok ? b0 : make_float2(INFINITY, INFINITY);
  }
}

// every bit-width of the set for one block of rho given as 8 packed pairs
template <int... Bs>
__device__ __forceinline__ void ttc_block_errors(const float2* v, float2* acc, BitSet<Bs...>) {
  const float m0 = ttc_min3(v[0].x, v[0].y, v[1].x), m1 = ttc_min3(v[1].y, v[2].x, v[2].y);
  const float m2 = ttc_min3(v[3].x, v[3].y, v[4].x), m3 = ttc_min3(v[4].y, v[5].x, v[5].y);
  const float m4 = ttc_min3(v[6].x, v[6].y, v[7].x);
  const float mn = fminf(ttc_min3(m0, m1, m2), ttc_min3(m3, m4, v[7].y));
  const float x0 = ttc_max3(v[0].x, v[0].y, v[1].x), x1 = ttc_max3(v[1].y, v[2].x, v[2].y);
  const float x2 = ttc_max3(v[3].x, v[3].y, v[4].x), x3 = ttc_max3(v[4].y, v[5].x, v[5].y);
  const float x4 = ttc_max3(v[6].x, v[6].y, v[7].x);
  const float mx = fmaxf(ttc_max3(x0, x1, x2), ttc_max3(x3, x4, v[7].y));
  const float lo = rd16(mn);
  const float2 nlo = make_float2(-lo, -lo);
  float2 d[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) d[j] = __fadd2_rn(v[j], nlo);
  int i = 0;
  (ttc_bit_error<Bs>(v, d, mx, lo, acc[i++]), ...);
}

__device__ __forceinline__ void ttc_epi_sync() { asm volatile("bar.sync 1, %0;" ::"n"(ttc::EPI_WARPS * 32) : "memory"); }

// grid (S x tiles, units), slices fastest; ttc::THREADS threads; ttc::SMEM bytes of dynamic
// shared memory.
// Registers: the SM's file is four partitions of 16K, one per scheduler, and the 18 warps put
// five on one partition, so a thread gets at most 96 (the launch bound makes ptxas keep to it).
template <typename TX, typename BITS>
__global__ void __launch_bounds__(ttc::THREADS, 1)
    table_tc_kernel(const __grid_constant__ CUtensorMap map_u, const __grid_constant__ CUtensorMap map_p,
                    TableTcArgs a) {
  using namespace ttc;
  extern __shared__ uint8_t ttc_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)ttc_raw + 1023) & ~(uintptr_t)1023);
  float* xs = reinterpret_cast<float*>(smem + STAGES * STAGE_BYTES);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + BAR_OFF);
  // full[STAGES] empty[STAGES] accfull[MAXT] accfree[MAXT] done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 2 * MAXT + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  __shared__ float sig[DIM];
  __shared__ float red[EPI_WARPS][MAXT * MAXC];

  const int T = a.cv.T, S = a.cv.S, NU = 2 * (a.cv.n_layers / a.cv.Lg);
  // slices fastest: the CTAs that run together share the token tile of U (one read from memory)
  const int s = blockIdx.x % S, tile = blockIdx.x / S, u = blockIdx.y;
  const int t0 = tile * ROWS;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const Cands& cd = a.cand;
  const int nT = cd.nT, nD = cd.nD, nB = cd.nB;
  const int klast = cd.rT[nT - 1];
  const int nkb = (klast + BK - 1) / BK;
  const uint32_t full0 = umma::smem_u32(bars), empty0 = full0 + 8 * STAGES, accfull0 = empty0 + 8 * STAGES;
  const uint32_t accfree0 = accfull0 + 8 * MAXT, done_bar = accfree0 + 8 * MAXT;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      umma::mbar_init(full0 + 8 * i, 1);
      umma::mbar_init(empty0 + 8 * i, 1);
    }
    for (int i = 0; i < MAXT; ++i) {
      umma::mbar_init(accfull0 + 8 * i, 1);
      umma::mbar_init(accfree0 + 8 * i, EPI_WARPS);
    }
    umma::mbar_init(done_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == EPI_WARPS) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(umma::smem_u32(tmem_slot)),
                 "n"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  for (int d = threadIdx.x; d < DIM; d += THREADS) sig[d] = rotation_sign(a.seed, u + a.cv.u0, d);
  umma::fence_before_sync();
  __syncthreads();
  umma::fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (warp == EPI_WARPS) {
    if (lane == 0) {
      // ---- TMA producer: for every candidate r_D, the K blocks of U and P' ----
      int it = 0;
      for (int iD = 0; iD < nD && !*abort_flag; ++iD) {
        const int ep = (iD * NU + u) * S + s;
        for (int j = 0; j < nkb; ++j, ++it) {
          const int st = it % STAGES;
          if (it >= STAGES && !umma::mbar_wait(empty0 + 8 * st, ((it / STAGES) & 1) ^ 1)) {
            *abort_flag = 1;
            break;
          }
          const uint32_t fb = full0 + 8 * st;
          const uint32_t sa = umma::smem_u32(smem + st * STAGE_BYTES);
          umma::mbar_expect_tx(fb, STAGE_BYTES);
          umma::tma_load_3d(sa, &map_u, j * BK, t0, u, fb);
          umma::tma_load_3d(sa + umma::BOX_BYTES, &map_u, j * BK, t0 + 64, u, fb);
          umma::tma_load_3d(sa + U_BYTES, &map_p, 0, j * BK, ep, fb);
          umma::tma_load_3d(sa + U_BYTES + umma::BOX_BYTES, &map_p, 64, j * BK, ep, fb);
        }
      }
    }
  } else if (warp == EPI_WARPS + 1) {
    if (lane == 0) {
      // ---- MMA issuer: K step k16 goes to the accumulator of the segment holding it ----
      constexpr uint32_t idesc = umma::instr_desc(DIM, false, true);
      int it = 0;
      for (int iD = 0; iD < nD && !*abort_flag; ++iD) {
        int seg = 0;
        for (int j = 0; j < nkb && !*abort_flag; ++j, ++it) {
          const int st = it % STAGES;
          if (!umma::mbar_wait(full0 + 8 * st, (it / STAGES) & 1)) {
            *abort_flag = 1;
            break;
          }
          umma::fence_after_sync();
          const uint32_t sa = umma::smem_u32(smem + st * STAGE_BYTES);
          for (int kk = 0; kk < BK / 16; ++kk) {
            const int k0 = j * BK + kk * 16;
            if (k0 >= klast) break;
            while (k0 >= cd.rT[seg]) ++seg;
            const int lo = seg ? cd.rT[seg - 1] : 0;
            if (k0 == lo && iD > 0) {
              // the previous candidate's epilogue must have read this segment
              if (!umma::mbar_wait(accfree0 + 8 * seg, (iD - 1) & 1)) {
                *abort_flag = 1;
                break;
              }
              umma::fence_after_sync();
            }
            const uint64_t ad = umma::smem_desc(sa + kk * 32, 16, 1024);
            const uint64_t bd = umma::smem_desc(sa + U_BYTES + kk * 2048, umma::BOX_BYTES, 1024);
            umma::mma_bf16(tmem + (uint32_t)(seg * DIM), ad, bd, idesc, k0 != lo ? 1u : 0u);
            if (k0 + 16 == cd.rT[seg]) umma::mma_commit(accfull0 + 8 * seg);
          }
          umma::mma_commit(empty0 + 8 * st);
        }
      }
      umma::mma_commit(done_bar);   // fires when every MMA issued above has completed
    }
  } else {
    // ---- epilogue: warp w owns TMEM lanes 32 (w % 4) .. +31 and columns EPI_COLS (w / 4) .. ----
    const int row = 32 * (warp & 3) + lane;
    const int cbase = EPI_COLS * (warp >> 2);
    const uint32_t lane_addr = (uint32_t)(32 * (warp & 3)) << 16;
    const BitConsts kb = bit_consts(cd);
    double* out = a.partial + (((long long)u * S + s) * a.tiles + tile) * (long long)(nD * nT * nB);
    const float* xrow = xs + row * XS_LD + cbase;
    ttc_rotate_tile<TX, EPI_WARPS * 32>(reinterpret_cast<const TX*>(a.cv.unit_ptr(u)) + (long long)s * T * DIM, T,
                                         t0, sig, xs);
    const float2 neg1 = make_float2(-1.f, -1.f);
    for (int iD = 0; iD < nD; ++iD) {
      float2 nrun[EPI_COLS / 2];   // minus the running sum of the finished segments
#pragma unroll
      for (int j = 0; j < EPI_COLS / 2; ++j) nrun[j] = make_float2(0.f, 0.f);
#pragma unroll 1
      for (int i = 0; i < nT; ++i) {
        bool ok = !*abort_flag && umma::mbar_wait(accfull0 + 8 * i, iD & 1);
        ok = __all_sync(0xffffffffu, ok);   // the TMEM loads below are warp-collective
        if (!ok) *abort_flag = 1;
        float err[MAXC];
#pragma unroll
        for (int b = 0; b < MAXC; ++b) err[b] = 0.f;
        float2 acc2[MAXC];   // packed partial sums of the fixed bit set (horizontal sum per cut)
#pragma unroll
        for (int b = 0; b < MAXC; ++b) acc2[b] = make_float2(0.f, 0.f);
        if (ok) {
          umma::fence_after_sync();
#pragma unroll
          for (int hh = 0; hh < EPI_COLS / 16; ++hh) {
            float seg[16];
            ttc_tmem_ld16(tmem + lane_addr + (uint32_t)(i * DIM + cbase + 16 * hh), seg);
            asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
            for (int j = 0; j < 8; ++j)
              nrun[8 * hh + j] = __ffma2_rn(make_float2(seg[2 * j], seg[2 * j + 1]), neg1, nrun[8 * hh + j]);
          }
          // the segment is in registers: release it to the next candidate's MMAs
          umma::fence_before_sync();
          __syncwarp();
          if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(accfree0 + 8 * i) : "memory");
          if (t0 + row < T) {
#pragma unroll
            for (int m = 0; m < EPI_COLS / 16; ++m) {
              float2 v2[8];
#pragma unroll
              for (int q = 0; q < 4; ++q) {
                const float4 xv = reinterpret_cast<const float4*>(xrow + 16 * m)[q];
                v2[2 * q] = __fadd2_rn(make_float2(xv.x, xv.y), nrun[8 * m + 2 * q]);
                v2[2 * q + 1] = __fadd2_rn(make_float2(xv.z, xv.w), nrun[8 * m + 2 * q + 1]);
              }
              if constexpr (std::is_same<BITS, void>::value) {
                block_errors(reinterpret_cast<const float*>(v2), kb, err);
              } else {
                ttc_block_errors(v2, acc2, BITS{});
              }
            }
          }
          if constexpr (!std::is_same<BITS, void>::value) {
#pragma unroll
            for (int b = 0; b < BITS::N; ++b) err[b] = acc2[b].x + acc2[b].y;
          }
        }
        // this cut's sums over the warp (every lane takes part, also after an abort)
#pragma unroll
        for (int b = 0; b < MAXC; ++b) {
          if (b >= nB) break;
          float v = err[b];
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
          if (lane == 0) red[warp][i * MAXC + b] = v;
        }
      }
      // over the epilogue warps in fixed order (fp64)
      ttc_epi_sync();
      if (threadIdx.x < nT * nB) {
        const int i = threadIdx.x / nB, b = threadIdx.x - i * nB;
        double v = 0.0;
        for (int w = 0; w < EPI_WARPS; ++w) v += (double)red[w][i * MAXC + b];
        out[(iD * nT + i) * nB + b] = v;
      }
      ttc_epi_sync();
    }
  }
  // every issued MMA has completed before tensor memory is freed
  __syncwarp();
  const bool drained = umma::mbar_wait(done_bar, 0);
  if ((*abort_flag || !drained) && threadIdx.x == 0 && a.status) atomicOr(a.status, DEV_ERR_TIMEOUT);
  umma::fence_before_sync();
  __syncthreads();
  if (warp == EPI_WARPS) {
    umma::fence_after_sync();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "n"(TMEM_COLS) : "memory");
  }
}

}  // namespace jolt

namespace jolt {
// ---------------------------------------------------------------------------------------
// Encoder on the tensor cores (D = 128): the chosen (r_T, r_D, b) of the unit from the blob's
// unit table; one CTA per 128 tokens of one slice.  The token-rank axis [0, r_T) is cut into
// 128-rank segments (two 64-rank K blocks accumulated in one accumulator) that rotate through
// the four TMEM accumulators.  The epilogue subtracts every finished segment from the rotated
// tile without rounding error (TwoSum into hi + lo), so the residual carries the fp32 error of
// one 128-rank segment, not of the whole sum; then it quantises rho = hi + lo block by block,
// packs the codes and writes codes and scales.
// Sixteen epilogue warps (four per TMEM lane quarter, 32 columns each).
// ---------------------------------------------------------------------------------------
namespace etc {
constexpr int EPI_WARPS = 16;
constexpr int THREADS = (EPI_WARPS + 2) * 32;
constexpr int COLS = ttc::DIM / (EPI_WARPS / 4);   // 32
// K blocks (64 ranks each) accumulated in one TMEM accumulator before the epilogue folds it
// into the residual: the residual carries the fp32 rounding of one 128-rank partial sum
constexpr int SEG_KB = 2;
}  // namespace etc

struct EncodeTcArgs {
  CacheView cv;
  int rTmax;
  Cands cand;
  uint64_t seed;
  unsigned char* blob;
  uint32_t* status;
};

template <typename TX>
__global__ void __launch_bounds__(etc::THREADS, 1)
    encode_tc_kernel(const __grid_constant__ CUtensorMap map_u, const __grid_constant__ CUtensorMap map_p,
                     EncodeTcArgs a) {
  using namespace ttc;
  extern __shared__ uint8_t etc_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)etc_raw + 1023) & ~(uintptr_t)1023);
  float* xs = reinterpret_cast<float*>(smem + STAGES * STAGE_BYTES);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + BAR_OFF);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 2 * MAXT + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  __shared__ float sig[DIM];

  const int T = a.cv.T, S = a.cv.S, NU = 2 * (a.cv.n_layers / a.cv.Lg);
  // slices fastest: the CTAs that run together share the token tile of U (one read from memory)
  const int s = blockIdx.x % S, tile = blockIdx.x / S, u = blockIdx.y;
  const BlobHeader* gh = reinterpret_cast<const BlobHeader*>(a.blob);
  const UnitHeader uh = reinterpret_cast<const UnitHeader*>(a.blob + sizeof(BlobHeader))[u];
  if (gh->status != 0 || uh.bits == 0) return;   // uniform over the CTA: nothing to write
  const int t0 = tile * ROWS;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rT = uh.r_T, b = uh.bits;
  int iD = 0;
  while (iD < a.cand.nD && a.cand.rD[iD] != uh.r_D) ++iD;
  const int nkb = (rT + BK - 1) / BK;     // K blocks of 64 ranks
  const int nseg = (nkb + etc::SEG_KB - 1) / etc::SEG_KB;   // segments of SEG_KB K blocks
  const uint32_t full0 = umma::smem_u32(bars), empty0 = full0 + 8 * STAGES, accfull0 = empty0 + 8 * STAGES;
  const uint32_t accfree0 = accfull0 + 8 * MAXT, done_bar = accfree0 + 8 * MAXT;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      umma::mbar_init(full0 + 8 * i, 1);
      umma::mbar_init(empty0 + 8 * i, 1);
    }
    for (int i = 0; i < MAXT; ++i) {
      umma::mbar_init(accfull0 + 8 * i, 1);
      umma::mbar_init(accfree0 + 8 * i, etc::EPI_WARPS);
    }
    umma::mbar_init(done_bar, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == etc::EPI_WARPS) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(umma::smem_u32(tmem_slot)),
                 "n"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  for (int d = threadIdx.x; d < DIM; d += etc::THREADS) sig[d] = rotation_sign(a.seed, u + a.cv.u0, d);
  umma::fence_before_sync();
  __syncthreads();
  umma::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  const int ep = (iD * NU + u) * S + s;

  if (warp == etc::EPI_WARPS) {
    if (lane == 0) {
      for (int j = 0; j < nkb; ++j) {
        const int st = j % STAGES;
        if (j >= STAGES && !umma::mbar_wait(empty0 + 8 * st, ((j / STAGES) & 1) ^ 1)) {
          *abort_flag = 1;
          break;
        }
        const uint32_t fb = full0 + 8 * st;
        const uint32_t sa = umma::smem_u32(smem + st * STAGE_BYTES);
        umma::mbar_expect_tx(fb, STAGE_BYTES);
        umma::tma_load_3d(sa, &map_u, j * BK, t0, u, fb);
        umma::tma_load_3d(sa + umma::BOX_BYTES, &map_u, j * BK, t0 + 64, u, fb);
        umma::tma_load_3d(sa + U_BYTES, &map_p, 0, j * BK, ep, fb);
        umma::tma_load_3d(sa + U_BYTES + umma::BOX_BYTES, &map_p, 64, j * BK, ep, fb);
      }
    }
  } else if (warp == etc::EPI_WARPS + 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = umma::instr_desc(DIM, false, true);
      for (int j = 0; j < nkb && !*abort_flag; ++j) {
        const int seg = j / etc::SEG_KB, jin = j - seg * etc::SEG_KB;
        const int st = j % STAGES, acc = seg % MAXT, use = seg / MAXT;
        if (!umma::mbar_wait(full0 + 8 * st, (j / STAGES) & 1)) {
          *abort_flag = 1;
          break;
        }
        // a segment's first K block waits until the epilogue has read the accumulator's last use
        if (jin == 0 && use > 0 && !umma::mbar_wait(accfree0 + 8 * acc, (use - 1) & 1)) {
          *abort_flag = 1;
          break;
        }
        umma::fence_after_sync();
        const uint32_t sa = umma::smem_u32(smem + st * STAGE_BYTES);
        for (int kk = 0; kk < BK / 16 && j * BK + kk * 16 < rT; ++kk) {
          const uint64_t ad = umma::smem_desc(sa + kk * 32, 16, 1024);
          const uint64_t bd = umma::smem_desc(sa + U_BYTES + kk * 2048, umma::BOX_BYTES, 1024);
          umma::mma_bf16(tmem + (uint32_t)(acc * DIM), ad, bd, idesc, (jin | kk) ? 1u : 0u);
        }
        if (jin == etc::SEG_KB - 1 || j == nkb - 1) umma::mma_commit(accfull0 + 8 * acc);
        umma::mma_commit(empty0 + 8 * st);
      }
      umma::mma_commit(done_bar);
    }
  } else {
    const int row = 32 * (warp & 3) + lane;
    const int cbase = etc::COLS * (warp >> 2);
    const uint32_t lane_addr = (uint32_t)(32 * (warp & 3)) << 16;
    ttc_rotate_tile<TX, etc::EPI_WARPS * 32>(reinterpret_cast<const TX*>(a.cv.unit_ptr(u)) + (long long)s * T * DIM,
                                             T, t0, sig, xs);
    float hi[etc::COLS], lo[etc::COLS];
#pragma unroll
    for (int j = 0; j < etc::COLS; ++j) {
      hi[j] = xs[row * XS_LD + cbase + j];
      lo[j] = 0.f;
    }
    for (int j = 0; j < nseg; ++j) {
      const int acc = j % MAXT, use = j / MAXT;
      bool ok = !*abort_flag && umma::mbar_wait(accfull0 + 8 * acc, use & 1);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) {
        *abort_flag = 1;
        break;
      }
      umma::fence_after_sync();
#pragma unroll
      for (int hh = 0; hh < etc::COLS / 16; ++hh) {
        float seg[16];
        ttc_tmem_ld16(tmem + lane_addr + (uint32_t)(acc * DIM + cbase + 16 * hh), seg);
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float sum, err;
          two_sum(hi[16 * hh + i], -seg[i], sum, err);
          hi[16 * hh + i] = sum;
          lo[16 * hh + i] = __fadd_rn(lo[16 * hh + i], err);
        }
      }
      umma::fence_before_sync();
      __syncwarp();
      if (lane == 0) asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(accfree0 + 8 * acc) : "memory");
    }
    const int t = t0 + row;
    if (!*abort_flag && t < T) {
      const float flev = (float)((1 << b) - 1);
      unsigned char* codes = a.blob + uh.off_codes;
      __half2* scales = reinterpret_cast<__half2*>(a.blob + uh.off_scales);
#pragma unroll
      for (int m = 0; m < etc::COLS / 16; ++m) {
        float v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = __fadd_rn(hi[16 * m + i], lo[16 * m + i]);
        float mn, mx;
        minmax16(v, mn, mx);
        const float l16 = rd16(mn);
        const float step = quant_step_cvt(mx, l16, b);
        const float inv = (step > 0.f && step <= kFp16Max) ? __frcp_rn(step) : 0.f;
        uint32_t w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
        for (int i = 0; i < 16; ++i) pack_code(w, i, b, block_code(v[i], l16, inv, flev));
        const long long blk = ((long long)s * T + t) * (DIM / 16) + cbase / 16 + m;
        unsigned char* dst = codes + blk * (2 * b);
        if (b == 8) *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
        else if (b == 4) *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
        else if (b == 2) *reinterpret_cast<uint32_t*>(dst) = w[0];
        else
          for (int byte = 0; byte < 2 * b; ++byte) dst[byte] = (unsigned char)(w[byte >> 2] >> ((byte & 3) * 8));
        scales[blk] = __halves2half2(__float2half_rn(l16), __float2half_rn(step));
      }
    }
  }
  __syncwarp();
  const bool drained = umma::mbar_wait(done_bar, 0);
  if ((*abort_flag || !drained) && threadIdx.x == 0 && a.status) atomicOr(a.status, DEV_ERR_TIMEOUT);
  umma::fence_before_sync();
  __syncthreads();
  if (warp == etc::EPI_WARPS) {
    umma::fence_after_sync();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "n"(TMEM_COLS) : "memory");
  }
}
}  // namespace jolt
