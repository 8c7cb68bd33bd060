// Streaming kernels of the compress / decompress path.
//
// The residual of every candidate is formed in the rotated basis: the cache tile is
// rotated once (sign flip + Walsh-Hadamard along the features), and the candidate's
// reconstruction U_s[:, :r_T] P'(r_D)[:r_T] comes straight out of the tensor cores with
// the rotation already folded into P' = bf16((C_s W_s^T) Phi).  The per-candidate work
// is then a subtraction, a 16-wide block min/max and the quantiser for every bit-width.
#pragma once

#include <type_traits>

#include "common.cuh"
#include "fp16_exact.cuh"
#include "gemm.cuh"

namespace jolt {

constexpr int MAXC = 8;   // candidates per set (token ranks, feature ranks, bit-widths)

struct CacheView {
  const void* k;          // [n_layers, H, T, D]
  const void* v;
  int dtype;              // 0 bf16, 1 fp32
  int n_layers, H, T, D, Lg, S;
  int u0;                 // global index of unit 0 (a shard of a larger cache): RNG streams use u + u0
  long long unit_elems;   // S * T * D
  __host__ __device__ const void* unit_ptr(int u) const {
    const char* base = (const char*)((u & 1) ? v : k);
    return base + (long long)(u >> 1) * unit_elems * (dtype ? 4 : 2);
  }
};

struct Cands {
  int nT, nD, nB;
  int rT[MAXC], rD[MAXC], bits[MAXC];
};

// ---------------------------------------------------------------------------------------
// fused residual / rotation / quantiser tile machinery (mma.sync m16n8k16 fragments)
//
// A CTA owns ROWS = 64 consecutive tokens of one slice (4 warps x 16 rows) and the full
// feature width D.  Thread (warp w, lane) holds rows g = lane/4 and g+8 of its warp's 16
// and, for every n8 tile j, columns 8j + 2(lane%4) + {0,1}.  A 16-wide quantisation block
// m is n8 tiles 2m and 2m+1: four values per thread, completed across the lane quad.
// ---------------------------------------------------------------------------------------
constexpr int TROWS = 64;
constexpr int TTHREADS = 128;
constexpr int KC = 64;  // token-rank chunk staged per pipeline step

// SPLIT = 2: two warps share a 16-row group, each holding half of the D columns (the table
// kernel, which runs eight warps per 64-row tile to halve the registers a thread holds)
template <int D, int SPLIT = 1>
struct TileFrag {
  static constexpr int NT = D / 8 / SPLIT;
  float v[2][NT][2];
};

// rotate the tile's rows (sigma, Walsh-Hadamard, 1/sqrt(D)) into smem as fp32
template <int D, typename TX>
__device__ __forceinline__ void rotate_tile_to_smem(const TX* X, int T, int t0, const float* sig, float* xs) {
  // xs: [TROWS][D + 4]
  for (int r = threadIdx.x; r < TROWS; r += blockDim.x) {
    float v[D];
    int t = t0 + r;
    if (t < T) {
      const TX* row = X + (long long)t * D;
#pragma unroll
      for (int d = 0; d < D; ++d) v[d] = ld_as_float(row + d) * sig[d];
    } else {
#pragma unroll
      for (int d = 0; d < D; ++d) v[d] = 0.f;
    }
    fwht_regs<D>(v);
    const float sc = (float)(1.0 / sqrt((double)D));
#pragma unroll
    for (int d = 0; d < D; ++d) xs[r * (D + 4) + d] = v[d] * sc;
  }
}

// the same rotation with the whole CTA working in shared memory: x * sigma staged, then the
// Walsh-Hadamard butterflies stage by stage (the order of fwht_regs, so the result is
// bit-identical), then the 1/sqrt(D) scale; keeps no row in registers
template <int D, typename TX>
__device__ __forceinline__ void rotate_tile_smem(const TX* X, int T, int t0, const float* sig, float* xs) {
  constexpr int LD = D + 4;
  for (int idx = threadIdx.x; idx < TROWS * D; idx += blockDim.x) {
    const int r = idx / D, d = idx - r * D, t = t0 + r;
    xs[r * LD + d] = t < T ? ld_as_float(X + (long long)t * D + d) * sig[d] : 0.f;
  }
  __syncthreads();
#pragma unroll
  for (int h = 1; h < D; h <<= 1) {
    for (int idx = threadIdx.x; idx < TROWS * D / 2; idx += blockDim.x) {
      const int r = idx / (D / 2), p = idx - r * (D / 2);
      const int i = (p / h) * 2 * h + (p % h);
      const float a = xs[r * LD + i], b = xs[r * LD + i + h];
      xs[r * LD + i] = a + b;
      xs[r * LD + i + h] = a - b;
    }
    __syncthreads();
  }
  const float sc = (float)(1.0 / sqrt((double)D));
  for (int idx = threadIdx.x; idx < TROWS * D; idx += blockDim.x) {
    const int r = idx / D, d = idx - r * D;
    xs[r * LD + d] *= sc;
  }
}

template <int D, int SPLIT = 1>
__device__ __forceinline__ void frag_from_smem(const float* xs, TileFrag<D, SPLIT>& f) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int NT = TileFrag<D, SPLIT>::NT;
  const int rg = warp / SPLIT, half = warp % SPLIT;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    int r = rg * 16 + (lane >> 2) + h * 8;
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      int c = (half * NT + j) * 8 + (lane & 3) * 2;
      f.v[h][j][0] = xs[r * (D + 4) + c];
      f.v[h][j][1] = xs[r * (D + 4) + c + 1];
    }
  }
}

// Staged operands for the reconstruction MMA:  sU [TROWS][KC] (K-contiguous, swizzled)
//                                             sP [KC][D]     (D-contiguous, swizzled)
template <int D>
struct ReconSmem {
  static constexpr int U_ELEMS = TROWS * KC;
  static constexpr int P_ELEMS = KC * D;
  static constexpr int STAGE = U_ELEMS + P_ELEMS;
};

__device__ __forceinline__ int su_off(int row, int ch) { return row * KC + ((ch ^ (row & 7)) << 3); }
template <int D>
__device__ __forceinline__ int sp_off(int krow, int ch) {
  constexpr int CH = D / 8;
  return krow * D + ((CH >= 8 ? (ch ^ (krow & 7)) : (ch ^ (krow & (CH - 1)))) << 3);
}

// issue cp.async of U rows [t0, t0+64) x k [k0, k0+KC) and P' rows k [k0, k0+KC)
template <int D>
__device__ __forceinline__ void recon_load_stage(bf16* st, const bf16* U, long long ldU, int T, int t0,
                                                 const bf16* P, int kmax, int k0) {
  using namespace gemm_detail;
  bf16* sU = st;
  bf16* sP = st + ReconSmem<D>::U_ELEMS;
  constexpr int UCH = TROWS * KC / 8;  // 512 chunks
  for (int c = threadIdx.x; c < UCH; c += blockDim.x) {
    int row = c / (KC / 8), ch = c % (KC / 8);
    int t = t0 + row, k = k0 + ch * 8;
    bool valid = (t < T) && (k < kmax);
    const bf16* src = valid ? U + (long long)t * ldU + k : U;
    cp_async16(smem_u32(sU + su_off(row, ch)), src, valid);
  }
  constexpr int PCH = KC * D / 8;
  for (int c = threadIdx.x; c < PCH; c += blockDim.x) {
    int krow = c / (D / 8), ch = c % (D / 8);
    int k = k0 + krow;
    bool valid = k < kmax;
    const bf16* src = valid ? P + (long long)k * D + ch * 8 : P;
    cp_async16(smem_u32(sP + sp_off<D>(krow, ch)), src, valid);
  }
}

// accumulate the k16 slab at chunk offset kk (absolute token rank kabs) of a staged chunk,
// keeping only the ranks in [klo, khi)
template <int D, int SPLIT = 1>
__device__ __forceinline__ void recon_mma_k16(const bf16* st, int kk, int kabs, int klo, int khi,
                                              float (*acc)[4]) {
  using namespace gemm_detail;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int rg = warp / SPLIT, half = warp % SPLIT;
  const bf16* sU = st;
  const bf16* sP = st + ReconSmem<D>::U_ELEMS;
  uint32_t a[4];
  {
    int row = rg * 16 + (lane & 15);
    int ch = (kk >> 3) + (lane >> 4);
    ldsm_x4(smem_u32(sU + su_off(row, ch)), a[0], a[1], a[2], a[3]);
  }
  if (klo > kabs || khi < kabs + 16) {
    // zero the bf16 halves whose k falls outside [klo, khi)
    int kq = kabs + (lane & 3) * 2;
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      int kb = kq + ((r >> 1) << 3);
      uint32_t m = 0;
      if (kb >= klo && kb < khi) m |= 0x0000FFFFu;
      if (kb + 1 >= klo && kb + 1 < khi) m |= 0xFFFF0000u;
      a[r] &= m;
    }
  }
  constexpr int NT = D / 8 / SPLIT;   // n8 tiles of this warp
#pragma unroll
  for (int np = 0; np < NT / 2; ++np) {
    uint32_t r0, r1, r2, r3;
    int krow = kk + (lane & 7) + (((lane >> 3) & 1) << 3);
    int ch = (half * NT / 2 + np) * 2 + (lane >> 4);
    ldsm_x4_t(smem_u32(sP + sp_off<D>(krow, ch)), r0, r1, r2, r3);
    mma16816(acc[np * 2 + 0], a, r0, r1);
    mma16816(acc[np * 2 + 1], a, r2, r3);
  }
}

// Walk the token-rank axis [0, kmax) in KC chunks; call epi(i) whenever the
// accumulated prefix reaches cut[i] (cuts ascending, all <= kmax), and fold() after every
// whole chunk (the encoder moves the chunk's sums out of the accumulator there).
template <int D, int SPLIT = 1, typename Epi, typename Fold>
__device__ __forceinline__ void recon_walk_fold(bf16* smem_stages, const bf16* U, long long ldU, int T, int t0,
                                                const bf16* P, int kmax, const int* cuts, int ncuts,
                                                float (*acc)[4], Epi&& epi, Fold&& fold) {
  using namespace gemm_detail;
  const int nchunks = (kmax + KC - 1) / KC;
  int ci = 0;
  while (ci < ncuts && cuts[ci] <= 0) { epi(ci); ++ci; }
  recon_load_stage<D>(smem_stages, U, ldU, T, t0, P, kmax, 0);
  cp_async_commit();
  for (int c = 0; c < nchunks; ++c) {
    if (c + 1 < nchunks)
      recon_load_stage<D>(smem_stages + ((c + 1) & 1) * ReconSmem<D>::STAGE, U, ldU, T, t0, P, kmax, (c + 1) * KC);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const bf16* st = smem_stages + (c & 1) * ReconSmem<D>::STAGE;
    for (int kk = 0; kk < KC; kk += 16) {
      int k = c * KC + kk;
      if (k >= kmax) break;
      int lo = k;
      while (lo < k + 16 && lo < kmax) {
        int hi = min(k + 16, kmax);
        if (ci < ncuts && cuts[ci] > lo && cuts[ci] < hi) hi = cuts[ci];
        recon_mma_k16<D, SPLIT>(st, kk, k, lo, hi, acc);
        lo = hi;
        while (ci < ncuts && cuts[ci] == lo) { epi(ci); ++ci; }
      }
    }
    if (ci < ncuts) fold();
    __syncthreads();
  }
  cp_async_wait<0>();
}

template <int D, int SPLIT = 1, typename Epi>
__device__ __forceinline__ void recon_walk(bf16* smem_stages, const bf16* U, long long ldU, int T, int t0,
                                           const bf16* P, int kmax, const int* cuts, int ncuts,
                                           float (*acc)[4], Epi&& epi) {
  recon_walk_fold<D, SPLIT>(smem_stages, U, ldU, T, t0, P, kmax, cuts, ncuts, acc, epi, [] {});
}

// error-free sum of two floats (Knuth's TwoSum): s + e == a + b exactly
__device__ __forceinline__ void two_sum(float a, float b, float& s, float& e) {
  s = __fadd_rn(a, b);
  const float bb = __fsub_rn(s, a);
  e = __fadd_rn(__fsub_rn(a, __fsub_rn(s, bb)), __fsub_rn(b, bb));
}

// ---------------------------------------------------------------------------------------
// residual tile in shared memory: the fragment owners write rho = x' - acc, then every
// thread quantises whole 16-wide blocks of one row (row = tid % 64, blocks of one half row)
// ---------------------------------------------------------------------------------------
template <int D, int THREADS = TTHREADS>
struct RhoTile {
  static constexpr int LD = D + 4;                 // row pitch (floats)
  static constexpr int BLK_PER_ROW = D / 16;
  static constexpr int BLOCKS = TROWS * BLK_PER_ROW;
  static constexpr int BLK_PER_THREAD = BLOCKS / THREADS;  // 4 for D = 128 and 128 threads
  static constexpr size_t BYTES = (size_t)TROWS * LD * 4;
};

template <int D, int SPLIT = 1>
__device__ __forceinline__ void write_rho(float* rho, const TileFrag<D, SPLIT>& xf, float (*acc)[4]) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int rg = warp / SPLIT, half = warp % SPLIT;
  constexpr int NT = TileFrag<D, SPLIT>::NT;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int r = rg * 16 + (lane >> 2) + h * 8;
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      const int c = (half * NT + j) * 8 + (lane & 3) * 2;
      float2 v = make_float2(xf.v[h][j][0] - acc[j][h * 2 + 0], xf.v[h][j][1] - acc[j][h * 2 + 1]);
      *reinterpret_cast<float2*>(rho + r * RhoTile<D>::LD + c) = v;
    }
  }
}

// blocks handled by this thread: row tid % 64, blocks [ (tid / 64) * BPT, +BPT ) of that row;
// with fewer blocks than threads, thread tid < BLOCKS holds block tid / 64 of row tid % 64
template <int D, int THREADS = TTHREADS>
__device__ __forceinline__ int block_row() { return threadIdx.x % TROWS; }
template <int D, int THREADS = TTHREADS>
__device__ __forceinline__ int block_first() {
  constexpr int BPT = RhoTile<D, THREADS>::BLK_PER_THREAD;
  return BPT > 0 ? (int)(threadIdx.x / TROWS) * BPT : (int)(threadIdx.x / TROWS);
}
template <int D, int THREADS = TTHREADS>
__host__ __device__ constexpr int blocks_per_thread() {
  return RhoTile<D, THREADS>::BLK_PER_THREAD > 0 ? RhoTile<D, THREADS>::BLK_PER_THREAD : 1;
}
template <int D, int THREADS = TTHREADS>
__device__ __forceinline__ bool has_blocks() {
  return RhoTile<D, THREADS>::BLK_PER_THREAD > 0 || (int)threadIdx.x < RhoTile<D, THREADS>::BLOCKS;
}

__device__ __forceinline__ void load16(const float* src, float* v) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    float4 t = reinterpret_cast<const float4*>(src)[q];
    v[4 * q + 0] = t.x;
    v[4 * q + 1] = t.y;
    v[4 * q + 2] = t.z;
    v[4 * q + 3] = t.w;
  }
}

__device__ __forceinline__ void minmax16(const float* v, float& mn, float& mx) {
  float a0 = fminf(v[0], v[1]), a1 = fminf(v[2], v[3]), a2 = fminf(v[4], v[5]), a3 = fminf(v[6], v[7]);
  float a4 = fminf(v[8], v[9]), a5 = fminf(v[10], v[11]), a6 = fminf(v[12], v[13]), a7 = fminf(v[14], v[15]);
  mn = fminf(fminf(fminf(a0, a1), fminf(a2, a3)), fminf(fminf(a4, a5), fminf(a6, a7)));
  float b0 = fmaxf(v[0], v[1]), b1 = fmaxf(v[2], v[3]), b2 = fmaxf(v[4], v[5]), b3 = fmaxf(v[6], v[7]);
  float b4 = fmaxf(v[8], v[9]), b5 = fmaxf(v[10], v[11]), b6 = fmaxf(v[12], v[13]), b7 = fmaxf(v[14], v[15]);
  mx = fmaxf(fmaxf(fmaxf(b0, b1), fmaxf(b2, b3)), fmaxf(fmaxf(b4, b5), fmaxf(b6, b7)));
}

// per-bit-width constants of the candidate set (b = 0 marks "no residual")
struct BitConsts {
  float flev[MAXC], inv[MAXC];
  int bits[MAXC];
  int n;
};
__device__ __forceinline__ BitConsts bit_consts(const Cands& cd) {
  BitConsts k;
  k.n = cd.nB;
#pragma unroll
  for (int i = 0; i < MAXC; ++i) {
    int b = i < cd.nB ? cd.bits[i] : 0;
    k.bits[i] = b;
    k.flev[i] = (float)((1 << b) - 1);
    k.inv[i] = b > 0 ? 1.0f / k.flev[i] : 0.f;
  }
  return k;
}

// squared quantisation error of one 16-wide block for every bit-width (added into err).
// The per-element work runs on packed fp32 pairs (FFMA2 / FADD2: the same IEEE round-to-
// nearest per lane as the scalar forms, half the instructions) with four partial sums, so
// the dependent accumulation chain is four deep instead of sixteen.
__device__ __forceinline__ void block_errors(const float* v, const BitConsts& k, float* err) {
  float mn, mx;
  minmax16(v, mn, mx);
  const float lo = rd16(mn);
  float2 d[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) d[j] = __fadd2_rn(make_float2(v[2 * j], v[2 * j + 1]), make_float2(-lo, -lo));
#pragma unroll
  for (int ib = 0; ib < MAXC; ++ib) {
    if (ib >= k.n) break;
    if (k.bits[ib] == 0) {
      float2 a0 = make_float2(0.f, 0.f), a1 = a0;
#pragma unroll
      for (int j = 0; j < 8; j += 2) {
        const float2 x0 = make_float2(v[2 * j], v[2 * j + 1]), x1 = make_float2(v[2 * j + 2], v[2 * j + 3]);
        a0 = __ffma2_rn(x0, x0, a0);
        a1 = __ffma2_rn(x1, x1, a1);
      }
      err[ib] += (a0.x + a0.y) + (a1.x + a1.y);
      continue;
    }
    const float step = quant_step(mx, lo, k.flev[ib], k.inv[ib]);
    if (!(isfinite(lo) && step <= kFp16Max)) {
      err[ib] = INFINITY;
      continue;
    }
    const float inv = step > 0.f ? __frcp_rn(step) : 0.f;
    const float2 inv2 = make_float2(inv, inv), nstep2 = make_float2(-step, -step);
    const float2 sh = make_float2(kRoundShift, kRoundShift), nsh = make_float2(-kRoundShift, -kRoundShift);
    float2 a0 = make_float2(0.f, 0.f), a1 = a0;
#pragma unroll
    for (int j = 0; j < 8; j += 2) {
      // code = rne(d / step) through the shift, e = d - code * step, e2 += e * e
      const float2 c0 = __fadd2_rn(__ffma2_rn(d[j], inv2, sh), nsh);
      const float2 c1 = __fadd2_rn(__ffma2_rn(d[j + 1], inv2, sh), nsh);
      const float2 e0 = __ffma2_rn(c0, nstep2, d[j]);
      const float2 e1 = __ffma2_rn(c1, nstep2, d[j + 1]);
      a0 = __ffma2_rn(e0, e0, a0);
      a1 = __ffma2_rn(e1, e1, a1);
    }
    err[ib] += (a0.x + a0.y) + (a1.x + a1.y);
  }
}

// The same errors for a bit-width set fixed at compile time (the default candidate set
// {0,1,2,3,4,8}): the per-width constants fold into the code and the loop over widths is
// unrolled without branches; the arithmetic of every width is the same as above.
template <int B>
__device__ __forceinline__ void bit_error(const float* v, const float2* d, float mx, float lo, float& err) {
  if constexpr (B == 0) {
    float2 a0 = make_float2(0.f, 0.f), a1 = a0;
#pragma unroll
    for (int j = 0; j < 8; j += 2) {
      const float2 x0 = make_float2(v[2 * j], v[2 * j + 1]), x1 = make_float2(v[2 * j + 2], v[2 * j + 3]);
      a0 = __ffma2_rn(x0, x0, a0);
      a1 = __ffma2_rn(x1, x1, a1);
    }
    err += (a0.x + a0.y) + (a1.x + a1.y);
  } else {
    constexpr float flev = (float)((1 << B) - 1);
    const float inv_lev = 1.0f / flev;
    const float step = quant_step(mx, lo, flev, inv_lev);
    if (!(isfinite(lo) && step <= kFp16Max)) {
      err = INFINITY;
      return;
    }
    const float inv = step > 0.f ? __frcp_rn(step) : 0.f;
    const float2 inv2 = make_float2(inv, inv), nstep2 = make_float2(-step, -step);
    const float2 sh = make_float2(kRoundShift, kRoundShift), nsh = make_float2(-kRoundShift, -kRoundShift);
    float2 a0 = make_float2(0.f, 0.f), a1 = a0;
#pragma unroll
    for (int j = 0; j < 8; j += 2) {
      const float2 c0 = __fadd2_rn(__ffma2_rn(d[j], inv2, sh), nsh);
      const float2 c1 = __fadd2_rn(__ffma2_rn(d[j + 1], inv2, sh), nsh);
      const float2 e0 = __ffma2_rn(c0, nstep2, d[j]);
      const float2 e1 = __ffma2_rn(c1, nstep2, d[j + 1]);
      a0 = __ffma2_rn(e0, e0, a0);
      a1 = __ffma2_rn(e1, e1, a1);
    }
    err += (a0.x + a0.y) + (a1.x + a1.y);
  }
}

template <int... Bs>
struct BitSet {
  static constexpr int N = sizeof...(Bs);
};
using DefaultBits = BitSet<0, 1, 2, 3, 4, 8>;

template <int... Bs>
__device__ __forceinline__ void block_errors_fixed(const float* v, float* err, BitSet<Bs...>) {
  float mn, mx;
  minmax16(v, mn, mx);
  const float lo = rd16(mn);
  float2 d[8];
#pragma unroll
  for (int j = 0; j < 8; ++j) d[j] = __fadd2_rn(make_float2(v[2 * j], v[2 * j + 1]), make_float2(-lo, -lo));
  int i = 0;
  (bit_error<Bs>(v, d, mx, lo, err[i++]), ...);
}

// ---------------------------------------------------------------------------------------
// distortion table kernel: grid (tiles, S, units); writes fp64 partial sums per CTA
// ---------------------------------------------------------------------------------------
struct TableArgs {
  CacheView cv;
  const bf16* U;        // [unit][T][ldU]
  long long ldU, sU;
  const bf16* P;        // [unit][iD][S][rTmax][D]
  long long sP_unit, sP_rd;
  int rTmax;
  Cands cand;
  uint64_t seed;
  double* partial;      // [unit][S][tiles][nD][nT][nB]
  int tiles;
};

template <int D>
inline size_t table_smem() {
  return RhoTile<D>::BYTES + 2 * (size_t)ReconSmem<D>::STAGE * sizeof(bf16);
}

// the table kernel runs 2 warps per 16-row group (each half of the columns) where D >= 32
template <int D>
__host__ __device__ constexpr int table_split() { return D >= 32 ? 2 : 1; }
template <int D>
__host__ __device__ constexpr int table_threads() { return TTHREADS * table_split<D>(); }

template <int D, typename TX, typename BITS>
__global__ void __launch_bounds__(table_threads<D>(), D >= 64 ? 2 : 1) table_kernel(TableArgs a) {
  constexpr int SPLIT = table_split<D>();
  constexpr int THREADS = table_threads<D>();
  extern __shared__ __align__(128) unsigned char smem_raw[];
  float* rho = reinterpret_cast<float*>(smem_raw);                                   // TROWS x LD
  bf16* stages = reinterpret_cast<bf16*>(smem_raw + RhoTile<D>::BYTES);                // 2 stages
  __shared__ float sig[D];
  __shared__ float red[THREADS / 32][MAXC];

  const int tile = blockIdx.x, s = blockIdx.y, u = blockIdx.z;
  const int T = a.cv.T;
  const int t0 = tile * TROWS;
  const TX* X = reinterpret_cast<const TX*>(a.cv.unit_ptr(u)) + (long long)s * T * D;
  for (int d = threadIdx.x; d < D; d += blockDim.x) sig[d] = rotation_sign(a.seed, u + a.cv.u0, d);
  __syncthreads();
  rotate_tile_smem<D, TX>(X, T, t0, sig, rho);   // x' staged through the rho buffer
  __syncthreads();
  TileFrag<D, SPLIT> xf;
  frag_from_smem<D, SPLIT>(rho, xf);
  __syncthreads();

  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const Cands& cd = a.cand;
  const BitConsts kb = bit_consts(cd);
  const bf16* U = a.U + (long long)u * a.sU;
  constexpr int NT = TileFrag<D, SPLIT>::NT;
  double* out = a.partial + (((long long)u * a.cv.S + s) * a.tiles + tile) * (long long)(cd.nD * cd.nT * cd.nB);
  const int brow = block_row<D, THREADS>();
  const bool mine = has_blocks<D, THREADS>();

  for (int iD = 0; iD < cd.nD; ++iD) {
    const bf16* P = a.P + (long long)u * a.sP_unit + iD * a.sP_rd + (long long)s * a.rTmax * D;
    float acc[NT][4];
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[j][e] = 0.f;

    auto epi = [&](int iT) {
      write_rho<D, SPLIT>(rho, xf, acc);
      __syncthreads();
      float err[MAXC];
#pragma unroll
      for (int ib = 0; ib < MAXC; ++ib) err[ib] = 0.f;
      if (mine) {
#pragma unroll 1
        for (int q = 0; q < blocks_per_thread<D, THREADS>(); ++q) {
          float v[16];
          load16(rho + brow * RhoTile<D>::LD + (block_first<D, THREADS>() + q) * 16, v);
          if constexpr (std::is_same<BITS, void>::value) block_errors(v, kb, err);
          else block_errors_fixed(v, err, BITS{});
        }
      }
      // reduce over the warp, then over the warps in fixed order (fp64)
#pragma unroll
      for (int ib = 0; ib < MAXC; ++ib) {
        if (ib >= cd.nB) break;
        float v = err[ib];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
        if (lane == 0) red[warp][ib] = v;
      }
      __syncthreads();
      if (threadIdx.x < cd.nB) {
        double v = 0.0;
        for (int w = 0; w < THREADS / 32; ++w) v += (double)red[w][threadIdx.x];
        out[(iD * cd.nT + iT) * cd.nB + threadIdx.x] = v;
      }
    };
    recon_walk<D, SPLIT>(stages, U, a.ldU, T, t0, P, cd.rT[cd.nT - 1], cd.rT, cd.nT, acc, epi);
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------------------
// unit record header (device layout of the compressed blob; 64 bytes each)
// ---------------------------------------------------------------------------------------
struct BlobHeader {      // 64 bytes at offset 0
  uint32_t magic, version, n_units, status;
  int32_t n_layers, n_heads, n_tokens, head_dim, layers_per_group, dtype, block, unit_offset;
  uint64_t seed, total_bytes;
};
struct UnitHeader {      // 64 bytes per unit after the global header
  int32_t r_T, r_D, bits, choice;
  uint64_t off_U, off_W, off_C, off_codes, off_scales;
  double distortion;
};
static_assert(sizeof(BlobHeader) == 64, "header");
static_assert(sizeof(UnitHeader) == 64, "unit header");
constexpr uint32_t kMagic = 0x544C4F4Au;  // "JOLT"
constexpr uint32_t kVersion = 1u;

// ---------------------------------------------------------------------------------------
// encode kernel: chosen (r_T, r_D, b) per unit from the blob's unit table
// grid (tiles, S, units)
// ---------------------------------------------------------------------------------------
struct EncodeArgs {
  CacheView cv;
  const bf16* U;
  long long ldU, sU;
  const bf16* P;
  long long sP_unit, sP_rd;
  int rTmax;
  Cands cand;
  uint64_t seed;
  unsigned char* blob;
};

template <int D, typename TX>
__global__ void __launch_bounds__(TTHREADS) encode_kernel(EncodeArgs a) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  float* rho = reinterpret_cast<float*>(smem_raw);
  bf16* stages = reinterpret_cast<bf16*>(smem_raw + RhoTile<D>::BYTES);
  __shared__ float sig[D];

  const int tile = blockIdx.x, s = blockIdx.y, u = blockIdx.z;
  const int T = a.cv.T;
  const int t0 = tile * TROWS;
  const UnitHeader uh = reinterpret_cast<const UnitHeader*>(a.blob + sizeof(BlobHeader))[u];
  const BlobHeader* gh = reinterpret_cast<const BlobHeader*>(a.blob);
  if (gh->status != 0) return;
  const int b = uh.bits;
  if (b == 0) return;
  int iD = 0;
  while (iD < a.cand.nD && a.cand.rD[iD] != uh.r_D) ++iD;

  const TX* X = reinterpret_cast<const TX*>(a.cv.unit_ptr(u)) + (long long)s * T * D;
  for (int d = threadIdx.x; d < D; d += blockDim.x) sig[d] = rotation_sign(a.seed, u + a.cv.u0, d);
  __syncthreads();
  rotate_tile_to_smem<D, TX>(X, T, t0, sig, rho);
  __syncthreads();
  TileFrag<D> xf;
  frag_from_smem<D>(rho, xf);
  __syncthreads();

  constexpr int NT = D / 8;
  const bf16* U = a.U + (long long)u * a.sU;
  const bf16* P = a.P + (long long)u * a.sP_unit + iD * a.sP_rd + (long long)s * a.rTmax * D;
  float acc[NT][4];
#pragma unroll
  for (int j = 0; j < NT; ++j)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[j][e] = 0.f;

  const float flev = (float)((1 << b) - 1);
  const float inv_lev = 1.0f / flev;
  unsigned char* codes = a.blob + uh.off_codes;
  __half2* scales = reinterpret_cast<__half2*>(a.blob + uh.off_scales);
  const int brow = block_row<D>();
  const bool has_blocks = (RhoTile<D>::BLK_PER_THREAD > 0) || threadIdx.x < TROWS;

  // the residual x' - U P' is kept as an unevaluated sum hi + lo: every whole chunk of token
  // ranks is subtracted from it without rounding error (TwoSum), so only the fp32 sums inside
  // one chunk round -- the reconstruction is subtracted from x' with a chunk's error, not the
  // error of the whole sum
  TileFrag<D> xl;
#pragma unroll
  for (int h = 0; h < 2; ++h)
#pragma unroll
    for (int j = 0; j < NT; ++j) xl.v[h][j][0] = xl.v[h][j][1] = 0.f;
  auto fold = [&]() {
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int j = 0; j < NT; ++j)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          float sum, err;
          two_sum(xf.v[h][j][e], -acc[j][h * 2 + e], sum, err);
          xf.v[h][j][e] = sum;
          xl.v[h][j][e] = __fadd_rn(xl.v[h][j][e], err);
          acc[j][h * 2 + e] = 0.f;
        }
  };
  auto epi = [&](int) {
    fold();
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int j = 0; j < NT; ++j)
#pragma unroll
        for (int e = 0; e < 2; ++e) xf.v[h][j][e] = __fadd_rn(xf.v[h][j][e], xl.v[h][j][e]);
    write_rho<D>(rho, xf, acc);
    __syncthreads();
    const int t = t0 + brow;
    if (!has_blocks || t >= T) return;
#pragma unroll 1
    for (int q = 0; q < blocks_per_thread<D>(); ++q) {
      const int m = block_first<D>() + q;
      float v[16];
      load16(rho + brow * RhoTile<D>::LD + m * 16, v);
      float mn, mx;
      minmax16(v, mn, mx);
      const float lo = rd16(mn);
      const float step = quant_step(mx, lo, flev, inv_lev);
      const float inv = (step > 0.f && step <= kFp16Max) ? __frcp_rn(step) : 0.f;
      uint32_t w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
      for (int j = 0; j < 16; ++j) pack_code(w, j, b, block_code(v[j], lo, inv, flev));
      const long long blk = ((long long)s * T + t) * (D / 16) + m;
      unsigned char* dst = codes + blk * (2 * b);
      // 2b bytes; the block start is 2b-aligned
      if (b == 8) {
        *reinterpret_cast<uint4*>(dst) = make_uint4(w[0], w[1], w[2], w[3]);
      } else if (b == 4) {
        *reinterpret_cast<uint2*>(dst) = make_uint2(w[0], w[1]);
      } else if (b == 2) {
        *reinterpret_cast<uint32_t*>(dst) = w[0];
      } else {
        for (int byte = 0; byte < 2 * b; ++byte) dst[byte] = (unsigned char)(w[byte >> 2] >> ((byte & 3) * 8));
      }
      scales[blk] = __halves2half2(__float2half_rn(lo), __float2half_rn(step));
    }
  };
  int cut = uh.r_T;
  recon_walk_fold<D>(stages, U, a.ldU, T, t0, P, cut, &cut, 1, acc, epi, fold);
}

// ---------------------------------------------------------------------------------------
// decode kernel: X_hat = (U P' + dequant) Phi^T ; grid (tiles, S, units)
// P' here is the decoder's own operator built from the stored core and feature factor
// ---------------------------------------------------------------------------------------
struct DecodeArgs {
  const unsigned char* blob;
  const bf16* U;         // [unit][T][ldU] aligned copy of the stored token factors
  long long ldU, sU;
  const bf16* P;         // [unit][S][rTmax][D]
  long long sP_unit;
  int rTmax;
  int T, S, Lg;
  int u0;                // global index of unit 0 (from the blob header)
  uint64_t seed;
  void* k_out;
  void* v_out;
  int out_f32;
};

template <int D>
__device__ __forceinline__ void fwht_frag_row(TileFrag<D>& f, int h) {
  // butterflies inside the thread: stride 1 (e) and strides 8..D/2 (n8 tile index)
  constexpr int NT = D / 8;
#pragma unroll
  for (int j = 0; j < NT; ++j) {
    float x0 = f.v[h][j][0], x1 = f.v[h][j][1];
    f.v[h][j][0] = x0 + x1;
    f.v[h][j][1] = x0 - x1;
  }
  // strides 2 and 4 across the lane quad
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int sh = 1; sh <= 2; sh <<= 1) {
    bool upper = (lane & sh) != 0;
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float mine = f.v[h][j][e];
        float other = __shfl_xor_sync(0xffffffffu, mine, sh);
        f.v[h][j][e] = upper ? other - mine : mine + other;
      }
  }
#pragma unroll
  for (int hs = 1; hs < NT; hs <<= 1) {
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      if (j & hs) continue;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float x0 = f.v[h][j][e], x1 = f.v[h][j + hs][e];
        f.v[h][j][e] = x0 + x1;
        f.v[h][j + hs][e] = x0 - x1;
      }
    }
  }
}

template <int D>
__global__ void __launch_bounds__(TTHREADS) decode_kernel(DecodeArgs a) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  bf16* stages = reinterpret_cast<bf16*>(smem_raw);
  __shared__ float sig[D];
  const int tile = blockIdx.x, s = blockIdx.y, u = blockIdx.z;
  const int T = a.T;
  const int t0 = tile * TROWS;
  const UnitHeader uh = reinterpret_cast<const UnitHeader*>(a.blob + sizeof(BlobHeader))[u];
  for (int d = threadIdx.x; d < D; d += blockDim.x) sig[d] = rotation_sign(a.seed, u + a.u0, d);
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  constexpr int NT = D / 8;
  const bf16* U = a.U + (long long)u * a.sU;
  const bf16* P = a.P + (long long)u * a.sP_unit + (long long)s * a.rTmax * D;
  float acc[NT][4];
#pragma unroll
  for (int j = 0; j < NT; ++j)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[j][e] = 0.f;
  int cut = uh.r_T;
  recon_walk<D>(stages, U, a.ldU, T, t0, P, uh.r_T, &cut, 1, acc, [](int) {});

  TileFrag<D> f;
  const int b = uh.bits;
  const int q = lane & 3;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    int t = t0 + warp * 16 + (lane >> 2) + h * 8;
    bool valid = t < T;
#pragma unroll
    for (int m = 0; m < D / 16; ++m) {
      float deq[4] = {0.f, 0.f, 0.f, 0.f};
      if (b > 0 && valid) {
        long long blk = ((long long)s * T + t) * (D / 16) + m;
        const unsigned char* src = a.blob + uh.off_codes + blk * (2 * b);
        uint32_t w[4] = {0u, 0u, 0u, 0u};
        for (int byte = 0; byte < 2 * b; ++byte) w[byte >> 2] |= (uint32_t)src[byte] << ((byte & 3) * 8);
        __half2 sc = reinterpret_cast<const __half2*>(a.blob + uh.off_scales)[blk];
        float lo = __low2float(sc), step = __high2float(sc);
#pragma unroll
        for (int i = 0; i < 4; ++i) deq[i] = fmaf((float)unpack_code(w, (i >> 1) * 8 + 2 * q + (i & 1), b), step, lo);
      }
      f.v[h][2 * m][0] = acc[2 * m][h * 2 + 0] + deq[0];
      f.v[h][2 * m][1] = acc[2 * m][h * 2 + 1] + deq[1];
      f.v[h][2 * m + 1][0] = acc[2 * m + 1][h * 2 + 0] + deq[2];
      f.v[h][2 * m + 1][1] = acc[2 * m + 1][h * 2 + 1] + deq[3];
    }
    fwht_frag_row<D>(f, h);
    if (!valid) continue;
    const float sc = (float)(1.0 / sqrt((double)D));
    const int g = u >> 1;
    long long row_off = ((long long)s * T + t) * D;          // row inside the unit
    long long unit_off = (long long)g * a.S * T * D;         // unit inside K or V
    void* outp = (u & 1) ? a.v_out : a.k_out;
#pragma unroll
    for (int j = 0; j < NT; ++j) {
      int c = j * 8 + 2 * q;
      float y0 = f.v[h][j][0] * sc * sig[c];
      float y1 = f.v[h][j][1] * sc * sig[c + 1];
      long long off = unit_off + row_off + c;
      if (a.out_f32) {
        float2* o = reinterpret_cast<float2*>(reinterpret_cast<float*>(outp) + off);
        *o = make_float2(y0, y1);
      } else {
        __nv_bfloat162* o = reinterpret_cast<__nv_bfloat162*>(reinterpret_cast<bf16*>(outp) + off);
        *o = __floats2bfloat162_rn(y0, y1);
      }
    }
  }
}

template <int D>
inline size_t decode_smem() {
  return 2 * (size_t)ReconSmem<D>::STAGE * sizeof(bf16);
}

}  // namespace jolt

namespace jolt {
// ---------------------------------------------------------------------------------------
// Per-block b-bit quantisation of the cache itself (no factors, no rotation): the plain
// quantisation baseline the pages set JoLT against ("A JoLT for the KV Cache ... Joint Tucker
// and JL-Residual Allocation for LLMs", introduction: the error is roughly an order of
// magnitude below cross-layer SVD and 4-bit quantisation).  Same quantiser as the residual:
// asymmetric min-max over 16 consecutive features with fp16 (lo, step).  Every thread takes
// whole blocks (consecutive threads consecutive blocks: coalesced 32- or 64-byte reads);
// per CTA and unit the fp64 sums of x^2 and of the squared error; codes and scales written
// when the output pointers are given (layout of the blob's residual arrays).
// grid (nblk, units); 256 threads.
// ---------------------------------------------------------------------------------------
template <typename TX>
__global__ void __launch_bounds__(256) quant_baseline_kernel(CacheView cv, int b, unsigned char* codes,
                                                             __half2* scales, double* part, int nblk) {
  const int u = blockIdx.y;
  const TX* X = reinterpret_cast<const TX*>(cv.unit_ptr(u));
  const long long nb = cv.unit_elems / 16;
  const float flev = (float)((1 << b) - 1), inv_lev = 1.0f / flev;
  double sx = 0.0, se = 0.0;
  for (long long q = blockIdx.x * (long long)blockDim.x + threadIdx.x; q < nb; q += (long long)nblk * blockDim.x) {
    float v[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = ld_as_float(X + q * 16 + i);
    float mn, mx;
    minmax16(v, mn, mx);
    const float lo = rd16(mn);
    const float step = quant_step(mx, lo, flev, inv_lev);
    const bool ok = isfinite(lo) && step <= kFp16Max;
    // codes and errors in fp64: v - lo, its quotient by the step and the rounding to the
    // nearest level (ties to even) are then those of the definition; the inputs of this
    // baseline are coarse (bf16 values, fp16 scales), so exact ties are common and a product
    // with a rounded reciprocal would settle them differently.  The kernel stays HBM-bound.
    uint32_t w[4] = {0u, 0u, 0u, 0u};
    double ex = 0.0, ee = 0.0;
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const double d = (double)v[i] - (double)lo;
      double c = (ok && step > 0.f) ? rint(d / (double)step) : 0.0;
      c = fmin(fmax(c, 0.0), (double)flev);
      pack_code(w, i, b, (uint32_t)c);
      const double e = (double)v[i] - fma(c, (double)step, (double)lo);
      ex = fma((double)v[i], (double)v[i], ex);
      ee = fma(e, e, ee);
    }
    sx += ex;
    se += ok ? ee : (double)INFINITY;
    if (codes) {
      unsigned char* dst = codes + ((long long)u * nb + q) * (2 * b);
      for (int byte = 0; byte < 2 * b; ++byte) dst[byte] = (unsigned char)(w[byte >> 2] >> ((byte & 3) * 8));
    }
    if (scales) scales[(long long)u * nb + q] = __halves2half2(__float2half_rn(lo), __float2half_rn(step));
  }
  __shared__ double s1[256], s2[256];
  s1[threadIdx.x] = sx;
  s2[threadIdx.x] = se;
  __syncthreads();
  for (int st = blockDim.x / 2; st > 0; st >>= 1) {
    if ((int)threadIdx.x < st) {
      s1[threadIdx.x] += s1[threadIdx.x + st];
      s2[threadIdx.x] += s2[threadIdx.x + st];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    part[((long long)u * nblk + blockIdx.x) * 2 + 0] = s1[0];
    part[((long long)u * nblk + blockIdx.x) * 2 + 1] = s2[0];
  }
}
}  // namespace jolt
