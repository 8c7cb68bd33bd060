// Batched, strided GEMMs used by the factor, sketch and core steps.
//
//   gemm_bf16 : C = alpha * A B (+ beta C), bf16 operands, fp32 accumulation on the tensor
//               cores (warp-level mma.sync m16n8k16, cp.async 3-stage pipeline).  Either
//               operand may be stored K-contiguous or M/N-contiguous, and both the K index
//               and the M/N index may be split into blocks with their own stride, which is
//               how the token unfolding X_(T) (column (l,h,d) -> slice stride T*D) and the
//               feature unfolding are read in place without a copy.
//   gemm_simt : the same contract for fp32 / fp64 operands on the CUDA cores (the small,
//               precision-sensitive products of the orthonormalisation steps).
#pragma once

#include "common.cuh"

namespace jolt {

struct GemmOperand {
  const void* ptr = nullptr;
  const void* ptr_odd = nullptr;  // if set: entry e reads (e odd ? ptr_odd : ptr) + (e/2) * sbatch
                                  // (the K / V alternation of units u = 2 g + kv)
  int bdiv = 1;                   // batch b uses entry e = b / bdiv (operands shared by bdiv batches)
  long long ld = 0;           // stride of the non-contiguous index inside a block
  long long sbatch = 0;       // stride between batch entries
  int kshift = 40;            // K index = kb * 2^kshift + kr
  long long skblk = 0;        //   -> kb * skblk + kr * (stride of K)
  int xshift = 40;            // M (or N) index split the same way
  long long sxblk = 0;
  bool kmajor = true;         // true: K is the contiguous index
};

struct GemmParams {
  int M = 0, N = 0, K = 0;
  int batch = 1;
  GemmOperand A, B;           // A is M x K, B is K x N (logical)
  void* C = nullptr;          // row-major M x N per batch / split
  long long ldc = 0, sbatchC = 0;
  int c_type = 0;             // 0: fp32, 1: bf16 (round to nearest), 2: fp64
  float alpha = 1.f, beta = 0.f;
  int splits = 1;             // split-K: split s covers [s*kchunk, (s+1)*kchunk)
  int kchunk = 0;
  long long ssplitC = 0;      // output stride between splits
  bool sym = false;           // C = A^T A (A = B): tiles above the diagonal are skipped (sgemm)
};

__host__ __device__ __forceinline__ long long opnd_offset(const GemmOperand& o, long long x, long long k) {
  long long xb = x >> o.xshift, xr = x & ((1LL << o.xshift) - 1);
  long long kb = k >> o.kshift, kr = k & ((1LL << o.kshift) - 1);
  long long off = xb * o.sxblk + kb * o.skblk;
  if (o.kmajor) off += xr * o.ld + kr;
  else off += xr + kr * o.ld;
  return off;
}

__host__ __device__ __forceinline__ const void* opnd_base_t(const GemmOperand& o, int b, int esize) {
  const int e = b / o.bdiv;
  const char* base = (const char*)((o.ptr_odd && (e & 1)) ? o.ptr_odd : o.ptr);
  long long idx = o.ptr_odd ? (long long)(e >> 1) : (long long)e;
  return base + idx * o.sbatch * esize;
}
__host__ __device__ __forceinline__ const void* opnd_base(const GemmOperand& o, int b) {
  return opnd_base_t(o, b, 2);
}

// ------------------------------------------------------------------------------------------
// bf16 tensor-core GEMM
// ------------------------------------------------------------------------------------------
namespace gemm_detail {
constexpr int BM = 128, BN = 128, BK = 32, STAGES = 3, THREADS = 256;
constexpr int TILE_ELEMS = BM * BK;  // 4096 bf16 = 8 KiB per operand tile

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  int sz = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(sz));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void mma16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Smem tile layouts (bf16 elements):
//   K-contiguous tile [128 rows][32 k]: 4 chunks of 16 B per row, chunk ^= (row>>1)&3
//   X-contiguous tile [32 k][128 x]  : 16 chunks per row, chunk ^= (row & 7)
__device__ __forceinline__ int kmaj_off(int row, int chunk) { return row * BK + ((chunk ^ ((row >> 1) & 3)) << 3); }
__device__ __forceinline__ int xmaj_off(int krow, int chunk) { return krow * BM + ((chunk ^ (krow & 7)) << 3); }

// issue the copies of one operand tile (rows x0.., k0..).  Whole in-range 16-byte chunks
// go through cp.async; a chunk that straddles the end of the contiguous index (or is not
// 16-byte aligned) is loaded element by element with zeros past the end, so no element
// beyond the logical extent is ever read.
__device__ __forceinline__ void load_tile(bf16* sm, const GemmOperand& o, const bf16* base, int x0, int k0,
                                          int Xext, int kend, int tid) {
#pragma unroll
  for (int it = 0; it < 2; ++it) {
    int c = tid + it * THREADS;  // 0..511
    int x, k, soff, cend, cpos;
    if (o.kmajor) {
      int row = c >> 2, ch = c & 3;
      x = x0 + row;
      k = k0 + ch * 8;
      soff = kmaj_off(row, ch);
      cpos = k;
      cend = kend;
    } else {
      int krow = c >> 4, ch = c & 15;
      x = x0 + ch * 8;
      k = k0 + krow;
      soff = xmaj_off(krow, ch);
      cpos = x;
      cend = Xext;
    }
    bool any = (x < Xext) && (k < kend);
    const bf16* src = any ? base + opnd_offset(o, x, k) : base;
    bool whole = any && (cpos + 8 <= cend) && ((reinterpret_cast<uintptr_t>(src) & 15) == 0);
    if (whole || !any) {
      cp_async16(smem_u32(sm + soff), src, whole);
    } else {
      __align__(16) bf16 v[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        int xe = o.kmajor ? x : x + e;
        int ke = o.kmajor ? k + e : k;
        bool ok = (o.kmajor ? (ke < kend) : (xe < Xext));
        v[e] = ok ? base[opnd_offset(o, xe, ke)] : __float2bfloat16_rn(0.f);
      }
      *reinterpret_cast<uint4*>(sm + soff) = *reinterpret_cast<const uint4*>(v);
    }
  }
}
}  // namespace gemm_detail

__global__ void __launch_bounds__(256) gemm_bf16_kernel(GemmParams p) {
  using namespace gemm_detail;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  bf16* sA = reinterpret_cast<bf16*>(smem_raw);
  bf16* sB = sA + STAGES * TILE_ELEMS;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int wm = warp >> 2, wn = warp & 3;  // 2 x 4 warps, warp tile 64 x 32
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  if (p.sym && blockIdx.x > blockIdx.y) return;   // mirrored from the tile below the diagonal
  const int bz = blockIdx.z;
  const int b = bz / p.splits, split = bz - b * p.splits;
  const int kbeg = split * p.kchunk;
  const int kend = min(p.K, kbeg + p.kchunk);

  const bf16* Ab = reinterpret_cast<const bf16*>(opnd_base(p.A, b));
  const bf16* Bb = reinterpret_cast<const bf16*>(opnd_base(p.B, b));

  float acc[4][4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.f;

  const int ntiles = kend > kbeg ? (int)ceil_div(kend - kbeg, BK) : 0;

#pragma unroll
  for (int s = 0; s < STAGES - 1; ++s) {
    if (s < ntiles) {
      load_tile(sA + s * TILE_ELEMS, p.A, Ab, m0, kbeg + s * BK, p.M, kend, tid);
      load_tile(sB + s * TILE_ELEMS, p.B, Bb, n0, kbeg + s * BK, p.N, kend, tid);
    }
    cp_async_commit();
  }

  for (int t = 0; t < ntiles; ++t) {
    cp_async_wait<STAGES - 2>();
    __syncthreads();
    {
      int tn = t + STAGES - 1;
      if (tn < ntiles) {
        int st = tn % STAGES;
        load_tile(sA + st * TILE_ELEMS, p.A, Ab, m0, kbeg + tn * BK, p.M, kend, tid);
        load_tile(sB + st * TILE_ELEMS, p.B, Bb, n0, kbeg + tn * BK, p.N, kend, tid);
      }
      cp_async_commit();
    }
    const bf16* tA = sA + (t % STAGES) * TILE_ELEMS;
    const bf16* tB = sB + (t % STAGES) * TILE_ELEMS;
#pragma unroll
    for (int kk = 0; kk < BK; kk += 16) {
      uint32_t af[4][4];
#pragma unroll
      for (int mt = 0; mt < 4; ++mt) {
        int mrow = wm * 64 + mt * 16;
        if (p.A.kmajor) {
          int row = mrow + (lane & 15);
          int ch = (kk >> 3) + (lane >> 4);
          ldsm_x4(smem_u32(tA + kmaj_off(row, ch)), af[mt][0], af[mt][1], af[mt][2], af[mt][3]);
        } else {
          int krow = kk + (lane & 7) + ((lane >> 4) << 3);
          int ch = (mrow >> 3) + ((lane >> 3) & 1);
          ldsm_x4_t(smem_u32(tA + xmaj_off(krow, ch)), af[mt][0], af[mt][1], af[mt][2], af[mt][3]);
        }
      }
      uint32_t bfr[4][2];
#pragma unroll
      for (int np = 0; np < 2; ++np) {
        int ncol = wn * 32 + np * 16;
        uint32_t r0, r1, r2, r3;
        if (p.B.kmajor) {
          int row = ncol + (lane & 7) + ((lane >> 4) << 3);
          int ch = (kk >> 3) + ((lane >> 3) & 1);
          ldsm_x4(smem_u32(tB + kmaj_off(row, ch)), r0, r1, r2, r3);
        } else {
          int krow = kk + (lane & 7) + (((lane >> 3) & 1) << 3);
          int ch = (ncol >> 3) + (lane >> 4);
          ldsm_x4_t(smem_u32(tB + xmaj_off(krow, ch)), r0, r1, r2, r3);
        }
        bfr[np * 2 + 0][0] = r0;
        bfr[np * 2 + 0][1] = r1;
        bfr[np * 2 + 1][0] = r2;
        bfr[np * 2 + 1][1] = r3;
      }
#pragma unroll
      for (int mt = 0; mt < 4; ++mt)
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) mma16816(acc[mt][nt], af[mt], bfr[nt][0], bfr[nt][1]);
    }
  }
  cp_async_wait<0>();

  // epilogue
  const long long cbase = (long long)b * p.sbatchC + (long long)split * p.ssplitC;
#pragma unroll
  for (int mt = 0; mt < 4; ++mt) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      int m = m0 + wm * 64 + mt * 16 + (lane >> 2) + h * 8;
      if (m >= p.M) continue;
#pragma unroll
      for (int nt = 0; nt < 4; ++nt) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          int n = n0 + wn * 32 + nt * 8 + (lane & 3) * 2 + e;
          if (n >= p.N) continue;
          float v = p.alpha * acc[mt][nt][h * 2 + e];
          long long off = cbase + (long long)m * p.ldc + n;
          if (p.c_type == 0) {
            float* C = reinterpret_cast<float*>(p.C) + off;
            *C = (p.beta != 0.f) ? v + p.beta * *C : v;
          } else if (p.c_type == 1) {
            bf16* C = reinterpret_cast<bf16*>(p.C) + off;
            *C = __float2bfloat16_rn(p.beta != 0.f ? v + p.beta * __bfloat162float(*C) : v);
          } else {
            double* C = reinterpret_cast<double*>(p.C) + off;
            *C = (p.beta != 0.f) ? (double)v + (double)p.beta * *C : (double)v;
          }
        }
      }
    }
  }
}

inline size_t gemm_bf16_smem() { return 2 * gemm_detail::STAGES * gemm_detail::TILE_ELEMS * sizeof(bf16); }

inline cudaError_t launch_gemm_bf16(const GemmParams& p, cudaStream_t st) {
  static bool attr_set = false;
  if (!attr_set) {
    cudaError_t e = cudaFuncSetAttribute(gemm_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)gemm_bf16_smem());
    if (e != cudaSuccess) return e;
    attr_set = true;
  }
  GemmParams q = p;
  if (q.kchunk <= 0) q.kchunk = q.K;
  dim3 grid((unsigned)ceil_div(q.N, gemm_detail::BN), (unsigned)ceil_div(q.M, gemm_detail::BM),
            (unsigned)(q.batch * q.splits));
  count_launch(), gemm_bf16_kernel<<<grid, gemm_detail::THREADS, gemm_bf16_smem(), st>>>(q);
  return cudaGetLastError();
}

// ------------------------------------------------------------------------------------------
// SIMT GEMM for fp32 / fp64 operands (accumulates in the type Acc)
// ------------------------------------------------------------------------------------------
template <typename TA, typename TB, typename Acc>
__global__ void __launch_bounds__(256) gemm_simt_kernel(GemmParams p) {
  constexpr int T = 64, TK = 16;
  __shared__ Acc sA[TK][T + 1];
  __shared__ Acc sB[TK][T + 1];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int m0 = blockIdx.y * T, n0 = blockIdx.x * T;
  const int bz = blockIdx.z;
  const int b = bz / p.splits, split = bz - b * p.splits;
  const int kbeg = split * p.kchunk;
  const int kend = min(p.K, kbeg + p.kchunk);
  const TA* A = reinterpret_cast<const TA*>(opnd_base_t(p.A, b, (int)sizeof(TA)));
  const TB* B = reinterpret_cast<const TB*>(opnd_base_t(p.B, b, (int)sizeof(TB)));
  Acc acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0;
  for (int k0 = kbeg; k0 < kend; k0 += TK) {
    for (int i = threadIdx.x; i < TK * T; i += 256) {
      int kk, xx;
      if (p.A.kmajor) { xx = i / TK; kk = i % TK; } else { kk = i / T; xx = i % T; }
      int m = m0 + xx, k = k0 + kk;
      sA[kk][xx] = (m < p.M && k < kend) ? (Acc)A[opnd_offset(p.A, m, k)] : (Acc)0;
      if (p.B.kmajor) { xx = i / TK; kk = i % TK; } else { kk = i / T; xx = i % T; }
      int n = n0 + xx;
      k = k0 + kk;
      sB[kk][xx] = (n < p.N && k < kend) ? (Acc)B[opnd_offset(p.B, n, k)] : (Acc)0;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      Acc a[4], bb[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = sA[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) bb[j] = sB[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] += a[i] * bb[j];
    }
    __syncthreads();
  }
  const long long cbase = (long long)b * p.sbatchC + (long long)split * p.ssplitC;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int m = m0 + ty + 16 * i;
    if (m >= p.M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      int n = n0 + tx + 16 * j;
      if (n >= p.N) continue;
      long long off = cbase + (long long)m * p.ldc + n;
      Acc v = (Acc)p.alpha * acc[i][j];
      if (p.c_type == 2) {
        double* C = reinterpret_cast<double*>(p.C) + off;
        *C = (p.beta != 0.f) ? (double)v + (double)p.beta * *C : (double)v;
      } else if (p.c_type == 0) {
        float* C = reinterpret_cast<float*>(p.C) + off;
        *C = (p.beta != 0.f) ? (float)v + p.beta * *C : (float)v;
      } else {
        bf16* C = reinterpret_cast<bf16*>(p.C) + off;
        *C = __float2bfloat16_rn((float)v + (p.beta != 0.f ? p.beta * __bfloat162float(*C) : 0.f));
      }
    }
  }
}

// ------------------------------------------------------------------------------------------
// fp32 x fp32 GEMM on the CUDA cores, register tiled: 128 x 128 CTA tile, 256 threads, 8 x 8
// outputs per thread (two 4 x 4 sub-blocks 64 apart), k-steps of 8 double-buffered in shared
// memory, 16-byte loads where an operand run is aligned and in range.
// ------------------------------------------------------------------------------------------
namespace sgemm_detail {
constexpr int BM = 128, BN = 128, BK = 8, THREADS = 256;

// The BK x 128 slice (k0.., x0..) of an operand, in two steps so that the global loads of the
// next slice are in flight while the current one is multiplied: fetch_slice reads this
// thread's four values into registers, store_slice puts them into s[BK][128] (x fastest).
__device__ __forceinline__ void fetch_slice(float* v, const GemmOperand& o, const float* base, int x0, int k0,
                                            int Xext, int kend, int tid) {
  v[0] = v[1] = v[2] = v[3] = 0.f;
  if (!o.kmajor) {
    // contiguous along x: thread -> (k row tid/32, four x from (tid%32)*4)
    const int kr = tid >> 5, xc = (tid & 31) * 4;
    const int k = k0 + kr, x = x0 + xc;
    if (k < kend) {
      const float* src = base + opnd_offset(o, x, k);
      const bool vec = (x + 3 < Xext) && (o.xshift >= 31 || ((x & ((1 << o.xshift) - 1)) + 3) < (1 << o.xshift)) &&
                       ((reinterpret_cast<uintptr_t>(src) & 15) == 0);
      if (vec) {
        float4 t = *reinterpret_cast<const float4*>(src);
        v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (x + e < Xext) v[e] = base[opnd_offset(o, x + e, k)];
      }
    }
  } else {
    // contiguous along k: thread -> (x row tid/2, four k from (tid%2)*4)
    const int xr = tid >> 1, kc = (tid & 1) * 4;
    const int x = x0 + xr, k = k0 + kc;
    if (x < Xext && k < kend) {
      const float* src = base + opnd_offset(o, x, k);
      const bool vec = (k + 3 < kend) && ((reinterpret_cast<uintptr_t>(src) & 15) == 0) &&
                       (o.kshift >= 31 || ((k & ((1 << o.kshift) - 1)) + 3) < (1 << o.kshift));
      if (vec) {
        float4 t = *reinterpret_cast<const float4*>(src);
        v[0] = t.x; v[1] = t.y; v[2] = t.z; v[3] = t.w;
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (k + e < kend) v[e] = base[opnd_offset(o, x, k + e)];
      }
    }
  }
}
__device__ __forceinline__ void store_slice(float (*s)[BM], const GemmOperand& o, const float* v, int tid) {
  if (!o.kmajor) {
    const int kr = tid >> 5, xc = (tid & 31) * 4;
    *reinterpret_cast<float4*>(&s[kr][xc]) = make_float4(v[0], v[1], v[2], v[3]);
  } else {
    // stored transposed
    const int xr = tid >> 1, kc = (tid & 1) * 4;
#pragma unroll
    for (int e = 0; e < 4; ++e) s[kc + e][xr] = v[e];
  }
}
}  // namespace sgemm_detail

__global__ void __launch_bounds__(256, 2) sgemm_kernel(GemmParams p) {
  using namespace sgemm_detail;
  __shared__ __align__(16) float As[2][BK][BM];
  __shared__ __align__(16) float Bs[2][BK][BN];
  const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  if (p.sym && blockIdx.x > blockIdx.y) return;   // mirrored from the tile below the diagonal
  const int bz = blockIdx.z;
  const int b = bz / p.splits, split = bz - b * p.splits;
  const int kbeg = split * p.kchunk;
  const int kend = min(p.K, kbeg + p.kchunk);
  const float* A = reinterpret_cast<const float*>(opnd_base_t(p.A, b, 4));
  const float* B = reinterpret_cast<const float*>(opnd_base_t(p.B, b, 4));
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
  const int ntiles = kend > kbeg ? (kend - kbeg + BK - 1) / BK : 0;
  float va[4], vb[4];
  if (ntiles > 0) {
    fetch_slice(va, p.A, A, m0, kbeg, p.M, kend, tid);
    fetch_slice(vb, p.B, B, n0, kbeg, p.N, kend, tid);
    store_slice(As[0], p.A, va, tid);
    store_slice(Bs[0], p.B, vb, tid);
  }
  __syncthreads();
  for (int t = 0; t < ntiles; ++t) {
    const int cur = t & 1;
    const bool more = t + 1 < ntiles;
    if (more) {
      fetch_slice(va, p.A, A, m0, kbeg + (t + 1) * BK, p.M, kend, tid);
      fetch_slice(vb, p.B, B, n0, kbeg + (t + 1) * BK, p.N, kend, tid);
    }
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float a[8], bb[8];
      const float4 a0 = *reinterpret_cast<const float4*>(&As[cur][kk][ty * 4]);
      const float4 a1 = *reinterpret_cast<const float4*>(&As[cur][kk][64 + ty * 4]);
      const float4 b0 = *reinterpret_cast<const float4*>(&Bs[cur][kk][tx * 4]);
      const float4 b1 = *reinterpret_cast<const float4*>(&Bs[cur][kk][64 + tx * 4]);
      a[0] = a0.x; a[1] = a0.y; a[2] = a0.z; a[3] = a0.w; a[4] = a1.x; a[5] = a1.y; a[6] = a1.z; a[7] = a1.w;
      bb[0] = b0.x; bb[1] = b0.y; bb[2] = b0.z; bb[3] = b0.w; bb[4] = b1.x; bb[5] = b1.y; bb[6] = b1.z; bb[7] = b1.w;
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], bb[j], acc[i][j]);
    }
    // the other buffer was last read before the previous barrier
    if (more) {
      store_slice(As[cur ^ 1], p.A, va, tid);
      store_slice(Bs[cur ^ 1], p.B, vb, tid);
    }
    __syncthreads();
  }
  const long long cbase = (long long)b * p.sbatchC + (long long)split * p.ssplitC;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int m = m0 + (i < 4 ? ty * 4 + i : 64 + ty * 4 + i - 4);
    if (m >= p.M) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int n = n0 + (j < 4 ? tx * 4 + j : 64 + tx * 4 + j - 4);
      if (n >= p.N) continue;
      const long long off = cbase + (long long)m * p.ldc + n;
      const float v = p.alpha * acc[i][j];
      if (p.c_type == 2) {
        double* C = reinterpret_cast<double*>(p.C) + off;
        *C = (p.beta != 0.f) ? (double)v + (double)p.beta * *C : (double)v;
      } else if (p.c_type == 0) {
        float* C = reinterpret_cast<float*>(p.C) + off;
        *C = (p.beta != 0.f) ? v + p.beta * *C : v;
      } else {
        bf16* C = reinterpret_cast<bf16*>(p.C) + off;
        *C = __float2bfloat16_rn(p.beta != 0.f ? v + p.beta * __bfloat162float(*C) : v);
      }
    }
  }
}

inline cudaError_t launch_sgemm(const GemmParams& p, cudaStream_t st) {
  GemmParams q = p;
  if (q.kchunk <= 0) q.kchunk = q.K;
  dim3 grid((unsigned)ceil_div(q.N, sgemm_detail::BN), (unsigned)ceil_div(q.M, sgemm_detail::BM),
            (unsigned)(q.batch * q.splits));
  count_launch();
  sgemm_kernel<<<grid, sgemm_detail::THREADS, 0, st>>>(q);
  return cudaGetLastError();
}

template <typename TA, typename TB, typename Acc>
inline cudaError_t launch_gemm_simt(const GemmParams& p, cudaStream_t st) {
  GemmParams q = p;
  if (q.kchunk <= 0) q.kchunk = q.K;
  dim3 grid((unsigned)ceil_div(q.N, 64), (unsigned)ceil_div(q.M, 64), (unsigned)(q.batch * q.splits));
  count_launch(), gemm_simt_kernel<TA, TB, Acc><<<grid, 256, 0, st>>>(q);
  return cudaGetLastError();
}

}  // namespace jolt
