// Cholesky QR of the sketch blocks: Q = Y L^{-T} with G = Y^T Y = L L^T (the factor kernels;
// the products run on the tensor cores).
//
// Three kernels, all in fp64 up to the last product:
//   chol_factor_kernel   one CTA per unit: the Cholesky factor L of the Gram, left-looking,
//                        blocked by 32 columns; it also inverts each 32 x 32 diagonal block;
//   tri_inv_kernel       one CTA per (32-column block, unit): that block column of W = L^{-1}
//                        by block forward substitution (the block columns are independent);
//   trsm_inv_kernel      one CTA per 64 rows of Y: Q = Y W^T in fp32 with every output
//                        column independent (no sequential dependency across columns).
// The Gram buffer G (column-major, ld gld, symmetric on entry) carries the factor between
// them: L's rows below its diagonal blocks go to the lower triangle, the inverses of the
// diagonal blocks to the upper triangle of their own diagonal block (W[i][c] at G[i*gld+c],
// c <= i), both places the factorisation no longer reads.
#pragma once


#include "common.cuh"

namespace jolt {

constexpr int CF_NB = 32;
constexpr int CF_MAXK = 256;
constexpr int CF_THREADS = 256;
constexpr int CF_P = CF_NB + 1;   // shared-memory pitch (doubles)

// asynchronous global -> shared copies (the staging loads of all three kernels stay in flight
// together instead of one round trip per element); src_bytes < size zero-fills the rest
__device__ __forceinline__ void cf_cp8(void* dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8;\n" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
               "l"(src)
               : "memory");
}
__device__ __forceinline__ void cf_cp16(void* dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"((uint32_t)__cvta_generic_to_shared(dst)),
               "l"(src), "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cf_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cf_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// Shared memory of the factor: the block column P (R x 32), the factored diagonal block L11,
// its inverse (stored transposed) and the finished columns left of the block column
// (R x J0, pitch J0 + 1), whose largest size for k <= 256 is 128 x 129 at J0 = 128.
constexpr int CF_LEFT_MAX = 128 * 129;
inline size_t chol_factor_smem() {
  return ((size_t)CF_MAXK * CF_P + 2 * (size_t)CF_NB * CF_P + CF_LEFT_MAX) * sizeof(double);
}

// Non-finite Gram entries (or one met earlier in the cache): G := I (so W = I) and
// DEV_ERR_NONFINITE.  A pivot that is not positive: DEV_ERR_FACTOR, the pivot taken as 1.
// Per block column J (rows J0..k, R of them), all 512 threads in every phase:
//   1. the finished columns 0..J0 of those rows are copied to shared memory in one batch;
//   2. the block column of the Gram minus their products (registers, 4 x 4 per thread,
//      the inner dimension split over the threads a short block column leaves idle);
//   3. the diagonal block factored column by column, one barrier per pivot;
//   4. its inverse by right-looking forward substitution, one barrier per row;
//   5. the rows below: L21 = A21 inv(L11)^T, 7 rows x 2 columns per thread;
//   6. L21 to the Gram's lower triangle, inv(L11) to the upper part of its diagonal block.
constexpr int CF_FT = 512;   // threads of the factor kernel
__global__ void __launch_bounds__(CF_FT, 1)
    chol_factor_kernel(double* G, int k, long long gld, long long sG, uint32_t* status) {
  extern __shared__ __align__(16) double cf_sm[];
  double* P = cf_sm;                      // [row - J0][col - J0]
  double* Ls = P + CF_MAXK * CF_P;        // L11 [r][c]
  double* XT = Ls + CF_NB * CF_P;         // inv(L11) transposed: XT[c][r] = inv(L11)[r][c]
  double* Lleft = XT + CF_NB * CF_P;      // [row - J0][q], q < J0
  __shared__ double rdiag[CF_NB];
  __shared__ int fail;
  constexpr int NW = CF_FT / 32;
  const int u = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  double* Gu = G + (long long)u * sG;
  const int nbk = (k + CF_NB - 1) / CF_NB;
  int bad = (tid == 0 && (*status & DEV_ERR_NONFINITE)) ? 1 : 0;
  if (tid == 0) fail = 0;

  for (int J = 0; J < nbk; ++J) {
    const int J0 = J * CF_NB, nb = min(CF_NB, k - J0), R = k - J0, lp = J0 + 1;
    // 1. L[J0 + lr][q], q < J0 (written before the barrier that ended block column q / 32)
    for (int q = warp; q < J0; q += NW) {
      const double* src = Gu + (long long)q * gld + J0;
#pragma unroll
      for (int t = 0; t < CF_MAXK / 32; ++t) {
        const int lr = lane + 32 * t;
        if (lr < R) cf_cp8(Lleft + lr * lp + q, src + lr);
      }
    }
    cf_commit();
    // 2. the Gram's block column through its symmetric upper part (never overwritten there),
    //    minus the products of the finished columns.  Thread tile: rows 4 trg .. 4 trg + 3,
    //    columns tcc + 8 j.  A short block column leaves tiles for fewer threads than the
    //    CTA has: the inner dimension is then split KS ways, split 0 starting from the Gram
    //    and the others from zero, and split 0 adds the others' partial sums in split order
    //    (they are parked in rows of P past R: at most 8192 doubles, P holds 8448).
    //    Every Gram entry is read here once up to symmetry, so the finiteness check is here.
    const int ntiles = 8 * ((R + 3) / 4);
    const int KS = max(1, CF_FT / ntiles);
    const int ti = tid % ntiles, ks = tid / ntiles, trg = ti >> 3, tcc = ti & 7;
    const bool act = ks < KS;
    double acc[4][4];
#pragma unroll
    for (int m = 0; m < 4; ++m)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int lr = 4 * trg + m, c = tcc + 8 * j;
        acc[m][j] = (ks == 0 && lr < R && c < nb) ? Gu[(long long)(J0 + lr) * gld + J0 + c] : 0.0;
        if (!isfinite(acc[m][j])) bad = 1;
      }
    cf_wait<0>();
    if (__syncthreads_or(bad)) {
      if (tid == 0) raise_status(status, DEV_ERR_NONFINITE);
      for (int c = warp; c < k; c += NW)
        for (int i = lane; i < k; i += 32) Gu[(long long)c * gld + i] = i == c ? 1.0 : 0.0;
      return;
    }
    if (act && J0 > 0) {
      const int qc = (J0 + KS - 1) / KS, qb = ks * qc, qe = min(J0, qb + qc);
#pragma unroll 2
      for (int q = qb; q < qe; ++q) {
        double b[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) b[j] = Lleft[(tcc + 8 * j) * lp + q];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          // rows past R would lie beyond the staged block
          const double a = 4 * trg + m < R ? Lleft[(4 * trg + m) * lp + q] : 0.0;
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[m][j] = fma(-a, b[j], acc[m][j]);
        }
      }
    }
    double* part = P + R * CF_P;   // partial sums of splits 1..KS-1
    if (act && ks > 0) {
#pragma unroll
      for (int m = 0; m < 4; ++m)
#pragma unroll
        for (int j = 0; j < 4; ++j) part[((ks - 1) * ntiles + ti) * 16 + m * 4 + j] = acc[m][j];
    }
    __syncthreads();
    if (ks == 0) {
      for (int s2 = 1; s2 < KS; ++s2)
#pragma unroll
        for (int m = 0; m < 4; ++m)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[m][j] += part[((s2 - 1) * ntiles + ti) * 16 + m * 4 + j];
    }
    __syncthreads();
    if (ks == 0) {
#pragma unroll
      for (int m = 0; m < 4; ++m)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int lr = 4 * trg + m, c = tcc + 8 * j;
          if (lr < R && c < nb) P[lr * CF_P + c] = acc[m][j];
        }
    }
    __syncthreads();
    // 3. diagonal block: thread (r = tid / 16, s = tid % 16) updates columns s and s + 16 of
    //    row r; a step reads only column c and writes only columns > c
    {
      const int r = tid >> 4, s16 = tid & 15;
      for (int c = 0; c < nb; ++c) {
        const double piv = P[c * CF_P + c];
        const bool ok = piv > 0.0 && isfinite(piv);
        const double rd = ok ? rsqrt(piv) : 1.0;
        if (r > c && r < nb) {
          const double lrc = P[r * CF_P + c] * rd;   // L[r][c]
#pragma unroll
          for (int i = 0; i < 2; ++i) {
            const int c2 = s16 + 16 * i;
            if (c2 > c && c2 <= r) P[r * CF_P + c2] = fma(-lrc, P[c2 * CF_P + c] * rd, P[r * CF_P + c2]);
          }
          if (s16 == 0) Ls[r * CF_P + c] = lrc;
        }
        if (tid == 0) {
          Ls[c * CF_P + c] = ok ? piv * rd : 1.0;
          rdiag[c] = rd;
          if (!ok) fail = 1;
        }
        __syncthreads();
      }
    }
    // 4. inv(L11): thread (column j = lane, rows w and w + 16) keeps its rows' running sums;
    //    row r is final once the rows above it are, and its owner publishes it
    {
      double x0 = (warp == lane && lane < nb) ? 1.0 : 0.0, x1 = (warp + 16 == lane && lane < nb) ? 1.0 : 0.0;
      for (int r = 0; r < nb; ++r) {
        if (warp == (r & 15)) XT[lane * CF_P + r] = (lane <= r) ? (r < 16 ? x0 : x1) * rdiag[r] : 0.0;
        __syncthreads();
        const double xr = XT[lane * CF_P + r];
        if (warp > r && warp < nb) x0 = fma(-Ls[warp * CF_P + r], xr, x0);
        if (warp + 16 > r && warp + 16 < nb) x1 = fma(-Ls[(warp + 16) * CF_P + r], xr, x1);
      }
    }
    // 5. rows below the diagonal block: L21[lr][c] = sum_{q <= c} A21[lr][q] inv(L11)[c][q];
    //    thread: columns cl and cl + 16, rows nb + rg + 32 t
    const int nbelow = R - nb, cl = tid & 15, rg = tid >> 4;
    constexpr int RT = (CF_MAXK - CF_NB) / 32;   // 7
    double o0[RT], o1[RT];
#pragma unroll
    for (int t = 0; t < RT; ++t) o0[t] = o1[t] = 0.0;
    if (nbelow > 0) {
#pragma unroll 2
      for (int q = 0; q < nb; ++q) {
        const double xa = XT[q * CF_P + cl], xb = XT[q * CF_P + cl + 16];   // inv(L11)[c][q]
#pragma unroll
        for (int t = 0; t < RT; ++t) {
          const int lr = nb + rg + 32 * t;
          if (32 * t < nbelow) {
            const double a = lr < R ? P[lr * CF_P + q] : 0.0;
            o0[t] = fma(a, xa, o0[t]);
            o1[t] = fma(a, xb, o1[t]);
          }
        }
      }
    }
    __syncthreads();
    // 6. outputs
#pragma unroll
    for (int t = 0; t < RT; ++t) {
      const int lr = nb + rg + 32 * t;
      if (lr < R) {
        if (cl < nb) P[lr * CF_P + cl] = o0[t];
        if (cl + 16 < nb) P[lr * CF_P + cl + 16] = o1[t];
      }
    }
    __syncthreads();
    for (int c = warp; c < nb; c += NW) {
      double* dst = Gu + (long long)(J0 + c) * gld + J0;
      for (int lr = nb + lane; lr < R; lr += 32) dst[lr] = P[lr * CF_P + c];
    }
    for (int idx = tid; idx < CF_NB * CF_NB; idx += CF_FT) {
      const int r = idx / CF_NB, c = idx % CF_NB;
      if (r < nb && c <= r) Gu[(long long)(J0 + r) * gld + J0 + c] = XT[c * CF_P + r];
    }
    __syncthreads();
  }
  if (tid == 0 && fail) raise_status(status, DEV_ERR_FACTOR);
}

// ------------------------------------------------------------------------------------------
// Block column J of W = L^{-1}:  W_JJ = inv(L_JJ),  W_IJ = -inv(L_II) sum_{J<=K<I} L_IK W_KJ.
// Written transposed and in fp32: WT[q][i] = W[i][q] for the rows q of block J (zeros for
// i < J0 and for i >= k up to the padded width ldw).
// ------------------------------------------------------------------------------------------
constexpr int TI_LP = CF_MAXK + 1;
inline size_t tri_inv_smem() {
  return ((size_t)CF_MAXK * CF_P + (size_t)CF_NB * TI_LP + 2 * (size_t)CF_NB * CF_P) * sizeof(double);
}

__global__ void __launch_bounds__(CF_THREADS, 1)
    tri_inv_kernel(const double* G, int k, long long gld, long long sG, float* WT, long long ldw, long long sW) {
  extern __shared__ __align__(16) double ti_sm[];
  double* X = ti_sm;                       // [i - J0][c]: rows of W's block column
  double* Ls = X + CF_MAXK * CF_P;         // [r][q - J0]: L's rows of block I
  double* Ds = Ls + CF_NB * TI_LP;         // inv(L_II)
  double* Ts = Ds + CF_NB * CF_P;          // sum_K L_IK W_KJ
  const int J = blockIdx.x, u = blockIdx.y, tid = threadIdx.x;
  const int J0 = J * CF_NB, nbJ = min(CF_NB, k - J0);
  const int nbk = (k + CF_NB - 1) / CF_NB;
  const double* Gu = G + (long long)u * sG;
  const int r = tid >> 3, cg = tid & 7;    // 32 x 32 outputs: row r, columns cg + 8 j

  // the inverse of the 32 x 32 diagonal block I (lower; W[I0 + r][I0 + c] at G[(I0 + r) * gld + I0 + c])
  auto stage_diag = [&](int I0, int nbI, double* dst) {
    for (int idx = tid; idx < CF_NB * CF_NB; idx += CF_THREADS) {
      const int rr = idx / CF_NB, c = idx % CF_NB;
      if (rr < nbI && c <= rr) cf_cp8(dst + rr * CF_P + c, Gu + (long long)(I0 + rr) * gld + I0 + c);
      else dst[rr * CF_P + c] = 0.0;
    }
  };
  stage_diag(J0, nbJ, X);
  cf_commit();
  for (int I = J + 1; I < nbk; ++I) {
    const int I0 = I * CF_NB, nbI = min(CF_NB, k - I0), KQ = I0 - J0;
    __syncthreads();
    for (int idx = tid; idx < KQ * CF_NB; idx += CF_THREADS) {
      const int q = idx / CF_NB, rr = idx % CF_NB;
      if (rr < nbI) cf_cp8(Ls + rr * TI_LP + q, Gu + (long long)(J0 + q) * gld + I0 + rr);
      else Ls[rr * TI_LP + q] = 0.0;
    }
    stage_diag(I0, nbI, Ds);
    cf_commit();
    cf_wait<0>();
    __syncthreads();
    double acc[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll 4
    for (int q = 0; q < KQ; ++q) {
      const double a = Ls[r * TI_LP + q];
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[j] = fma(a, X[q * CF_P + cg + 8 * j], acc[j]);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) Ts[r * CF_P + cg + 8 * j] = acc[j];
    __syncthreads();
    double out[4] = {0.0, 0.0, 0.0, 0.0};
    for (int s = 0; s <= r; ++s) {
      const double d = Ds[r * CF_P + s];
#pragma unroll
      for (int j = 0; j < 4; ++j) out[j] = fma(d, Ts[s * CF_P + cg + 8 * j], out[j]);
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) X[(KQ + r) * CF_P + cg + 8 * j] = r < nbI ? -out[j] : 0.0;
  }
  cf_wait<0>();
  __syncthreads();
  float* Wu = WT + (long long)u * sW;
  for (int c = tid >> 5; c < nbJ; c += CF_THREADS / 32)
    for (int i = tid & 31; i < ldw; i += 32)
      Wu[(long long)(J0 + c) * ldw + i] = (i >= J0 && i < k) ? (float)X[(i - J0) * CF_P + c] : 0.f;
}

// ------------------------------------------------------------------------------------------
// Q = Y W^T in place, W lower triangular (k <= 256): a CTA keeps 64 rows of Y in shared
// memory and stages WT 16 rows at a time (the next chunk in flight while the current one is
// used); warp w computes rows 8w..8w+7, lane l the columns l + 32 j.  Column blocks j with
// 32 j + 31 < q0 meet only zeros of W in the chunk at q0 and are skipped.
// ------------------------------------------------------------------------------------------
constexpr int TI_RB = 64;
constexpr int TI_QC = 16;   // rows of WT per staged chunk (double-buffered)
inline int trsm_inv_pitch(int kq) { return kq + 4; }
inline size_t trsm_inv_smem(int kq) {
  return ((size_t)TI_RB * trsm_inv_pitch(kq) + 2 * (size_t)TI_QC * kq) * sizeof(float);
}

__global__ void __launch_bounds__(CF_THREADS, 2)
    trsm_inv_kernel(float* Y, long long m, int k, long long ld, long long sY, const float* WT, long long ldw,
                    long long sW) {
  extern __shared__ __align__(16) float tv_sm[];
  const int kq = (k + 31) & ~31, P = kq + 4, nj = kq / 32;
  float* panel = tv_sm;                                      // TI_RB x P
  float* const wt0 = panel + TI_RB * P;                      // two buffers TI_QC x kq
  const int u = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long long r0 = (long long)blockIdx.x * TI_RB;
  float* Yu = Y + (long long)u * sY;
  const float* Wu = WT + (long long)u * sW;
  // rows r0.. of Y (16-byte copies: ld is a multiple of 4 floats; columns >= k and rows >= m
  // are zero-filled)
  for (int rr = warp; rr < TI_RB; rr += CF_THREADS / 32)
    for (int c = 4 * lane; c < kq; c += 128) {
      const bool row_ok = r0 + rr < m;
      const int nbytes = row_ok ? 4 * max(0, min(4, k - c)) : 0;
      cf_cp16(panel + rr * P + c, nbytes > 0 ? Yu + (r0 + rr) * ld + c : Yu, nbytes);
    }
  auto stage = [&](int q0, float* buf) {
    for (int q = warp; q < TI_QC; q += CF_THREADS / 32)
      for (int c = 4 * lane; c < kq; c += 128) {
        const bool ok = q0 + q < k;
        cf_cp16(buf + q * kq + c, ok ? Wu + (long long)(q0 + q) * ldw + c : Wu, ok ? 16 : 0);
      }
    cf_commit();
  };
  stage(0, wt0);   // committed together with the panel
  // accumulators of column blocks 2p and 2p + 1 side by side: packed fp32 FMAs (two IEEE
  // fmas each, in the same order as scalar ones)
  float2 acc[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int p = 0; p < 4; ++p) acc[i][p] = make_float2(0.f, 0.f);
  const int nch = (k + TI_QC - 1) / TI_QC;
  for (int ch = 0; ch < nch; ++ch) {
    const int q0 = ch * TI_QC;
    // the buffer of chunk ch + 1 was last read before the barrier ending chunk ch - 1
    if (ch + 1 < nch) {
      stage(q0 + TI_QC, wt0 + ((ch + 1) & 1) * (TI_QC * kq));
      cf_wait<1>();
    } else {
      cf_wait<0>();
    }
    __syncthreads();
    const float* wt = wt0 + (ch & 1) * (TI_QC * kq);
    // column blocks j with 32 j + 31 < q0 meet only zeros of W: a pair is skipped when both
    // of its blocks are (an inactive block of a live pair adds 0 * y = +0)
    const int jmin = q0 / 32;
#pragma unroll 1
    for (int q = 0; q < TI_QC; q += 4) {
      float2 w[4][4];
#pragma unroll
      for (int pr = 0; pr < 4; ++pr)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j0 = 2 * pr, j1 = 2 * pr + 1;
          w[pr][e] = make_float2((j0 >= jmin && j0 < nj) ? wt[(q + e) * kq + lane + 32 * j0] : 0.f,
                                 (j1 >= jmin && j1 < nj) ? wt[(q + e) * kq + lane + 32 * j1] : 0.f);
        }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float4 y = *reinterpret_cast<const float4*>(panel + (warp * 8 + i) * P + q0 + q);
#pragma unroll
        for (int pr = 0; pr < 4; ++pr) {
          if (2 * pr + 1 >= jmin && 2 * pr < nj) {
            float2 a = acc[i][pr];
            a = __ffma2_rn(make_float2(y.x, y.x), w[pr][0], a);
            a = __ffma2_rn(make_float2(y.y, y.y), w[pr][1], a);
            a = __ffma2_rn(make_float2(y.z, y.z), w[pr][2], a);
            a = __ffma2_rn(make_float2(y.w, y.w), w[pr][3], a);
            acc[i][pr] = a;
          }
        }
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const long long rr = r0 + warp * 8 + i;
    if (rr >= m) continue;
#pragma unroll
    for (int pr = 0; pr < 4; ++pr) {
      const int c0 = lane + 64 * pr, c1 = c0 + 32;
      if (2 * pr < nj && c0 < k) Yu[rr * ld + c0] = acc[i][pr].x;
      if (2 * pr + 1 < nj && c1 < k) Yu[rr * ld + c1] = acc[i][pr].y;
    }
  }
}

}  // namespace jolt

namespace jolt {

// ------------------------------------------------------------------------------------------
// W = L^{-1} for any k (the block-column recursion of tri_inv_kernel with the block column
// kept in global fp64 scratch instead of shared memory; each sum over K split over TI_G thread
// groups and added in group order):
//   W_JJ = inv(L_JJ),   W_IJ = -inv(L_II) sum_{J <= K < I} L_IK W_KJ   (I > J).
// G: L's blocks below the diagonal in the lower triangle, inv(L_II) in the upper part of
// the diagonal blocks.  One CTA per (block column J, unit), TI_G x 256 threads (dynamic
// shared memory tri_inv_large_smem()); thread (r, cg) of a group computes entries (r, cg + 8 j)
// of each 32 x 32 block.  scr: per unit and block column a kq32 x 32 fp64 slab (row i of the
// slab = row i of W).  Output as tri_inv_kernel: WT[q][i] = W[i][q] in fp32 at pitch ldw, zeros
// for i < J0 and for k <= i < ldw.
// ------------------------------------------------------------------------------------------
constexpr int TI_G = 4;   // K blocks of one sum formed at once, one thread group of CF_THREADS each
inline size_t tri_inv_large_smem() { return sizeof(double) * (3 * TI_G + 1) * CF_NB * CF_P; }
__global__ void __launch_bounds__(CF_THREADS * TI_G) tri_inv_large_kernel(const double* G, int k, long long gld,
                                                                         long long sG, double* scr, int kq32, float* WT,
                                                                         long long ldw, long long sW) {
  extern __shared__ double ti_sm[];
  double(*Ls)[CF_NB][CF_P] = reinterpret_cast<double(*)[CF_NB][CF_P]>(ti_sm);   // [TI_G] L_IK, [r][q]
  double(*Xs)[CF_NB][CF_P] = Ls + TI_G;                                          // [TI_G] W_KJ, [q][c]
  double(*Tg)[CF_NB][CF_P] = Xs + TI_G;                                          // [TI_G] partial sums
  double(*Ds)[CF_P] = reinterpret_cast<double(*)[CF_P]>(Tg + TI_G);            // inv(L_II)
  const int J = blockIdx.x, u = blockIdx.y, tid = threadIdx.x;
  const int g = tid / CF_THREADS, lt = tid - g * CF_THREADS;
  const int nbk = (k + CF_NB - 1) / CF_NB;
  const int J0 = J * CF_NB, nbJ = min(CF_NB, k - J0);
  const double* Gu = G + (long long)u * sG;
  double* X = scr + ((long long)u * nbk + J) * (long long)kq32 * CF_NB;   // X[i * 32 + c]
  const int r = lt >> 3, cg = lt & 7;
  // W_JJ
  for (int idx = tid; idx < CF_NB * CF_NB; idx += blockDim.x) {
    const int rr = idx / CF_NB, c = idx % CF_NB;
    X[(long long)(J0 + rr) * CF_NB + c] =
        (rr < nbJ && c < nbJ && c <= rr) ? Gu[(long long)(J0 + rr) * gld + J0 + c] : 0.0;
  }
  __syncthreads();
  for (int I = J + 1; I < nbk; ++I) {
    const int I0 = I * CF_NB, nbI = min(CF_NB, k - I0);
    // group g sums the K blocks J + g, J + g + TI_G, ... (its own barrier: the trip counts differ)
    double acc[4] = {0.0, 0.0, 0.0, 0.0};
    for (int K = J + g; K < I; K += TI_G) {
      const int K0 = K * CF_NB, nbK = min(CF_NB, k - K0);
      for (int idx = lt; idx < CF_NB * CF_NB; idx += CF_THREADS) {
        const int a = idx / CF_NB, b = idx % CF_NB;
        // L_IK[b][a] = L[I0 + b][K0 + a], column-major at G[(K0 + a) * gld + I0 + b]: consecutive
        // threads read consecutive rows of one column
        Ls[g][b][a] = (b < nbI && a < nbK) ? Gu[(long long)(K0 + a) * gld + I0 + b] : 0.0;
        Xs[g][a][b] = a < nbK ? X[(long long)(K0 + a) * CF_NB + b] : 0.0;
      }
      asm volatile("bar.sync %0, %1;" ::"r"(1 + g), "n"(CF_THREADS) : "memory");
#pragma unroll 8
      for (int q = 0; q < CF_NB; ++q) {
        const double l = Ls[g][r][q];
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[j] = fma(l, Xs[g][q][cg + 8 * j], acc[j]);
      }
      asm volatile("bar.sync %0, %1;" ::"r"(1 + g), "n"(CF_THREADS) : "memory");
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) Tg[g][r][cg + 8 * j] = acc[j];
    for (int idx = tid; idx < CF_NB * CF_NB; idx += blockDim.x) {
      const int rr = idx / CF_NB, s2 = idx % CF_NB;
      Ds[rr][s2] = (rr < nbI && s2 <= rr) ? Gu[(long long)(I0 + rr) * gld + I0 + s2] : 0.0;
    }
    __syncthreads();
    if (g == 0) {
      // W_IJ = -inv(L_II) (sum over the groups, in group order)
      double out[4] = {0.0, 0.0, 0.0, 0.0};
      for (int s2 = 0; s2 <= r; ++s2) {
        const double d = Ds[r][s2];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          double t = Tg[0][s2][cg + 8 * j];
#pragma unroll
          for (int gg = 1; gg < TI_G; ++gg) t += Tg[gg][s2][cg + 8 * j];
          out[j] = fma(d, t, out[j]);
        }
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) X[(long long)(I0 + r) * CF_NB + cg + 8 * j] = r < nbI ? -out[j] : 0.0;
    }
    __syncthreads();
  }
  float* Wu = WT + (long long)u * sW;
  for (int c = tid >> 5; c < nbJ; c += blockDim.x / 32)
    for (int i = tid & 31; i < ldw; i += 32)
      Wu[(long long)(J0 + c) * ldw + i] = (i >= J0 && i < k) ? (float)X[(long long)i * CF_NB + c] : 0.f;
}

}  // namespace jolt

namespace jolt {
// ------------------------------------------------------------------------------------------
// Cholesky factor for 256 < k <= 1024 as a sequence of small steps over all matrices at once,
// right-looking by 32-column block columns J (the blocked arithmetic of chol_factor_kernel,
// with every block of a step handled by its own CTA, so the whole GPU works on each step):
//   chol_step_diag_kernel   L_JJ = chol(A_JJ) and inv(L_JJ) (one warp per matrix);
//   chol_step_panel_kernel  L_IJ = A_IJ inv(L_JJ)^T for I > J (one CTA per block);
//   chol_step_update_kernel A_IK -= L_IJ L_KJ^T for J < K <= I (one CTA per block pair).
// Output as chol_factor_kernel: L below the diagonal blocks in the lower triangle, inv(L_JJ)
// in the upper part of its diagonal block (W[r][c] at row J0 + c, column J0 + r).  A pivot
// that is not positive raises DEV_ERR_FACTOR and is taken as 1.  G column-major, pitch gld,
// matrix stride sG.
// ------------------------------------------------------------------------------------------
// grid (matrices), 32 threads
__global__ void __launch_bounds__(32) chol_step_diag_kernel(double* G, int k, long long gld, long long sG, int J,
                                                            uint32_t* status) {
  __shared__ double Ls[CF_NB][CF_P];
  const int lane = threadIdx.x;
  double* Gu = G + (long long)blockIdx.x * sG;
  const int J0 = J * CF_NB, nbJ = min(CF_NB, k - J0);
  auto at = [&](int r, int c) -> double& { return Gu[(long long)c * gld + r]; };
  for (int c = 0; c < CF_NB; ++c) Ls[lane][c] = (lane < nbJ && c < nbJ) ? at(J0 + lane, J0 + c) : (lane == c ? 1.0 : 0.0);
  __syncwarp();
  bool bad = false;
  // lane r holds row r
  for (int c = 0; c < CF_NB; ++c) {
    double d = Ls[c][c];
    if (!(d > 0.0) || !isfinite(d)) {
      if (c < nbJ) bad = true;
      d = 1.0;
    }
    d = sqrt(d);
    __syncwarp();
    if (lane == c) Ls[c][c] = d;
    if (lane > c) Ls[lane][c] /= d;
    __syncwarp();
    if (lane > c)
      for (int s = c + 1; s <= lane; ++s) Ls[lane][s] -= Ls[lane][c] * Ls[s][c];
    __syncwarp();
  }
  // inverse: lane c solves L x = e_c
  double x[CF_NB];
#pragma unroll
  for (int r = 0; r < CF_NB; ++r) {
    double v = (r == lane) ? 1.0 : 0.0;
#pragma unroll
    for (int p = 0; p < r; ++p) v = fma(-Ls[r][p], x[p], v);
    x[r] = v / Ls[r][r];
  }
  // W[r][lane] = x[r] (r >= lane) at row J0 + lane, column J0 + r
#pragma unroll
  for (int r = 0; r < CF_NB; ++r)
    if (r >= lane && r < nbJ && lane < nbJ) at(J0 + lane, J0 + r) = x[r];
  if (bad && status) raise_status(status, DEV_ERR_FACTOR);
}

// grid (blocks below J, matrices), CF_THREADS threads
__global__ void __launch_bounds__(CF_THREADS) chol_step_panel_kernel(double* G, int k, long long gld, long long sG,
                                                                     int J) {
  __shared__ double As[CF_NB][CF_P];
  __shared__ double Wi[CF_NB][CF_P];
  const int tid = threadIdx.x;
  double* Gu = G + (long long)blockIdx.y * sG;
  const int J0 = J * CF_NB, nbJ = min(CF_NB, k - J0);
  const int I = J + 1 + blockIdx.x, I0 = I * CF_NB, nbI = min(CF_NB, k - I0);
  auto at = [&](int r, int c) -> double& { return Gu[(long long)c * gld + r]; };
  for (int idx = tid; idx < CF_NB * CF_NB; idx += blockDim.x) {
    const int r = idx % CF_NB, c = idx / CF_NB;
    As[r][c] = (r < nbI && c < nbJ) ? at(I0 + r, J0 + c) : 0.0;
    // inv(L_JJ)[c][r] sits at row J0 + r, column J0 + c (r <= c)
    Wi[c][r] = (r <= c && c < nbJ) ? at(J0 + r, J0 + c) : 0.0;
  }
  __syncthreads();
  // L_IJ[r][c] = sum_s A_IJ[r][s] inv(L_JJ)[c][s]  (s <= c)
  const int r = tid & 31, cg0 = tid >> 5;   // row r, columns cg0 + 8 jj (coalesced writes)
#pragma unroll
  for (int jj = 0; jj < 4; ++jj) {
    const int c = cg0 + 8 * jj;
    double acc = 0.0;
    for (int s2 = 0; s2 <= c; ++s2) acc = fma(As[r][s2], Wi[c][s2], acc);
    if (r < nbI && c < nbJ) at(I0 + r, J0 + c) = acc;
  }
}

// grid (block pairs (I, K) with J < K <= I < nbk, matrices), CF_THREADS threads
__global__ void __launch_bounds__(CF_THREADS) chol_step_update_kernel(double* G, int k, long long gld, long long sG,
                                                                      int J) {
  __shared__ double Li[CF_NB][CF_P];
  __shared__ double Lk[CF_NB][CF_P];
  const int tid = threadIdx.x;
  double* Gu = G + (long long)blockIdx.y * sG;
  const int J0 = J * CF_NB, nbJ = min(CF_NB, k - J0);
  // pair index -> (i, kk) with 0 <= kk <= i: row-major lower triangle
  const int idx = blockIdx.x;
  int i = (int)((sqrt(8.0 * idx + 1.0) - 1.0) * 0.5);
  while ((i + 1) * (i + 2) / 2 <= idx) ++i;
  while (i * (i + 1) / 2 > idx) --i;
  const int kk = idx - i * (i + 1) / 2;
  const int I = J + 1 + i, K = J + 1 + kk;
  const int I0 = I * CF_NB, K0 = K * CF_NB, nbI = min(CF_NB, k - I0), nbK = min(CF_NB, k - K0);
  auto at = [&](int r, int c) -> double& { return Gu[(long long)c * gld + r]; };
  for (int e = tid; e < CF_NB * CF_NB; e += blockDim.x) {
    const int r = e % CF_NB, c = e / CF_NB;
    Li[r][c] = (r < nbI && c < nbJ) ? at(I0 + r, J0 + c) : 0.0;
    Lk[r][c] = (r < nbK && c < nbJ) ? at(K0 + r, J0 + c) : 0.0;
  }
  const int r = tid & 31, cg0 = tid >> 5;
  double aold[4];
#pragma unroll
  for (int jj = 0; jj < 4; ++jj) {
    const int c = cg0 + 8 * jj;
    aold[jj] = (r < nbI && c < nbK) ? at(I0 + r, K0 + c) : 0.0;
  }
  __syncthreads();
#pragma unroll
  for (int jj = 0; jj < 4; ++jj) {
    const int c = cg0 + 8 * jj;
    double acc = 0.0;
#pragma unroll 8
    for (int s2 = 0; s2 < CF_NB; ++s2) acc = fma(Li[r][s2], Lk[c][s2], acc);
    if (r < nbI && c < nbK) at(I0 + r, K0 + c) = aold[jj] - acc;
  }
}
}  // namespace jolt
