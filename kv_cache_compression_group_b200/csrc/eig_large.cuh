// Symmetric eigen-decomposition of batched fp64 matrices of order 256 < n <= 1024 (the
// FlashJoLT Rayleigh-Ritz step at sketch widths above 256, the exact token factor up to 1024
// tokens).  The same algorithm as the cluster solver of eig_cluster.cuh -- Householder
// tridiagonalisation, multisection on Sturm counts, inverse iteration, the back-transformation
// -- with the matrix in global memory (it does not fit the shared memory of a cluster):
//   1. tridiag_gm_kernel: one cluster of 8 CTAs of 1024 threads per matrix; CTA q owns the
//      columns c with c % 8 == q (contiguous in the column-major matrix).  Per column j: the
//      owner forms the reflector and writes it into every CTA's shared memory (distributed
//      shared memory) and to global memory; every CTA computes p = beta A v on its columns
//      (one warp per column), applying the previous step's rank-2 update to the column in the
//      same pass, and sends p and its warps' partial p.v to all.  Two cluster barriers per
//      column; vectors alternate between two buffers (as in eig_cluster.cuh).
//   2. tri_eig_kernel: 128 eigenvalues per CTA by multisection (8 threads each), then their
//      eigenvectors of T by inverse iteration (one thread each, the factors in global memory).
//   3. tight_mgs_kernel: vectors of eigenvalues closer than 1e-10 ||T|| orthonormalised in
//      order by one warp (they span their cluster's invariant subspace).
//   4. wy_tfactor_kernel, wy_apply_kernel: V = H_0 ... H_{n-3} Z with the reflectors taken 32 at
//      a time in compact WY form (I - Y T Y^T), 16 eigenvectors per CTA in shared memory.
// Output as the cluster solver: w ascending; V[r * n + i] = component r of eigenvector i.
// Non-finite input raises DEV_ERR_NONFINITE (the matrices are sanitised before, so the
// arithmetic stays finite).  Every thread of every CTA of a cluster passes the same cluster
// barriers.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"
#include "eig_cluster.cuh"

namespace jolt {
namespace eigl {
namespace cg = cooperative_groups;
constexpr int CL = 8;             // CTAs per matrix in the tridiagonalisation
constexpr int MAXN = 1024;
constexpr int THREADS = 256;
constexpr int WARPS = THREADS / 32;
// the tridiagonalisation runs 1024 threads per CTA: one warp per column in the matrix-vector
// product and the update, so that many loads of the (L2-resident) matrix are in flight
constexpr int TRI_THREADS = 1024;
constexpr int TRI_WARPS = TRI_THREADS / 32;
constexpr int TRED = CL * TRI_WARPS;   // partial sums of p.v: one per warp of the cluster
// tridiagonalisation shared memory (doubles): v[2][MAXN] | p[2][MAXN] | red[2][TRED] | beta[2] | tmp[TRI_WARPS]
constexpr size_t TRI_SMEM = sizeof(double) * (4 * (size_t)MAXN + 2 * TRED + 2 + TRI_WARPS);
// per matrix global scratch (doubles): reflectors n*n | LU factors 5*n*n | d, e, beta 3*n
__host__ __device__ inline size_t scratch_doubles(int n) { return (size_t)6 * n * n + 3 * (size_t)n; }
constexpr int EV_PER_CTA = 128;   // eigenvalues / eigenvectors per CTA of tri_eig_kernel
// back-transformation in blocks of WY_NB reflectors (compact WY form I - Y T Y^T)
constexpr int WY_NB = 32;
constexpr int WY_COLS = 16;       // eigenvectors per CTA
constexpr int WY_ROWS = 128;      // rows of Y staged together
constexpr int WY_THREADS = 256;
}  // namespace eigl

__device__ __forceinline__ double eigl_block_sum(double v, double* tmp) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = eigc::warp_sum(v);
  __syncthreads();
  if (lane == 0) tmp[warp] = v;
  __syncthreads();
  double s = 0.0;
  for (int i = 0; i < (int)(blockDim.x >> 5); ++i) s += tmp[i];
  __syncthreads();
  return s;
}

// copy the lower triangle of every column-major matrix onto its upper triangle
__global__ void symmetrize_lower_kernel(double* A, int n, long long sA) {
  double* M = A + (long long)blockIdx.y * sA;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < (long long)n * n;
       idx += (long long)gridDim.x * blockDim.x) {
    const int c = (int)(idx / n), r = (int)(idx - (long long)c * n);
    if (r < c) M[idx] = M[(long long)r * n + c];   // (r, c) above the diagonal <- (c, r)
  }
}

// grid (8 * matrices), clusters of 8, eigl::TRI_THREADS threads, eigl::TRI_SMEM dynamic shared
// memory.  A: n x n symmetric, column-major (both triangles), stride sA, overwritten.
//
// Look-ahead order: the rank-2 update of step j - 1, A -= v w^T + w v^T, is not applied in a
// pass of its own; at step j the owner of column j first applies it to that column and forms
// the reflector v_j from it, and then every CTA applies it to each of its columns c > j in the
// same pass over the column that forms p_c = beta_j (column c) . v_j.  One read and one write
// of the trailing matrix per step, two cluster barriers.
__global__ void __cluster_dims__(eigl::CL, 1, 1) __launch_bounds__(eigl::TRI_THREADS)
    tridiag_gm_kernel(double* A, int n, long long sA, double* scr) {
  using namespace eigl;
  cg::cluster_group cluster = cg::this_cluster();
  const int q = (int)cluster.block_rank();
  const int u = blockIdx.x / CL;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  extern __shared__ double tg_sm[];
  double* vb = tg_sm;                     // [2][MAXN] reflectors v_j (by the parity of j)
  double* pb = vb + 2 * MAXN;             // [2][MAXN] p_j
  double* red = pb + 2 * MAXN;            // [2][TRED]
  double* sbeta = red + 2 * TRED;         // [2]
  double* tmp = sbeta + 2;                // [TRI_WARPS]
  double* Au = A + (long long)u * sA;
  double* base = scr + (long long)u * scratch_doubles(n);
  double* refl = base;                    // [n][n]
  double* dg = base + 6 * (long long)n * n;
  double* eg = dg + n;
  double* bg = eg + n;
  for (int i = tid; i < 4 * MAXN; i += blockDim.x) tg_sm[i] = 0.0;
  cluster.sync();
  double Kp = 0.0;   // K of the previous step (the same in every thread)
  for (int j = 0; j + 2 < n; ++j) {
    const int cur = j & 1, prv = cur ^ 1;
    const double* vp = vb + prv * MAXN;   // v_{j-1} (zero at j = 0)
    const double* pp = pb + prv * MAXN;   // p_{j-1} (zero at j = 0)
    if (j % CL == q) {
      // column j brought up to date (update j - 1 on rows >= j), then its reflector
      double* col = Au + (long long)j * n;
      if (j > 0) {
        const double vj = vp[j], wj = fma(-Kp, vj, pp[j]);
        for (int r = j + tid; r < n; r += blockDim.x) col[r] = col[r] - (vp[r] * wj + fma(-Kp, vp[r], pp[r]) * vj);
        __syncthreads();
      }
      double part = 0.0;
      for (int r = j + 2 + tid; r < n; r += blockDim.x) part = fma(col[r], col[r], part);
      const double tail2 = eigl_block_sum(part, tmp);
      const double x0 = col[j + 1];
      double beta = 0.0, alpha = x0;
      if (tail2 > 0.0) {
        const double nrm = sqrt(fma(x0, x0, tail2));
        alpha = x0 > 0.0 ? -nrm : nrm;
        const double v0 = x0 - alpha;
        beta = 2.0 / fma(v0, v0, tail2);
      }
      for (int r = tid; r < MAXN; r += blockDim.x) {
        const double v = (r <= j || r >= n) ? 0.0 : (r == j + 1 ? x0 - alpha : col[r]);
        for (int t = 0; t < CL; ++t) cluster.map_shared_rank(vb, t)[cur * MAXN + r] = v;
        if (r < n) refl[(long long)j * n + r] = v;
      }
      if (tid == 0) {
        for (int t = 0; t < CL; ++t) cluster.map_shared_rank(sbeta, t)[cur] = beta;
        dg[j] = col[j];
        eg[j] = alpha;
        bg[j] = beta;
      }
    }
    cluster.sync();   // (A) v_j and beta_j everywhere
    const double beta = sbeta[cur];
    const double* v = vb + cur * MAXN;
    // my first column after j (the columns c with c % CL == q), then every CL-th; warp w takes
    // the columns cf + CL (w + TRI_WARPS i); one warp per column, lanes over rows
    const int cf = j + 1 + ((q - (j + 1)) % CL + CL) % CL;
    double pv = 0.0;
    for (int c = cf + CL * warp; c < n; c += CL * TRI_WARPS) {
      double* col = Au + (long long)c * n;
      const double vc = vp[c], wc = fma(-Kp, vc, pp[c]);
      double s0 = 0.0, s1 = 0.0, s2 = 0.0, s3 = 0.0;
      int r = j + 1 + lane;
      if (j > 0) {
        for (; r + 96 < n; r += 128) {
          const double a0 = col[r], a1 = col[r + 32], a2 = col[r + 64], a3 = col[r + 96];
          const double b0 = a0 - (vp[r] * wc + fma(-Kp, vp[r], pp[r]) * vc);
          const double b1 = a1 - (vp[r + 32] * wc + fma(-Kp, vp[r + 32], pp[r + 32]) * vc);
          const double b2 = a2 - (vp[r + 64] * wc + fma(-Kp, vp[r + 64], pp[r + 64]) * vc);
          const double b3 = a3 - (vp[r + 96] * wc + fma(-Kp, vp[r + 96], pp[r + 96]) * vc);
          col[r] = b0;
          col[r + 32] = b1;
          col[r + 64] = b2;
          col[r + 96] = b3;
          s0 = fma(b0, v[r], s0);
          s1 = fma(b1, v[r + 32], s1);
          s2 = fma(b2, v[r + 64], s2);
          s3 = fma(b3, v[r + 96], s3);
        }
        for (; r < n; r += 32) {
          const double b0 = col[r] - (vp[r] * wc + fma(-Kp, vp[r], pp[r]) * vc);
          col[r] = b0;
          s0 = fma(b0, v[r], s0);
        }
      } else {
        for (; r + 96 < n; r += 128) {
          s0 = fma(col[r], v[r], s0);
          s1 = fma(col[r + 32], v[r + 32], s1);
          s2 = fma(col[r + 64], v[r + 64], s2);
          s3 = fma(col[r + 96], v[r + 96], s3);
        }
        for (; r < n; r += 32) s0 = fma(col[r], v[r], s0);
      }
      const double pc = beta * eigc::warp_sum((s0 + s1) + (s2 + s3));
      if (lane < CL) cluster.map_shared_rank(pb, lane)[cur * MAXN + c] = pc;
      pv = fma(pc, v[c], pv);   // the same on every lane
    }
    if (lane < CL) cluster.map_shared_rank(red, lane)[cur * TRED + q * TRI_WARPS + warp] = pv;
    cluster.sync();   // (B) p_j and the partial sums of p_j . v_j everywhere
    // K_j = beta_j p_j . v_j / 2, summed in the same order in every warp of every CTA
    double ptv = 0.0;
#pragma unroll
    for (int t = 0; t < TRED / 32; ++t) ptv += red[cur * TRED + lane * (TRED / 32) + t];
    Kp = 0.5 * beta * eigc::warp_sum(ptv);
  }
  // the last update on the last two columns, then the last 2 x 2 block of T
  {
    const int jl = n - 3, cur = jl & 1;
    const double* vp = vb + cur * MAXN;
    const double* pp = pb + cur * MAXN;
    for (int c = n - 2; c < n; ++c) {
      if (c % CL != q) continue;
      double* col = Au + (long long)c * n;
      const double vc = vp[c], wc = fma(-Kp, vc, pp[c]);
      for (int r = n - 2 + tid; r < n; r += blockDim.x) col[r] = col[r] - (vp[r] * wc + fma(-Kp, vp[r], pp[r]) * vc);
    }
    __syncthreads();
  }
  if (tid == 0) {
    const int c2 = n - 2, c1 = n - 1;
    if (c2 % CL == q) {
      dg[c2] = Au[(long long)c2 * n + c2];
      eg[c2] = Au[(long long)c2 * n + c1];
      bg[c2] = 0.0;
    }
    if (c1 % CL == q) {
      dg[c1] = Au[(long long)c1 * n + c1];
      eg[c1] = 0.0;
      bg[c1] = 0.0;
    }
  }
}

// grid (ceil(n / 128), matrices), eigl::THREADS threads.  Eigenvalues i in [128 bx, 128 bx + 128)
// by multisection, then their eigenvectors of T by inverse iteration into V (row-major).
__global__ void __launch_bounds__(eigl::THREADS) tri_eig_kernel(int n, double* w, long long sw, double* V,
                                                                double* scr) {
  using namespace eigl;
  __shared__ double sd[MAXN], se[MAXN], e2[MAXN];
  const int u = blockIdx.y, tid = threadIdx.x;
  double* base = scr + (long long)u * scratch_doubles(n);
  double* U0 = base + (long long)n * n;
  double* U1 = U0 + (long long)n * n;
  double* U2 = U1 + (long long)n * n;
  double* Lm = U2 + (long long)n * n;
  double* Pv = Lm + (long long)n * n;
  const double* dg = base + 6 * (long long)n * n;
  const double* eg = dg + n;
  double* wu = w + (long long)u * sw;
  double* Vu = V + (long long)u * n * n;
  for (int k = tid; k < n; k += blockDim.x) {
    sd[k] = dg[k];
    se[k] = k < n - 1 ? eg[k] : 0.0;
    e2[k] = k < n - 1 ? eg[k] * eg[k] : 0.0;
  }
  __syncthreads();
  double glo = INFINITY, ghi = -INFINITY, e2max = 0.0;
  for (int k = 0; k < n; ++k) {
    const double rad = (k + 1 < n ? fabs(se[k]) : 0.0) + (k ? fabs(se[k - 1]) : 0.0);
    glo = fmin(glo, sd[k] - rad);
    ghi = fmax(ghi, sd[k] + rad);
    e2max = fmax(e2max, e2[k]);
  }
  const double pivmin = 2.2250738585072014e-308 * fmax(1.0, e2max);
  const int i0 = blockIdx.x * EV_PER_CTA;
  __shared__ double wl[EV_PER_CTA];
  constexpr int SUB = 8;
  for (int pass = 0; pass < EV_PER_CTA / (THREADS / SUB); ++pass) {
    const int i = i0 + pass * (THREADS / SUB) + tid / SUB, sub = tid % SUB;
    const int gbase = (tid & 31) & ~(SUB - 1);
    double a = glo, b = ghi;
    for (int it = 0; it < 24; ++it) {
      const bool done = b - a <= 2.220446049250313e-16 * fmax(fabs(a), fabs(b)) + pivmin;
      if (__all_sync(0xffffffffu, done)) break;
      const double x = a + (b - a) * (double)(sub + 1) / (double)(SUB + 1);
      const int cnt = (i < n && !done) ? eigc::sturm_count(sd, e2, n, x, pivmin) : 0;
      double na = a, nb = b;
#pragma unroll
      for (int s2 = 0; s2 < SUB; ++s2) {
        const double xs = __shfl_sync(0xffffffffu, x, gbase + s2);
        const int cs = __shfl_sync(0xffffffffu, cnt, gbase + s2);
        if (cs <= i) na = fmax(na, xs);
        else nb = fmin(nb, xs);
      }
      if (!done) {
        a = na;
        b = nb;
      }
    }
    if (sub == 0 && i < n) {
      wu[i] = 0.5 * (a + b);
      wl[i - i0] = 0.5 * (a + b);
    }
  }
  __syncthreads();
  // the tolerance of the inverse iteration from the spectrum's ends
  const double norm = fmax(fabs(glo), fabs(ghi));
  const double tiny = 2.220446049250313e-16 * fmax(norm, 2.2250738585072014e-308);
  if (tid < EV_PER_CTA && i0 + tid < n) {
    const int i = i0 + tid;
    eigc::tri_lu(sd, se, n, wl[tid], tiny, U0, U1, U2, Lm, Pv, i);
    for (int k = 0; k < n; ++k) Vu[(long long)k * n + i] = eigc::start_value(i, k);
    for (int it = 0; it < 2; ++it) eigc::tri_solve_normalise(U0, U1, U2, Lm, Pv, n, Vu, i);
  }
}

// one warp per matrix: eigenvalues closer than 1e-10 ||T|| -- their vectors orthonormalised in
// order (modified Gram-Schmidt)
__global__ void tight_mgs_kernel(int n, const double* w, long long sw, double* V) {
  const int u = blockIdx.x, lane = threadIdx.x;
  const double* wu = w + (long long)u * sw;
  double* Vu = V + (long long)u * n * n;
  const double norm = fmax(fabs(wu[0]), fabs(wu[n - 1]));
  const double ctol = 1e-10 * norm;
  int cs0 = 0;
  double wprev = wu[0];
  for (int i = 1; i < n; ++i) {
    const double wi = wu[i];
    const bool tight = wi - wprev < ctol;
    wprev = wi;
    if (!tight) {
      cs0 = i;
      continue;
    }
    for (int jj = cs0; jj < i; ++jj) {
      double dot = 0.0;
      for (int k = lane; k < n; k += 32) dot = fma(Vu[(long long)k * n + jj], Vu[(long long)k * n + i], dot);
      dot = eigc::warp_sum(dot);
      for (int k = lane; k < n; k += 32) Vu[(long long)k * n + i] = fma(-dot, Vu[(long long)k * n + jj], Vu[(long long)k * n + i]);
      __syncwarp();
    }
    double nrm = 0.0;
    for (int k = lane; k < n; k += 32) nrm = fma(Vu[(long long)k * n + i], Vu[(long long)k * n + i], nrm);
    nrm = eigc::warp_sum(nrm);
    const double inv = nrm > 0.0 ? 1.0 / sqrt(nrm) : 0.0;
    for (int k = lane; k < n; k += 32) Vu[(long long)k * n + i] *= inv;
    __syncwarp();
  }
}

// ---- back-transformation V = H_0 H_1 ... H_{n-3} Z in blocks of 32 reflectors ----
// The product of the reflectors j0 .. j0 + jn - 1 of a block is I - Y T Y^T (Y = [v_j0 ..], T
// upper triangular: T_ii = beta_i, T[0:i, i] = -beta_i T[0:i, 0:i] Y[:, 0:i]^T v_i, the forward
// accumulation of Schreiber and Van Loan's compact WY form).  V = P_0 (P_1 (... (P_last Z))).
// T of block b goes to the scratch area of the inverse-iteration factors (free by then).
inline __host__ __device__ int wy_blocks(int n) { return (n - 2 + eigl::WY_NB - 1) / eigl::WY_NB; }

// grid (wy_blocks(n), matrices), eigl::WY_THREADS threads
__global__ void __launch_bounds__(eigl::WY_THREADS) wy_tfactor_kernel(int n, double* scr) {
  using namespace eigl;
  constexpr int TF_ROWS = 64;   // rows of Y staged together (static shared memory stays under 48 KB)
  __shared__ double Yc[TF_ROWS][WY_NB + 1];
  __shared__ double Ss[WY_NB][WY_NB + 1];
  __shared__ double Ts[WY_NB][WY_NB + 1];
  const int u = blockIdx.y, b = blockIdx.x, tid = threadIdx.x;
  double* base = scr + (long long)u * scratch_doubles(n);
  const double* refl = base;
  const double* bg = base + 6 * (long long)n * n + 2 * (long long)n;
  double* Tg = base + (long long)n * n + (long long)b * WY_NB * WY_NB;
  const int j0 = b * WY_NB, jn = min(WY_NB, n - 2 - j0), r0 = j0 + 1;
  // S = Y^T Y: thread (i, mg) accumulates S[i][mg + 8 k]
  const int i = tid >> 3, mg = tid & 7;
  double sacc[4] = {0.0, 0.0, 0.0, 0.0};
  for (int rc = r0; rc < n; rc += TF_ROWS) {
    const int nr = min(TF_ROWS, n - rc);
    __syncthreads();
    for (int idx = tid; idx < WY_NB * TF_ROWS; idx += blockDim.x) {
      const int ii = idx / TF_ROWS, rr = idx - ii * TF_ROWS;
      Yc[rr][ii] = (ii < jn && rr < nr) ? refl[(long long)(j0 + ii) * n + rc + rr] : 0.0;
    }
    __syncthreads();
    for (int rr = 0; rr < nr; ++rr) {
      const double y = Yc[rr][i];
#pragma unroll
      for (int k = 0; k < 4; ++k) sacc[k] = fma(y, Yc[rr][mg + 8 * k], sacc[k]);
    }
  }
#pragma unroll
  for (int k = 0; k < 4; ++k) Ss[i][mg + 8 * k] = sacc[k];
  __syncthreads();
  if (tid < 32) {
    // T column by column; lane l owns row l (and reads only its own row of T)
    const int l = tid;
    for (int c = 0; c < WY_NB; ++c) {
      double t = 0.0;
      if (c < jn) {
        const double tau = bg[j0 + c];
        if (l < c) {
          double acc = 0.0;
          for (int m = l; m < c; ++m) acc = fma(Ts[l][m], Ss[m][c], acc);
          t = -tau * acc;
        } else if (l == c) {
          t = tau;
        }
      }
      Ts[l][c] = t;
    }
  }
  __syncthreads();
  for (int idx = tid; idx < WY_NB * WY_NB; idx += blockDim.x) Tg[idx] = Ts[idx / WY_NB][idx % WY_NB];
}

inline size_t wy_apply_smem(int n) {
  using namespace eigl;
  return sizeof(double) * ((size_t)n * WY_COLS + (size_t)WY_ROWS * (WY_NB + 1) + WY_NB * WY_COLS +
                           WY_NB * (WY_NB + 1));
}

// grid (ceil(n / 16), matrices), eigl::WY_THREADS threads, wy_apply_smem(n) bytes of dynamic
// shared memory.  Z (16 eigenvectors of T) in shared memory; for every block from the last:
// W = Y^T Z, W = T W, Z -= Y W, with Y staged 128 rows at a time.
__global__ void __launch_bounds__(eigl::WY_THREADS) wy_apply_kernel(int n, double* V, const double* scr) {
  using namespace eigl;
  extern __shared__ double wy_sm[];
  double* Z = wy_sm;                                                  // [n][WY_COLS]
  double(*Yc)[WY_NB + 1] = reinterpret_cast<double(*)[WY_NB + 1]>(Z + (size_t)n * WY_COLS);   // [WY_ROWS]
  double* Wb = reinterpret_cast<double*>(Yc + WY_ROWS);               // [WY_NB][WY_COLS]
  double* Tb = Wb + WY_NB * WY_COLS;                                  // [WY_NB][WY_NB + 1]
  const int u = blockIdx.y, c0 = blockIdx.x * WY_COLS, tid = threadIdx.x;
  const double* base = scr + (long long)u * scratch_doubles(n);
  const double* refl = base;
  double* Vu = V + (long long)u * n * n;
  for (int idx = tid; idx < n * WY_COLS; idx += blockDim.x) {
    const int r = idx / WY_COLS, c = idx - r * WY_COLS;
    Z[idx] = c0 + c < n ? Vu[(long long)r * n + c0 + c] : 0.0;
  }
  const int iw = tid >> 3, cp = (tid & 7) * 2;     // W phase: row iw of W, columns cp, cp + 1
  const int cu = tid & 15, rg = tid >> 4;          // update phase: column cu, rows rg + 16 k
  auto load_y = [&](int j0, int jn, int rc, int nr) {
    __syncthreads();
    for (int idx = tid; idx < WY_NB * WY_ROWS; idx += blockDim.x) {
      const int ii = idx / WY_ROWS, rr = idx - ii * WY_ROWS;
      Yc[rr][ii] = (ii < jn && rr < nr) ? refl[(long long)(j0 + ii) * n + rc + rr] : 0.0;
    }
    __syncthreads();
  };
  for (int b = wy_blocks(n) - 1; b >= 0; --b) {
    const int j0 = b * WY_NB, jn = min(WY_NB, n - 2 - j0), r0 = j0 + 1;
    const double* Tg = base + (long long)n * n + (long long)b * WY_NB * WY_NB;
    for (int idx = tid; idx < WY_NB * WY_NB; idx += blockDim.x) Tb[(idx / WY_NB) * (WY_NB + 1) + idx % WY_NB] = Tg[idx];
    // W = Y^T Z
    double w0 = 0.0, w1 = 0.0;
    for (int rc = r0; rc < n; rc += WY_ROWS) {
      const int nr = min(WY_ROWS, n - rc);
      load_y(j0, jn, rc, nr);
      for (int rr = 0; rr < nr; ++rr) {
        const double y = Yc[rr][iw];
        const double2 z = *reinterpret_cast<const double2*>(Z + (size_t)(rc + rr) * WY_COLS + cp);
        w0 = fma(y, z.x, w0);
        w1 = fma(y, z.y, w1);
      }
    }
    Wb[iw * WY_COLS + cp] = w0;
    Wb[iw * WY_COLS + cp + 1] = w1;
    __syncthreads();
    // W = T W (T upper triangular)
    double a0 = 0.0, a1 = 0.0;
    for (int m = iw; m < WY_NB; ++m) {
      const double t = Tb[iw * (WY_NB + 1) + m];
      a0 = fma(t, Wb[m * WY_COLS + cp], a0);
      a1 = fma(t, Wb[m * WY_COLS + cp + 1], a1);
    }
    __syncthreads();
    Wb[iw * WY_COLS + cp] = a0;
    Wb[iw * WY_COLS + cp + 1] = a1;
    __syncthreads();
    double wc[WY_NB];
#pragma unroll
    for (int m = 0; m < WY_NB; ++m) wc[m] = Wb[m * WY_COLS + cu];
    // Z -= Y W
    for (int rc = r0; rc < n; rc += WY_ROWS) {
      const int nr = min(WY_ROWS, n - rc);
      load_y(j0, jn, rc, nr);
#pragma unroll 2
      for (int k = 0; k < WY_ROWS / 16; ++k) {
        const int rr = rg + 16 * k;
        if (rr < nr) {
          double acc = 0.0;
#pragma unroll
          for (int m = 0; m < WY_NB; ++m) acc = fma(Yc[rr][m], wc[m], acc);
          Z[(size_t)(rc + rr) * WY_COLS + cu] -= acc;
        }
      }
    }
    __syncthreads();
  }
  __syncthreads();
  for (int idx = tid; idx < n * WY_COLS; idx += blockDim.x) {
    const int r = idx / WY_COLS, c = idx - r * WY_COLS;
    if (c0 + c < n) Vu[(long long)r * n + c0 + c] = Z[idx];
  }
}

}  // namespace jolt
