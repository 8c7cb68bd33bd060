// Symmetric eigen-decomposition of batched fp64 matrices of order 256 < n <= 1024 (the
// FlashJoLT Rayleigh-Ritz step at sketch widths above 256, the exact token factor up to 1024
// tokens).  The same algorithm as the cluster solver of eig_cluster.cuh -- Householder
// tridiagonalisation, multisection on Sturm counts, inverse iteration, the back-transformation
// -- with the matrix in global memory (it does not fit the shared memory of a cluster):
//   1. tridiag_gm_kernel: one cluster of 8 CTAs per matrix; CTA q owns the columns c with
//      c % 8 == q (contiguous in the column-major matrix).  Per column j: the owner forms the
//      reflector and writes it into every CTA's shared memory (distributed shared memory) and
//      to global memory; every CTA computes p = beta A v on its columns and sends p and its
//      partial p.v to all; every CTA applies the rank-2 update to its columns.  Two cluster
//      barriers per column; vectors alternate between two buffers (as in eig_cluster.cuh).
//   2. tri_eig_kernel: 128 eigenvalues per CTA by multisection (8 threads each), then their
//      eigenvectors of T by inverse iteration (one thread each, the factors in global memory).
//   3. tight_mgs_kernel: vectors of eigenvalues closer than 1e-10 ||T|| orthonormalised in
//      order by one warp (they span their cluster's invariant subspace).
//   4. backtransform_kernel: V = H_0 ... H_{n-3} Z on 16 eigenvectors per CTA, the vectors in
//      shared memory, the reflectors staged 8 at a time, one warp per two vectors.
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
constexpr int RED = CL * WARPS;
// tridiagonalisation shared memory (doubles): v[2][MAXN] | p[2][MAXN] | red[2][RED] | beta[2] | tmp[THREADS]
constexpr size_t TRI_SMEM = sizeof(double) * (4 * (size_t)MAXN + 2 * RED + 2 + THREADS);
// per matrix global scratch (doubles): reflectors n*n | LU factors 5*n*n | d, e, beta 3*n
__host__ __device__ inline size_t scratch_doubles(int n) { return (size_t)6 * n * n + 3 * (size_t)n; }
constexpr int EV_PER_CTA = 128;   // eigenvalues / eigenvectors per CTA of tri_eig_kernel
constexpr int BT_COLS = 16;       // eigenvectors per CTA of the back-transformation
constexpr int BT_REFL = 8;        // reflectors staged together
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

// grid (8 * matrices), clusters of 8, eigl::THREADS threads, eigl::TRI_SMEM dynamic shared
// memory.  A: n x n symmetric, column-major (both triangles), stride sA, overwritten.
__global__ void __cluster_dims__(eigl::CL, 1, 1) __launch_bounds__(eigl::THREADS)
    tridiag_gm_kernel(double* A, int n, long long sA, double* scr) {
  using namespace eigl;
  cg::cluster_group cluster = cg::this_cluster();
  const int q = (int)cluster.block_rank();
  const int u = blockIdx.x / CL;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  extern __shared__ double tg_sm[];
  double* vb = tg_sm;                     // [2][MAXN]
  double* pb = vb + 2 * MAXN;             // [2][MAXN]
  double* red = pb + 2 * MAXN;            // [2][RED]
  double* sbeta = red + 2 * RED;          // [2]
  double* tmp = sbeta + 2;                // [THREADS]
  double* Au = A + (long long)u * sA;
  double* base = scr + (long long)u * scratch_doubles(n);
  double* refl = base;                    // [n][n]
  double* dg = base + 6 * (long long)n * n;
  double* eg = dg + n;
  double* bg = eg + n;
  for (int i = tid; i < 4 * MAXN; i += blockDim.x) tg_sm[i] = 0.0;
  cluster.sync();
  for (int j = 0; j + 2 < n; ++j) {
    const int buf = j & 1;
    if (j % CL == q) {
      // the reflector of column j (rows j+1 .. n-1); every thread takes part in the sums
      const double* col = Au + (long long)j * n;
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
        for (int t = 0; t < CL; ++t) cluster.map_shared_rank(vb, t)[buf * MAXN + r] = v;
        if (r < n) refl[(long long)j * n + r] = v;
      }
      if (tid == 0) {
        for (int t = 0; t < CL; ++t) cluster.map_shared_rank(sbeta, t)[buf] = beta;
        dg[j] = col[j];
        eg[j] = alpha;
        bg[j] = beta;
      }
    }
    cluster.sync();   // (A) v and beta everywhere
    const double beta = sbeta[buf];
    const double* v = vb + buf * MAXN;
    if (beta != 0.0) {
      // p_c = beta * (column c) . v on my columns c > j: 8 threads per column
      double pv = 0.0;
      const int part = tid & 7;
      // the same trip count on every lane (the shuffles below take the whole warp)
      const int iters = (n + CL * (THREADS / 8) - 1) / (CL * (THREADS / 8));
      for (int it = 0; it < iters; ++it) {
        const int c = q + CL * (tid >> 3) + CL * (THREADS / 8) * it;
        double s = 0.0;
        if (c > j && c < n) {
          const double* col = Au + (long long)c * n;
          for (int r = j + 1 + part; r < n; r += 8) s = fma(col[r], v[r], s);
        }
#pragma unroll
        for (int o = 4; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (part == 0 && c > j && c < n) {
          const double pc = beta * s;
          for (int t = 0; t < CL; ++t) cluster.map_shared_rank(pb, t)[buf * MAXN + c] = pc;
          pv = fma(pc, v[c], pv);
        }
      }
      pv = eigc::warp_sum(pv);
      if (lane == 0)
        for (int t = 0; t < CL; ++t) cluster.map_shared_rank(red, t)[buf * RED + q * WARPS + warp] = pv;
    }
    cluster.sync();   // (B) p and the partial sums of p.v everywhere
    if (beta != 0.0) {
      double ptv = 0.0;
      for (int t = 0; t < RED; ++t) ptv += red[buf * RED + t];
      const double K = 0.5 * beta * ptv;
      const double* pf = pb + buf * MAXN;
      // A -= v w^T + w v^T on my columns, w = p - K v; one warp per column, lanes over rows
      for (int c = q + CL * warp; c < n; c += CL * WARPS) {
        if (c <= j) continue;
        double* col = Au + (long long)c * n;
        const double vc = v[c], wc = fma(-K, vc, pf[c]);
        for (int r = j + 1 + lane; r < n; r += 32) col[r] = col[r] - (v[r] * wc + fma(-K, v[r], pf[r]) * vc);
      }
    }
    __syncthreads();
  }
  // the last 2 x 2 block of T
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

// grid (ceil(n / 16), matrices), eigl::THREADS threads, dynamic shared memory backtransform_smem(n).
// Z (16 eigenvectors of T) staged in shared memory; H_{n-3} .. H_0 applied in turn, 8
// reflectors staged together; warp w updates vectors 2w and 2w + 1, lanes over rows.
inline size_t backtransform_smem(int n) {
  return sizeof(double) * ((size_t)n * eigl::BT_COLS + (size_t)eigl::BT_REFL * n);
}
__global__ void __launch_bounds__(eigl::THREADS) backtransform_kernel(int n, double* V, const double* scr) {
  using namespace eigl;
  extern __shared__ double bt_sm[];
  double* Z = bt_sm;                      // [n][BT_COLS]
  double* R = Z + (size_t)n * BT_COLS;    // [BT_REFL][n]
  const int u = blockIdx.y, c0 = blockIdx.x * BT_COLS, tid = threadIdx.x;
  const int lane = tid & 31, warp = tid >> 5;
  const double* base = scr + (long long)u * scratch_doubles(n);
  const double* refl = base;
  const double* bg = base + 6 * (long long)n * n + 2 * (long long)n;
  double* Vu = V + (long long)u * n * n;
  for (int idx = tid; idx < n * BT_COLS; idx += blockDim.x) {
    const int r = idx / BT_COLS, c = idx - r * BT_COLS;
    Z[idx] = c0 + c < n ? Vu[(long long)r * n + c0 + c] : 0.0;
  }
  for (int jh = n - 3; jh >= 0; jh -= BT_REFL) {
    const int jl = jh - BT_REFL + 1 > 0 ? jh - BT_REFL + 1 : 0;   // reflectors jh, jh-1, .., jl
    __syncthreads();
    for (int idx = tid; idx < (jh - jl + 1) * n; idx += blockDim.x) {
      const int k = idx / n, r = idx - k * n;
      R[k * n + r] = refl[(long long)(jh - k) * n + r];
    }
    __syncthreads();
    for (int k = 0; k <= jh - jl; ++k) {
      const int j = jh - k;
      const double bj = bg[j];
      const double* v = R + k * n;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        const int c = 2 * warp + cc;
        double s = 0.0;
        for (int r = j + 1 + lane; r < n; r += 32) s = fma(v[r], Z[r * BT_COLS + c], s);
        s = eigc::warp_sum(s) * bj;
        for (int r = j + 1 + lane; r < n; r += 32) Z[r * BT_COLS + c] = fma(-s, v[r], Z[r * BT_COLS + c]);
      }
    }
  }
  __syncthreads();
  for (int idx = tid; idx < n * BT_COLS; idx += blockDim.x) {
    const int r = idx / BT_COLS, c = idx - r * BT_COLS;
    if (c0 + c < n) Vu[(long long)r * n + c0 + c] = Z[idx];
  }
}

}  // namespace jolt
