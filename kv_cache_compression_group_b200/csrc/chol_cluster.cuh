// Cholesky factor G = L L^T of one symmetric positive definite n x n fp64 matrix
// (n <= 256) per thread-block cluster of 8 CTAs, for the orthonormalisation step of
// Cholesky QR.  CTA q keeps columns [32q, 32q + 32) of G in its shared memory.  Panel step
// J (J = 0 .. 7): CTA J factors its 32 columns (the diagonal block by one warp, the rows
// below by a triangular solve per row) and writes the finished panel into the shared memory of every CTA to its right
// (distributed shared memory; two panel buffers alternate), one cluster barrier, then every
// CTA to the right subtracts the panel's rank-32 update from its own columns.  At the end
// every CTA writes its columns of L as fp32 (row-major, zeros above the diagonal) and the
// inverse of its 32 x 32 diagonal block (fp64 forward substitution, rounded to fp32): the
// operands of the row-panel triangular solve.  A non-positive or non-finite pivot raises
// DEV_ERR_FACTOR (the pivot is replaced by 1 so the cluster finishes), a non-finite entry
// DEV_ERR_NONFINITE.  Every thread of every CTA passes the same sequence of cluster barriers.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"

namespace jolt {

namespace cholc {
namespace cg = cooperative_groups;
constexpr int CL = 8;
constexpr int NC = 32;
constexpr int MAXN = CL * NC;
constexpr int THREADS = 256;
constexpr int LD = NC + 1;
// shared memory (doubles): A [MAXN][LD] | panel[2][MAXN][LD]
constexpr size_t SMEM_DOUBLES = (size_t)3 * MAXN * LD;
inline size_t smem_bytes() { return SMEM_DOUBLES * sizeof(double); }
}  // namespace cholc

// grid: 8 CTAs per matrix in clusters of 8, cholc::THREADS threads, cholc::smem_bytes().
// G: symmetric matrices (lower triangle of column-major, leading dimension gld, stride sG);
// Lr: fp32 row-major L (leading dimension ldl, stride sL); Dinv: fp32 inverses of the 32 x 32
// diagonal blocks ([block][32][32], stride sD per matrix).
__global__ void __cluster_dims__(cholc::CL, 1, 1) __launch_bounds__(cholc::THREADS)
    chol_cluster_kernel(const double* G, int n, long long gld, long long sG, float* Lr, long long ldl, long long sL,
                        float* Dinv, long long sD, uint32_t* status) {
  using namespace cholc;
  cg::cluster_group cluster = cg::this_cluster();
  const int q = (int)cluster.block_rank();
  const int u = blockIdx.x / CL;
  const int tid = threadIdx.x;
  extern __shared__ double cholc_sm[];
  double* As = cholc_sm;                  // [MAXN][LD]: my columns
  double* pb = As + MAXN * LD;            // [2][MAXN][LD]: received panels
  const double* Gu = G + (long long)u * sG;
  const int c0 = q * NC;
  const int nblk = (n + NC - 1) / NC;

  bool bad = false;
  for (int idx = tid; idx < MAXN * NC; idx += blockDim.x) {
    const int r = idx / NC, lc = idx - r * NC, c = c0 + lc;
    const double a = (r < n && c < n && r >= c) ? Gu[(long long)c * gld + r] : 0.0;
    if (!isfinite(a)) bad = true;
    As[r * LD + lc] = a;
  }
  if (bad) raise_status(status, DEV_ERR_NONFINITE);
  __syncthreads();

  for (int J = 0; J < CL; ++J) {
    const int buf = J & 1;
    if (q == J && J < nblk) {
      // factor my 32 columns: the 32 x 32 diagonal block by warp 0 (lane = row), then every
      // row below solves x L_JJ^T = a (one thread per row)
      const int nb = min(NC, n - c0);
      if (tid < 32) {
        const int lane = tid;
        for (int jj = 0; jj < nb; ++jj) {
          double d = As[(c0 + jj) * LD + jj];
          if (!(d > 0.0) || !isfinite(d)) {
            if (lane == 0) raise_status(status, DEV_ERR_FACTOR);
            d = 1.0;
          }
          d = sqrt(d);
          __syncwarp();
          if (lane == jj) As[(c0 + jj) * LD + jj] = d;
          if (lane > jj && lane < nb) As[(c0 + lane) * LD + jj] /= d;
          __syncwarp();
          if (lane > jj && lane < nb) {
            const double lij = As[(c0 + lane) * LD + jj];
            for (int p = jj + 1; p <= lane; ++p)
              As[(c0 + lane) * LD + p] = fma(-lij, As[(c0 + p) * LD + jj], As[(c0 + lane) * LD + p]);
          }
          __syncwarp();
        }
      }
      __syncthreads();
      for (int r = c0 + nb + tid; r < n; r += blockDim.x) {
        double x[NC];
#pragma unroll
        for (int jj = 0; jj < NC; ++jj) x[jj] = jj < nb ? As[r * LD + jj] : 0.0;
#pragma unroll
        for (int jj = 0; jj < NC; ++jj) {
          if (jj < nb) {
            double v = x[jj];
#pragma unroll
            for (int p = 0; p < jj; ++p) v = fma(-x[p], As[(c0 + jj) * LD + p], v);
            x[jj] = v / As[(c0 + jj) * LD + jj];
          }
        }
#pragma unroll
        for (int jj = 0; jj < NC; ++jj)
          if (jj < nb) As[r * LD + jj] = x[jj];
      }
      __syncthreads();
      // the finished panel to every CTA on my right
      for (int t = q + 1; t < CL; ++t) {
        double* dst = cluster.map_shared_rank(pb, t) + buf * MAXN * LD;
        for (int idx = tid; idx < MAXN * NC; idx += blockDim.x) {
          const int r = idx / NC, lc = idx - r * NC;
          dst[r * LD + lc] = As[r * LD + lc];
        }
      }
    }
    cluster.sync();
    if (q > J && J < nblk && c0 < n) {
      // rank-32 update of my columns with panel J: A[r][c] -= sum_p P[r][p] P[c][p], r >= c
      const double* P = pb + buf * MAXN * LD;
      const int lc = tid & (NC - 1);
      const int c = c0 + lc;
      if (c < n) {
        double pc[NC];
#pragma unroll
        for (int p = 0; p < NC; ++p) pc[p] = P[c * LD + p];
        for (int r = c + (tid >> 5); r < n; r += blockDim.x / NC) {
          double s = 0.0;
#pragma unroll
          for (int p = 0; p < NC; ++p) s = fma(P[r * LD + p], pc[p], s);
          As[r * LD + lc] -= s;
        }
      }
    }
    __syncthreads();
  }

  // outputs: my columns of L in fp32 (row-major, zeros above the diagonal), and the inverse
  // of my diagonal block
  if (c0 < n) {
    float* Lu = Lr + (long long)u * sL;
    for (int idx = tid; idx < n * NC; idx += blockDim.x) {
      const int r = idx / NC, lc = idx - r * NC, c = c0 + lc;
      if (c < n) Lu[(long long)r * ldl + c] = r >= c ? (float)As[r * LD + lc] : 0.f;
    }
    if (tid < 32) {
      const int lane = tid, nb = min(NC, n - c0);
      double x[NC];
#pragma unroll
      for (int r = 0; r < NC; ++r) {
        double v = (r == lane) ? 1.0 : 0.0;
        if (r < nb && lane < nb) {
#pragma unroll
          for (int p = 0; p < r; ++p) v = fma(-As[(c0 + r) * LD + p], x[p], v);
          x[r] = lane <= r ? v / As[(c0 + r) * LD + r] : 0.0;
        } else {
          x[r] = 0.0;
        }
      }
      float* D = Dinv + (long long)u * sD + (long long)q * NC * NC;
#pragma unroll
      for (int r = 0; r < NC; ++r) D[r * NC + lane] = (float)x[r];
    }
  }
}

}  // namespace jolt
