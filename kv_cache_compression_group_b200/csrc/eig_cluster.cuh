// Symmetric eigen-decomposition of one n x n fp64 matrix (2 <= n <= 256) per thread-block
// cluster of 8 CTAs, for the Rayleigh-Ritz step of FlashJoLT (n = sketch width):
//   1. Householder reduction to tridiagonal form.  CTA q of the cluster keeps columns
//      [32q, 32q + 32) of the symmetric matrix in its shared memory; the owner of column j
//      forms the reflector and writes it into every CTA's shared memory (distributed shared
//      memory), every CTA computes p = beta A v on its columns and sends them, with its
//      partial sum of p.v, to every CTA; then every CTA forms w = p - K v and applies the
//      rank-2 update to its columns.  Two cluster barriers per column; the vectors alternate
//      between two buffers so a CTA one step ahead never overwrites what a slower one still
//      reads.  The reflectors also go to global memory.
//   2. every eigenvalue of T by multisection on Sturm counts (8 threads per eigenvalue, each
//      round shrinks the bracket ninefold);
//   3. every eigenvector of T by inverse iteration (one thread each: tridiagonal LU with
//      partial pivoting, two solves from a splitmix64 start vector); the vectors of
//      eigenvalues closer than 1e-10 ||T|| span their cluster's invariant subspace and are
//      orthonormalised in order by one warp (modified Gram-Schmidt);
//   4. back-transformation V = H_0 ... H_{n-3} Z, CTA q on eigenvectors [32q, 32q + 32).
// Output: w ascending; V[r * n + i] = component r of the unit eigenvector of w[i].
// Non-finite input raises DEV_ERR_NONFINITE.  Every thread of every CTA passes the same
// sequence of cluster barriers (all loops around them have cluster-uniform trip counts).
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"

namespace jolt {

namespace eigc {
namespace cg = cooperative_groups;
constexpr int CL = 8;            // CTAs per matrix
constexpr int NC = 32;           // columns (and eigenvectors) per CTA
constexpr int MAXN = CL * NC;    // 256
constexpr int THREADS = 256;
constexpr int SUB = 8;           // threads per eigenvalue in the multisection
// shared memory (doubles): A [MAXN][NC + 1] | v[2][MAXN] | w[2][MAXN] | d | e | beta [MAXN] |
// p [NC] | red[2][RED] | tmp[THREADS]
constexpr int A_LD = NC + 1;
constexpr int WARPS = THREADS / 32;
constexpr int RED = CL * WARPS;  // partial-sum slots per buffer: one per (CTA, warp)
constexpr size_t SMEM_DOUBLES = (size_t)MAXN * A_LD + 4 * MAXN + 3 * MAXN + NC + 2 * RED + THREADS;
inline size_t smem_bytes() { return SMEM_DOUBLES * sizeof(double); }
// global scratch per matrix (doubles): reflectors n*n | LU 5*n*n
__host__ __device__ inline size_t scratch_doubles(int n) { return (size_t)6 * n * n; }

__device__ __forceinline__ double block_sum(double v, double* tmp) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  __syncthreads();
  if (lane == 0) tmp[warp] = v;
  __syncthreads();
  double s = 0.0;
  for (int i = 0; i < nw; ++i) s += tmp[i];
  __syncthreads();
  return s;
}

__device__ __forceinline__ int sturm_count(const double* d, const double* e2, int n, double x, double pivmin) {
  double q = d[0] - x;
  int c = q < 0.0;
  for (int k = 1; k < n; ++k) {
    if (fabs(q) < pivmin) q = -pivmin;
    q = d[k] - x - e2[k - 1] / q;
    c += q < 0.0;
  }
  return c;
}

// LU factors (partial pivoting) of T - lam I for column i of the interleaved arrays
__device__ void tri_lu(const double* d, const double* e, int n, double lam, double tiny, double* U0, double* U1,
                       double* U2, double* L, double* P, int i) {
  double u0 = d[0] - lam, u1 = e[0], u2 = 0.0;
  for (int k = 0; k + 1 < n; ++k) {
    const double a = e[k], b = d[k + 1] - lam, c = (k + 2 < n) ? e[k + 1] : 0.0;
    const long long o = (long long)k * n + i;
    double l, n0, n1;
    if (fabs(a) > fabs(u0)) {
      P[o] = 1.0;
      U0[o] = a;
      U1[o] = b;
      U2[o] = c;
      l = u0 / a;
      n0 = u1 - l * b;
      n1 = u2 - l * c;
    } else {
      if (u0 == 0.0) u0 = tiny;
      P[o] = 0.0;
      U0[o] = u0;
      U1[o] = u1;
      U2[o] = u2;
      l = a / u0;
      n0 = b - l * u1;
      n1 = c - l * u2;
    }
    L[o] = l;
    u0 = n0;
    u1 = n1;
    u2 = 0.0;
  }
  U0[(long long)(n - 1) * n + i] = u0 != 0.0 ? u0 : tiny;
}

// x <- (T - lam I)^{-1} x (column i, stride n), normalised
__device__ void tri_solve_normalise(const double* U0, const double* U1, const double* U2, const double* L,
                                    const double* P, int n, double* x, int i) {
  for (int k = 0; k + 1 < n; ++k) {
    const long long o = (long long)k * n + i;
    double bk = x[o], bk1 = x[o + n];
    if (P[o] != 0.0) {
      const double t = bk;
      bk = bk1;
      bk1 = t;
    }
    bk1 -= L[o] * bk;
    x[o] = bk;
    x[o + n] = bk1;
  }
  double x1 = 0.0, x2 = 0.0, nrm = 0.0;
  for (int k = n - 1; k >= 0; --k) {
    const long long o = (long long)k * n + i;
    double s = x[o];
    if (k + 1 < n) s -= U1[o] * x1;
    if (k + 2 < n) s -= U2[o] * x2;
    s /= U0[o];
    x[o] = s;
    nrm = fma(s, s, nrm);
    x2 = x1;
    x1 = s;
  }
  const double inv = nrm > 0.0 && isfinite(nrm) ? 1.0 / sqrt(nrm) : 0.0;
  for (int k = 0; k < n; ++k) x[(long long)k * n + i] *= inv;
}

// the same solve with the vector in shared memory (x[k * xs + il]) and the factors of global
// column i
__device__ void tri_solve_normalise_sm(const double* U0, const double* U1, const double* U2, const double* L,
                                       const double* P, int n, double* x, int il, int xs, int i) {
  for (int k = 0; k + 1 < n; ++k) {
    const long long o = (long long)k * n + i;
    double bk = x[k * xs + il], bk1 = x[(k + 1) * xs + il];
    if (P[o] != 0.0) {
      const double t = bk;
      bk = bk1;
      bk1 = t;
    }
    bk1 -= L[o] * bk;
    x[k * xs + il] = bk;
    x[(k + 1) * xs + il] = bk1;
  }
  double x1 = 0.0, x2 = 0.0, nrm = 0.0;
  for (int k = n - 1; k >= 0; --k) {
    const long long o = (long long)k * n + i;
    double s = x[k * xs + il];
    if (k + 1 < n) s -= U1[o] * x1;
    if (k + 2 < n) s -= U2[o] * x2;
    s /= U0[o];
    x[k * xs + il] = s;
    nrm = fma(s, s, nrm);
    x2 = x1;
    x1 = s;
  }
  const double inv = nrm > 0.0 && isfinite(nrm) ? 1.0 / sqrt(nrm) : 0.0;
  for (int k = 0; k < n; ++k) x[k * xs + il] *= inv;
}

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ double start_value(int i, int k) {
  const uint64_t h = splitmix64_mix(((uint64_t)(i + 1) << 32) ^ (uint64_t)(k + 0x9E37));
  return ((double)(h >> 11) * 0x1.0p-53) * 2.0 - 1.0;
}
}  // namespace eigc

// grid: (8 * matrices) CTAs of eigc::THREADS threads in clusters of 8; dynamic shared memory
// eigc::smem_bytes().  A: input matrices (lower triangle of column-major n x n, stride sA);
// w: eigenvalues (stride sw); V: eigenvectors (row-major n x n per matrix, stride n*n);
// scr: eigc::scratch_doubles(n) per matrix.
__global__ void __cluster_dims__(eigc::CL, 1, 1) __launch_bounds__(eigc::THREADS, 2)
    sym_eig_cluster_kernel(const double* A, int n, long long sA, double* w, long long sw, double* V, double* scr,
                           uint32_t* status) {
  using namespace eigc;
  cg::cluster_group cluster = cg::this_cluster();
  const int q = (int)cluster.block_rank();
  const int u = blockIdx.x / CL;
  const int tid = threadIdx.x;
  extern __shared__ double eigc_sm[];
  double* As = eigc_sm;                    // [MAXN][A_LD]
  double* vb = As + MAXN * A_LD;           // [2][MAXN]
  double* wb = vb + 2 * MAXN;              // [2][MAXN]
  double* sd = wb + 2 * MAXN;              // [MAXN]
  double* se = sd + MAXN;                  // [MAXN]
  double* sb = se + MAXN;                  // [MAXN]
  double* sp = sb + MAXN;                  // [NC]
  double* red = sp + NC;                   // [2][RED]
  double* tmp = red + 2 * RED;             // [THREADS]
  const double* Au = A + (long long)u * sA;
  double* wu = w + (long long)u * sw;
  double* Vu = V + (long long)u * n * n;
  double* refl = scr + (long long)u * scratch_doubles(n);
  double* U0 = refl + (long long)n * n;
  double* U1 = U0 + (long long)n * n;
  double* U2 = U1 + (long long)n * n;
  double* Lm = U2 + (long long)n * n;
  double* Pv = Lm + (long long)n * n;
  const int c0 = q * NC;

  // 0. my columns of the symmetric matrix (lower triangle of the column-major input)
  bool bad = false;
  for (int idx = tid; idx < MAXN * NC; idx += blockDim.x) {
    const int r = idx / NC, lc = idx - r * NC, c = c0 + lc;
    double a = 0.0;
    if (r < n && c < n) a = r >= c ? Au[(long long)c * n + r] : Au[(long long)r * n + c];
    if (!isfinite(a)) bad = true;
    As[r * A_LD + lc] = a;
  }
  for (int idx = tid; idx < 7 * MAXN; idx += blockDim.x) vb[idx] = 0.0;   // v, w, d, e, beta
  if (bad) raise_status(status, DEV_ERR_NONFINITE);
  cluster.sync();

  // 1. tridiagonalisation
  for (int j = 0; j + 2 < n; ++j) {
    const int buf = j & 1, owner = j / NC, lc = j - owner * NC;
    if (q == owner) {
      // every warp forms the same norm (same order), so no CTA barrier is needed here
      double part = 0.0;
      for (int r = j + 2 + (tid & 31); r < n; r += 32) {
        const double x = As[r * A_LD + lc];
        part = fma(x, x, part);
      }
      const double tail2 = warp_sum(part);
      const double x0 = As[(j + 1) * A_LD + lc];
      double beta = 0.0, alpha = x0;
      if (tail2 > 0.0) {
        const double nrm = sqrt(fma(x0, x0, tail2));
        alpha = x0 > 0.0 ? -nrm : nrm;
        const double v0 = x0 - alpha;
        beta = 2.0 / fma(v0, v0, tail2);
      }
      // v to every CTA (and to global memory for the back-transformation)
      for (int r = tid; r < MAXN; r += blockDim.x) {
        const double v = r <= j || r >= n ? 0.0 : (r == j + 1 ? x0 - alpha : As[r * A_LD + lc]);
        for (int t = 0; t < CL; ++t) cluster.map_shared_rank(vb, t)[buf * MAXN + r] = v;
        if (r < n) refl[(long long)j * n + r] = v;
      }
      if (tid == 0) {
        const double dj = As[j * A_LD + lc];
        for (int t = 0; t < CL; ++t) {
          cluster.map_shared_rank(sd, t)[j] = dj;
          cluster.map_shared_rank(se, t)[j] = alpha;
          cluster.map_shared_rank(sb, t)[j] = beta;
        }
      }
    }
    cluster.sync();   // (A) v, beta everywhere
    const double beta = sb[j];
    const double* v = vb + buf * MAXN;
    double* pfull = wb + buf * MAXN;   // p of every column, gathered from all CTAs
    if (beta != 0.0) {
      // p_c = beta * sum_r A[r][c] v_r on my columns c >= j+1: 8 threads per column
      const int lcol = tid >> 3, part = tid & 7, c = c0 + lcol;
      double s = 0.0;
      if (c > j && c < n)
        for (int r = j + 1 + part; r < n; r += 8) s = fma(As[r * A_LD + lcol], v[r], s);
#pragma unroll
      for (int o = 4; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      const double pc = (c > j && c < n) ? beta * s : 0.0;
      if (part == 0)
        for (int t = 0; t < CL; ++t) cluster.map_shared_rank(wb, t)[buf * MAXN + c] = pc;
      // one partial sum of p.v per warp, into slot (q, warp) of every CTA
      const double pv = warp_sum(part == 0 ? pc * v[c] : 0.0);
      if ((tid & 31) == 0)
        for (int t = 0; t < CL; ++t) cluster.map_shared_rank(red, t)[buf * RED + q * WARPS + (tid >> 5)] = pv;
    }
    cluster.sync();   // (B) p and the partial sums of p.v everywhere
    if (beta != 0.0) {
      double ptv = 0.0;
      for (int t = 0; t < RED; ++t) ptv += red[buf * RED + t];
      const double K = 0.5 * beta * ptv;
      // A -= v w^T + w v^T with w = p - K v (each CTA forms w itself from the gathered p)
      const int lcol = tid & (NC - 1), c = c0 + lcol;
      if (c > j && c < n) {
        const double vc = v[c], wc = fma(-K, vc, pfull[c]);
        for (int r = j + 1 + (tid >> 5); r < n; r += blockDim.x / NC) {
          const int o = r * A_LD + lcol;
          As[o] = As[o] - (v[r] * wc + fma(-K, v[r], pfull[r]) * vc);
        }
      }
    }
    __syncthreads();
  }
  // the last 2 x 2 block of T
  if (tid == 0) {
    const int cl2 = n - 2, cl1 = n - 1;
    if (cl2 / NC == q) {
      const double a = As[cl2 * A_LD + (cl2 - c0)], b = As[cl1 * A_LD + (cl2 - c0)];
      for (int t = 0; t < CL; ++t) {
        cluster.map_shared_rank(sd, t)[cl2] = a;
        cluster.map_shared_rank(se, t)[cl2] = b;
      }
    }
    if (cl1 / NC == q) {
      const double a = As[cl1 * A_LD + (cl1 - c0)];
      for (int t = 0; t < CL; ++t) cluster.map_shared_rank(sd, t)[cl1] = a;
    }
  }
  __threadfence();
  cluster.sync();   // d, e complete everywhere; reflectors in global memory

  // 2. eigenvalues by multisection: thread group of SUB on eigenvalue c0 + tid / SUB
  double* e2 = vb;   // reuse: e^2
  for (int k = tid; k < MAXN; k += blockDim.x) e2[k] = k < n - 1 ? se[k] * se[k] : 0.0;
  __syncthreads();
  double glo = INFINITY, ghi = -INFINITY, e2max = 0.0;
  for (int k = 0; k < n; ++k) {
    const double rad = (k + 1 < n ? fabs(se[k]) : 0.0) + (k ? fabs(se[k - 1]) : 0.0);
    glo = fmin(glo, sd[k] - rad);
    ghi = fmax(ghi, sd[k] + rad);
    e2max = fmax(e2max, e2[k]);
  }
  const double pivmin = 2.2250738585072014e-308 * fmax(1.0, e2max);
  {
    const int i = c0 + tid / SUB, sub = tid % SUB;
    const int gbase = (tid & 31) & ~(SUB - 1);   // first lane of this thread's group
    double a = glo, b = ghi;
    // a fixed number of rounds (9^24 ~ 8e22 shrinks any bracket to the fp64 resolution), so
    // every lane of the warp takes part in every shuffle
    for (int it = 0; it < 24; ++it) {
      const bool done = b - a <= 2.220446049250313e-16 * fmax(fabs(a), fabs(b)) + pivmin;
      if (__all_sync(0xffffffffu, done)) break;   // the whole warp has converged
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
    if (sub == 0 && i < n) wu[i] = 0.5 * (a + b);
  }
  __threadfence();
  cluster.sync();   // every eigenvalue in global memory
  const double norm = fmax(fabs(wu[0]), fabs(wu[n - 1]));
  const double tiny = 2.220446049250313e-16 * fmax(norm, 2.2250738585072014e-308);
  const double ctol = 1e-10 * norm;

  // 3. eigenvectors of T (one thread per eigenvector of this CTA; the iterate in shared
  //    memory, the factors in global memory), two solves, then into V
  if (tid < NC && c0 + tid < n) {
    const int i = c0 + tid;
    double* xs = As;   // [MAXN][NC], free until the back-transformation
    eigc::tri_lu(sd, se, n, wu[i], tiny, U0, U1, U2, Lm, Pv, i);
    for (int k = 0; k < n; ++k) xs[k * NC + tid] = eigc::start_value(i, k);
    for (int it = 0; it < 2; ++it) eigc::tri_solve_normalise_sm(U0, U1, U2, Lm, Pv, n, xs, tid, NC, i);
    for (int k = 0; k < n; ++k) Vu[(long long)k * n + i] = xs[k * NC + tid];
  }
  __threadfence();
  cluster.sync();
  // eigenvalues closer than ctol: their vectors span the cluster's invariant subspace; one
  // warp of the cluster orthonormalises them in order (modified Gram-Schmidt)
  if (q == 0 && tid < 32) {
    const int lane = tid;
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
  __threadfence();
  cluster.sync();

  // 4. back-transformation of my eigenvectors: Z staged in shared memory (As reused)
  double* Zs = As;   // [MAXN][A_LD]
  for (int idx = tid; idx < MAXN * NC; idx += blockDim.x) {
    const int r = idx / NC, il = idx - r * NC;
    Zs[r * A_LD + il] = (r < n && c0 + il < n) ? Vu[(long long)r * n + c0 + il] : 0.0;
  }
  __syncthreads();
  {
    const int il = tid & (NC - 1), part = tid >> 5;   // 8 row groups per eigenvector
    double* vj = vb;                                    // reflector staging
    for (int j = n - 3; j >= 0; --j) {
      for (int r = tid; r < n; r += blockDim.x) vj[r] = r > j ? refl[(long long)j * n + r] : 0.0;
      __syncthreads();
      const double bj = sb[j];
      double s = 0.0;
      for (int r = j + 1 + part; r < n; r += 8) s = fma(vj[r], Zs[r * A_LD + il], s);
      tmp[part * NC + il] = s;
      __syncthreads();
      double tot = 0.0;
#pragma unroll
      for (int g = 0; g < 8; ++g) tot += tmp[g * NC + il];
      tot *= bj;
      for (int r = j + 1 + part; r < n; r += 8) Zs[r * A_LD + il] = fma(-tot, vj[r], Zs[r * A_LD + il]);
      __syncthreads();
    }
  }
  for (int idx = tid; idx < MAXN * NC; idx += blockDim.x) {
    const int r = idx / NC, il = idx - r * NC;
    if (r < n && c0 + il < n) Vu[(long long)r * n + c0 + il] = Zs[r * A_LD + il];
  }
}

}  // namespace jolt
