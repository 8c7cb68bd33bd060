// Small kernels around the factor, allocation and packing steps.
#pragma once

#include "common.cuh"
#include "kernels.cuh"

namespace jolt {

// out[b][i] = sum_s part[b][s][i]  in a fixed order (s ascending), fp64
template <typename TP>
__global__ void reduce_splits_kernel(const TP* part, double* out, int nbatch, int nsplit, long long n) {
  long long total = (long long)nbatch * n;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    long long b = idx / n, i = idx - b * n;
    const TP* p = part + b * nsplit * n + i;
    double acc = 0.0;
    for (int s = 0; s < nsplit; ++s) acc += (double)p[(long long)s * n];
    out[idx] = acc;
  }
}

// the same sum for a symmetric k x k result whose split partials hold only the tiles on and
// below the diagonal (tile edge te): entry (r, c) of an upper tile is read at (c, r)
template <typename TP>
__global__ void reduce_splits_sym_kernel(const TP* part, double* out, int nbatch, int nsplit, int k, long long ld,
                                         int te) {
  const long long n = (long long)k * ld;
  const long long total = (long long)nbatch * k * k;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    const long long b = idx / ((long long)k * k), rem = idx - b * k * k;
    const int r = (int)(rem / k), c = (int)(rem - (long long)r * k);
    const long long src = (c / te > r / te) ? (long long)c * ld + r : (long long)r * ld + c;
    const TP* p = part + b * nsplit * n + src;
    double acc = 0.0;
    for (int s = 0; s < nsplit; ++s) acc += (double)p[(long long)s * n];
    out[b * n + (long long)r * ld + c] = acc;
  }
}

// every diagonal entry of the unit's feature Gram must be finite (a NaN/Inf anywhere in
// the cache reaches the diagonal through x*x)
__global__ void gram_diag_check_kernel(const double* G, int n, int nunits, uint32_t* status) {
  int u = blockIdx.x;
  if (u >= nunits) return;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    double v = G[(long long)u * n * n + (long long)i * n + i];
    if (!isfinite(v)) raise_status(status, DEV_ERR_NONFINITE);
  }
}

// Leading r eigenvectors in descending eigenvalue order (ties: lower original index first)
// from an ascending eigen-solver output (eigenvectors in columns, column-major, lda),
// the entry of largest magnitude made positive (ties: lowest row).
// Writes row-major n x ldo fp32 (optional), bf16 (optional) and the eigenvalues (optional).
// eigenvector i of matrix u is vecs[u * svec + i * lda + row * inc]
__global__ void eig_select_kernel(const double* vals, const double* vecs, int n, long long lda, long long inc,
                                  long long sval, long long svec, int r, float* out_f32, bf16* out_bf16,
                                  long long ldo, long long sout, double* out_vals) {
  const int j = blockIdx.x, u = blockIdx.y;
  const double* w = vals + (long long)u * sval;
  // the j-th largest: with ties broken towards the lower index, descending order of an
  // ascending list is position n-1-j unless equal neighbours exist; resolve exactly.
  __shared__ int src;
  if (threadIdx.x == 0) {
    // count of entries strictly greater, then pick among equals the lowest index
    int pos = n - 1 - j;
    double v = w[pos];
    int first_eq = pos;
    while (first_eq > 0 && w[first_eq - 1] == v) --first_eq;
    int last_eq = pos;
    while (last_eq < n - 1 && w[last_eq + 1] == v) ++last_eq;
    int rank_in_group = (last_eq - pos);  // 0 for the first (largest-position) in descending walk
    src = first_eq + rank_in_group;
    if (out_vals) out_vals[(long long)u * r + j] = v;
  }
  __syncthreads();
  const double* col = vecs + (long long)u * svec + (long long)src * lda;
  __shared__ double bestv[256];
  __shared__ int besti[256];
  double bv = -1.0;
  int bi = 0x7fffffff;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    double a = fabs(col[i * inc]);
    if (a > bv || (a == bv && i < bi)) { bv = a; bi = i; }
  }
  bestv[threadIdx.x] = bv;
  besti[threadIdx.x] = bi;
  __syncthreads();
  for (int st = blockDim.x / 2; st > 0; st >>= 1) {
    if ((int)threadIdx.x < st) {
      double ov = bestv[threadIdx.x + st];
      int oi = besti[threadIdx.x + st];
      if (ov > bestv[threadIdx.x] || (ov == bestv[threadIdx.x] && oi < besti[threadIdx.x])) {
        bestv[threadIdx.x] = ov;
        besti[threadIdx.x] = oi;
      }
    }
    __syncthreads();
  }
  // no finite entry (a non-finite input, already reported in the status word): sign +1
  const int piv = besti[0] < n ? besti[0] : 0;
  const double sgn = col[(long long)piv * inc] < 0 ? -1.0 : 1.0;
  for (int i = threadIdx.x; i < n; i += blockDim.x) {
    double v = sgn * col[i * inc];
    long long o = (long long)u * sout + (long long)i * ldo + j;
    if (out_f32) out_f32[o] = (float)v;
    if (out_bf16) out_bf16[o] = __float2bfloat16_rn((float)v);
  }
}

// Same sign convention on the columns j < r of every unit's row-major fp32 matrix (n rows,
// pitch lda, unit stride sA), in place, plus a bf16 copy; three coalesced passes:
//   sign_key_kernel   per column the largest |a| with its first row, as one 64-bit key
//                     (|a|'s bits above the complement of the row: the atomic maximum of the
//                     keys is the largest magnitude, ties to the lowest row; non-finite
//                     magnitudes never win, a column without any keeps the key 0);
//   sign_of_kernel    the sign of the entry the key names (+1 for key 0);
//   sign_apply_kernel a *= sign, bf16 copy.
// keys: [units][r] uint64, zeroed before sign_key_kernel; signs: [units][r] fp32.
constexpr int SK_ROWS = 512;   // rows per CTA of sign_key_kernel
// grid (ceil(n / SK_ROWS), units), 256 threads
__global__ void __launch_bounds__(256) sign_key_kernel(const float* A, long long lda, long long sA, int n, int r,
                                                       unsigned long long* keys) {
  const int u = blockIdx.y, i0 = blockIdx.x * SK_ROWS, i1 = min(n, i0 + SK_ROWS);
  const float* a = A + (long long)u * sA;
  for (int c = threadIdx.x; c < r; c += blockDim.x) {
    unsigned long long best = 0ull;
    for (int i = i0; i < i1; ++i) {
      const float x = fabsf(a[(long long)i * lda + c]);
      if (!(x <= 3.402823466e38f)) continue;   // NaN or infinite: never the pivot
      const unsigned long long key =
          ((unsigned long long)__float_as_uint(x) << 32) | (unsigned long long)(0xFFFFFFFFu - (unsigned)i);
      best = key > best ? key : best;
    }
    if (best) atomicMax(keys + (long long)u * r + c, best);
  }
}
// grid (units), 1024 threads
__global__ void sign_of_kernel(const float* A, long long lda, long long sA, int r, const unsigned long long* keys,
                               float* signs) {
  const int u = blockIdx.x;
  const float* a = A + (long long)u * sA;
  for (int c = threadIdx.x; c < r; c += blockDim.x) {
    const unsigned long long key = keys[(long long)u * r + c];
    float sg = 1.f;
    if (key) {
      const long long piv = (long long)(0xFFFFFFFFu - (unsigned)(key & 0xFFFFFFFFull));
      sg = a[piv * lda + c] < 0.f ? -1.f : 1.f;
    }
    signs[(long long)u * r + c] = sg;
  }
}
// grid-stride over units x n x r (4 columns per thread; lda, ldo, r multiples of 4)
__global__ void sign_apply_kernel(float* A, long long lda, long long sA, int n, int r, const float* signs,
                                  bf16* out_bf16, long long ldo, long long so, int nunits) {
  const int r4 = r / 4;
  const long long per = (long long)n * r4, total = per * nunits;
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const int u = (int)(e / per);
    const long long rem = e - (long long)u * per;
    const long long i = rem / r4;
    const int c = (int)(rem - i * r4) * 4;
    float4* pa = reinterpret_cast<float4*>(A + (long long)u * sA + i * lda + c);
    const float4 sg = *reinterpret_cast<const float4*>(signs + (long long)u * r + c);
    float4 v = *pa;
    v.x *= sg.x;
    v.y *= sg.y;
    v.z *= sg.z;
    v.w *= sg.w;
    *pa = v;
    if (out_bf16) {
      __nv_bfloat162 h0 = __floats2bfloat162_rn(v.x, v.y), h1 = __floats2bfloat162_rn(v.z, v.w);
      uint2 w;
      w.x = *reinterpret_cast<uint32_t*>(&h0);
      w.y = *reinterpret_cast<uint32_t*>(&h1);
      *reinterpret_cast<uint2*>(out_bf16 + (long long)u * so + i * ldo + c) = w;
    }
  }
}

// FlashJoLT test matrix: Omega[m][j] = bf16(gaussian(seed, OMEGA stream of unit, m*k + j)),
// zero in the padding columns k <= j < ld
__global__ void omega_kernel(bf16* om, int M, int k, long long ld, long long sunit, uint64_t seed, int unit0,
                             int nunits) {
  long long total = (long long)nunits * M * ld;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    long long u = idx / ((long long)M * ld);
    long long rem = idx - u * M * ld;
    long long m = rem / ld, j = rem - m * ld;
    // one rounding from double to bf16 (round to nearest even)
    om[u * sunit + m * ld + j] =
        j < k ? __double2bfloat16(gaussian(seed, stream_id(kStreamOmega, unit0 + (int)u), (uint64_t)(m * k + j)))
              : __float2bfloat16_rn(0.f);
  }
}

// fp32 -> bf16 hi + bf16 lo with hi + lo ~ x (2^-17 relative)
__global__ void split_bf16_kernel(const float* x, bf16* hi, bf16* lo, long long n) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    float v = x[i];
    bf16 h = __float2bfloat16_rn(v);
    hi[i] = h;
    lo[i] = __float2bfloat16_rn(v - __bfloat162float(h));
  }
}

// the same split of a row-major block of pitch ld, columns k..ld written as zeros (they enter
// tensor-core K blocks that must contribute nothing)
__global__ void split_bf16_cols_kernel(const float* x, bf16* hi, bf16* lo, long long n, int ld, int k) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const float v = (int)(i % ld) < k ? x[i] : 0.f;
    bf16 h = __float2bfloat16_rn(v);
    hi[i] = h;
    lo[i] = __float2bfloat16_rn(v - __bfloat162float(h));
  }
}


// zero the strict upper triangle of column-major n x n matrices (lda)
__global__ void tril_zero_kernel(double* A, int n, long long lda, long long sA, int nbatch) {
  long long total = (long long)nbatch * n * n;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    long long b = idx / ((long long)n * n);
    long long rem = idx - b * n * n;
    long long col = rem / n, row = rem - col * n;
    if (row < col) A[b * sA + col * lda + row] = 0.0;
  }
}

// Guard in front of every eigen / Cholesky call: if the cache was flagged non-finite, or the
// matrix itself holds a NaN / Inf, the matrix is replaced by the identity (the status word
// records the error), so the solver only ever sees finite input.  One block per call.
__global__ void sanitize_sym_kernel(double* A, int n, long long lda, uint32_t* status) {
  __shared__ int bad;
  if (threadIdx.x == 0) bad = (*status & DEV_ERR_NONFINITE) ? 1 : 0;
  __syncthreads();
  for (long long i = threadIdx.x; i < (long long)n * n && !bad; i += blockDim.x) {
    long long r = i / n, c = i - r * n;
    if (!isfinite(A[c * lda + r])) bad = 1;
  }
  __syncthreads();
  if (!bad) return;
  if (threadIdx.x == 0) raise_status(status, DEV_ERR_NONFINITE);
  for (long long i = threadIdx.x; i < (long long)n * n; i += blockDim.x) {
    long long r = i / n, c = i - r * n;
    A[c * lda + r] = (r == c) ? 1.0 : 0.0;
  }
}

// batched guard: one block per matrix (stride sA between matrices)
__global__ void sanitize_sym_batched_kernel(double* A, int n, long long lda, long long sA, uint32_t* status) {
  double* M = A + blockIdx.x * sA;
  __shared__ int bad;
  if (threadIdx.x == 0) bad = (*status & DEV_ERR_NONFINITE) ? 1 : 0;
  __syncthreads();
  // column by column (consecutive threads read consecutive rows)
  for (long long i = threadIdx.x; i < (long long)n * n && !bad; i += blockDim.x) {
    long long c = i / n, r = i - c * n;
    if (!isfinite(M[c * lda + r])) bad = 1;
  }
  __syncthreads();
  if (!bad) return;
  if (threadIdx.x == 0) raise_status(status, DEV_ERR_NONFINITE);
  for (long long i = threadIdx.x; i < (long long)n * n; i += blockDim.x) {
    long long c = i / n, r = i - c * n;
    M[c * lda + r] = (r == c) ? 1.0 : 0.0;
  }
}

__global__ void info_check_kernel(const int* info, int n, uint32_t* status, uint32_t bits) {
  int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n && info[i] != 0) raise_status(status, bits);
}

// fp32 -> fp64 copy (for the eigen solver input) with optional scale per column
__global__ void f32_to_f64_kernel(const float* in, double* out, long long n) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
    out[i] = (double)in[i];
}

// V[:, j] *= 1/sqrt(lambda_j) (row-major n x ld fp32) and flag non-positive eigenvalues
__global__ void scale_cols_kernel(float* V, const double* lam, int n, int r, long long ld, long long sV,
                                  long long slam, int nunits, uint32_t* status) {
  long long total = (long long)nunits * n * r;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < total;
       idx += (long long)gridDim.x * blockDim.x) {
    long long u = idx / ((long long)n * r);
    long long rem = idx - u * n * r;
    long long i = rem / r, j = rem - i * r;
    double l = lam[u * slam + j];
    if (!(l > 0.0)) {
      raise_status(status, DEV_ERR_FACTOR);
      l = 1.0;
    }
    V[u * sV + i * ld + j] = (float)((double)V[u * sV + i * ld + j] / sqrt(l));
  }
}

// the core from the token-major product, Ct[u][i][s * ldw + c], into its stored layout
// core[u][s][i][c] (c < ldc <= ldw)
__global__ void core_permute_kernel(const bf16* Ct, bf16* core, int nunits, int S, int rT, int ldw, int ldc) {
  const long long total = (long long)nunits * S * rT * ldc;
  for (long long e = blockIdx.x * (long long)blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const int c = (int)(e % ldc);
    long long r = e / ldc;
    const int i = (int)(r % rT);
    r /= rT;
    const int s = (int)(r % S);
    const long long u = r / S;
    core[e] = Ct[(u * rT + i) * ((long long)S * ldw) + (long long)s * ldw + c];
  }
}

// ------------------------------------------------------------------------------------------
// distortion table finalisation, byte table and the Lagrangian dual
// ------------------------------------------------------------------------------------------
// table[u][(iT*nD + iD)*nB + ib] = sum over (slice, tile) of partial[u][s][tile][(iD*nT+iT)*nB+ib]
// grid (units x choices), 256 threads: the partial sums of every (slice, tile) of one table
// entry, strided over the threads, then a fixed-order tree (the same order on every call)
__global__ void __launch_bounds__(256) table_reduce_kernel(const double* partial, double* table, int nunits, int S,
                                                           int tiles, int nT, int nD, int nB) {
  __shared__ double red[256];
  const int nc = nT * nD * nB;
  const int idx = blockIdx.x;
  const int u = idx / nc, c = idx - u * nc;
  const int ib = c % nB, iD = (c / nB) % nD, iT = c / (nB * nD);
  const int pc = (iD * nT + iT) * nB + ib;
  const double* p = partial + (long long)u * S * tiles * nc + pc;
  double acc = 0.0;
  for (long long st = threadIdx.x; st < (long long)S * tiles; st += blockDim.x) acc += p[st * nc];
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int w = blockDim.x / 2; w > 0; w >>= 1) {
    if ((int)threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) table[idx] = red[0];
}

__host__ __device__ inline unsigned long long pad16u(unsigned long long n) { return (n + 15ull) / 16ull * 16ull; }

// stored bytes of one unit for (r_T, r_D, b): U, W, core in bf16, codes (2b bytes per block
// of 16) and one fp16 (lo, step) pair per block, each array padded to 16 bytes
__host__ __device__ inline unsigned long long unit_payload_bytes(int T, int D, int S, int rT, int rD, int b) {
  unsigned long long n = pad16u(2ull * T * rT) + pad16u(2ull * D * rD) + pad16u(2ull * S * rT * rD);
  if (b > 0) {
    unsigned long long nblk = (unsigned long long)S * T * (D / 16);
    n += pad16u(nblk * 2ull * b) + pad16u(nblk * 4ull);
  }
  return n;
}

__global__ void bytes_table_kernel(unsigned long long* B, int nunits, int T, int D, int S, Cands cd) {
  const int nc = cd.nT * cd.nD * cd.nB;
  int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= nunits * nc) return;
  int c = idx % nc;
  int ib = c % cd.nB, iD = (c / cd.nB) % cd.nD, iT = c / (cd.nB * cd.nD);
  B[idx] = unit_payload_bytes(T, D, S, cd.rT[iT], cd.rD[iD], cd.bits[ib]);
}

// Per unit, argmin_c D[c] + lam*B[c] with two separate roundings (no fused multiply-add);
// ties go to fewer bytes, then to the lower choice index.  D is finite or +inf and lam*B is
// finite or +inf, so no NaN is compared.
struct AllocArgs {
  const double* D;
  const unsigned long long* B;
  int nunits, nc;
  unsigned long long budget;       // bytes available to the payload (headers already taken out)
  int* choice;                     // [nunits]
  double* lambda;                  // [1]
  uint32_t* status;
  // blob filling (optional)
  unsigned char* blob;
  unsigned long long blob_cap;
  unsigned long long header_bytes;
  int T, D_, S;
  Cands cd;
  BlobHeader hdr;                  // global header prototype (passed by value)
  const int32_t* forced;           // optional caller choices: skip the search, fill the headers
};

// F(lam): every unit's Lagrangian choice (one warp per unit, lanes over the choices, then a
// lexicographic (value, bytes, index) reduction), and the total bytes
__device__ unsigned long long alloc_F(const AllocArgs& a, double lam, int* sch, unsigned long long* sB) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  for (int u = warp; u < a.nunits; u += nwarps) {
    const double* Dr = a.D + (long long)u * a.nc;
    const unsigned long long* Br = a.B + (long long)u * a.nc;
    double bv = 0.0;
    unsigned long long bb = 0ull;
    int bc = -1;
    for (int c = lane; c < a.nc; c += 32) {
      double v = __dadd_rn(Dr[c], __dmul_rn(lam, (double)Br[c]));
      bool better = (bc < 0) || (v < bv) || (v == bv && Br[c] < bb);
      if (better) { bv = v; bb = Br[c]; bc = c; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      double ov = __shfl_xor_sync(0xffffffffu, bv, o);
      unsigned long long ob = __shfl_xor_sync(0xffffffffu, bb, o);
      int oc = __shfl_xor_sync(0xffffffffu, bc, o);
      bool take = (oc >= 0) && ((bc < 0) || (ov < bv) || (ov == bv && (ob < bb || (ob == bb && oc < bc))));
      if (take) { bv = ov; bb = ob; bc = oc; }
    }
    if (lane == 0) {
      sch[u] = bc;
      sB[u] = Br[bc];
    }
  }
  __syncthreads();
  unsigned long long tot = 0ull;
  for (int u = 0; u < a.nunits; ++u) tot += sB[u];
  __syncthreads();
  return tot;
}

// one CTA: the bisection on lambda, then the unit headers and byte offsets of the blob
__global__ void allocate_kernel(AllocArgs a) {
  extern __shared__ unsigned char sm[];
  int* sch = reinterpret_cast<int*>(sm);
  unsigned long long* sB = reinterpret_cast<unsigned long long*>(sm + ((a.nunits * 4 + 15) / 16) * 16);
  __shared__ double s_lam;
  __shared__ int s_state;  // 0 ok, 1 infeasible
  // feasibility: every unit at its fewest-bytes choice
  if (a.forced) {
    for (int u = threadIdx.x; u < a.nunits; u += blockDim.x) sch[u] = a.forced[u];
    __syncthreads();
    if (threadIdx.x == 0) s_lam = 0.0;
    __syncthreads();
  }
  if (threadIdx.x == 0 && !a.forced) {
    unsigned long long minB = 0ull;
    for (int u = 0; u < a.nunits; ++u) {
      unsigned long long m = ~0ull;
      for (int c = 0; c < a.nc; ++c) m = min(m, a.B[(long long)u * a.nc + c]);
      minB += m;
    }
    s_state = minB > a.budget ? 1 : 0;
  }
  if (a.forced && threadIdx.x == 0) s_state = 0;
  __syncthreads();
  if (s_state) {
    if (threadIdx.x == 0) {
      raise_status(a.status, DEV_ERR_INFEASIBLE);
      a.lambda[0] = __longlong_as_double(0x7ff0000000000000LL);
      if (a.blob) {
        BlobHeader h = a.hdr;
        h.status = DEV_ERR_INFEASIBLE;
        h.total_bytes = 0;
        *reinterpret_cast<BlobHeader*>(a.blob) = h;
      }
    }
    return;
  }
  double lam = 0.0;
  unsigned long long F = a.forced ? 0ull : alloc_F(a, 0.0, sch, sB);
  if (!a.forced && F > a.budget) {
    double lo = 0.0, hi = 1.0;
    for (int it = 0; it < 2100; ++it) {
      if (alloc_F(a, hi, sch, sB) <= a.budget) break;
      hi = __dmul_rn(hi, 2.0);
    }
    for (int it = 0; it < 200; ++it) {
      double mid = __dadd_rn(lo, __dmul_rn(__dadd_rn(hi, -lo), 0.5));
      if (alloc_F(a, mid, sch, sB) <= a.budget) hi = mid;
      else lo = mid;
    }
    lam = hi;
    F = alloc_F(a, hi, sch, sB);
  }
  if (threadIdx.x == 0) s_lam = lam;
  __syncthreads();
  if (!a.forced) {
    for (int u = threadIdx.x; u < a.nunits; u += blockDim.x) a.choice[u] = sch[u];
    if (threadIdx.x == 0) a.lambda[0] = s_lam;
  }
  if (!a.blob || threadIdx.x != 0) return;
  // unit headers and payload offsets, in unit order
  unsigned long long off = a.header_bytes;
  UnitHeader* uh = reinterpret_cast<UnitHeader*>(a.blob + sizeof(BlobHeader));
  for (int u = 0; u < a.nunits; ++u) {
    int c = sch[u];
    int ib = c % a.cd.nB, iD = (c / a.cd.nB) % a.cd.nD, iT = c / (a.cd.nB * a.cd.nD);
    int rT = a.cd.rT[iT], rD = a.cd.rD[iD], b = a.cd.bits[ib];
    UnitHeader h;
    h.r_T = rT;
    h.r_D = rD;
    h.bits = b;
    h.choice = c;
    h.off_U = off;
    h.off_W = h.off_U + pad16u(2ull * a.T * rT);
    h.off_C = h.off_W + pad16u(2ull * a.D_ * rD);
    h.off_codes = h.off_C + pad16u(2ull * a.S * rT * rD);
    unsigned long long nblk = (unsigned long long)a.S * a.T * (a.D_ / 16);
    h.off_scales = h.off_codes + (b > 0 ? pad16u(nblk * 2ull * b) : 0ull);
    h.distortion = a.D[(long long)u * a.nc + c];
    uh[u] = h;
    off += a.B[(long long)u * a.nc + c];
  }
  BlobHeader g = a.hdr;
  g.total_bytes = off;
  g.status = off > a.blob_cap ? DEV_ERR_CAPACITY : 0u;
  if (g.status) raise_status(a.status, DEV_ERR_CAPACITY);
  *reinterpret_cast<BlobHeader*>(a.blob) = g;
}

// copy the chosen prefixes of U (T x r_T), W (D x r_D) and the core (S x r_T x r_D) into the blob
__global__ void copy_factors_kernel(unsigned char* blob, const bf16* U, long long ldU, long long sU,
                                    const bf16* W, long long ldW, long long sW, const bf16* C, long long ldC,
                                    long long sC_slice, long long sC_unit, int T, int D, int S) {
  const int u = blockIdx.y;
  const BlobHeader* gh = reinterpret_cast<const BlobHeader*>(blob);
  if (gh->status != 0) return;
  const UnitHeader h = reinterpret_cast<const UnitHeader*>(blob + sizeof(BlobHeader))[u];
  bf16* oU = reinterpret_cast<bf16*>(blob + h.off_U);
  bf16* oW = reinterpret_cast<bf16*>(blob + h.off_W);
  bf16* oC = reinterpret_cast<bf16*>(blob + h.off_C);
  long long nU = (long long)T * h.r_T, nW = (long long)D * h.r_D, nC = (long long)S * h.r_T * h.r_D;
  long long tot = nU + nW + nC;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < tot; i += (long long)gridDim.x * blockDim.x) {
    if (i < nU) {
      long long t = i / h.r_T, j = i - t * h.r_T;
      oU[i] = U[u * sU + t * ldU + j];
    } else if (i < nU + nW) {
      long long k = i - nU;
      long long d = k / h.r_D, j = k - d * h.r_D;
      oW[k] = W[u * sW + d * ldW + j];
    } else {
      long long k = i - nU - nW;
      long long s = k / ((long long)h.r_T * h.r_D);
      long long rem = k - s * h.r_T * h.r_D;
      long long r = rem / h.r_D, q = rem - r * h.r_D;
      oC[k] = C[u * sC_unit + s * sC_slice + r * ldC + q];
    }
  }
}

__global__ void iota_kernel(int* out, int n, int first) {
  int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = first + i;
}

// device-side errors of the factor stage go into the blob header status word
__global__ void fold_status_kernel(const uint32_t* status, unsigned char* blob) {
  BlobHeader* h = reinterpret_cast<BlobHeader*>(blob);
  uint32_t s = *status;
  if (s) h->status |= s;
}

// dense rows x cols bf16 (ld = cols) -> rows x ldo, zero padded columns
__global__ void copy2d_kernel(const bf16* src, long long rows, int cols, bf16* dst, long long ldo) {
  long long tot = rows * ldo;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < tot; i += (long long)gridDim.x * blockDim.x) {
    long long r = i / ldo, j = i - r * ldo;
    dst[i] = j < cols ? src[r * cols + j] : __float2bfloat16_rn(0.f);
  }
}

// copy a unit's U from the blob (T x r_T) into an aligned workspace (T x ld)
__global__ void unpack_u_kernel(const unsigned char* blob, bf16* out, long long ld, long long sunit, int T) {
  const int u = blockIdx.y;
  const UnitHeader h = reinterpret_cast<const UnitHeader*>(blob + sizeof(BlobHeader))[u];
  const bf16* src = reinterpret_cast<const bf16*>(blob + h.off_U);
  long long tot = (long long)T * ld;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < tot; i += (long long)gridDim.x * blockDim.x) {
    long long t = i / ld, j = i - t * ld;
    out[u * sunit + i] = j < h.r_T ? src[t * h.r_T + j] : __float2bfloat16_rn(0.f);
  }
}

// per-unit sums of squares of X and of X - Y over one of K / V (grid (nblk, groups));
// partial sums land at part[(unit * nblk + block) * 2 + {0, 1}] with unit = 2 g + kv
template <typename TX, typename TY>
__global__ void frob_partial_kernel(const TX* X, const TY* Y, long long n_per_unit, int kv, double* part, int nblk) {
  const int g = blockIdx.y, u = 2 * g + kv;
  __shared__ double s1[256], s2[256];
  double a = 0.0, b = 0.0;
  const TX* x = X + (long long)g * n_per_unit;
  const TY* y = Y ? Y + (long long)g * n_per_unit : nullptr;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n_per_unit; i += (long long)nblk * blockDim.x) {
    double xv = (double)ld_as_float(x + i);
    a += xv * xv;
    if (y) {
      double d = xv - (double)ld_as_float(y + i);
      b += d * d;
    }
  }
  s1[threadIdx.x] = a;
  s2[threadIdx.x] = b;
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

__global__ void frob_final_kernel(const double* part, int nunits, int nblk, double* sq) {
  int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= nunits * 2) return;
  int u = i >> 1, w = i & 1;
  double acc = 0.0;
  for (int b = 0; b < nblk; ++b) acc += part[((long long)u * nblk + b) * 2 + w];
  sq[i] = acc;
}

// ---------------------------------------------------------------------------------------
// FP32-pipe rate probe (measurement only): every thread runs `iters` rounds of FP32_CHAINS
// independent fused multiply-add chains, scalar (FFMA) or on packed pairs (FFMA2, two lanes'
// worth of FMAs per instruction).  The chains start at 1 and contract towards 1, so no value
// overflows or goes subnormal; one value per thread is stored only when it is impossible, so
// the work is kept without memory traffic.
// ---------------------------------------------------------------------------------------
constexpr int FP32_CHAINS = 8;
__global__ void __launch_bounds__(256) fma_probe_kernel(float* sink, int iters, int packed, float a, float b) {
  if (packed) {
    float2 x[FP32_CHAINS];
#pragma unroll
    for (int i = 0; i < FP32_CHAINS; ++i) x[i] = make_float2(1.f + i * 1e-3f, 1.f - i * 1e-3f);
    const float2 a2 = make_float2(a, a), b2 = make_float2(b, b);
    for (int it = 0; it < iters; ++it)
#pragma unroll
      for (int i = 0; i < FP32_CHAINS; ++i) x[i] = __ffma2_rn(x[i], a2, b2);
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < FP32_CHAINS; ++i) s += x[i].x + x[i].y;
    if (s == -1.f) sink[blockIdx.x * blockDim.x + threadIdx.x] = s;
  } else {
    float x[FP32_CHAINS];
#pragma unroll
    for (int i = 0; i < FP32_CHAINS; ++i) x[i] = 1.f + i * 1e-3f;
    for (int it = 0; it < iters; ++it)
#pragma unroll
      for (int i = 0; i < FP32_CHAINS; ++i) x[i] = fmaf(x[i], a, b);
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < FP32_CHAINS; ++i) s += x[i];
    if (s == -1.f) sink[blockIdx.x * blockDim.x + threadIdx.x] = s;
  }
}

}  // namespace jolt

namespace jolt {
// Symmetric Gram from the tensor-core partial products: G[u][i * gld + j] (fp64, i, j < k) =
// sum over the nsplit partial slots s of part[u][s] at the upper entry (min(i,j), max(i,j)),
// added in fp64 (only the tiles on and above the diagonal were computed).
__global__ void reduce_upper_sym_kernel(const float* part, double* G, int nbatch, int nsplit, int k, long long gld) {
  const long long per = (long long)k * k, n = (long long)nbatch * per;
  for (long long idx = blockIdx.x * (long long)blockDim.x + threadIdx.x; idx < n;
       idx += (long long)gridDim.x * blockDim.x) {
    const int u = (int)(idx / per);
    const long long r = idx - u * per;
    const int i = (int)(r / k), j = (int)(r - (long long)i * k);
    const int a = i < j ? i : j, b = i < j ? j : i;
    const float* p = part + (long long)u * nsplit * k * gld + (long long)a * gld + b;
    double s = 0.0;
    for (int q = 0; q < nsplit; ++q) s += (double)p[(long long)q * k * gld];
    G[(long long)u * k * gld + (long long)i * gld + j] = s;
  }
}
}  // namespace jolt

namespace jolt {
// ---------------------------------------------------------------------------------------
// Rotated reconstruction operator in fp64:  P'[b][i][:] = bf16_rn( (C_b[i][:rD] W_u[:, :rD]^T)
// diag(sigma_u) H_D / sqrt(D) ), every step in fp64 (products of bf16 operands, fp64 sums,
// the Walsh-Hadamard butterflies in the order of strides 1, 2, ..., D/2, the division by
// sqrt(D)) and one round-to-nearest-even to 8 significant bits at the end.  Only the sums'
// order differs from a plain fp64 evaluation, so the bf16 result equals the exactly rounded
// operator except at ties closer than about 1e-16 relative.
// grid (ceil(rT / 32), batch entries); 256 threads; entry b uses W of unit u = umap[b / S].
// ---------------------------------------------------------------------------------------
__device__ __forceinline__ bf16 bf16_rn_from_f64(double x) {
  // round to 8 significant bits (quantum at least 2^-133, the bf16 subnormal step) with ties
  // to even, then the now exact conversion
  if (x == 0.0 || !isfinite(x)) return __float2bfloat16_rn((float)x);
  int e;
  (void)frexp(x, &e);                 // x = m 2^e, 0.5 <= |m| < 1
  const int qe = e - 8 > -133 ? e - 8 : -133;
  const double y = rint(ldexp(x, -qe));
  return __float2bfloat16_rn((float)ldexp(y, qe));
}

constexpr int PX_ROWS = 32;
template <int D>
__global__ void __launch_bounds__(256) pmat_exact_kernel(const bf16* C, long long ldC, long long sC, int rT, int rD,
                                                         const bf16* W, long long ldW, long long sW, int S,
                                                         const int* umap, uint64_t seed, bf16* out, long long sOut) {
  constexpr int CPT = D >= 32 ? D / 32 : 1;   // columns per thread (and per lane in the rotation)
  constexpr int LANES = D / CPT;              // lanes that hold columns (32, or D when D < 32)
  constexpr int CS_BYTES = PX_ROWS * (128 + 8) * 2, WT_BYTES = 128 * (D + 8) * 2, PS_BYTES = PX_ROWS * (D + 1) * 8;
  constexpr int BYTES = CS_BYTES + WT_BYTES > PS_BYTES ? CS_BYTES + WT_BYTES : PS_BYTES;
  __shared__ __align__(16) unsigned char px_sm[BYTES];
  auto cs = reinterpret_cast<bf16(*)[128 + 8]>(px_sm);                 // C rows of the tile
  auto wt = reinterpret_cast<bf16(*)[D + 8]>(px_sm + CS_BYTES);        // W^T: wt[q][d]
  auto ps = reinterpret_cast<double(*)[D + 1]>(px_sm);                 // the products (after the GEMM)
  const int b = blockIdx.y, i0 = blockIdx.x * PX_ROWS, tid = threadIdx.x;
  const int u = umap[b / S];
  const bf16* Cb = C + (long long)b * sC;
  const bf16* Wu = W + (long long)(b / S) * sW;
  for (int idx = tid; idx < PX_ROWS * rD; idx += 256) {
    const int r = idx / rD, q = idx - r * rD;
    cs[r][q] = (i0 + r < rT) ? Cb[(long long)(i0 + r) * ldC + q] : __float2bfloat16_rn(0.f);
  }
  for (int idx = tid; idx < D * rD; idx += 256) {
    const int d = idx / rD, q = idx - d * rD;
    wt[q][d] = Wu[(long long)d * ldW + q];
  }
  __syncthreads();
  const int rg = tid >> 5, cg = tid & 31;   // rows 4 rg .. 4 rg + 3, columns CPT cg .. + CPT - 1
  double acc[4][CPT];
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int e = 0; e < CPT; ++e) acc[r][e] = 0.0;
  for (int q = 0; q < rD && cg < LANES; ++q) {
    double cv[4], wv[CPT];
#pragma unroll
    for (int r = 0; r < 4; ++r) cv[r] = (double)__bfloat162float(cs[4 * rg + r][q]);
#pragma unroll
    for (int e = 0; e < CPT; ++e) wv[e] = (double)__bfloat162float(wt[q][CPT * cg + e]);
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int e = 0; e < CPT; ++e) acc[r][e] = fma(cv[r], wv[e], acc[r][e]);
  }
  __syncthreads();   // ps overlays cs and wt
  if (cg < LANES)
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int e = 0; e < CPT; ++e) ps[4 * rg + r][CPT * cg + e] = acc[r][e];
  __syncthreads();
  // rotation: warp w takes rows 4w .. 4w + 3, lane l holds columns CPT l .. CPT l + CPT - 1
  const int lane = tid & 31, warp = tid >> 5;
  double sg[CPT];
#pragma unroll
  for (int e = 0; e < CPT; ++e) sg[e] = lane < LANES ? (double)rotation_sign(seed, u, CPT * lane + e) : 0.0;
  const double rs = sqrt((double)D);
  for (int rr = 0; rr < 4; ++rr) {
    const int r = 4 * warp + rr;
    double v[CPT];
#pragma unroll
    for (int e = 0; e < CPT; ++e) v[e] = lane < LANES ? ps[r][CPT * lane + e] * sg[e] : 0.0;
#pragma unroll
    for (int h = 1; h < CPT; h <<= 1)
#pragma unroll
      for (int e = 0; e < CPT; ++e)
        if (!(e & h)) {
          const double a = v[e], c = v[e + h];
          v[e] = a + c;
          v[e + h] = a - c;
        }
#pragma unroll
    for (int hl = 1; hl < LANES; hl <<= 1) {
      const bool upper = (lane & hl) != 0;
#pragma unroll
      for (int e = 0; e < CPT; ++e) {
        const double mine = v[e], other = __shfl_xor_sync(0xffffffffu, mine, hl);
        v[e] = upper ? other - mine : mine + other;
      }
    }
    if (i0 + r < rT && lane < LANES) {
      bf16* o = out + (long long)b * sOut + (long long)(i0 + r) * D + CPT * lane;
#pragma unroll
      for (int e = 0; e < CPT; ++e) o[e] = bf16_rn_from_f64(v[e] / rs);
    }
  }
}
}  // namespace jolt
