// Host side of the JoLT C ABI: argument checks, workspace plan and launch sequences.
#include <cusolverDn.h>

#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "jolt.h"
#include "common.cuh"
#include "gemm.cuh"
#include "kernels.cuh"
#include "misc.cuh"

using namespace jolt;

namespace {

thread_local std::string g_err;

jolt_status fail(jolt_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  g_err = buf;
  return s;
}

#define CUDA_TRY(x)                                                                         \
  do {                                                                                      \
    cudaError_t e_ = (x);                                                                   \
    if (e_ != cudaSuccess) return fail(JOLT_ERR_CUDA, "%s: %s", #x, cudaGetErrorString(e_)); \
  } while (0)
#define SOLVER_TRY(x)                                                               \
  do {                                                                              \
    cusolverStatus_t s_ = (x);                                                      \
    if (s_ != CUSOLVER_STATUS_SUCCESS) return fail(JOLT_ERR_CUDA, "%s: cusolver status %d", #x, (int)s_); \
  } while (0)
#define JTRY(x)                    \
  do {                             \
    jolt_status j_ = (x);          \
    if (j_ != JOLT_OK) return j_;  \
  } while (0)

// ------------------------------------------------------------------------------------------
// cuSOLVER handle (one per thread and device)
// ------------------------------------------------------------------------------------------
struct Solver {
  cusolverDnHandle_t h = nullptr;
  cusolverDnParams_t params = nullptr;
  int device = -1;
  std::vector<char> host_ws;
};
thread_local Solver g_solver;

jolt_status solver_get(cudaStream_t st, Solver** out) {
  int dev = 0;
  CUDA_TRY(cudaGetDevice(&dev));
  if (g_solver.h == nullptr || g_solver.device != dev) {
    if (g_solver.h) {
      cusolverDnDestroyParams(g_solver.params);
      cusolverDnDestroy(g_solver.h);
    }
    SOLVER_TRY(cusolverDnCreate(&g_solver.h));
    SOLVER_TRY(cusolverDnCreateParams(&g_solver.params));
    g_solver.device = dev;
  }
  SOLVER_TRY(cusolverDnSetStream(g_solver.h, st));
  *out = &g_solver;
  return JOLT_OK;
}

// ------------------------------------------------------------------------------------------
// plan: derived sizes and workspace layout
// ------------------------------------------------------------------------------------------
struct Bump {
  size_t off = 0;
  size_t take(size_t bytes) {
    size_t o = off;
    off += (bytes + 255) / 256 * 256;
    return o;
  }
};

struct Plan {
  int nL, H, T, D, Lg, S, G, NU, M, dtype;
  Cands cd;
  int nC, rTmax, rDmax, ldU, ldW, ldC, method, q, k, kp;
  bool m_side;            // exact token factor through the M x M Gram (T > M)
  int gd_split;           // split-K of the feature Gram
  int gt_split;           // split-K of the token Gram
  size_t solver_dev;      // cuSOLVER device workspace
  size_t solver_host;
  // workspace offsets (bytes)
  size_t o_status, o_gd_part, o_gd, o_evals, o_Wf, o_Ws, o_Uf, o_Us, o_core, o_zc, o_ptmp, o_P, o_partial,
      o_table, o_bytes, o_choice, o_lambda, o_hdr, o_umap, o_info, o_solver;
  // token factor scratch (per unit, reused)
  size_t o_gt_part, o_gt, o_vsel, o_lam, o_omega, o_Y, o_Yt, o_Zm, o_Zt, o_h, o_l, o_Bm, o_G;
  size_t ws_total;
  int tiles;
  size_t blob_max;
  // decompress workspace
  size_t d_U, d_W, d_C, d_ptmp, d_P, d_umap, dws_total;
};

int max_in(const int32_t* v, int n) {
  int m = 0;
  for (int i = 0; i < n; ++i) m = v[i] > m ? v[i] : m;
  return m;
}

jolt_status check_list(const int32_t* v, int n, int lo, int hi, const char* name) {
  if (n < 1 || n > JOLT_MAX_CANDIDATES) return fail(JOLT_ERR_INVALID_ARG, "%s: count %d not in [1, 8]", name, n);
  for (int i = 0; i < n; ++i) {
    if (v[i] < lo || v[i] > hi) return fail(JOLT_ERR_INVALID_ARG, "%s[%d] = %d not in [%d, %d]", name, i, v[i], lo, hi);
    if (i && v[i] <= v[i - 1]) return fail(JOLT_ERR_INVALID_ARG, "%s must be strictly ascending", name);
  }
  return JOLT_OK;
}

jolt_status make_plan(const jolt_shape* sh, const jolt_options* op, Plan* p) {
  if (!sh || !op) return fail(JOLT_ERR_INVALID_ARG, "null shape or options");
  if (sh->dtype != JOLT_BF16 && sh->dtype != JOLT_F32) return fail(JOLT_ERR_INVALID_ARG, "dtype %d", sh->dtype);
  if (sh->n_layers < 1 || sh->n_heads < 1 || sh->n_tokens < 1 || sh->layers_per_group < 1)
    return fail(JOLT_ERR_INVALID_ARG, "non-positive dimension");
  const int D = sh->head_dim;
  if (D != 16 && D != 32 && D != 64 && D != 128)
    return fail(JOLT_ERR_UNSUPPORTED_SHAPE, "head_dim %d not in {16, 32, 64, 128}", D);
  if (sh->n_layers % sh->layers_per_group)
    return fail(JOLT_ERR_UNSUPPORTED_SHAPE, "n_layers %% layers_per_group != 0");
  if (sh->n_tokens % 16) return fail(JOLT_ERR_UNSUPPORTED_SHAPE, "n_tokens %d not a multiple of 16", sh->n_tokens);
  p->nL = sh->n_layers;
  p->H = sh->n_heads;
  p->T = sh->n_tokens;
  p->D = D;
  p->Lg = sh->layers_per_group;
  p->S = p->Lg * p->H;
  p->G = p->nL / p->Lg;
  p->NU = 2 * p->G;
  p->M = p->S * D;
  p->dtype = sh->dtype;
  if ((long long)p->S * p->T * D >= (1LL << 40)) return fail(JOLT_ERR_UNSUPPORTED_SHAPE, "unit too large");
  if (op->method != JOLT_EXACT && op->method != JOLT_RANDOMIZED)
    return fail(JOLT_ERR_INVALID_ARG, "method %d", op->method);
  const int rcap = p->T < p->M ? p->T : p->M;
  JTRY(check_list(op->token_ranks, op->n_token_ranks, 1, rcap, "token_ranks"));
  JTRY(check_list(op->feature_ranks, op->n_feature_ranks, 1, D, "feature_ranks"));
  JTRY(check_list(op->bits, op->n_bits, 0, 8, "bits"));
  p->cd.nT = op->n_token_ranks;
  p->cd.nD = op->n_feature_ranks;
  p->cd.nB = op->n_bits;
  for (int i = 0; i < MAXC; ++i) {
    p->cd.rT[i] = i < op->n_token_ranks ? op->token_ranks[i] : 0;
    p->cd.rD[i] = i < op->n_feature_ranks ? op->feature_ranks[i] : 0;
    p->cd.bits[i] = i < op->n_bits ? op->bits[i] : 0;
  }
  p->nC = p->cd.nT * p->cd.nD * p->cd.nB;
  p->rTmax = max_in(op->token_ranks, op->n_token_ranks);
  p->rDmax = max_in(op->feature_ranks, op->n_feature_ranks);
  if (p->rTmax % 8 || p->rDmax % 8)
    return fail(JOLT_ERR_UNSUPPORTED_SHAPE, "largest token / feature rank must be a multiple of 8");
  p->ldU = p->rTmax;
  p->ldW = p->rDmax;
  p->ldC = p->rDmax;
  p->method = op->method;
  p->q = op->power_iters;
  p->k = 0;
  p->kp = 0;
  if (op->method == JOLT_RANDOMIZED) {
    if (op->oversample < 0 || op->power_iters < 0 || op->power_iters > 16)
      return fail(JOLT_ERR_INVALID_ARG, "oversample / power_iters out of range");
    p->k = p->rTmax + op->oversample;
    if (p->k > rcap) return fail(JOLT_ERR_UNSUPPORTED_SHAPE, "sketch width %d exceeds min(T, M) = %d", p->k, rcap);
    p->kp = (int)round_up(p->k, 8);
  }
  p->m_side = p->T > p->M;
  p->tiles = (int)ceil_div(p->T, TROWS);

  // split-K of the Grams (fixed: results do not depend on the device)
  long long rows = (long long)p->S * p->T;
  p->gd_split = (int)ceil_div(rows, 1024);
  if (p->gd_split > 64) p->gd_split = 64;
  p->gt_split = p->m_side ? (int)ceil_div(p->T, 4096) : (p->S < 16 ? p->S : 16);
  if (p->gt_split > 64) p->gt_split = 64;

  // cuSOLVER device workspace: a bound of twice the LAPACK syevd requirement
  // (1 + 6n + 2n^2 doubles) for the largest eigenproblem; the actual need is queried and
  // checked against it at run time, so the plan itself never touches the GPU.
  {
    long long nmax = D;
    if (op->method == JOLT_EXACT) nmax = p->m_side ? p->M : p->T;
    else nmax = p->k > nmax ? p->k : nmax;
    if (nmax < D) nmax = D;
    p->solver_dev = (size_t)(2 * (1 + 6 * nmax + 2 * nmax * nmax) * 8 + (4 << 20));
    p->solver_host = 0;
  }

  const int NU = p->NU, T = p->T, S = p->S, M = p->M;
  Bump b;
  p->o_status = b.take(256);
  p->o_gd_part = b.take((size_t)NU * p->gd_split * D * D * 4);
  p->o_gd = b.take((size_t)NU * D * D * 8);
  {
    long long ntok = op->method == JOLT_EXACT ? (p->m_side ? M : T) : p->kp;
    long long nev = (long long)NU * D > ntok ? (long long)NU * D : ntok;
    p->o_evals = b.take((size_t)nev * 8 + 256);
  }
  p->o_Wf = b.take((size_t)NU * D * p->ldW * 4);
  p->o_Ws = b.take((size_t)NU * D * p->ldW * 2);
  p->o_Uf = b.take((size_t)NU * T * p->ldU * 4);
  p->o_Us = b.take((size_t)NU * T * p->ldU * 2);
  p->o_core = b.take((size_t)NU * S * p->rTmax * p->ldC * 2);
  p->o_zc = b.take((size_t)S * T * p->ldW * 2);                        // per unit, reused
  p->o_ptmp = b.take((size_t)S * p->rTmax * D * 4);                    // per unit, reused
  p->o_P = b.take((size_t)NU * p->cd.nD * S * p->rTmax * D * 2);
  p->o_partial = b.take((size_t)NU * S * p->tiles * p->nC * 8);
  p->o_table = b.take((size_t)NU * p->nC * 8);
  p->o_bytes = b.take((size_t)NU * p->nC * 8);
  p->o_choice = b.take((size_t)NU * 4);
  p->o_lambda = b.take(8);
  p->o_hdr = b.take(64);
  p->o_umap = b.take((size_t)NU * S * 4 + 64);
  p->o_info = b.take(64);
  p->o_solver = b.take(p->solver_dev + 256);
  // token factor scratch
  p->o_gt_part = p->o_gt = p->o_vsel = p->o_lam = p->o_omega = 0;
  p->o_Y = p->o_Yt = p->o_Zm = p->o_Zt = p->o_h = p->o_l = p->o_Bm = p->o_G = 0;
  if (op->method == JOLT_EXACT) {
    long long n = p->m_side ? M : T;
    p->o_gt_part = b.take((size_t)p->gt_split * n * n * 4);
    p->o_gt = b.take((size_t)n * n * 8);
    p->o_lam = b.take((size_t)p->rTmax * 8 + 256);
    if (p->m_side) {
      p->o_vsel = b.take((size_t)M * p->ldU * 4);
      p->o_h = b.take((size_t)M * p->ldU * 2);
      p->o_l = b.take((size_t)M * p->ldU * 2);
      p->o_Yt = b.take((size_t)T * p->ldU * 4);
      p->o_G = b.take((size_t)p->ldU * p->ldU * 8);
    }
  } else {
    const int kp = p->kp;
    long long big = M > T ? M : T;
    p->o_omega = b.take((size_t)M * kp * 2);
    p->o_Y = b.take((size_t)T * kp * 4);
    p->o_Yt = b.take((size_t)big * kp * 4);
    p->o_Zm = b.take((size_t)M * kp * 4);
    p->o_h = b.take((size_t)big * kp * 2);
    p->o_l = b.take((size_t)big * kp * 2);
    p->o_Bm = b.take((size_t)kp * M * 4);
    p->o_G = b.take((size_t)kp * kp * 8);
    p->o_vsel = b.take((size_t)kp * p->ldU * 4);
  }
  p->ws_total = b.off;

  // largest possible blob
  unsigned long long mx = 0;
  for (int i = 0; i < p->cd.nT; ++i)
    for (int j = 0; j < p->cd.nD; ++j)
      for (int l = 0; l < p->cd.nB; ++l) {
        unsigned long long v = unit_payload_bytes(T, D, S, p->cd.rT[i], p->cd.rD[j], p->cd.bits[l]);
        mx = v > mx ? v : mx;
      }
  p->blob_max = 64 + 64 * (size_t)NU + (size_t)NU * mx;

  Bump d;
  d.take(256);
  p->d_U = d.take((size_t)NU * T * p->ldU * 2);
  p->d_W = d.take((size_t)NU * D * p->ldW * 2);
  p->d_C = d.take((size_t)NU * S * p->rTmax * p->ldC * 2);
  p->d_ptmp = d.take((size_t)S * p->rTmax * D * 4);
  p->d_P = d.take((size_t)NU * S * p->rTmax * D * 2);
  p->d_umap = d.take((size_t)NU * S * 4 + 64);
  p->dws_total = d.off;
  return JOLT_OK;
}

// ------------------------------------------------------------------------------------------
// GEMM dispatch on operand element types (0 bf16, 1 fp32, 2 fp64)
// ------------------------------------------------------------------------------------------
jolt_status gemm(const GemmParams& p, int ta, int tb, cudaStream_t st) {
  cudaError_t e;
  const bool dacc = p.c_type == 2;
  if (ta == 0 && tb == 0) e = launch_gemm_bf16(p, st);
#define GEMM_CASE(A, B, TA, TB)                                                              \
  else if (ta == A && tb == B) e = dacc ? launch_gemm_simt<TA, TB, double>(p, st)           \
                                        : launch_gemm_simt<TA, TB, float>(p, st);
  GEMM_CASE(1, 1, float, float)
  GEMM_CASE(1, 0, float, bf16)
  GEMM_CASE(0, 1, bf16, float)
  GEMM_CASE(1, 2, float, double)
  GEMM_CASE(2, 1, double, float)
  GEMM_CASE(2, 2, double, double)
#undef GEMM_CASE
  else return fail(JOLT_ERR_INVALID_ARG, "gemm type combination %d/%d", ta, tb);
  if (e != cudaSuccess) return fail(JOLT_ERR_CUDA, "gemm launch: %s", cudaGetErrorString(e));
  return JOLT_OK;
}

unsigned grid1d(long long n, int threads = 256) {
  long long g = ceil_div(n, threads);
  if (g > 148 * 32) g = 148 * 32;
  if (g < 1) g = 1;
  return (unsigned)g;
}

struct Ctx {
  const Plan& p;
  unsigned char* ws;
  cudaStream_t st;
  const void* k;
  const void* v;
  uint64_t seed;
  template <typename T>
  T* at(size_t off) const { return reinterpret_cast<T*>(ws + off); }
  uint32_t* status() const { return at<uint32_t>(p.o_status); }
  CacheView view() const {
    CacheView c;
    c.k = k;
    c.v = v;
    c.dtype = p.dtype;
    c.n_layers = p.nL;
    c.H = p.H;
    c.T = p.T;
    c.D = p.D;
    c.Lg = p.Lg;
    c.S = p.S;
    c.unit_elems = (long long)p.S * p.T * p.D;
    return c;
  }
};

// X_(T) as operand: (row t, col (s,d))  -> offset s*T*D + t*D + d
GemmOperand xt_rowmajor(const Ctx& c, const void* x) {
  GemmOperand o;
  o.ptr = x;
  o.kmajor = true;       // as A (T x M): contiguous along the M index inside a slice
  o.ld = c.p.D;
  o.kblk = c.p.D;
  o.skblk = (long long)c.p.T * c.p.D;
  return o;
}

// ------------------------------------------------------------------------------------------
// symmetric eigen solve (cuSOLVER, fp64), one matrix at a time
// ------------------------------------------------------------------------------------------
// the solver's device workspace must fit the plan's bound; host workspace grows on demand
jolt_status solver_ws(const Ctx& c, Solver* s, size_t dv, size_t hv, void** host) {
  if (dv > c.p.solver_dev)
    return fail(JOLT_ERR_WORKSPACE_TOO_SMALL, "cuSOLVER needs %zu device bytes, plan holds %zu", dv, c.p.solver_dev);
  if (s->host_ws.size() < hv) s->host_ws.resize(hv);
  *host = hv ? s->host_ws.data() : nullptr;
  return JOLT_OK;
}

jolt_status sym_eig(const Ctx& c, double* A, int64_t n, double* w) {
  Solver* s = nullptr;
  JTRY(solver_get(c.st, &s));
  size_t dv = 0, hv = 0;
  SOLVER_TRY(cusolverDnXsyevd_bufferSize(s->h, s->params, CUSOLVER_EIG_MODE_VECTOR, CUBLAS_FILL_MODE_LOWER, n,
                                         CUDA_R_64F, A, n, CUDA_R_64F, w, CUDA_R_64F, &dv, &hv));
  void* host = nullptr;
  JTRY(solver_ws(c, s, dv, hv, &host));
  SOLVER_TRY(cusolverDnXsyevd(s->h, s->params, CUSOLVER_EIG_MODE_VECTOR, CUBLAS_FILL_MODE_LOWER, n, CUDA_R_64F, A, n,
                              CUDA_R_64F, w, CUDA_R_64F, c.at<void>(c.p.o_solver), dv, host, hv,
                              c.at<int>(c.p.o_info)));
  info_check_kernel<<<1, 32, 0, c.st>>>(c.at<int>(c.p.o_info), 1, c.status(), DEV_ERR_FACTOR);
  CUDA_TRY(cudaGetLastError());
  return JOLT_OK;
}

// Q = Y R^{-1} with R^T R = Y^T Y (Cholesky QR), twice; Y is m x k fp32 row-major (ld),
// overwritten by Q.  tmp: m x ld fp32; G: k x k fp64 (ld = gld)
jolt_status cholqr2(const Ctx& c, float* Y, int64_t m, int k, int ld, float* tmp, double* G, int gld) {
  Solver* s = nullptr;
  JTRY(solver_get(c.st, &s));
  size_t dv1 = 0, hv1 = 0, dv2 = 0, hv2 = 0;
  SOLVER_TRY(cusolverDnXpotrf_bufferSize(s->h, s->params, CUBLAS_FILL_MODE_LOWER, k, CUDA_R_64F, G, gld, CUDA_R_64F,
                                         &dv1, &hv1));
  SOLVER_TRY(cusolverDnXtrtri_bufferSize(s->h, CUBLAS_FILL_MODE_LOWER, CUBLAS_DIAG_NON_UNIT, k, CUDA_R_64F, G, gld,
                                         &dv2, &hv2));
  void* host1 = nullptr;
  JTRY(solver_ws(c, s, dv1 > dv2 ? dv1 : dv2, hv1 > hv2 ? hv1 : hv2, &host1));
  for (int pass = 0; pass < 2; ++pass) {
    CUDA_TRY(cudaMemsetAsync(G, 0, (size_t)gld * gld * 8, c.st));
    CUDA_TRY(cudaMemsetAsync(tmp, 0, (size_t)m * ld * 4, c.st));
    GemmParams g;
    g.M = k;
    g.N = k;
    g.K = (int)m;
    g.A.ptr = Y;
    g.A.kmajor = false;
    g.A.ld = ld;
    g.B.ptr = Y;
    g.B.kmajor = false;
    g.B.ld = ld;
    g.C = G;
    g.ldc = gld;
    g.c_type = 2;
    JTRY(gemm(g, 1, 1, c.st));
    SOLVER_TRY(cusolverDnXpotrf(s->h, s->params, CUBLAS_FILL_MODE_LOWER, k, CUDA_R_64F, G, gld, CUDA_R_64F,
                                c.at<void>(c.p.o_solver), dv1, host1, hv1, c.at<int>(c.p.o_info)));
    info_check_kernel<<<1, 32, 0, c.st>>>(c.at<int>(c.p.o_info), 1, c.status(), DEV_ERR_FACTOR);
    SOLVER_TRY(cusolverDnXtrtri(s->h, CUBLAS_FILL_MODE_LOWER, CUBLAS_DIAG_NON_UNIT, k, CUDA_R_64F, G, gld,
                                c.at<void>(c.p.o_solver), dv2, host1, hv2, c.at<int>(c.p.o_info)));
    info_check_kernel<<<1, 32, 0, c.st>>>(c.at<int>(c.p.o_info), 1, c.status(), DEV_ERR_FACTOR);
    tril_zero_kernel<<<grid1d((long long)k * k), 256, 0, c.st>>>(G, k, gld, 0, 1);
    // Q = Y L^{-T}: B(kk, n) = Linv(n, kk) stored column-major at n + kk*gld
    GemmParams q;
    q.M = (int)m;
    q.N = k;
    q.K = k;
    q.A.ptr = Y;
    q.A.kmajor = true;
    q.A.ld = ld;
    q.B.ptr = G;
    q.B.kmajor = false;
    q.B.ld = gld;
    q.C = tmp;
    q.ldc = ld;
    q.c_type = 0;
    JTRY(gemm(q, 1, 2, c.st));
    CUDA_TRY(cudaMemcpyAsync(Y, tmp, (size_t)m * ld * 4, cudaMemcpyDeviceToDevice, c.st));
  }
  CUDA_TRY(cudaGetLastError());
  return JOLT_OK;
}

// C (m x n fp32) = X-product with an fp32 operand F given as bf16 hi + lo splits, or
// directly when the cache is fp32.  Operand roles are given by the caller.
jolt_status gemm_xf(const Ctx& c, GemmParams g, bool f_is_A, const float* F, long long nF, int fld_unused) {
  (void)fld_unused;
  const bool xbf = c.p.dtype == JOLT_BF16;
  if (!xbf) {
    if (f_is_A) g.A.ptr = F;
    else g.B.ptr = F;
    return gemm(g, f_is_A ? 1 : 1, 1, c.st);
  }
  bf16* hi = c.at<bf16>(c.p.o_h);
  bf16* lo = c.at<bf16>(c.p.o_l);
  split_bf16_kernel<<<grid1d(nF), 256, 0, c.st>>>(F, hi, lo, nF);
  CUDA_TRY(cudaGetLastError());
  GemmParams g1 = g, g2 = g;
  if (f_is_A) {
    g1.A.ptr = hi;
    g2.A.ptr = lo;
  } else {
    g1.B.ptr = hi;
    g2.B.ptr = lo;
  }
  g1.beta = 0.f;
  g2.beta = 1.f;
  JTRY(gemm(g1, 0, 0, c.st));
  JTRY(gemm(g2, 0, 0, c.st));
  return JOLT_OK;
}

int xtype(const Ctx& c) { return c.p.dtype == JOLT_BF16 ? 0 : 1; }

// ------------------------------------------------------------------------------------------
// stage 1a: feature factor W of every unit
// ------------------------------------------------------------------------------------------
jolt_status run_feature_factor(const Ctx& c, float* Wf, long long ldWf, bf16* Ws, long long ldWs) {
  const Plan& p = c.p;
  const int D = p.D;
  float* part = c.at<float>(p.o_gd_part);
  const long long rows = (long long)p.S * p.T;
  const int kchunk = (int)round_up(ceil_div(rows, p.gd_split), 32);
  for (int kv = 0; kv < 2; ++kv) {
    GemmParams g;
    g.M = D;
    g.N = D;
    g.K = (int)rows;
    g.batch = p.G;
    g.A.ptr = kv ? c.v : c.k;
    g.A.kmajor = false;
    g.A.ld = D;
    g.A.sbatch = rows * D;
    g.B = g.A;
    g.C = part + (size_t)kv * p.gd_split * D * D;
    g.ldc = D;
    g.sbatchC = 2LL * p.gd_split * D * D;
    g.ssplitC = (long long)D * D;
    g.splits = p.gd_split;
    g.kchunk = kchunk;
    g.c_type = 0;
    JTRY(gemm(g, xtype(c), xtype(c), c.st));
  }
  double* G = c.at<double>(p.o_gd);
  reduce_splits_kernel<float><<<grid1d((long long)p.NU * D * D), 256, 0, c.st>>>(part, G, p.NU, p.gd_split,
                                                                                 (long long)D * D);
  gram_diag_check_kernel<<<p.NU, 128, 0, c.st>>>(G, D, p.NU, c.status());
  CUDA_TRY(cudaGetLastError());
  double* w = c.at<double>(p.o_evals);
  for (int u = 0; u < p.NU; ++u) {
    JTRY(sym_eig(c, G + (size_t)u * D * D, D, w + (size_t)u * D));
  }
  eig_select_kernel<<<dim3(p.rDmax, p.NU), 128, 0, c.st>>>(w, G, D, D, D, (long long)D * D, p.rDmax, Wf, Ws, ldWf,
                                                           (long long)D * ldWf, nullptr);
  CUDA_TRY(cudaGetLastError());
  (void)ldWs;
  return JOLT_OK;
}

// ------------------------------------------------------------------------------------------
// stage 1b: token factor U of one unit (exact or randomized)
// ------------------------------------------------------------------------------------------
jolt_status run_token_exact(const Ctx& c, int u, float* Uf, long long ldUf) {
  const Plan& p = c.p;
  const int T = p.T, M = p.M, D = p.D;
  const void* X = c.view().unit_ptr(u);
  const int n = p.m_side ? M : T;
  float* part = c.at<float>(p.o_gt_part);
  double* G = c.at<double>(p.o_gt);
  GemmParams g;
  g.C = part;
  g.ldc = n;
  g.c_type = 0;
  g.splits = p.gt_split;
  g.ssplitC = (long long)n * n;
  if (!p.m_side) {
    g.M = T;
    g.N = T;
    g.K = M;
    g.A = xt_rowmajor(c, X);
    g.B = g.A;  // B = X_(T)^T is K-major with the same addressing
    g.kchunk = (int)round_up(ceil_div(M, p.gt_split), D);
  } else {
    g.M = M;
    g.N = M;
    g.K = T;
    GemmOperand a;
    a.ptr = X;
    a.kmajor = false;     // contiguous along the (s,d) index inside a slice
    a.ld = D;             // t stride
    a.xblk = D;
    a.sxblk = (long long)T * D;
    g.A = a;
    g.B = a;
    g.kchunk = (int)round_up(ceil_div(T, p.gt_split), 32);
  }
  JTRY(gemm(g, xtype(c), xtype(c), c.st));
  reduce_splits_kernel<float><<<grid1d((long long)n * n), 256, 0, c.st>>>(part, G, 1, p.gt_split, (long long)n * n);
  CUDA_TRY(cudaGetLastError());
  double* w = c.at<double>(p.o_evals);
  JTRY(sym_eig(c, G, n, w));
  if (!p.m_side) {
    eig_select_kernel<<<dim3(p.rTmax, 1), 256, 0, c.st>>>(w, G, n, n, 0, 0, p.rTmax, Uf, nullptr, ldUf, 0, nullptr);
    CUDA_TRY(cudaGetLastError());
    return JOLT_OK;
  }
  // T > M: U = X_(T) V Lambda^{-1/2}, then Cholesky-QR re-orthonormalisation
  float* V = c.at<float>(p.o_vsel);
  double* lam = c.at<double>(p.o_lam);
  eig_select_kernel<<<dim3(p.rTmax, 1), 256, 0, c.st>>>(w, G, n, n, 0, 0, p.rTmax, V, nullptr, p.ldU, 0, lam);
  scale_cols_kernel<<<grid1d((long long)M * p.rTmax), 256, 0, c.st>>>(V, lam, M, p.rTmax, p.ldU, 0, 0, 1, c.status());
  CUDA_TRY(cudaGetLastError());
  GemmParams y;
  y.M = T;
  y.N = p.rTmax;
  y.K = M;
  y.A = xt_rowmajor(c, X);
  y.B.kmajor = false;
  y.B.ld = p.ldU;
  y.C = Uf;
  y.ldc = ldUf;
  y.c_type = 0;
  if (xtype(c) == 0) JTRY(gemm_xf(c, y, false, V, (long long)M * p.ldU, p.ldU));
  else {
    y.B.ptr = V;
    JTRY(gemm(y, 1, 1, c.st));
  }
  JTRY(cholqr2(c, Uf, T, p.rTmax, (int)ldUf, c.at<float>(p.o_Yt), c.at<double>(p.o_G), p.ldU));
  return JOLT_OK;
}

jolt_status run_token_randomized(const Ctx& c, int u, float* Uf, long long ldUf) {
  const Plan& p = c.p;
  const int T = p.T, M = p.M, D = p.D, k = p.k, kp = p.kp;
  const void* X = c.view().unit_ptr(u);
  bf16* Om = c.at<bf16>(p.o_omega);
  float* Y = c.at<float>(p.o_Y);
  float* tmp = c.at<float>(p.o_Yt);
  float* Z = c.at<float>(p.o_Zm);
  double* G = c.at<double>(p.o_G);
  CUDA_TRY(cudaMemsetAsync(Y, 0, (size_t)T * kp * 4, c.st));
  CUDA_TRY(cudaMemsetAsync(Z, 0, (size_t)M * kp * 4, c.st));
  omega_kernel<<<grid1d((long long)M * kp), 256, 0, c.st>>>(Om, M, k, kp, 0, c.seed, u, 1);
  CUDA_TRY(cudaGetLastError());
  // Y = X_(T) Omega
  GemmParams g;
  g.M = T;
  g.N = k;
  g.K = M;
  g.A = xt_rowmajor(c, X);
  g.B.ptr = Om;
  g.B.kmajor = false;
  g.B.ld = kp;
  g.C = Y;
  g.ldc = kp;
  g.c_type = 0;
  JTRY(gemm(g, xtype(c), 0, c.st));
  JTRY(cholqr2(c, Y, T, k, kp, tmp, G, kp));
  // X_(T)^T as A (M x T): contiguous along (s,d) inside a slice, t stride D
  GemmOperand xtT;
  xtT.ptr = X;
  xtT.kmajor = false;
  xtT.ld = D;
  xtT.xblk = D;
  xtT.sxblk = (long long)T * D;
  for (int it = 0; it < p.q; ++it) {
    GemmParams z;
    z.M = M;
    z.N = k;
    z.K = T;
    z.A = xtT;
    z.B.kmajor = false;
    z.B.ld = kp;
    z.C = Z;
    z.ldc = kp;
    z.c_type = 0;
    JTRY(gemm_xf(c, z, false, Y, (long long)T * kp, kp));
    JTRY(cholqr2(c, Z, M, k, kp, tmp, G, kp));
    GemmParams y = g;
    y.B.kmajor = false;
    y.B.ld = kp;
    JTRY(gemm_xf(c, y, false, Z, (long long)M * kp, kp));
    JTRY(cholqr2(c, Y, T, k, kp, tmp, G, kp));
  }
  // B = Q^T X_(T) (k x M), then the k x k matrix B B^T
  float* Bm = c.at<float>(p.o_Bm);
  GemmParams bq;
  bq.M = k;
  bq.N = M;
  bq.K = T;
  bq.A.kmajor = false;  // A(i, t) = Q[t][i]
  bq.A.ld = kp;
  GemmOperand xn;       // B(t, (s,d)) = X[s][t][d]: contiguous along (s,d) inside a slice
  xn.ptr = X;
  xn.kmajor = false;
  xn.ld = D;
  xn.xblk = D;
  xn.sxblk = (long long)T * D;
  bq.B = xn;
  bq.C = Bm;
  bq.ldc = M;
  bq.c_type = 0;
  JTRY(gemm_xf(c, bq, true, Y, (long long)T * kp, kp));
  CUDA_TRY(cudaMemsetAsync(G, 0, (size_t)kp * kp * 8, c.st));
  GemmParams gg;
  gg.M = k;
  gg.N = k;
  gg.K = M;
  gg.A.ptr = Bm;
  gg.A.kmajor = true;
  gg.A.ld = M;
  gg.B.ptr = Bm;
  gg.B.kmajor = true;
  gg.B.ld = M;
  gg.C = G;
  gg.ldc = k;
  gg.c_type = 2;
  JTRY(gemm(gg, 1, 1, c.st));
  double* w = c.at<double>(p.o_evals);
  JTRY(sym_eig(c, G, k, w));
  float* V = c.at<float>(p.o_vsel);
  eig_select_kernel<<<dim3(p.rTmax, 1), 256, 0, c.st>>>(w, G, k, k, 0, 0, p.rTmax, V, nullptr, p.ldU, 0, nullptr);
  CUDA_TRY(cudaGetLastError());
  // U = Q V
  GemmParams uq;
  uq.M = T;
  uq.N = p.rTmax;
  uq.K = k;
  uq.A.ptr = Y;
  uq.A.kmajor = true;
  uq.A.ld = kp;
  uq.B.ptr = V;
  uq.B.kmajor = false;
  uq.B.ld = p.ldU;
  uq.C = Uf;
  uq.ldc = ldUf;
  uq.c_type = 0;
  JTRY(gemm(uq, 1, 1, c.st));
  return JOLT_OK;
}

jolt_status run_factor(const Ctx& c, float* Uf, long long ldUf, float* Wf, long long ldWf, bf16* Us, bf16* Ws) {
  const Plan& p = c.p;
  CUDA_TRY(cudaMemsetAsync(c.status(), 0, 4, c.st));
  JTRY(run_feature_factor(c, Wf, ldWf, Ws, ldWf));
  for (int u = 0; u < p.NU; ++u) {
    float* U = Uf + (size_t)u * p.T * ldUf;
    if (p.method == JOLT_EXACT) JTRY(run_token_exact(c, u, U, ldUf));
    else JTRY(run_token_randomized(c, u, U, ldUf));
  }
  // sign convention of the token factor columns (the randomized and back-projected routes
  // need it; for the eigenvector route it is already in place) and the bf16 copy
  col_sign_fix_kernel<<<dim3(p.rTmax, p.NU), 256, 0, c.st>>>(Uf, ldUf, (long long)p.T * ldUf, p.T, p.rTmax, Us,
                                                             ldUf, (long long)p.T * ldUf);
  CUDA_TRY(cudaGetLastError());
  return JOLT_OK;
}

// ------------------------------------------------------------------------------------------
// stage 2: stored core, rotated reconstruction operators and the distortion table
// ------------------------------------------------------------------------------------------
jolt_status run_core(const Ctx& c, const bf16* Us, long long ldU, const bf16* Ws, long long ldW, bf16* core) {
  const Plan& p = c.p;
  const int T = p.T, D = p.D, S = p.S;
  bf16* Zc = c.at<bf16>(p.o_zc);
  for (int u = 0; u < p.NU; ++u) {
    const void* X = c.view().unit_ptr(u);
    // Z = bf16(X_(D) W_s)   ((S T) x rDmax)
    GemmParams z;
    z.M = S * T;
    z.N = p.rDmax;
    z.K = D;
    z.A.ptr = X;
    z.A.kmajor = true;
    z.A.ld = D;
    z.B.ptr = Ws + (size_t)u * D * ldW;
    z.B.kmajor = false;
    z.B.ld = ldW;
    z.C = Zc;
    z.ldc = p.ldW;
    z.c_type = 1;
    JTRY(gemm(z, xtype(c), 0, c.st));
    // C_s = bf16(U_s^T Z_s) per slice  (rTmax x rDmax)
    GemmParams cc;
    cc.M = p.rTmax;
    cc.N = p.rDmax;
    cc.K = T;
    cc.batch = S;
    cc.A.ptr = Us + (size_t)u * T * ldU;
    cc.A.kmajor = false;
    cc.A.ld = ldU;
    cc.A.sbatch = 0;
    cc.B.ptr = Zc;
    cc.B.kmajor = false;
    cc.B.ld = p.ldW;
    cc.B.sbatch = (long long)T * p.ldW;
    cc.C = core + (size_t)u * S * p.rTmax * p.ldC;
    cc.ldc = p.ldC;
    cc.sbatchC = (long long)p.rTmax * p.ldC;
    cc.c_type = 1;
    JTRY(gemm(cc, 0, 0, c.st));
  }
  return JOLT_OK;
}

template <int D>
void launch_rotate_rows(const float* in, bf16* out, long long nrows, long long rows_per_unit, const int* umap,
                        uint64_t seed, cudaStream_t st) {
  rotate_rows_kernel<D><<<(unsigned)ceil_div(nrows, 64), 64, 0, st>>>(in, out, nrows, rows_per_unit, umap, seed);
}

jolt_status rotate_rows(const Ctx& c, const float* in, bf16* out, long long nrows, long long rows_per_unit,
                        const int* umap) {
  switch (c.p.D) {
    case 16: launch_rotate_rows<16>(in, out, nrows, rows_per_unit, umap, c.seed, c.st); break;
    case 32: launch_rotate_rows<32>(in, out, nrows, rows_per_unit, umap, c.seed, c.st); break;
    case 64: launch_rotate_rows<64>(in, out, nrows, rows_per_unit, umap, c.seed, c.st); break;
    default: launch_rotate_rows<128>(in, out, nrows, rows_per_unit, umap, c.seed, c.st); break;
  }
  CUDA_TRY(cudaGetLastError());
  return JOLT_OK;
}

// P'(r_D) for one unit: bf16(rotate(C_s[:, :rT, :r_D] W_s[:, :r_D]^T)), rows rT of every slice
// out layout [S][rTslice][D] (rows >= rT of a slice are not written meaningfully)
jolt_status pmat_unit(const Ctx& c, int u, const bf16* core_u, long long ldC, int rT, int rTslice, const bf16* Ws_u,
                      long long ldW, int rD, float* ptmp, bf16* out, const int* umap) {
  const Plan& p = c.p;
  GemmParams g;
  g.M = rT;
  g.N = p.D;
  g.K = rD;
  g.batch = p.S;
  g.A.ptr = core_u;
  g.A.kmajor = true;
  g.A.ld = ldC;
  g.A.sbatch = (long long)rT * ldC;
  g.B.ptr = Ws_u;
  g.B.kmajor = true;  // B(j, d) = W_s[d][j]
  g.B.ld = ldW;
  g.C = ptmp;
  g.ldc = p.D;
  g.sbatchC = (long long)rTslice * p.D;
  g.c_type = 0;
  JTRY(gemm(g, 0, 0, c.st));
  JTRY(rotate_rows(c, ptmp, out, (long long)p.S * rTslice, (long long)p.S * rTslice, umap + u));
  return JOLT_OK;
}

jolt_status fill_umap(const Ctx& c, int* umap, int n) {
  iota_kernel<<<(unsigned)ceil_div(n, 128), 128, 0, c.st>>>(umap, n);
  CUDA_TRY(cudaGetLastError());
  return JOLT_OK;
}

template <int D, typename TX>
jolt_status launch_table_T(const Ctx& c, const TableArgs& a) {
  size_t sm = table_smem<D>();
  CUDA_TRY(cudaFuncSetAttribute(table_kernel<D, TX>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm));
  table_kernel<D, TX><<<dim3(c.p.tiles, c.p.S, c.p.NU), TTHREADS, sm, c.st>>>(a);
  CUDA_TRY(cudaGetLastError());
  return JOLT_OK;
}

template <int D>
jolt_status launch_table_D(const Ctx& c, const TableArgs& a) {
  return c.p.dtype == JOLT_BF16 ? launch_table_T<D, bf16>(c, a) : launch_table_T<D, float>(c, a);
}

jolt_status run_table(const Ctx& c, const bf16* Us, long long ldU, const bf16* Ws, long long ldW, bf16* core,
                      double* table) {
  const Plan& p = c.p;
  JTRY(run_core(c, Us, ldU, Ws, ldW, core));
  bf16* P = c.at<bf16>(p.o_P);
  int* umap = c.at<int>(p.o_umap);
  JTRY(fill_umap(c, umap, p.NU));
  const long long sP_rd = (long long)p.S * p.rTmax * p.D;
  const long long sP_unit = p.cd.nD * sP_rd;
  for (int u = 0; u < p.NU; ++u)
    for (int iD = 0; iD < p.cd.nD; ++iD)
      JTRY(pmat_unit(c, u, core + (size_t)u * p.S * p.rTmax * p.ldC, p.ldC, p.rTmax, p.rTmax,
                     Ws + (size_t)u * p.D * ldW, ldW, p.cd.rD[iD], c.at<float>(p.o_ptmp), P + u * sP_unit + iD * sP_rd,
                     umap));
  TableArgs a;
  a.cv = c.view();
  a.U = Us;
  a.ldU = ldU;
  a.sU = (long long)p.T * ldU;
  a.P = P;
  a.sP_unit = sP_unit;
  a.sP_rd = sP_rd;
  a.rTmax = p.rTmax;
  a.cand = p.cd;
  a.seed = c.seed;
  a.partial = c.at<double>(p.o_partial);
  a.tiles = p.tiles;
  switch (p.D) {
    case 16: JTRY(launch_table_D<16>(c, a)); break;
    case 32: JTRY(launch_table_D<32>(c, a)); break;
    case 64: JTRY(launch_table_D<64>(c, a)); break;
    default: JTRY(launch_table_D<128>(c, a)); break;
  }
  table_reduce_kernel<<<(unsigned)ceil_div((long long)p.NU * p.nC, 128), 128, 0, c.st>>>(
      a.partial, table, p.NU, p.S, p.tiles, p.cd.nT, p.cd.nD, p.cd.nB);
  CUDA_TRY(cudaGetLastError());
  return JOLT_OK;
}

// ------------------------------------------------------------------------------------------
// stage 4: encode
// ------------------------------------------------------------------------------------------
template <int D, typename TX>
jolt_status launch_encode_T(const Ctx& c, const EncodeArgs& a) {
  size_t sm = table_smem<D>();
  CUDA_TRY(cudaFuncSetAttribute(encode_kernel<D, TX>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm));
  encode_kernel<D, TX><<<dim3(c.p.tiles, c.p.S, c.p.NU), TTHREADS, sm, c.st>>>(a);
  CUDA_TRY(cudaGetLastError());
  return JOLT_OK;
}
template <int D>
jolt_status launch_encode_D(const Ctx& c, const EncodeArgs& a) {
  return c.p.dtype == JOLT_BF16 ? launch_encode_T<D, bf16>(c, a) : launch_encode_T<D, float>(c, a);
}

BlobHeader header_proto(const Plan& p, uint64_t seed) {
  BlobHeader h;
  memset(&h, 0, sizeof h);
  h.magic = kMagic;
  h.version = kVersion;
  h.n_units = (uint32_t)p.NU;
  h.status = 0;
  h.n_layers = p.nL;
  h.n_heads = p.H;
  h.n_tokens = p.T;
  h.head_dim = p.D;
  h.layers_per_group = p.Lg;
  h.dtype = p.dtype;
  h.block = 16;
  h.seed = seed;
  return h;
}

jolt_status run_allocate(const Ctx& c, const double* table, unsigned long long budget_payload, unsigned char* blob,
                         size_t blob_cap, const int32_t* forced_choice) {
  const Plan& p = c.p;
  unsigned long long* B = c.at<unsigned long long>(p.o_bytes);
  bytes_table_kernel<<<(unsigned)ceil_div((long long)p.NU * p.nC, 128), 128, 0, c.st>>>(B, p.NU, p.T, p.D, p.S, p.cd);
  CUDA_TRY(cudaGetLastError());
  AllocArgs a;
  memset(&a, 0, sizeof a);
  a.D = table;
  a.B = B;
  a.nunits = p.NU;
  a.nc = p.nC;
  a.budget = forced_choice ? ~0ull : budget_payload;
  a.choice = c.at<int>(p.o_choice);
  a.lambda = c.at<double>(p.o_lambda);
  a.status = c.status();
  a.blob = blob;
  a.blob_cap = blob_cap;
  a.header_bytes = 64ull + 64ull * p.NU;
  a.T = p.T;
  a.D_ = p.D;
  a.S = p.S;
  a.cd = p.cd;
  a.hdr = header_proto(p, c.seed);
  size_t sm = (size_t)((p.NU * 4 + 15) / 16) * 16 + (size_t)p.NU * 8;
  a.forced = forced_choice;  // caller's choices (jolt_encode): same header filling, no search
  allocate_kernel<<<1, 128, sm, c.st>>>(a);
  CUDA_TRY(cudaGetLastError());
  return JOLT_OK;
}

jolt_status run_encode(const Ctx& c, const bf16* Us, long long ldU, const bf16* Ws, long long ldW, const bf16* core,
                       unsigned char* blob) {
  const Plan& p = c.p;
  EncodeArgs a;
  a.cv = c.view();
  a.U = Us;
  a.ldU = ldU;
  a.sU = (long long)p.T * ldU;
  a.P = c.at<bf16>(p.o_P);
  a.sP_rd = (long long)p.S * p.rTmax * p.D;
  a.sP_unit = p.cd.nD * a.sP_rd;
  a.rTmax = p.rTmax;
  a.cand = p.cd;
  a.seed = c.seed;
  a.blob = blob;
  switch (p.D) {
    case 16: JTRY(launch_encode_D<16>(c, a)); break;
    case 32: JTRY(launch_encode_D<32>(c, a)); break;
    case 64: JTRY(launch_encode_D<64>(c, a)); break;
    default: JTRY(launch_encode_D<128>(c, a)); break;
  }
  copy_factors_kernel<<<dim3(64, p.NU), 256, 0, c.st>>>(blob, Us, ldU, (long long)p.T * ldU, Ws, ldW,
                                                         (long long)p.D * ldW, core, p.ldC, (long long)p.rTmax * p.ldC,
                                                         (long long)p.S * p.rTmax * p.ldC, p.T, p.D, p.S);
  CUDA_TRY(cudaGetLastError());
  return JOLT_OK;
}

jolt_status check_ws(const Plan& p, void* ws, size_t ws_bytes) {
  if (!ws) return fail(JOLT_ERR_INVALID_ARG, "null workspace");
  if (ws_bytes < p.ws_total)
    return fail(JOLT_ERR_WORKSPACE_TOO_SMALL, "workspace %zu bytes, need %zu", ws_bytes, p.ws_total);
  if (reinterpret_cast<uintptr_t>(ws) % 256) return fail(JOLT_ERR_INVALID_ARG, "workspace not 256-byte aligned");
  return JOLT_OK;
}

jolt_status check_inputs(const Plan& p, const void* k, const void* v) {
  if (!k || !v) return fail(JOLT_ERR_INVALID_ARG, "null cache pointer");
  if (reinterpret_cast<uintptr_t>(k) % 16 || reinterpret_cast<uintptr_t>(v) % 16)
    return fail(JOLT_ERR_INVALID_ARG, "cache pointers must be 16-byte aligned");
  (void)p;
  return JOLT_OK;
}

jolt_status check_aligned(const void* q, const char* name) {
  if (!q) return fail(JOLT_ERR_INVALID_ARG, "null %s", name);
  if (reinterpret_cast<uintptr_t>(q) % 16) return fail(JOLT_ERR_INVALID_ARG, "%s must be 16-byte aligned", name);
  return JOLT_OK;
}

}  // namespace

// ==========================================================================================
// C ABI
// ==========================================================================================
extern "C" {

const char* jolt_version(void) { return "jolt-b200 1.0 (sm_100a)"; }

const char* jolt_last_error(void) { return g_err.c_str(); }

jolt_status jolt_workspace_size(const jolt_shape* shape, const jolt_options* opts, size_t* ws_bytes,
                                size_t* blob_bytes, size_t* dws_bytes) {
  Plan p;
  JTRY(make_plan(shape, opts, &p));
  if (ws_bytes) *ws_bytes = p.ws_total;
  if (blob_bytes) *blob_bytes = p.blob_max;
  if (dws_bytes) *dws_bytes = p.dws_total;
  return JOLT_OK;
}

jolt_status jolt_counts(const jolt_shape* shape, const jolt_options* opts, int32_t* n_units, int32_t* n_choices) {
  Plan p;
  JTRY(make_plan(shape, opts, &p));
  if (n_units) *n_units = p.NU;
  if (n_choices) *n_choices = p.nC;
  return JOLT_OK;
}

jolt_status jolt_choice_bytes(const jolt_shape* shape, const jolt_options* opts, uint64_t* bytes_host) {
  Plan p;
  JTRY(make_plan(shape, opts, &p));
  if (!bytes_host) return fail(JOLT_ERR_INVALID_ARG, "null output");
  for (int c = 0; c < p.nC; ++c) {
    int ib = c % p.cd.nB, iD = (c / p.cd.nB) % p.cd.nD, iT = c / (p.cd.nB * p.cd.nD);
    bytes_host[c] = unit_payload_bytes(p.T, p.D, p.S, p.cd.rT[iT], p.cd.rD[iD], p.cd.bits[ib]);
  }
  return JOLT_OK;
}

jolt_status jolt_factor(const jolt_shape* shape, const void* k_dev, const void* v_dev, const jolt_options* opts,
                        uint64_t seed, float* u_dev, int64_t ld_u, float* w_dev, int64_t ld_w, void* ws_dev,
                        size_t ws_bytes, void* stream) {
  Plan p;
  JTRY(make_plan(shape, opts, &p));
  JTRY(check_ws(p, ws_dev, ws_bytes));
  JTRY(check_inputs(p, k_dev, v_dev));
  if (!u_dev || !w_dev || ld_u < p.rTmax || ld_w < p.rDmax) return fail(JOLT_ERR_INVALID_ARG, "factor outputs");
  Ctx c{p, (unsigned char*)ws_dev, (cudaStream_t)stream, k_dev, v_dev, seed};
  return run_factor(c, u_dev, ld_u, w_dev, ld_w, nullptr, nullptr);
}

jolt_status jolt_table(const jolt_shape* shape, const void* k_dev, const void* v_dev, const jolt_options* opts,
                       uint64_t seed, const void* u_bf16_dev, int64_t ld_u, const void* w_bf16_dev, int64_t ld_w,
                       void* core_dev, double* table_dev, void* ws_dev, size_t ws_bytes, void* stream) {
  Plan p;
  JTRY(make_plan(shape, opts, &p));
  JTRY(check_ws(p, ws_dev, ws_bytes));
  JTRY(check_inputs(p, k_dev, v_dev));
  JTRY(check_aligned(u_bf16_dev, "u_bf16"));
  JTRY(check_aligned(w_bf16_dev, "w_bf16"));
  JTRY(check_aligned(core_dev, "core"));
  JTRY(check_aligned(table_dev, "table"));
  if (ld_u < p.rTmax || ld_w < p.rDmax || ld_u % 8 || ld_w % 8)
    return fail(JOLT_ERR_INVALID_ARG, "ld_u / ld_w must cover the largest rank and be multiples of 8");
  Ctx c{p, (unsigned char*)ws_dev, (cudaStream_t)stream, k_dev, v_dev, seed};
  CUDA_TRY(cudaMemsetAsync(c.status(), 0, 4, c.st));
  return run_table(c, (const bf16*)u_bf16_dev, ld_u, (const bf16*)w_bf16_dev, ld_w, (bf16*)core_dev, table_dev);
}

jolt_status jolt_allocate(const double* dist_dev, const uint64_t* bytes_dev, int32_t n_units, int32_t n_choices,
                          uint64_t budget_bytes, int32_t* choice_dev, double* lambda_dev, uint32_t* status_dev,
                          void* stream) {
  if (!dist_dev || !bytes_dev || !choice_dev || !lambda_dev || !status_dev || n_units < 1 || n_choices < 1)
    return fail(JOLT_ERR_INVALID_ARG, "jolt_allocate arguments");
  cudaStream_t st = (cudaStream_t)stream;
  CUDA_TRY(cudaMemsetAsync(status_dev, 0, 4, st));
  AllocArgs a;
  memset(&a, 0, sizeof a);
  a.D = dist_dev;
  a.B = (const unsigned long long*)bytes_dev;
  a.nunits = n_units;
  a.nc = n_choices;
  a.budget = budget_bytes;
  a.choice = choice_dev;
  a.lambda = lambda_dev;
  a.status = status_dev;
  size_t sm = (size_t)((n_units * 4 + 15) / 16) * 16 + (size_t)n_units * 8;
  allocate_kernel<<<1, 128, sm, st>>>(a);
  CUDA_TRY(cudaGetLastError());
  return JOLT_OK;
}

jolt_status jolt_encode(const jolt_shape* shape, const void* k_dev, const void* v_dev, const jolt_options* opts,
                        uint64_t seed, const void* u_bf16_dev, int64_t ld_u, const void* w_bf16_dev, int64_t ld_w,
                        const void* core_dev, const int32_t* choice_dev, const double* dist_dev, void* blob_dev,
                        size_t blob_cap, void* ws_dev, size_t ws_bytes, void* stream) {
  Plan p;
  JTRY(make_plan(shape, opts, &p));
  JTRY(check_ws(p, ws_dev, ws_bytes));
  JTRY(check_inputs(p, k_dev, v_dev));
  JTRY(check_aligned(u_bf16_dev, "u_bf16"));
  JTRY(check_aligned(w_bf16_dev, "w_bf16"));
  JTRY(check_aligned(core_dev, "core"));
  JTRY(check_aligned(blob_dev, "blob"));
  if (!choice_dev || !dist_dev) return fail(JOLT_ERR_INVALID_ARG, "null pointer");
  if (ld_u < p.rTmax || ld_w < p.rDmax || ld_u % 8 || ld_w % 8)
    return fail(JOLT_ERR_INVALID_ARG, "ld_u / ld_w must cover the largest rank and be multiples of 8");
  Ctx c{p, (unsigned char*)ws_dev, (cudaStream_t)stream, k_dev, v_dev, seed};
  CUDA_TRY(cudaMemsetAsync(c.status(), 0, 4, c.st));
  // P' of every feature rank from the given core (the encoder's reconstruction operators)
  bf16* P = c.at<bf16>(p.o_P);
  int* umap = c.at<int>(p.o_umap);
  JTRY(fill_umap(c, umap, p.NU));
  const long long sP_rd = (long long)p.S * p.rTmax * p.D;
  const bf16* core = (const bf16*)core_dev;
  const bf16* Ws = (const bf16*)w_bf16_dev;
  for (int u = 0; u < p.NU; ++u)
    for (int iD = 0; iD < p.cd.nD; ++iD)
      JTRY(pmat_unit(c, u, core + (size_t)u * p.S * p.rTmax * p.ldC, p.ldC, p.rTmax, p.rTmax,
                     Ws + (size_t)u * p.D * ld_w, ld_w, p.cd.rD[iD], c.at<float>(p.o_ptmp),
                     P + u * p.cd.nD * sP_rd + iD * sP_rd, umap));
  JTRY(run_allocate(c, dist_dev, 0, (unsigned char*)blob_dev, blob_cap, choice_dev));
  return run_encode(c, (const bf16*)u_bf16_dev, ld_u, Ws, ld_w, core, (unsigned char*)blob_dev);
}

jolt_status jolt_compress(const jolt_shape* shape, const void* k_dev, const void* v_dev, const jolt_options* opts,
                          uint64_t budget_bytes, uint64_t seed, void* blob_dev, size_t blob_cap, void* ws_dev,
                          size_t ws_bytes, void* stream) {
  Plan p;
  JTRY(make_plan(shape, opts, &p));
  JTRY(check_ws(p, ws_dev, ws_bytes));
  JTRY(check_inputs(p, k_dev, v_dev));
  if (!blob_dev) return fail(JOLT_ERR_INVALID_ARG, "null blob");
  if (reinterpret_cast<uintptr_t>(blob_dev) % 16) return fail(JOLT_ERR_INVALID_ARG, "blob not 16-byte aligned");
  if (blob_cap < budget_bytes && blob_cap < p.blob_max)
    return fail(JOLT_ERR_OUTPUT_TOO_SMALL, "blob capacity %zu below budget %llu", blob_cap,
                (unsigned long long)budget_bytes);
  const unsigned long long hdr = 64ull + 64ull * p.NU;
  if (budget_bytes < hdr) return fail(JOLT_ERR_BUDGET_INFEASIBLE, "budget below the headers (%llu bytes)", hdr);
  Ctx c{p, (unsigned char*)ws_dev, (cudaStream_t)stream, k_dev, v_dev, seed};
  float* Uf = c.at<float>(p.o_Uf);
  float* Wf = c.at<float>(p.o_Wf);
  bf16* Us = c.at<bf16>(p.o_Us);
  bf16* Ws = c.at<bf16>(p.o_Ws);
  JTRY(run_factor(c, Uf, p.ldU, Wf, p.ldW, Us, Ws));
  bf16* core = c.at<bf16>(p.o_core);
  double* table = c.at<double>(p.o_table);
  JTRY(run_table(c, Us, p.ldU, Ws, p.ldW, core, table));
  JTRY(run_allocate(c, table, budget_bytes - hdr, (unsigned char*)blob_dev, blob_cap, nullptr));
  JTRY(run_encode(c, Us, p.ldU, Ws, p.ldW, core, (unsigned char*)blob_dev));
  // device-side errors of the factor stage are folded into the header status
  fold_status_kernel<<<1, 1, 0, c.st>>>(c.status(), (unsigned char*)blob_dev);
  CUDA_TRY(cudaGetLastError());
  return JOLT_OK;
}

jolt_status jolt_read_header(const void* blob_dev, jolt_shape* shape_out, uint64_t* total_bytes,
                             jolt_unit_record* records, int32_t cap, void* stream) {
  if (!blob_dev) return fail(JOLT_ERR_INVALID_ARG, "null blob");
  cudaStream_t st = (cudaStream_t)stream;
  BlobHeader h;
  CUDA_TRY(cudaMemcpyAsync(&h, blob_dev, sizeof h, cudaMemcpyDeviceToHost, st));
  CUDA_TRY(cudaStreamSynchronize(st));
  if (h.magic != kMagic || h.version != kVersion || h.n_units == 0 || h.n_units > 1u << 20)
    return fail(JOLT_ERR_BAD_BLOB, "bad blob header");
  if (shape_out) {
    shape_out->n_layers = h.n_layers;
    shape_out->n_heads = h.n_heads;
    shape_out->n_tokens = h.n_tokens;
    shape_out->head_dim = h.head_dim;
    shape_out->layers_per_group = h.layers_per_group;
    shape_out->dtype = h.dtype;
  }
  if (total_bytes) *total_bytes = h.total_bytes;
  if (records && cap > 0) {
    int n = (int)h.n_units < cap ? (int)h.n_units : cap;
    CUDA_TRY(cudaMemcpyAsync(records, (const char*)blob_dev + sizeof(BlobHeader), n * sizeof(UnitHeader),
                             cudaMemcpyDeviceToHost, st));
    CUDA_TRY(cudaStreamSynchronize(st));
  }
  if (h.status & DEV_ERR_INFEASIBLE) return fail(JOLT_ERR_BUDGET_INFEASIBLE, "budget infeasible (device)");
  if (h.status & (DEV_ERR_NONFINITE | DEV_ERR_FACTOR))
    return fail(JOLT_ERR_NUMERIC, "non-finite input or factorisation breakdown (status %u)", h.status);
  if (h.status & DEV_ERR_CAPACITY) return fail(JOLT_ERR_OUTPUT_TOO_SMALL, "blob capacity below payload");
  if (h.status) return fail(JOLT_ERR_BAD_BLOB, "blob status %u", h.status);
  return JOLT_OK;
}

jolt_status jolt_decompress(const void* blob_dev, int32_t out_dtype, void* k_out_dev, void* v_out_dev, void* ws_dev,
                            size_t ws_bytes, void* stream) {
  if (out_dtype != JOLT_BF16 && out_dtype != JOLT_F32) return fail(JOLT_ERR_INVALID_ARG, "out_dtype %d", out_dtype);
  if (!k_out_dev || !v_out_dev || !ws_dev) return fail(JOLT_ERR_INVALID_ARG, "null pointer");
  cudaStream_t st = (cudaStream_t)stream;
  jolt_shape sh;
  uint64_t total = 0;
  BlobHeader h;
  CUDA_TRY(cudaMemcpyAsync(&h, blob_dev, sizeof h, cudaMemcpyDeviceToHost, st));
  CUDA_TRY(cudaStreamSynchronize(st));
  if (h.magic != kMagic || h.version != kVersion || h.n_units == 0 || h.n_units > 4096)
    return fail(JOLT_ERR_BAD_BLOB, "bad blob header");
  std::vector<jolt_unit_record> rec(h.n_units);
  JTRY(jolt_read_header(blob_dev, &sh, &total, rec.data(), (int32_t)h.n_units, stream));
  // a plan for this shape with candidate sets made of the ranks actually stored
  jolt_options op;
  memset(&op, 0, sizeof op);
  int rTm = 8, rDm = 8;
  for (auto& r : rec) {
    if (r.r_T < 1 || r.r_T > sh.n_tokens || r.r_D < 1 || r.r_D > sh.head_dim || r.bits < 0 || r.bits > 8)
      return fail(JOLT_ERR_BAD_BLOB, "unit record out of range");
    if (r.off_U + 2ull * sh.n_tokens * r.r_T > total) return fail(JOLT_ERR_BAD_BLOB, "unit record offsets");
    rTm = r.r_T > rTm ? r.r_T : rTm;
    rDm = r.r_D > rDm ? r.r_D : rDm;
  }
  op.n_token_ranks = 1;
  op.token_ranks[0] = (int)round_up(rTm, 8) > sh.n_tokens ? rTm : (int)round_up(rTm, 8);
  op.n_feature_ranks = 1;
  op.feature_ranks[0] = (int)round_up(rDm, 8) > sh.head_dim ? rDm : (int)round_up(rDm, 8);
  op.n_bits = 1;
  op.method = JOLT_EXACT;
  Plan p;
  JTRY(make_plan(&sh, &op, &p));
  if (ws_bytes < p.dws_total)
    return fail(JOLT_ERR_WORKSPACE_TOO_SMALL, "decompress workspace %zu bytes, need %zu", ws_bytes, p.dws_total);
  Ctx c{p, (unsigned char*)ws_dev, st, nullptr, nullptr, h.seed};
  bf16* Ucp = c.at<bf16>(p.d_U);
  bf16* Wcp = c.at<bf16>(p.d_W);
  bf16* Ccp = c.at<bf16>(p.d_C);
  float* ptmp = c.at<float>(p.d_ptmp);
  bf16* P = c.at<bf16>(p.d_P);
  int* umap = c.at<int>(p.d_umap);
  JTRY(fill_umap(c, umap, p.NU));
  CUDA_TRY(cudaMemsetAsync(ptmp, 0, (size_t)p.S * p.rTmax * p.D * 4, st));
  const unsigned char* blob = (const unsigned char*)blob_dev;
  const long long sP_unit = (long long)p.S * p.rTmax * p.D;
  for (int u = 0; u < p.NU; ++u) {
    const jolt_unit_record& r = rec[u];
    bf16* Uu = Ucp + (size_t)u * p.T * p.ldU;
    bf16* Wu = Wcp + (size_t)u * p.D * p.ldW;
    bf16* Cu = Ccp + (size_t)u * p.S * p.rTmax * p.ldC;
    copy2d_kernel<<<grid1d((long long)p.T * p.ldU), 256, 0, st>>>((const bf16*)(blob + r.off_U), p.T, r.r_T, Uu, p.ldU);
    copy2d_kernel<<<grid1d((long long)p.D * p.ldW), 256, 0, st>>>((const bf16*)(blob + r.off_W), p.D, r.r_D, Wu, p.ldW);
    copy2d_kernel<<<grid1d((long long)p.S * r.r_T * p.ldC), 256, 0, st>>>((const bf16*)(blob + r.off_C),
                                                                          (long long)p.S * r.r_T, r.r_D, Cu, p.ldC);
    CUDA_TRY(cudaGetLastError());
    JTRY(pmat_unit(c, u, Cu, p.ldC, r.r_T, p.rTmax, Wu, p.ldW, r.r_D, ptmp, P + u * sP_unit, umap));
  }
  DecodeArgs a;
  a.blob = blob;
  a.U = Ucp;
  a.ldU = p.ldU;
  a.sU = (long long)p.T * p.ldU;
  a.P = P;
  a.sP_unit = sP_unit;
  a.rTmax = p.rTmax;
  a.T = p.T;
  a.S = p.S;
  a.Lg = p.Lg;
  a.seed = h.seed;
  a.k_out = k_out_dev;
  a.v_out = v_out_dev;
  a.out_f32 = out_dtype == JOLT_F32;
  dim3 grid(p.tiles, p.S, p.NU);
  switch (p.D) {
#define DEC_CASE(DD)                                                                                     \
  case DD: {                                                                                             \
    CUDA_TRY(cudaFuncSetAttribute(decode_kernel<DD>, cudaFuncAttributeMaxDynamicSharedMemorySize,        \
                                  (int)decode_smem<DD>()));                                              \
    decode_kernel<DD><<<grid, TTHREADS, decode_smem<DD>(), st>>>(a);                                     \
    break;                                                                                               \
  }
    DEC_CASE(16)
    DEC_CASE(32)
    DEC_CASE(64)
    DEC_CASE(128)
#undef DEC_CASE
    default: return fail(JOLT_ERR_BAD_BLOB, "head_dim");
  }
  CUDA_TRY(cudaGetLastError());
  return JOLT_OK;
}

jolt_status jolt_frobenius(const jolt_shape* shape, const void* k_dev, const void* v_dev, const void* ky_dev,
                           const void* vy_dev, int32_t ydtype, double* sq_dev, void* ws_dev, size_t ws_bytes,
                           void* stream) {
  if (!shape || !k_dev || !v_dev || !sq_dev || !ws_dev) return fail(JOLT_ERR_INVALID_ARG, "null pointer");
  if ((ky_dev == nullptr) != (vy_dev == nullptr)) return fail(JOLT_ERR_INVALID_ARG, "give both or neither of ky, vy");
  if (shape->n_layers < 1 || shape->layers_per_group < 1 || shape->n_layers % shape->layers_per_group)
    return fail(JOLT_ERR_INVALID_ARG, "shape");
  const int G = shape->n_layers / shape->layers_per_group, NU = 2 * G, nblk = 64;
  if (ws_bytes < (size_t)NU * nblk * 16) return fail(JOLT_ERR_WORKSPACE_TOO_SMALL, "frobenius workspace");
  const long long n = (long long)shape->layers_per_group * shape->n_heads * shape->n_tokens * shape->head_dim;
  cudaStream_t st = (cudaStream_t)stream;
  double* part = (double*)ws_dev;
  for (int kv = 0; kv < 2; ++kv) {
    const void* X = kv ? v_dev : k_dev;
    const void* Y = kv ? vy_dev : ky_dev;
    dim3 grid(nblk, G);
    if (shape->dtype == JOLT_BF16) {
      if (ydtype == JOLT_F32)
        frob_partial_kernel<bf16, float><<<grid, 256, 0, st>>>((const bf16*)X, (const float*)Y, n, kv, part, nblk);
      else
        frob_partial_kernel<bf16, bf16><<<grid, 256, 0, st>>>((const bf16*)X, (const bf16*)Y, n, kv, part, nblk);
    } else {
      if (ydtype == JOLT_F32)
        frob_partial_kernel<float, float><<<grid, 256, 0, st>>>((const float*)X, (const float*)Y, n, kv, part, nblk);
      else
        frob_partial_kernel<float, bf16><<<grid, 256, 0, st>>>((const float*)X, (const bf16*)Y, n, kv, part, nblk);
    }
    CUDA_TRY(cudaGetLastError());
  }
  frob_final_kernel<<<(unsigned)ceil_div(2 * NU, 128), 128, 0, st>>>(part, NU, nblk, sq_dev);
  CUDA_TRY(cudaGetLastError());
  return JOLT_OK;
}

}  // extern "C"
