// Decode-side attention over the stored factors ("A JoLT for the KV cache: Near-Lossless KV
// Cache Compression via Joint Rank-bit Allocation", abstract: the decode path evaluates
// attention directly over the stored factors, without forming dense K and V tensors).
//
// One decode step of n_q query heads against every cached token of one layer l (layer group
// g = l / L_g, local layer ll, GQA: query head j reads KV head h = j / (n_q / H)).  With the
// rotation Phi = diag(sigma) H_D / sqrt(D) the decoder stores a slice as
//   X_hat = (U_s P' + rho_hat) Phi^T,     rho_hat = lo + code * step per 16-wide block,
// so, with q' = Phi^T q (the query rotated as a row):
//   scores  s_t = U_K[t, :] (P'_K q') + rho_hat_K[t, :] . q'      (scaled by 1 / sqrt(D))
//   output  y   = ( (p^T U_V) P'_V + p^T rho_hat_V ) Phi_V^T       (p = softmax of the scores)
// where rho_hat . q' is taken block by block from the codes and the fp16 (lo, step) pair.  No
// dense K or V row is formed: the kernels read the stored token factors, codes and scales once.
//
// Three kernels:
//   attend_query_kernel   one CTA per query head: q' (fp32 Walsh-Hadamard in shared memory)
//                         and a = P'_K q' (r_T of K values);
//   attend_chunk_kernel   one CTA per (token chunk, KV head) for all query heads of that KV
//                         head: 64-token tiles, scores from the U_K tile (staged in shared
//                         memory 128 ranks at a time) and the K codes, an online softmax
//                         (running max, rescaled sums), and the running sums p^T U_V and
//                         p^T rho_hat_V; one partial record per (chunk, query head);
//   attend_combine_kernel one CTA per query head: the chunks' records merged under the
//                         global max, times P'_V, un-rotated.
// All arithmetic in fp32 (exp by expf).
#pragma once

#include "common.cuh"
#include "fp16_exact.cuh"
#include "kernels.cuh"

namespace jolt {
namespace att {
constexpr int TT = 64;          // tokens per tile
constexpr int RC = 128;         // token-factor ranks staged per step
constexpr int THREADS = 128;
constexpr int MAXG = 8;         // query heads per KV head
constexpr int MAXR = 1024;      // largest stored token rank
}  // namespace att

struct AttendArgs {
  const unsigned char* blob;
  const bf16* U;          // [unit][T][ldU] aligned copies of the stored token factors
  long long ldU, sU;
  const bf16* P;          // [unit][S][rTmax][D] rotated operators
  long long sP_unit;
  int rTmax;
  int T, S, H, D, Lg, u0;
  uint64_t seed;
  int layer;              // global layer index
  int nq, G;              // query heads, query heads per KV head
  const float* q;         // [nq][D]
  float* qrot;            // [nq][D]   scratch: q'
  float* a;               // [nq][rTmax] scratch: P'_K q'
  float* part;            // [H][nch][G][2 + rTmax + D] scratch: chunk records
  int nch;                // token chunks per KV head
  float* out;             // [nq][D]
};

__device__ __forceinline__ const UnitHeader& att_unit(const unsigned char* blob, int u) {
  return reinterpret_cast<const UnitHeader*>(blob + sizeof(BlobHeader))[u];
}

// q' = Phi_K^T q as a row (sign flip, Walsh-Hadamard, 1/sqrt(D)) and a = P'_K q'
template <int D>
__global__ void __launch_bounds__(att::THREADS) attend_query_kernel(AttendArgs A) {
  __shared__ float qs[D];
  const int j = blockIdx.x, tid = threadIdx.x;
  const int h = j / A.G, g = A.layer / A.Lg, ll = A.layer - g * A.Lg, uK = 2 * g;
  for (int d = tid; d < D; d += blockDim.x) qs[d] = A.q[(long long)j * D + d] * rotation_sign(A.seed, uK + A.u0, d);
  __syncthreads();
  for (int hw = 1; hw < D; hw <<= 1) {
    for (int p = tid; p < D / 2; p += blockDim.x) {
      const int i = (p / hw) * 2 * hw + (p % hw);
      const float x = qs[i], y = qs[i + hw];
      qs[i] = x + y;
      qs[i + hw] = x - y;
    }
    __syncthreads();
  }
  const float sc = (float)(1.0 / sqrt((double)D));
  for (int d = tid; d < D; d += blockDim.x) {
    qs[d] *= sc;
    A.qrot[(long long)j * D + d] = qs[d];
  }
  __syncthreads();
  const int rT = att_unit(A.blob, uK).r_T;
  const bf16* P = A.P + (long long)uK * A.sP_unit + ((long long)(ll * A.H + h) * A.rTmax) * D;
  for (int r = tid; r < rT; r += blockDim.x) {
    const bf16* row = P + (long long)r * D;
    float s = 0.f;
    for (int d = 0; d < D; ++d) s = fmaf(__bfloat162float(row[d]), qs[d], s);
    A.a[(long long)j * A.rTmax + r] = s;
  }
}

// dequantised residual block (16 values) of token t, block b of one slice
__device__ __forceinline__ void att_block(const unsigned char* blob, const UnitHeader& uh, long long blk, float* v) {
  const int b = uh.bits;
  const unsigned char* src = blob + uh.off_codes + blk * (2 * b);
  uint32_t w[4] = {0u, 0u, 0u, 0u};
  for (int byte = 0; byte < 2 * b; ++byte) w[byte >> 2] |= (uint32_t)src[byte] << ((byte & 3) * 8);
  const __half2 sc = reinterpret_cast<const __half2*>(blob + uh.off_scales)[blk];
  const float lo = __low2float(sc), step = __high2float(sc);
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = fmaf((float)unpack_code(w, i, b), step, lo);
}

// grid (nch, H); att::THREADS threads; dynamic shared memory attend_chunk_smem(D, rTmax, G)
template <int D>
__global__ void __launch_bounds__(att::THREADS) attend_chunk_kernel(AttendArgs A) {
  using namespace att;
  extern __shared__ __align__(16) float at_sm[];
  const int c = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
  const int G = A.G, T = A.T;
  const int g = A.layer / A.Lg, ll = A.layer - g * A.Lg, uK = 2 * g, uV = 2 * g + 1;
  const int s = ll * A.H + h;   // slice inside the unit
  const UnitHeader hK = att_unit(A.blob, uK), hV = att_unit(A.blob, uV);
  const int rK = hK.r_T, rV = hV.r_T;
  // shared memory: a[G][rTmax] | qrot[G][D] | tile of U (TT x RC bf16) |
  // scores / weights p[G][TT] | dequantised V residual [TT][D] | z[G][rTmax] | w[G][D] | m, e
  float* as = at_sm;
  float* qr = as + G * A.rTmax;
  bf16* ut = reinterpret_cast<bf16*>(qr + G * D);
  float* ps = reinterpret_cast<float*>(ut + TT * (RC + 8));
  float* rv = ps + G * TT;
  float* zs = rv + TT * (D + 4);
  float* ws = zs + G * A.rTmax;
  float* ms = ws + G * D;       // [G] running max
  float* es = ms + G;           // [G] running sum
  float* al = es + G;           // [G] rescale factor of this tile
  const int j0 = h * G;
  for (int i = tid; i < G * A.rTmax; i += blockDim.x) {
    as[i] = A.a[(long long)j0 * A.rTmax + i];
    zs[i] = 0.f;
  }
  for (int i = tid; i < G * D; i += blockDim.x) {
    qr[i] = A.qrot[(long long)j0 * D + i];
    ws[i] = 0.f;
  }
  if (tid < G) {
    ms[tid] = -INFINITY;
    es[tid] = 0.f;
  }
  const int per = (T + A.nch - 1) / A.nch;
  const int tb = c * per, te = min(T, tb + per);
  const bf16* UK = A.U + (long long)uK * A.sU;
  const bf16* UV = A.U + (long long)uV * A.sU;
  const float isq = (float)(1.0 / sqrt((double)D));
  __syncthreads();
  for (int t0 = tb; t0 < te; t0 += TT) {
    const int nt = min(TT, te - t0);
    // ---- scores: thread (token tt = tid / 2, half) ----
    const int tt = tid >> 1, half = tid & 1;
    float sacc[MAXG];
#pragma unroll
    for (int jj = 0; jj < MAXG; ++jj) sacc[jj] = 0.f;
    for (int r0 = 0; r0 < rK; r0 += RC) {
      for (int idx = tid; idx < TT * (RC / 8); idx += blockDim.x) {
        const int row = idx / (RC / 8), ch = idx - row * (RC / 8), r = r0 + ch * 8;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (row < nt && r < rK) v = *reinterpret_cast<const uint4*>(UK + (long long)(t0 + row) * A.ldU + r);
        *reinterpret_cast<uint4*>(ut + row * (RC + 8) + ch * 8) = v;
      }
      __syncthreads();
      const int rlo = half * (RC / 2), rhi = min(RC, rK - r0);
      for (int r = rlo; r < rlo + RC / 2 && r < rhi; ++r) {
        const float u = __bfloat162float(ut[tt * (RC + 8) + r]);
#pragma unroll
        for (int jj = 0; jj < MAXG; ++jj)
          if (jj < G) sacc[jj] = fmaf(u, as[jj * A.rTmax + r0 + r], sacc[jj]);
      }
      __syncthreads();
    }
    // residual of K: blocks half * D/32 .. of the token's row
    if (hK.bits > 0 && tt < nt) {
      const long long row = (long long)s * T + (t0 + tt);
      constexpr int NB = D / 16;
      for (int bb = half * (NB / 2); bb < (half ? NB : NB / 2); ++bb) {
        float v[16];
        att_block(A.blob, hK, row * NB + bb, v);
#pragma unroll
        for (int jj = 0; jj < MAXG; ++jj) {
          if (jj >= G) break;
          float dot = 0.f;
#pragma unroll
          for (int i = 0; i < 16; ++i) dot = fmaf(v[i], qr[jj * D + 16 * bb + i], dot);
          sacc[jj] += dot;
        }
      }
    }
#pragma unroll
    for (int jj = 0; jj < MAXG; ++jj) sacc[jj] += __shfl_xor_sync(0xffffffffu, sacc[jj], 1);
    if (half == 0)
#pragma unroll
      for (int jj = 0; jj < MAXG; ++jj)
        if (jj < G) ps[jj * TT + tt] = tt < nt ? sacc[jj] * isq : -INFINITY;
    // dequantised V residual rows of the tile (zero rows past the end)
    if (hV.bits > 0) {
      const int ddh = half * (D / 2);
      for (int bb = ddh / 16; bb < (ddh + D / 2) / 16; ++bb) {
        float v[16];
        if (tt < nt) att_block(A.blob, hV, ((long long)s * T + (t0 + tt)) * (D / 16) + bb, v);
        else
#pragma unroll
          for (int i = 0; i < 16; ++i) v[i] = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) rv[tt * (D + 4) + 16 * bb + i] = v[i];
      }
    }
    __syncthreads();
    // ---- online softmax: warp jj < G takes query head jj ----
    const int warp = tid >> 5, lane = tid & 31;
    for (int jj = warp; jj < G; jj += blockDim.x / 32) {
      float mx = -INFINITY;
      for (int t = lane; t < TT; t += 32) mx = fmaxf(mx, ps[jj * TT + t]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      const float mnew = fmaxf(ms[jj], mx);
      float sum = 0.f;
      for (int t = lane; t < TT; t += 32) {
        const float p = ps[jj * TT + t] == -INFINITY ? 0.f : expf(ps[jj * TT + t] - mnew);
        ps[jj * TT + t] = p;
        sum += p;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      __syncwarp();
      if (lane == 0) {
        const float alpha = ms[jj] == -INFINITY ? 0.f : expf(ms[jj] - mnew);
        al[jj] = alpha;
        es[jj] = es[jj] * alpha + sum;
        ms[jj] = mnew;
      }
    }
    __syncthreads();
    // ---- values: z[j][r] = alpha z + sum_t p_t U_V[t, r]; thread owns rank r0 + tid ----
    for (int r0 = 0; r0 < rV; r0 += RC) {
      for (int idx = tid; idx < TT * (RC / 8); idx += blockDim.x) {
        const int row = idx / (RC / 8), ch = idx - row * (RC / 8), r = r0 + ch * 8;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (row < nt && r < rV) v = *reinterpret_cast<const uint4*>(UV + (long long)(t0 + row) * A.ldU + r);
        *reinterpret_cast<uint4*>(ut + row * (RC + 8) + ch * 8) = v;
      }
      __syncthreads();
      const int r = r0 + tid;
      if (tid < RC && r < rV) {
        float acc[MAXG];
#pragma unroll
        for (int jj = 0; jj < MAXG; ++jj) acc[jj] = 0.f;
        for (int t = 0; t < TT; ++t) {
          const float u = __bfloat162float(ut[t * (RC + 8) + tid]);
#pragma unroll
          for (int jj = 0; jj < MAXG; ++jj)
            if (jj < G) acc[jj] = fmaf(ps[jj * TT + t], u, acc[jj]);
        }
#pragma unroll
        for (int jj = 0; jj < MAXG; ++jj)
          if (jj < G) zs[jj * A.rTmax + r] = fmaf(zs[jj * A.rTmax + r], al[jj], acc[jj]);
      }
      __syncthreads();
    }
    // ---- w[j][d] = alpha w + sum_t p_t rho_hat_V[t, d]; thread owns d ----
    for (int d = tid; d < D; d += blockDim.x) {
      float acc[MAXG];
#pragma unroll
      for (int jj = 0; jj < MAXG; ++jj) acc[jj] = 0.f;
      if (hV.bits > 0)
        for (int t = 0; t < TT; ++t) {
          const float v = rv[t * (D + 4) + d];
#pragma unroll
          for (int jj = 0; jj < MAXG; ++jj)
            if (jj < G) acc[jj] = fmaf(ps[jj * TT + t], v, acc[jj]);
        }
#pragma unroll
      for (int jj = 0; jj < MAXG; ++jj)
        if (jj < G) ws[jj * D + d] = fmaf(ws[jj * D + d], al[jj], acc[jj]);
    }
    __syncthreads();
  }
  // the chunk's record per query head: m, e, z[rTmax], w[D]
  const long long rec = 2 + A.rTmax + D;
  for (int jj = 0; jj < G; ++jj) {
    float* o = A.part + (((long long)h * A.nch + c) * G + jj) * rec;
    if (tid == 0) {
      o[0] = ms[jj];
      o[1] = es[jj];
    }
    for (int r = tid; r < A.rTmax; r += blockDim.x) o[2 + r] = r < rV ? zs[jj * A.rTmax + r] : 0.f;
    for (int d = tid; d < D; d += blockDim.x) o[2 + A.rTmax + d] = ws[jj * D + d];
  }
}

inline size_t attend_chunk_smem(int D, int rTmax, int G) {
  using namespace att;
  return sizeof(float) * ((size_t)G * rTmax + G * D) + sizeof(bf16) * TT * (RC + 8) +
         sizeof(float) * ((size_t)G * TT + TT * (D + 4) + (size_t)G * rTmax + G * D + 3 * G) + 64;
}

// y' = (Z / E) P'_V + W / E over the chunks' records, then y = y' Phi_V^T; one CTA per query head
template <int D>
__global__ void __launch_bounds__(att::THREADS) attend_combine_kernel(AttendArgs A) {
  __shared__ float zsh[att::MAXR];
  __shared__ float ysh[D];
  __shared__ float wgt[64];
  __shared__ float stat[2];
  const int j = blockIdx.x, tid = threadIdx.x;
  const int h = j / A.G, jj = j - h * A.G;
  const int g = A.layer / A.Lg, ll = A.layer - g * A.Lg, uV = 2 * g + 1;
  const int rV = att_unit(A.blob, uV).r_T;
  const long long rec = 2 + A.rTmax + D;
  auto R = [&](int c) { return A.part + (((long long)h * A.nch + c) * A.G + jj) * rec; };
  if (tid == 0) {
    float M = -INFINITY;
    for (int c = 0; c < A.nch; ++c) M = fmaxf(M, R(c)[0]);
    float E = 0.f;
    for (int c = 0; c < A.nch; ++c) {
      const float m = R(c)[0];
      const float f = m == -INFINITY ? 0.f : expf(m - M);
      wgt[c] = f;
      E = fmaf(R(c)[1], f, E);
    }
    stat[0] = M;
    stat[1] = 1.f / E;
  }
  __syncthreads();
  const float inv = stat[1];
  for (int r = tid; r < rV; r += blockDim.x) {
    float z = 0.f;
    for (int c = 0; c < A.nch; ++c) z = fmaf(R(c)[2 + r], wgt[c], z);
    zsh[r] = z * inv;
  }
  __syncthreads();
  const bf16* P = A.P + (long long)uV * A.sP_unit + ((long long)(ll * A.H + h) * A.rTmax) * D;
  for (int d = tid; d < D; d += blockDim.x) {
    float y = 0.f;
    for (int c = 0; c < A.nch; ++c) y = fmaf(R(c)[2 + A.rTmax + d], wgt[c], y);
    y *= inv;
    for (int r = 0; r < rV; ++r) y = fmaf(zsh[r], __bfloat162float(P[(long long)r * D + d]), y);
    ysh[d] = y;
  }
  __syncthreads();
  for (int hw = 1; hw < D; hw <<= 1) {
    for (int p = tid; p < D / 2; p += blockDim.x) {
      const int i = (p / hw) * 2 * hw + (p % hw);
      const float x = ysh[i], y = ysh[i + hw];
      ysh[i] = x + y;
      ysh[i + hw] = x - y;
    }
    __syncthreads();
  }
  const float sc = (float)(1.0 / sqrt((double)D));
  for (int d = tid; d < D; d += blockDim.x)
    A.out[(long long)j * D + d] = ysh[d] * sc * rotation_sign(A.seed, uV + A.u0, d);
}

}  // namespace jolt
