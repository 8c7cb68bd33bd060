// Exact fp16 directed rounding, the quantiser step, codes and code packing of the b-bit
// block quantiser.
// Host and device: the device code is what the table and encode kernels run; the host
// copy of the same source lets a CPU check compare it with the float64 definition.
#pragma once

#include <cuda_fp16.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

namespace jolt {

__host__ __device__ __forceinline__ uint32_t f32_bits(float x) {
#ifdef __CUDA_ARCH__
  return __float_as_uint(x);
#else
  uint32_t u;
  memcpy(&u, &x, sizeof u);
  return u;
#endif
}
__host__ __device__ __forceinline__ float bits_f32(uint32_t u) {
#ifdef __CUDA_ARCH__
  return __uint_as_float(u);
#else
  float x;
  memcpy(&x, &u, sizeof x);
  return x;
#endif
}

// ---------------------------------------------------------------------------------------
// exact fp16 directed rounding and the quantiser step, in FP32-pipe integer / float ops
// (fp16 normal values are the floats whose low 13 mantissa bits are zero; other ranges
// go through the conversion instructions)
// ---------------------------------------------------------------------------------------
constexpr float kFp16MinNormal = 6.103515625e-05f;  // 2^-14
constexpr float kFp16Max = 65504.f;

// fp16 round toward -inf (as __float2half_rd)
__host__ __device__ __forceinline__ float rd16(float x) {
  const float ax = fabsf(x);
  if (ax >= kFp16MinNormal && ax <= kFp16Max) {
    uint32_t u = f32_bits(x);
    if (x >= 0.f) u &= ~0x1FFFu;
    else if (u & 0x1FFFu) u = (u | 0x1FFFu) + 1u;
    return bits_f32(u);
  }
  return __half2float(__float2half_rd(x));
}

// fp16 round toward +inf of a positive float (as __float2half_ru)
__host__ __device__ __forceinline__ float ru16_pos(float q) {
  if (q >= kFp16MinNormal && q <= kFp16Max) {
    uint32_t u = f32_bits(q);
    if (u & 0x1FFFu) u = (u | 0x1FFFu) + 1u;
    return bits_f32(u);
  }
  return __half2float(__float2half_ru(q));
}

// neighbouring fp16 values of a positive fp16 value s
__host__ __device__ __forceinline__ float next16_up(float s) {
  if (s >= kFp16MinNormal && s < kFp16Max) return bits_f32(f32_bits(s) + 0x2000u);
  return __half2float(__ushort_as_half((unsigned short)(__half_as_ushort(__float2half_rn(s)) + 1)));
}
__host__ __device__ __forceinline__ float next16_down(float s) {
  if (s > kFp16MinNormal && s <= kFp16Max) return bits_f32(f32_bits(s) - 0x2000u);
  unsigned short h = __half_as_ushort(__float2half_rn(s));
  return h ? __half2float(__ushort_as_half((unsigned short)(h - 1))) : 0.f;
}

// a >= mx - lo, decided exactly (R is the rounded difference)
__host__ __device__ __forceinline__ bool ge_exact(float a, float mx, float lo, float R) {
  if (a > R * 1.0000002384185791f) return true;
  if (a < R * 0.9999997615814209f) return false;
  return (double)a >= (double)mx - (double)lo;
}

// quantiser step: the smallest fp16 s with s * levels >= mx - lo exactly (the fp16
// round-up of (mx - lo)/levels); 0 when mx <= lo.  A float estimate is corrected by one
// fp16 step where needed.
__host__ __device__ __forceinline__ float quant_step(float mx, float lo, float flev, float inv_lev) {
  if (!(mx > lo)) return 0.f;
  const float R = mx - lo;
  float s = ru16_pos(R * inv_lev);
  if (!(s <= kFp16Max)) return s;  // +inf: this block cannot be stored with this many bits
  if (!ge_exact(s * flev, mx, lo, R)) {
    s = next16_up(s);
  } else {
    float sp = next16_down(s);
    if (sp > 0.f && ge_exact(sp * flev, mx, lo, R)) s = sp;
  }
  return s;
}

// The same step as quant_step, decided without data-dependent branches where the float
// comparisons are conclusive (the common case): the fp16 round-up of (max - lo) / levels in
// the normal fp16 range by bit operations, then the one-step corrections of quant_step chosen
// by selects.  Where a comparison is inconclusive, or the value leaves the range where the
// neighbouring fp16 numbers are one bit step away, it calls quant_step itself; so the result
// is quant_step's in every case.
__host__ __device__ __forceinline__ float quant_step_sel(float mx, float lo, float flev, float inv_lev) {
  const float R = mx - lo;
  const float q = R * inv_lev;
  const bool inside = (mx > lo) && q >= 2.0f * kFp16MinNormal && q <= 16384.f;
  uint32_t u = f32_bits(q);
  u = (u & 0x1FFFu) ? ((u | 0x1FFFu) + 1u) : u;
  const float s = bits_f32(u), sp = bits_f32(u - 0x2000u), su = bits_f32(u + 0x2000u);
  const float a = s * flev, ap = sp * flev;
  const float Rhi = R * 1.0000002384185791f, Rlo = R * 0.9999997615814209f;
  const bool a_ge = a > Rhi, a_lt = a < Rlo;
  const bool ap_ge = ap > Rhi, ap_lt = ap < Rlo;
  const bool sure = inside && (a_lt || (a_ge && (ap_ge || ap_lt)));
  if (!sure) return quant_step(mx, lo, flev, inv_lev);
  return a_lt ? su : (ap_ge ? sp : s);
}

// 1 / (2^b - 1) rounded down and up to fp32, b = 1 .. 8 (hexadecimal float literals)
__host__ __device__ __forceinline__ float inv_levels_rd(int b) {
  switch (b) {
    case 1: return 0x1.000000p+0f;
    case 2: return 0x1.555554p-2f;
    case 3: return 0x1.249248p-3f;
    case 4: return 0x1.111110p-4f;
    case 5: return 0x1.084210p-5f;
    case 6: return 0x1.041040p-6f;
    case 7: return 0x1.020408p-7f;
    default: return 0x1.010100p-8f;
  }
}
__host__ __device__ __forceinline__ float inv_levels_ru(int b) {
  switch (b) {
    case 1: return 0x1.000000p+0f;
    case 2: return 0x1.555556p-2f;
    case 3: return 0x1.24924ap-3f;
    case 4: return 0x1.111112p-4f;
    case 5: return 0x1.084212p-5f;
    case 6: return 0x1.041042p-6f;
    case 7: return 0x1.02040ap-7f;
    default: return 0x1.010102p-8f;
  }
}

// The same step as quant_step, from a bracket of the quotient: lower and upper fp32 bounds of
// (mx - lo) / levels (directed roundings of the difference and of the product with the
// directed reciprocal), each rounded up to fp16 by the conversion instruction.  When the two
// agree, the fp16 round-up of the exact quotient is that value (the round-up is monotone);
// otherwise (the quotient lies within a few fp32 ulps of an fp16 number) quant_step decides.
// The conversion also covers the fp16 subnormal range and the overflow to +inf.  On the host
// the bracket is widened by one ulp on each side in place of the directed roundings.
__host__ __device__ __forceinline__ float quant_step_cvt(float mx, float lo, int b) {
  if (!(mx > lo)) return 0.f;
#ifdef __CUDA_ARCH__
  const float rlo = __fsub_rd(mx, lo), rhi = __fsub_ru(mx, lo);
  const float qlo = __fmul_rd(rlo, inv_levels_rd(b)), qhi = __fmul_ru(rhi, inv_levels_ru(b));
#else
  const float r = mx - lo;
  const float rlo = nextafterf(r, -INFINITY), rhi = nextafterf(r, INFINITY);
  const float qlo = nextafterf(fmaxf(rlo, 0.f) * inv_levels_rd(b), -INFINITY);
  const float qhi = nextafterf(rhi * inv_levels_ru(b), INFINITY);
#endif
  const __half hlo = __float2half_ru(qlo), hhi = __float2half_ru(qhi);
  if (__half_as_ushort(hlo) != __half_as_ushort(hhi)) {
    const float flev = (float)((1 << b) - 1);
    return quant_step(mx, lo, flev, 1.0f / flev);
  }
  return __half2float(hlo);
}

// ---------------------------------------------------------------------------------------
// codes of the b-bit block quantiser and their packing
// ---------------------------------------------------------------------------------------
// round-half-even of d * inv to an integer-valued float: one FMA onto the 1.5*2^23 shift
constexpr float kRoundShift = 12582912.0f;
__host__ __device__ __forceinline__ float code_of(float d, float inv) {
#ifdef __CUDA_ARCH__
  return __fsub_rn(__fmaf_rn(d, inv, kRoundShift), kRoundShift);
#else
  volatile float t = fmaf(d, inv, kRoundShift);   // one rounding, then an exact subtraction
  return t - kRoundShift;
#endif
}

// code of one value: round((v - lo) * inv) clamped to [0, levels]; inv is the correctly
// rounded reciprocal of the fp16 step
__host__ __device__ __forceinline__ uint32_t block_code(float v, float lo, float inv, float flev) {
  float c = code_of(v - lo, inv);
  c = fminf(fmaxf(c, 0.f), flev);
  return (uint32_t)c;
}

// code j of a block occupies bits [j b, (j + 1) b) of the block's little-endian bit string,
// held as four 32-bit words (2 b bytes for 16 codes)
__host__ __device__ __forceinline__ void pack_code(uint32_t* w, int j, int b, uint32_t code) {
  const int pos = j * b;
  w[pos >> 5] |= code << (pos & 31);
  if ((pos & 31) + b > 32) w[(pos >> 5) + 1] |= code >> (32 - (pos & 31));
}
__host__ __device__ __forceinline__ uint32_t unpack_code(const uint32_t* w, int j, int b) {
  const int pos = j * b;
  uint32_t code = w[pos >> 5] >> (pos & 31);
  if ((pos & 31) + b > 32) code |= w[(pos >> 5) + 1] << (32 - (pos & 31));
  return code & ((1u << b) - 1u);
}

}  // namespace jolt
