// Shared device helpers of the JoLT library: the counter-based random numbers that
// draw the rotation signs and the FlashJoLT sketch matrix, rounding helpers, and the
// device status word kernels raise errors through.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>

namespace jolt {

// number of kernels this library has launched in the process (all threads)
inline std::atomic<unsigned long long>& launch_counter() {
  static std::atomic<unsigned long long> n{0};
  return n;
}
// while this thread captures a CUDA graph, its launches are counted here instead (they run
// when the graph is launched, and are added to the process count at every launch)
inline unsigned long long*& capture_counter() {
  thread_local unsigned long long* c = nullptr;
  return c;
}
inline void count_launch() {
  if (capture_counter()) ++*capture_counter();
  else launch_counter().fetch_add(1, std::memory_order_relaxed);
}

typedef __nv_bfloat16 bf16;

// ---- device status bits (OR-ed into a 32-bit word in the workspace) -------------------
enum : uint32_t {
  DEV_ERR_NONFINITE = 1u,     // NaN / Inf met in the input cache
  DEV_ERR_FACTOR = 2u,        // Cholesky / eigen breakdown
  DEV_ERR_INFEASIBLE = 4u,    // budget below the fewest-bytes choice of every unit
  DEV_ERR_BLOB = 8u,          // a compressed record failed validation
  DEV_ERR_CAPACITY = 16u,     // output buffer smaller than the chosen payload
  DEV_ERR_TIMEOUT = 32u,      // a bounded device-side wait gave up
};

// ---- splitmix64 (Steele, Lea & Flood, OOPSLA 2014) ------------------------------------
constexpr uint64_t kGoldenGamma = 0x9E3779B97F4A7C15ull;
constexpr uint64_t kIndexMult = 0xD1B54A32D192ED03ull;
constexpr uint32_t kStreamOmega = 1u;
constexpr uint32_t kStreamSign = 2u;

__host__ __device__ __forceinline__ uint64_t splitmix64_mix(uint64_t z) {
  z += kGoldenGamma;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

__host__ __device__ __forceinline__ uint64_t stream_id(uint32_t kind, int unit) {
  return ((uint64_t)kind << 32) | (uint32_t)unit;
}

__host__ __device__ __forceinline__ uint64_t hash64(uint64_t seed, uint64_t stream, uint64_t idx) {
  return splitmix64_mix((seed ^ (stream * kGoldenGamma)) + idx * kIndexMult);
}

// sigma_d = -1 when the low bit of the hash is set
__host__ __device__ __forceinline__ float rotation_sign(uint64_t seed, int unit, int d) {
  return (hash64(seed, stream_id(kStreamSign, unit), (uint64_t)d) & 1ull) ? -1.0f : 1.0f;
}

// Box-Muller in double precision on two independent 53-bit uniforms
__device__ __forceinline__ double gaussian(uint64_t seed, uint64_t stream, uint64_t idx) {
  uint64_t h1 = hash64(seed, stream, idx);
  uint64_t h2 = hash64(seed, stream, idx | (1ull << 63));
  double u1 = (double)((h1 >> 11) + 1ull) * 0x1p-53;
  double u2 = (double)(h2 >> 11) * 0x1p-53;
  return sqrt(-2.0 * log(u1)) * cos((2.0 * 3.14159265358979323846) * u2);
}

__device__ __forceinline__ float ld_as_float(const bf16* p) { return __bfloat162float(*p); }
__device__ __forceinline__ float ld_as_float(const float* p) { return *p; }

__device__ __forceinline__ void raise_status(uint32_t* status, uint32_t bits) {
  if (status) atomicOr(status, bits);
}

// In-register unnormalised Walsh-Hadamard transform of N values (Sylvester order)
template <int N>
__device__ __forceinline__ void fwht_regs(float* v) {
#pragma unroll
  for (int h = 1; h < N; h <<= 1) {
#pragma unroll
    for (int i = 0; i < N; i += 2 * h) {
#pragma unroll
      for (int j = i; j < i + h; ++j) {
        float a = v[j], b = v[j + h];
        v[j] = a + b;
        v[j + h] = a - b;
      }
    }
  }
}

__host__ __device__ __forceinline__ long long ceil_div(long long a, long long b) { return (a + b - 1) / b; }
__host__ __device__ __forceinline__ long long round_up(long long a, long long b) { return ceil_div(a, b) * b; }

}  // namespace jolt
