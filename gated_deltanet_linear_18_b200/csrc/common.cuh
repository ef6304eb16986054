// Shared device helpers of the gated delta rule library (one translation unit: gdn_api.cu).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace gdn {

// Per-device error word.  Kernels that give up on a bounded wait OR a bit in here and skip the rest
// of their work; gdn_check_error reads and clears it.  Statically allocated with the module.
__device__ unsigned int g_error_word = 0u;

enum : unsigned int { kErrTimeout = 1u };

__device__ __forceinline__ void record_error(unsigned int bits) { atomicOr(&g_error_word, bits); }

template <typename T> __device__ __forceinline__ float to_f(T x);
template <> __device__ __forceinline__ float to_f<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) {
  return __bfloat162float(x);
}

template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

__device__ __forceinline__ float sigmoidf_(float x) { return 1.0f / (1.0f + expf(-x)); }

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Two fp32 lanes in one 64-bit register pair, for the paired fp32 instructions of sm_100 (each lane
// is the IEEE round-to-nearest operation of its scalar counterpart).
using f2_t = unsigned long long;
__device__ __forceinline__ f2_t pk2(float a, float b) {
  f2_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ void up2(f2_t r, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(r));
}
__device__ __forceinline__ f2_t fma2(f2_t a, f2_t b, f2_t c) {   // a b + c
  f2_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ f2_t mul2(f2_t a, f2_t b) {
  f2_t r;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ f2_t add2(f2_t a, f2_t b) {
  f2_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}
__device__ __forceinline__ f2_t splat2(float a) { return pk2(a, a); }
__device__ __forceinline__ float hsum2(f2_t r) {
  float a, b;
  up2(r, a, b);
  return a + b;
}

// Rows of sequence s: of [B, T, ...] tensors (cu == nullptr), rows s T .. s T + T - 1; packed
// (cu != nullptr), rows cu[s] .. cu[s + 1] - 1 of [T, ...] tensors (T = total rows), clamped to
// the tensor and cut at max_len, so that malformed offsets cannot reach outside it.
struct RowSpan {
  long row0;
  int len;
};
__device__ __forceinline__ RowSpan row_span(const int* __restrict__ cu, int s, int T,
                                            int max_len) {
  if (!cu) return RowSpan{(long)s * T, T};
  const int a = min(max(cu[s], 0), T);
  const int b = min(max(cu[s + 1], a), min(T, a + max_len));
  return RowSpan{(long)a, b - a};
}

}  // namespace gdn
