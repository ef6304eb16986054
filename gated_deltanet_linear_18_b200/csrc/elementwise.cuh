// Bandwidth-bound prologue and epilogue of the Gated DeltaNet layer.
//
// Prologue ("L'attention hybride", "Le décompte": a causal convolution with 4 taps per channel
// and no bias over the q, k and v channels; "Les briques d'un réseau de neurones", 2.: SiLU):
//   y[t, c] = SiLU( sum_{j<4} w[c, j] x[t - 3 + j, c] ),  x[t < 0] = 0,
// then each q and k head vector is divided by sqrt(|y|^2 + eps).
// Epilogue (same pages: swish output gate, one dv-wide gain; 4.: RMSNorm):
//   y = o / sqrt(mean(o^2) + eps) * w (.) z sigmoid(z).
#pragma once

#include "common.cuh"

namespace gdn {

constexpr int kPrologueTokens = 64;     // tokens per CTA

// Vectors of 16 bytes: 8 bf16 or 4 fp32 values.
template <typename T> struct Vec16;
template <> struct Vec16<float> {
  static constexpr int N = 4;
  static __device__ __forceinline__ void load(const float* p, float (&v)[4]) {
    const float4 a = *reinterpret_cast<const float4*>(p);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  }
  static __device__ __forceinline__ void store(float* p, const float (&v)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  }
};
template <> struct Vec16<__nv_bfloat16> {
  static constexpr int N = 8;
  static __device__ __forceinline__ void load(const __nv_bfloat16* p, float (&v)[8]) {
    const uint4 a = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = __uint_as_float(w[i] << 16);
      v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, const float (&v)[8]) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      __nv_bfloat162 h = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
      w[i] = *reinterpret_cast<uint32_t*>(&h);
    }
    *reinterpret_cast<uint4*>(p) = make_uint4(w[0], w[1], w[2], w[3]);
  }
};

__device__ __forceinline__ float silu_fast(float x) { return __fdividef(x, 1.0f + __expf(-x)); }

// grid: (ceil(T / kPrologueTokens), 2*Hk + Hv, B); block: 128 threads.  One CTA takes one head
// (d channels) of kPrologueTokens tokens: the raw rows of those tokens and of the three before
// them (zeros before t = 0) come into shared memory by 16-byte asynchronous copies, all issued at
// once (so each SM keeps many tiles' worth of loads in flight), then every token is convolved from
// shared memory.  A head row of d channels is held by L = d / N threads (N channels of one 16-byte
// vector each); the 128 / L row groups of the CTA take every (128 / L)-th token.  The L2 norm of a
// q or k row is a shuffle reduction over its L threads (one warp).
template <typename Tio>
__global__ void __launch_bounds__(128)
prologue_kernel(const Tio* __restrict__ xq, const Tio* __restrict__ xk,
                const Tio* __restrict__ xv, const float* __restrict__ wq,
                const float* __restrict__ wk, const float* __restrict__ wv,
                Tio* __restrict__ yq, Tio* __restrict__ yk, Tio* __restrict__ yv, int T, int Hk,
                int Hv, int dk, int dv, float eps) {
  constexpr int N = Vec16<Tio>::N;
  constexpr int R = kPrologueTokens + 3;      // staged rows: 3 history tokens, then the tile
  extern __shared__ __align__(16) uint8_t pro_smem[];
  Tio* tile = reinterpret_cast<Tio*>(pro_smem);
  const int slot = blockIdx.y;
  const long b = blockIdx.z;
  const Tio* x;
  const float* w;
  Tio* y;
  int d, head, width;
  bool l2;
  if (slot < Hk) {
    x = xq; w = wq; y = yq; d = dk; head = slot; width = Hk * dk; l2 = true;
  } else if (slot < 2 * Hk) {
    x = xk; w = wk; y = yk; d = dk; head = slot - Hk; width = Hk * dk; l2 = true;
  } else {
    x = xv; w = wv; y = yv; d = dv; head = slot - 2 * Hk; width = Hv * dv; l2 = false;
  }
  const int L = d / N;                        // 2 .. 32, a power of two
  const long t0 = (long)blockIdx.x * kPrologueTokens;
  const Tio* xh = x + b * T * (long)width + (long)head * d;
  // stage rows t0 - 3 .. t0 + kPrologueTokens - 1 (row r holds token t0 - 3 + r)
  for (int i = threadIdx.x; i < R * L; i += 128) {
    const int r = i / L, c = i - r * L;
    const long t = t0 - 3 + r;
    const bool in = t >= 0 && t < T;
    const Tio* src = in ? xh + t * width + c * N : xh;
    const uint32_t dst = static_cast<uint32_t>(__cvta_generic_to_shared(tile + (long)r * d + c * N));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
                 "r"(in ? 16 : 0) : "memory");
  }
  asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;" ::: "memory");
  const int grp = threadIdx.x / L, lc = threadIdx.x % L, ngrp = 128 / L;
  const long c0 = (long)head * d + lc * N;    // first channel of this thread
  float wt[N][4];
#pragma unroll
  for (int i = 0; i < N; ++i)                 // weights need only 4-byte alignment
#pragma unroll
    for (int j = 0; j < 4; ++j) wt[i][j] = w[(c0 + i) * 4 + j];
  __syncthreads();
  const long rem = T - t0;
  const int nt = rem < kPrologueTokens ? (int)rem : kPrologueTokens;
  for (int i = grp; i < kPrologueTokens; i += ngrp) {   // same trip count within a warp
    float h[4][N];
#pragma unroll
    for (int j = 0; j < 4; ++j) Vec16<Tio>::load(tile + (long)(i + j) * d + lc * N, h[j]);
    float yv_[N];
    float ss = 0.f;
#pragma unroll
    for (int j = 0; j < N; ++j) {
      const float pre = wt[j][0] * h[0][j] + wt[j][1] * h[1][j] + wt[j][2] * h[2][j] +
                        wt[j][3] * h[3][j];
      yv_[j] = silu_fast(pre);
      ss += yv_[j] * yv_[j];
    }
    if (l2) {
      for (int o = L >> 1; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      const float inv = rsqrtf(ss + eps);
#pragma unroll
      for (int j = 0; j < N; ++j) yv_[j] *= inv;
    }
    if (i < nt) Vec16<Tio>::store(y + (b * T + t0 + i) * width + c0, yv_);
  }
}

// Shared memory of one prologue CTA for heads of d channels.
inline size_t prologue_smem_bytes(int d, size_t elem) {
  return (size_t)(kPrologueTokens + 3) * d * elem;
}

// One warp per row of dv <= 128 values, 4 consecutive channels per lane.  `o` may be wider than
// z / y (the layer keeps o in fp32).
template <typename T4> struct Vec4;
template <> struct Vec4<float> {
  static __device__ __forceinline__ void load(const float* p, float (&v)[4]) {
    const float4 a = *reinterpret_cast<const float4*>(p);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  }
  static __device__ __forceinline__ void store(float* p, const float (&v)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  }
};
template <> struct Vec4<__nv_bfloat16> {
  static __device__ __forceinline__ void load(const __nv_bfloat16* p, float (&v)[4]) {
    const uint2 a = *reinterpret_cast<const uint2*>(p);
    v[0] = __uint_as_float(a.x << 16); v[1] = __uint_as_float(a.x & 0xFFFF0000u);
    v[2] = __uint_as_float(a.y << 16); v[3] = __uint_as_float(a.y & 0xFFFF0000u);
  }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, const float (&v)[4]) {
    __nv_bfloat162 h0 = __floats2bfloat162_rn(v[0], v[1]), h1 = __floats2bfloat162_rn(v[2], v[3]);
    *reinterpret_cast<uint2*>(p) =
        make_uint2(*reinterpret_cast<uint32_t*>(&h0), *reinterpret_cast<uint32_t*>(&h1));
  }
};

template <typename To, typename Tz, typename Ty = Tz>
__global__ void __launch_bounds__(256)
out_norm_kernel(const To* __restrict__ o, const Tz* __restrict__ z, const float* __restrict__ w,
                Ty* __restrict__ y, long long rows, int dv, float eps) {
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const int c = 4 * lane;
  const bool active = c < dv;
  float ov[4] = {0.f, 0.f, 0.f, 0.f}, zv[4] = {0.f, 0.f, 0.f, 0.f};
  if (active) {
    Vec4<To>::load(o + row * dv + c, ov);
    Vec4<Tz>::load(z + row * dv + c, zv);
  }
  float ss = (ov[0] * ov[0] + ov[1] * ov[1]) + (ov[2] * ov[2] + ov[3] * ov[3]);
  ss = warp_sum(ss);
  const float inv = rsqrtf(ss / dv + eps);
  if (active) {
    const float ww[4] = {w[c], w[c + 1], w[c + 2], w[c + 3]};
    float yv[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) yv[e] = ov[e] * inv * ww[e] * silu_fast(zv[e]);
    Vec4<Ty>::store(y + row * dv + c, yv);
  }
}

// Gates from the in_proj_ba outputs: beta = sigmoid(b), log alpha = -softplus(-a), one thread per
// (token, value head); rows of 2 Hv inputs and Hv outputs, so both sides are read and written
// contiguously across the threads of a warp.
template <typename Tin>
__global__ void gates_kernel(const Tin* __restrict__ ba, float* __restrict__ log_alpha,
                             float* __restrict__ beta, long long rows, int Hv) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= rows * Hv) return;
  const long long r = i / Hv;
  const int h = (int)(i - r * Hv);
  const float b = to_f(ba[r * 2 * Hv + h]), a = to_f(ba[r * 2 * Hv + Hv + h]);
  beta[i] = 1.0f / (1.0f + expf(-b));
  // -softplus(-a), written so that neither branch overflows
  log_alpha[i] = a >= 0.f ? -log1pf(expf(-a)) : a - log1pf(expf(a));
}

}  // namespace gdn
