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
constexpr int kPrologueGroup = 8;       // tokens reduced together per barrier

// grid: (ceil(T / 64), 2*Hk + Hv, B); block: 128 threads, thread = channel within the head.
template <typename Tio>
__global__ void __launch_bounds__(128)
prologue_kernel(const Tio* __restrict__ xq, const Tio* __restrict__ xk,
                const Tio* __restrict__ xv, const float* __restrict__ wq,
                const float* __restrict__ wk, const float* __restrict__ wv,
                Tio* __restrict__ yq, Tio* __restrict__ yk, Tio* __restrict__ yv, int T, int Hk,
                int Hv, int dk, int dv, float eps) {
  const int slot = blockIdx.y;
  const long b = blockIdx.z;
  const int c = threadIdx.x;
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
  const bool active = c < d;
  const long ch = (long)head * d + c;
  float w0 = 0.f, w1 = 0.f, w2 = 0.f, w3 = 0.f;
  if (active) { w0 = w[ch * 4 + 0]; w1 = w[ch * 4 + 1]; w2 = w[ch * 4 + 2]; w3 = w[ch * 4 + 3]; }

  const long t0 = (long)blockIdx.x * kPrologueTokens;
  const long tend = min((long)T, t0 + kPrologueTokens);
  auto load = [&](long t) -> float {
    return (active && t >= 0 && t < T) ? to_f(x[(b * T + t) * width + ch]) : 0.f;
  };
  float h3 = load(t0 - 3), h2 = load(t0 - 2), h1 = load(t0 - 1);   // x[t-3], x[t-2], x[t-1]

  __shared__ float red[2][kPrologueGroup][4];
  int buf = 0;
  for (long tg = t0; tg < tend; tg += kPrologueGroup) {
    float yv_[kPrologueGroup];
#pragma unroll
    for (int g = 0; g < kPrologueGroup; ++g) {
      const float xt = load(tg + g);
      const float pre = w0 * h3 + w1 * h2 + w2 * h1 + w3 * xt;
      h3 = h2; h2 = h1; h1 = xt;
      yv_[g] = active ? pre * sigmoidf_(pre) : 0.f;
    }
    if (l2) {
#pragma unroll
      for (int g = 0; g < kPrologueGroup; ++g) {
        const float s = warp_sum(yv_[g] * yv_[g]);
        if ((c & 31) == 0) red[buf][g][c >> 5] = s;
      }
      __syncthreads();
#pragma unroll
      for (int g = 0; g < kPrologueGroup; ++g) {
        const float ss = red[buf][g][0] + red[buf][g][1] + red[buf][g][2] + red[buf][g][3];
        yv_[g] *= rsqrtf(ss + eps);
      }
      buf ^= 1;
    }
    if (active) {
#pragma unroll
      for (int g = 0; g < kPrologueGroup; ++g)
        if (tg + g < tend) y[(b * T + tg + g) * width + ch] = from_f<Tio>(yv_[g]);
    }
  }
}

// One warp per row of dv <= 128 values.  `o` may be wider than z / y (the layer keeps o in fp32).
template <typename To, typename Tio>
__global__ void __launch_bounds__(256)
out_norm_kernel(const To* __restrict__ o, const Tio* __restrict__ z, const float* __restrict__ w,
                Tio* __restrict__ y, long long rows, int dv, float eps) {
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const To* orow = o + row * dv;
  const Tio* zrow = z + row * dv;
  float ov[4];
  float ss = 0.f;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int cidx = lane + 32 * e;
    ov[e] = cidx < dv ? to_f(orow[cidx]) : 0.f;
    ss += ov[e] * ov[e];
  }
  ss = warp_sum(ss);
  const float inv = rsqrtf(ss / dv + eps);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int cidx = lane + 32 * e;
    if (cidx < dv) {
      const float zz = to_f(zrow[cidx]);
      y[row * dv + cidx] = from_f<Tio>(ov[e] * inv * w[cidx] * (zz * sigmoidf_(zz)));
    }
  }
}

}  // namespace gdn
