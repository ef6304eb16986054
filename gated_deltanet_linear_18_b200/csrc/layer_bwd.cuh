// Backward of the layer's pieces around the recurrence: the gated RMSNorm, the causal conv + SiLU
// (+ L2 norm for q and k) prologue and the gates from in_proj_ba.  Each is the chain rule through
// its forward definition ("L'attention hybride", "Les 48 couches Gated DeltaNet": conv kernel 4,
// swish output gate; "Le décompte": 4 conv weights per channel, one norm gain; "Les briques d'un
// réseau de neurones", 2.: SiLU(x) = x sigmoid(x), 4.: RMSNorm).  Weight gradients (norm gain,
// conv taps) are sums over tokens: every CTA writes its partial sums and col_sum_kernel adds them
// in a fixed order, so results do not depend on scheduling.
#pragma once

#include "common.cuh"

namespace gdn {
namespace lbwd {

__device__ __forceinline__ float sigm(float x) { return 1.0f / (1.0f + expf(-x)); }
// d/dx of x sigmoid(x)
__device__ __forceinline__ float silu_grad(float x) {
  const float s = sigm(x);
  return s * (1.0f + x * (1.0f - s));
}

constexpr int kNormWarps = 8;

// Gated RMSNorm backward, y = o inv w SiLU(z), inv = 1 / sqrt(mean(o^2) + eps), one warp per row of
// dv <= 128 (4 columns per lane), rows strided over a fixed grid:
//   g = dy w SiLU(z);  do = inv g - o inv^3 (g . o) / dv;  dz = dy o inv w SiLU'(z);
//   dw += dy o inv SiLU(z)  (per CTA: dw_part[blockIdx.x][dv]).
template <typename Tz, typename Ty>
__global__ void __launch_bounds__(32 * kNormWarps)
out_norm_bwd_kernel(const float* __restrict__ o, const Tz* __restrict__ z,
                    const float* __restrict__ w, const Ty* __restrict__ dy,
                    float* __restrict__ d_o, float* __restrict__ dz, float* __restrict__ dw_part,
                    long long rows, int dv, float eps) {
  __shared__ float part[kNormWarps][128];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, c = 4 * lane;
  const bool active = c < dv;
  float ww[4] = {0.f, 0.f, 0.f, 0.f}, acc[4] = {0.f, 0.f, 0.f, 0.f};
  if (active)
    for (int e = 0; e < 4; ++e) ww[e] = w[c + e];
  for (long long row = (long long)blockIdx.x * kNormWarps + warp; row < rows;
       row += (long long)gridDim.x * kNormWarps) {
    float ov[4] = {0.f, 0.f, 0.f, 0.f}, zv[4] = {0.f, 0.f, 0.f, 0.f}, gv[4] = {0.f, 0.f, 0.f, 0.f};
    if (active)
      for (int e = 0; e < 4; ++e) {
        ov[e] = o[row * dv + c + e];
        zv[e] = to_f(z[row * dv + c + e]);
        gv[e] = to_f(dy[row * dv + c + e]);
      }
    float ss = 0.f;
    for (int e = 0; e < 4; ++e) ss = fmaf(ov[e], ov[e], ss);
    ss = warp_sum(ss);
    const float inv = 1.0f / sqrtf(ss / dv + eps);
    float g[4], go = 0.f;
    for (int e = 0; e < 4; ++e) {
      const float sz = zv[e] * sigm(zv[e]);
      g[e] = gv[e] * ww[e] * sz;
      go = fmaf(g[e], ov[e], go);
      acc[e] = fmaf(gv[e] * ov[e] * inv, sz, acc[e]);
    }
    go = warp_sum(go);
    if (active)
      for (int e = 0; e < 4; ++e) {
        d_o[row * dv + c + e] = inv * g[e] - ov[e] * inv * inv * inv * go / dv;
        dz[row * dv + c + e] = gv[e] * ov[e] * inv * ww[e] * silu_grad(zv[e]);
      }
  }
  if (active)
    for (int e = 0; e < 4; ++e) part[warp][c + e] = acc[e];
  __syncthreads();
  for (int j = threadIdx.x; j < dv; j += blockDim.x) {
    float s = 0.f;
    for (int wp = 0; wp < kNormWarps; ++wp) s += part[wp][j];
    dw_part[(long long)blockIdx.x * dv + j] = s;
  }
}

// out[j] = sum over i < n of part[i * m + j] (in order of i).
__global__ void col_sum_kernel(const float* __restrict__ part, float* __restrict__ out, int n,
                               int m) {
  const int j = blockIdx.x * blockDim.x + threadIdx.x;
  if (j >= m) return;
  float s = 0.f;
  for (int i = 0; i < n; ++i) s += part[(long)i * m + j];
  out[j] = s;
}

// Prologue backward, step 1: the gradient at the convolution's output (pre), one warp per
// (token, head) row of d channels (d / 32 per lane, d in {32, 64, 128}; 16: lanes 0..15).
//   s = SiLU(pre);  q, k (normalize): y = s / n, n = sqrt(s . s + eps),
//   ds = dy / n - s (s . dy) / n^3;  v: ds = dy;  dpre = ds SiLU'(pre).
// x: raw inputs [B, T, heads * d]; dy: [B, T, heads, d] fp32; dpre: [B, T, heads * d] fp32.
template <typename Tin>
__global__ void __launch_bounds__(256)
conv_dpre_kernel(const Tin* __restrict__ x, const float* __restrict__ w,
                 const float* __restrict__ dy, float* __restrict__ dpre, long long rows, int T,
                 int heads, int d, int normalize, float eps) {
  const long long row = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);   // (b * T + t) * heads + h
  const int lane = threadIdx.x & 31;
  if (row >= rows) return;
  const int h = (int)(row % heads);
  const long long bt = row / heads;
  const int t = (int)(bt % T);
  const int C = heads * d;
  constexpr int kMax = 4;                             // channels per lane (d <= 128)
  float pre[kMax], s[kMax], g[kMax];
  float ss = 0.f, sd = 0.f;
  const int per = d >= 32 ? d / 32 : 1;
  const bool lane_on = d >= 32 || lane < d;
  for (int e = 0; e < kMax; ++e) {
    pre[e] = s[e] = g[e] = 0.f;
    if (e >= per || !lane_on) continue;
    const int ch = h * d + lane * per + e;
    float acc = 0.f;
    for (int j = 0; j < 4; ++j) {
      const int u = t - 3 + j;
      if (u >= 0) acc = fmaf(w[ch * 4 + j], to_f(x[(bt - t + u) * C + ch]), acc);
    }
    pre[e] = acc;
    s[e] = acc * sigm(acc);
    g[e] = dy[row * d + lane * per + e];
    ss = fmaf(s[e], s[e], ss);
    sd = fmaf(s[e], g[e], sd);
  }
  float n = 1.f, n3 = 1.f;
  if (normalize) {
    ss = warp_sum(ss);
    sd = warp_sum(sd);
    n = sqrtf(ss + eps);
    n3 = n * n * n;
  }
  for (int e = 0; e < per && lane_on; ++e) {
    const float ds = normalize ? g[e] / n - s[e] * sd / n3 : g[e];
    dpre[bt * C + h * d + lane * per + e] = ds * silu_grad(pre[e]);
  }
}

constexpr int kConvTok = 64;    // tokens per CTA of conv_bwd_kernel

// Prologue backward, step 2: through the 4-tap convolution, one thread per channel of a
// 128-channel block over kConvTok tokens:  dx[t] = sum_j w[j] dpre[t + 3 - j]  (t + 3 - j < T),
//   dw[j] += dpre[t] x[t - 3 + j]  (t - 3 + j >= 0), per CTA: dw_part[cta][C][4], cta over
//   (token tile, batch).  grid (ceil(C / 128), ceil(T / kConvTok), B).
template <typename Tin>
__global__ void __launch_bounds__(128)
conv_bwd_kernel(const Tin* __restrict__ x, const float* __restrict__ w,
                const float* __restrict__ dpre, float* __restrict__ dx,
                float* __restrict__ dw_part, int T, int C) {
  const int c = blockIdx.x * 128 + threadIdx.x;
  const long b = blockIdx.z;
  const int t0 = blockIdx.y * kConvTok;
  const long cta = (long)blockIdx.z * gridDim.y + blockIdx.y;
  if (c >= C) return;
  const float w0 = w[c * 4], w1 = w[c * 4 + 1], w2 = w[c * 4 + 2], w3 = w[c * 4 + 3];
  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
  const int t1 = min(T, t0 + kConvTok);
  auto P = [&](int t) -> float { return t < T ? dpre[(b * T + t) * C + c] : 0.f; };
  auto X = [&](int t) -> float { return t >= 0 ? to_f(x[(b * T + t) * C + c]) : 0.f; };
  for (int t = t0; t < t1; ++t) {
    // tap j multiplies x[t - 3 + j] in the output at t, so x[t] feeds outputs t + 3 - j
    dx[(b * T + t) * C + c] = fmaf(w0, P(t + 3), fmaf(w1, P(t + 2), fmaf(w2, P(t + 1), w3 * P(t))));
    const float p = P(t);
    a0 = fmaf(p, X(t - 3), a0);
    a1 = fmaf(p, X(t - 2), a1);
    a2 = fmaf(p, X(t - 1), a2);
    a3 = fmaf(p, X(t), a3);
  }
  float* dp = dw_part + (cta * C + c) * 4;
  dp[0] = a0;
  dp[1] = a1;
  dp[2] = a2;
  dp[3] = a3;
}

// Gates backward: db = dbeta beta (1 - beta), da = dlog_alpha sigmoid(-a), one thread per (token,
// value head); dba [rows, 2 Hv] fp32 (the b gradients, then the a gradients).
template <typename Tin>
__global__ void gates_bwd_kernel(const Tin* __restrict__ ba, const float* __restrict__ dla,
                                 const float* __restrict__ dbeta, float* __restrict__ dba,
                                 long long rows, int Hv) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= rows * Hv) return;
  const long long r = i / Hv;
  const int h = (int)(i - r * Hv);
  const float b = to_f(ba[r * 2 * Hv + h]), a = to_f(ba[r * 2 * Hv + Hv + h]);
  const float sb = sigm(b);
  dba[r * 2 * Hv + h] = dbeta[i] * sb * (1.0f - sb);
  dba[r * 2 * Hv + Hv + h] = dla[i] * sigm(-a);
}

}  // namespace lbwd
}  // namespace gdn
