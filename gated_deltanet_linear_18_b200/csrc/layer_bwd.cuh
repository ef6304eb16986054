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

// Vectors of PER consecutive values (PER in 1, 2, 4) as fp32: PER x 4 bytes of fp32 or PER x 2 of
// bf16, read with one load (the pointer aligned to that size).
template <int PER, typename T>
__device__ __forceinline__ void vload(const T* p, float (&v)[PER]) {
  if constexpr (sizeof(T) == 4) {
    if constexpr (PER == 4) {
      const float4 a = *reinterpret_cast<const float4*>(p);
      v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    } else if constexpr (PER == 2) {
      const float2 a = *reinterpret_cast<const float2*>(p);
      v[0] = a.x; v[1] = a.y;
    } else {
      v[0] = to_f(p[0]);
    }
  } else {
    if constexpr (PER == 4) {
      const uint2 a = *reinterpret_cast<const uint2*>(p);
      v[0] = __uint_as_float(a.x << 16); v[1] = __uint_as_float(a.x & 0xFFFF0000u);
      v[2] = __uint_as_float(a.y << 16); v[3] = __uint_as_float(a.y & 0xFFFF0000u);
    } else if constexpr (PER == 2) {
      const uint32_t a = *reinterpret_cast<const uint32_t*>(p);
      v[0] = __uint_as_float(a << 16); v[1] = __uint_as_float(a & 0xFFFF0000u);
    } else {
      v[0] = to_f(p[0]);
    }
  }
}
template <int PER>
__device__ __forceinline__ void vstore(float* p, const float (&v)[PER]) {
  if constexpr (PER == 4) *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  else if constexpr (PER == 2) *reinterpret_cast<float2*>(p) = make_float2(v[0], v[1]);
  else p[0] = v[0];
}

// Gated RMSNorm backward, y = o inv w SiLU(z), inv = 1 / sqrt(mean(o^2) + eps), one warp per row of
// dv <= 128 (4 columns per lane, read and written as vectors), rows strided over a fixed grid:
//   g = dy w SiLU(z);  do = inv g - o inv^3 (g . o) / dv;  dz = dy o inv w SiLU'(z);
//   dw += dy o inv SiLU(z)  (per CTA: dw_part[blockIdx.x][dv]).
// dz is written as one 16-byte vector per lane when dz_vec (the caller's dz 16-byte aligned), else
// value by value.
template <typename Tz, typename Ty>
__global__ void __launch_bounds__(32 * kNormWarps)
out_norm_bwd_kernel(const float* __restrict__ o, const Tz* __restrict__ z,
                    const float* __restrict__ w, const Ty* __restrict__ dy,
                    float* __restrict__ d_o, float* __restrict__ dz, float* __restrict__ dw_part,
                    long long rows, int dv, float eps, int dz_vec) {
  __shared__ float part[kNormWarps][128];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, c = 4 * lane;
  const bool active = c < dv;
  float ww[4] = {0.f, 0.f, 0.f, 0.f}, acc[4] = {0.f, 0.f, 0.f, 0.f};
  if (active)
    for (int e = 0; e < 4; ++e) ww[e] = w[c + e];
  for (long long row = (long long)blockIdx.x * kNormWarps + warp; row < rows;
       row += (long long)gridDim.x * kNormWarps) {
    float ov[4] = {0.f, 0.f, 0.f, 0.f}, zv[4] = {0.f, 0.f, 0.f, 0.f}, gv[4] = {0.f, 0.f, 0.f, 0.f};
    if (active) {
      vload<4>(o + row * dv + c, ov);
      vload<4>(z + row * dv + c, zv);
      vload<4>(dy + row * dv + c, gv);
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
    if (active) {
      float dov[4], dzv[4];
      for (int e = 0; e < 4; ++e) {
        dov[e] = inv * g[e] - ov[e] * inv * inv * inv * go / dv;
        dzv[e] = gv[e] * ov[e] * inv * ww[e] * silu_grad(zv[e]);
      }
      vstore<4>(d_o + row * dv + c, dov);
      if (dz_vec) vstore<4>(dz + row * dv + c, dzv);
      else
        for (int e = 0; e < 4; ++e) dz[row * dv + c + e] = dzv[e];
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

constexpr int kDpreTok = 64;    // tokens per CTA of conv_dpre_kernel (16 per warp)

// Prologue backward, step 1: the gradient at the convolution's output (pre).  grid (heads,
// ceil(T / kDpreTok), B), 128 threads: warp w takes 16 consecutive tokens of one head, lane l the
// channels l PER .. l PER + PER - 1 of it (d = 32 PER; for d = 16, PER = 1 and lanes 16.. idle),
// with the weights loaded once and the 4-tap window of raw inputs in a ring of four register rows
// (token t reads slots t .. t + 3 mod 4, the loop unrolled by four):
//   s = SiLU(pre);  q, k (normalize): y = s / n, n = sqrt(s . s + eps),
//   ds = dy / n - s (s . dy) / n^3;  v: ds = dy;  dpre = ds SiLU'(pre).
// x: raw inputs [B, T, heads * d]; dy: [B, T, heads, d] fp32; dpre: [B, T, heads * d] fp32; x, dy
// and dpre aligned to PER values.  Sequences as in row_span (cu: packed rows of T in all, grid z
// over the sequences, y over ceil(max_len / kDpreTok) tiles).
template <typename Tin, int PER>
__global__ void __launch_bounds__(128)
conv_dpre_kernel(const Tin* __restrict__ x, const float* __restrict__ w,
                 const float* __restrict__ dy, float* __restrict__ dpre, int T, int heads, int d,
                 int normalize, float eps, const int* __restrict__ cu, int max_len) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int h = blockIdx.x;
  const RowSpan sp = row_span(cu, (int)blockIdx.z, T, max_len);   // this sequence's rows
  const long r0 = sp.row0;
  const int Ts = sp.len;
  const int tb = blockIdx.y * kDpreTok + warp * (kDpreTok / 4);
  const int C = heads * d;
  const bool on = lane * PER < d;
  const int ch0 = h * d + lane * PER;         // this lane's first channel
  float wt[PER][4];
#pragma unroll
  for (int e = 0; e < PER; ++e)
#pragma unroll
    for (int j = 0; j < 4; ++j) wt[e][j] = on ? w[(ch0 + e) * 4 + j] : 0.f;
  const Tin* xb = x + r0 * C + ch0;
  auto row_in = [&](int t, float (&v)[PER]) {  // raw inputs of token t (zeros outside 0 .. Ts - 1)
#pragma unroll
    for (int e = 0; e < PER; ++e) v[e] = 0.f;
    if (on && t >= 0 && t < Ts) vload<PER>(xb + (long)t * C, v);
  };
  float r[4][PER];
  row_in(tb - 3, r[0]);
  row_in(tb - 2, r[1]);
  row_in(tb - 1, r[2]);
#pragma unroll 1
  for (int t4 = 0; t4 < kDpreTok / 4; t4 += 4) {
#pragma unroll
    for (int sl = 0; sl < 4; ++sl) {
      const int t = tb + t4 + sl;
      if (t >= Ts) break;                     // uniform over the warp
      const int q0 = sl, r1 = (sl + 1) & 3, r2 = (sl + 2) & 3, r3 = (sl + 3) & 3;
      row_in(t, r[r3]);
      const long row = (r0 + t) * heads + h;
      float pre[PER], s[PER], g[PER];
#pragma unroll
      for (int e = 0; e < PER; ++e) g[e] = 0.f;
      if (on) vload<PER>(dy + row * d + lane * PER, g);
      float ss = 0.f, sd = 0.f;
#pragma unroll
      for (int e = 0; e < PER; ++e) {
        // the taps in order (w[.., 3] on token t), as the forward's sum; a zero-history tap adds
        // nothing
        float acc = 0.f;
        if (t - 3 >= 0) acc = fmaf(wt[e][0], r[q0][e], acc);
        if (t - 2 >= 0) acc = fmaf(wt[e][1], r[r1][e], acc);
        if (t - 1 >= 0) acc = fmaf(wt[e][2], r[r2][e], acc);
        acc = fmaf(wt[e][3], r[r3][e], acc);
        pre[e] = acc;
        s[e] = acc * sigm(acc);
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
      if (on) {
        float out[PER];
#pragma unroll
        for (int e = 0; e < PER; ++e) {
          const float ds = normalize ? g[e] / n - s[e] * sd / n3 : g[e];
          out[e] = ds * silu_grad(pre[e]);
        }
        vstore<PER>(dpre + (r0 + t) * (long)C + ch0, out);
      }
    }
  }
}

constexpr int kConvTok = 64;    // tokens per CTA of conv_bwd_kernel

// Prologue backward, step 2: through the 4-tap convolution, one thread per channel of a
// 128-channel block over kConvTok tokens, dpre and x in rings of four registers (each read once):
//   dx[t] = sum_j w[j] dpre[t + 3 - j]  (t + 3 - j < T),
//   dw[j] += dpre[t] x[t - 3 + j]  (t - 3 + j >= 0), per CTA: dw_part[cta][C][4], cta over
//   (token tile, batch).  grid (ceil(C / 128), ceil(T / kConvTok), B); packed sequences as in
//   conv_dpre_kernel (a tile past its sequence's end writes zero partial sums).
template <typename Tin>
__global__ void __launch_bounds__(128)
conv_bwd_kernel(const Tin* __restrict__ x, const float* __restrict__ w,
                const float* __restrict__ dpre, float* __restrict__ dx,
                float* __restrict__ dw_part, int T, int C, const int* __restrict__ cu,
                int max_len) {
  const int c = blockIdx.x * 128 + threadIdx.x;
  const RowSpan sp = row_span(cu, (int)blockIdx.z, T, max_len);   // this sequence's rows
  const long r0 = sp.row0;
  const int Ts = sp.len;
  const int t0 = blockIdx.y * kConvTok;
  const long cta = (long)blockIdx.z * gridDim.y + blockIdx.y;
  if (c >= C) return;
  const float w0 = w[c * 4], w1 = w[c * 4 + 1], w2 = w[c * 4 + 2], w3 = w[c * 4 + 3];
  float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
  const int t1 = min(Ts, t0 + kConvTok);
  auto P = [&](int t) -> float { return t < Ts ? dpre[(r0 + t) * C + c] : 0.f; };
  auto X = [&](int t) -> float { return t >= 0 && t < Ts ? to_f(x[(r0 + t) * C + c]) : 0.f; };
  // p[t mod 4] = dpre[t] for t .. t + 3, xr[t mod 4] = x[t - 3 + ...] for t - 3 .. t
  float p[4], xr[4];
  p[0] = P(t0); p[1] = P(t0 + 1); p[2] = P(t0 + 2);
  xr[0] = X(t0 - 3); xr[1] = X(t0 - 2); xr[2] = X(t0 - 1);
#pragma unroll 1
  for (int t4 = 0; t4 < kConvTok; t4 += 4) {
#pragma unroll
    for (int sl = 0; sl < 4; ++sl) {
      const int t = t0 + t4 + sl;
      if (t >= t1) break;
      const int q0 = sl, r1 = (sl + 1) & 3, r2 = (sl + 2) & 3, r3 = (sl + 3) & 3;
      p[r3] = P(t + 3);
      xr[r3] = X(t);
      // tap j multiplies x[t - 3 + j] in the output at t, so x[t] feeds outputs t + 3 - j
      dx[(r0 + t) * C + c] = fmaf(w0, p[r3], fmaf(w1, p[r2], fmaf(w2, p[r1], w3 * p[q0])));
      a0 = fmaf(p[q0], xr[q0], a0);
      a1 = fmaf(p[q0], xr[r1], a1);
      a2 = fmaf(p[q0], xr[r2], a2);
      a3 = fmaf(p[q0], xr[r3], a3);
    }
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
