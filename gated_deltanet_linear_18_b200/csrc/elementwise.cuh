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

// SiLU of the 4-tap convolution in fp64, the definition the bf16 rounding follows:
// acc = sum_k w_k x_k, SiLU(acc) = acc / (1 + e^-acc).  x: the oldest of the 4 staged rows of one
// channel, the next rows `d` elements apart.
__device__ __forceinline__ double silu_conv_fp64(const __nv_bfloat16* x, int d, const float* w4) {
  double acc = 0.0;
#pragma unroll
  for (int k = 0; k < 4; ++k) acc += (double)w4[k] * (double)__bfloat162float(x[(long)k * d]);
  return acc * (1.0 / (1.0 + exp(-acc)));
}
__device__ __forceinline__ uint32_t bf16_pair_rn(double a, double b) {
  return (uint32_t)__bfloat16_as_ushort(__double2bfloat16(a)) |
         ((uint32_t)__bfloat16_as_ushort(__double2bfloat16(b)) << 16);
}

// Whether every value within e of y rounds to the same bf16 value as y: the rounding boundary of
// y's bf16 cell (the midpoint, low 16 bits 0x8000) is farther than e, and e is below a quarter of
// the cell (so no neighbouring cell's boundary is within reach either).  NaN is never decided.
__device__ __forceinline__ bool bf16_decided(float y, float e) {
  const float mid = __uint_as_float((__float_as_uint(y) & 0xFFFF0000u) | 0x8000u);
  return fabsf(y - mid) > e && e < fabsf(y) * 0.0009765625f;
}

// Fast approximations of 2^x and 1/x (the SFU instructions).  The rounding decision below budgets
// 8 units of fp32 roundoff (2^-21 relative) for each of them, more than the maximum relative
// errors the PTX ISA documents for ex2.approx and rcp.approx.
__device__ __forceinline__ float ex2_fast(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rcp_fast(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

constexpr int kPrologueList = 1024;     // undecided values one CTA redoes in fp64 afterwards

// The staged tile of one prologue CTA: the raw rows of tokens t0 - 3 .. t0 + kPrologueTokens - 1
// of one head of d channels, row r holding token t0 - 3 + r, brought in by 16-byte asynchronous
// copies that are all issued at once (many tiles in flight per SM).  Tokens -3 .. -1 come from the
// carried history hh (the raw rows of the three tokens before this call, oldest first, at the same
// row width), or are zeros when there is none; tokens from T on are zeros.
template <typename Tio>
__device__ __forceinline__ void prologue_stage(Tio* tile, const Tio* xh, const Tio* hh, long t0,
                                               int T, int width, int d) {
  constexpr int N = Vec16<Tio>::N;
  const int L = d / N, lgL = __ffs(L) - 1;    // 16-byte pieces per row (a power of two)
  for (int i = threadIdx.x; i < (kPrologueTokens + 3) * L; i += blockDim.x) {
    const int r = i >> lgL, c = i & (L - 1);
    const long t = t0 - 3 + r;
    const bool hist = t < 0 && hh != nullptr;
    const bool in = (t >= 0 && t < T) || hist;
    const Tio* src = !in ? xh : (t >= 0 ? xh + t * width + c * N : hh + (t + 3) * width + c * N);
    const uint32_t dst = static_cast<uint32_t>(__cvta_generic_to_shared(tile + (long)r * d + c * N));
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
                 "r"(in ? 16 : 0) : "memory");
  }
  asm volatile("cp.async.commit_group;\ncp.async.wait_group 0;" ::: "memory");
}

// Vectors of 4 values: 16 bytes of fp32 or 8 of bf16.
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

// Whether every value within 2^-24 E of y rounds to the same bf16 value as y, tested as: the
// midpoint next to y's truncation to bf16 (low 16 bits 0x8000; the cell boundary nearest y unless y
// sits at the start of its binade) is farther than twice that.  Every other boundary is at least
// half that distance away (the nearest one below a binade's start, where the cell below is half
// as wide, included), so all are farther than 2^-24 E.  The scaling by 2^23 is exact; E = 0 (an
// exact y) is decided, NaN never.
__device__ __forceinline__ bool bf16_decided_e24(float y, float E) {
  const float mid = __uint_as_float((__float_as_uint(y) & 0xFFFF0000u) | 0x8000u);
  return fabsf(y - mid) * 8388608.0f > E;
}

// Prologue of the v channels (no normalisation): grid (Hv, ceil(T / kPrologueTokens), B), head
// slots fastest, so that CTAs that run together read neighbouring parts of the same token rows;
// block: 128 threads.  One CTA takes one head of dv channels over kPrologueTokens tokens: a head
// row is held by L = dv / 4 threads (4 channels each) and the 128 / L row groups take consecutive
// spans of tokens, carrying the conv window in registers (a ring of four rows).
//
// bf16 outputs: rounding to bf16 is a quantising decision, taken here as the exact result would
// take it, i.e. as rounding the fp64 value does.  The fp32 value s = SiLU(pre) is within
// 2^-24 ((20 + 2 |pre|) |s| + 1.2 P) of the exact value, P = |p0| + |p1| + |p2| + |pre| the
// magnitudes of the conv's partial sums (each of its four FMAs rounds once, by at most a unit of
// its result, carried through SiLU' <= 1.1): the exponent's argument rounds with the constant
// log2 e (2 |pre| units of s, relative), ex2.approx and rcp.approx are budgeted 8 units each (more
// than the maximum errors the PTX ISA documents), the remaining operations one unit each.
// Values whose rounding that leaves open (about 0.2 %, bf16_decided_e24) are marked in a
// per-thread bit mask, gathered into a shared-memory list after the loop and redone in fp64 after
// the tile is stored, so the rare fp64 work and its bookkeeping stay off the common path.
template <typename Tio>
__global__ void __launch_bounds__(128, 6)
prologue_v_kernel(const Tio* __restrict__ x, const Tio* __restrict__ hist,
                  const float* __restrict__ w, Tio* __restrict__ y, int T, int Hv, int dv,
                  const int* __restrict__ cu, int max_len) {
  constexpr bool kBf16 = sizeof(Tio) == 2;
  extern __shared__ __align__(16) uint8_t pro_smem[];
  Tio* tile = reinterpret_cast<Tio*>(pro_smem);
  __shared__ uint16_t list[kPrologueList];    // undecided (token << 8 | channel)
  __shared__ int nlist;
  const int head = blockIdx.x, d = dv, width = Hv * dv;
  const long b = blockIdx.z;
  const long t0 = (long)blockIdx.y * kPrologueTokens;
  const RowSpan sp = row_span(cu, (int)b, T, max_len);
  if (t0 >= sp.len) return;                   // past this sequence's end (uniform, no barrier yet)
  const int L = d / 4, grp = threadIdx.x / L, lc = threadIdx.x % L, ngrp = 128 / L;
  const int tpg = kPrologueTokens / ngrp, i0 = grp * tpg;  // this row group's tokens
  if (threadIdx.x == 0) nlist = 0;
  prologue_stage(tile, x + sp.row0 * width + (long)head * d,
                 hist ? hist + b * 3 * (long)width + (long)head * d : nullptr, t0, sp.len, width,
                 d);
  const long c0 = (long)head * d + lc * 4;    // first channel of this thread
  float wk[4][4];                             // [channel][tap]
#pragma unroll
  for (int c = 0; c < 4; ++c)
#pragma unroll
    for (int k = 0; k < 4; ++k) wk[c][k] = w[(c0 + c) * 4 + k];   // 4-byte alignment only
  __syncthreads();
  const long rem = sp.len - t0;
  const int nt = rem < kPrologueTokens ? (int)rem : kPrologueTokens;
  Tio* const yt = y + (sp.row0 + t0) * width + c0;        // this thread's channels of token t0
  const Tio* const xr = tile + lc * 4;                    // ... of tile row 0
  // The four channels run as two pairs on sm_100's paired fp32 instructions (each lane the IEEE
  // operation of the scalar form, so every value and every rounding decision is that of the
  // scalar arithmetic): weights and window rows are held as channel pairs.
  f2_t w2[2][4];                              // [channel pair][tap]
#pragma unroll
  for (int jp = 0; jp < 2; ++jp)
#pragma unroll
    for (int k = 0; k < 4; ++k) w2[jp][k] = pk2(wk[2 * jp][k], wk[2 * jp + 1][k]);
  // token i reads tile rows i .. i + 3 at ring slots i .. i + 3 (mod 4): with the token loop
  // unrolled by four no row is ever moved
  f2_t h[4][2];
  auto load_row = [&](long row, f2_t (&hr)[2]) {
    float v[4];
    Vec4<Tio>::load(xr + row * d, v);
    hr[0] = pk2(v[0], v[1]);
    hr[1] = pk2(v[2], v[3]);
  };
#pragma unroll
  for (int r = 0; r < 3; ++r) load_row(i0 + r, h[r]);
  const f2_t neg_log2e = splat2(-1.4426950408889634f), one2 = splat2(1.0f);
  unsigned long long umask = 0ull;            // undecided values: bit 4 (i - i0) + channel
#pragma unroll 1
  for (int t4 = 0; t4 < tpg; t4 += 4) {
    unsigned m16 = 0u;
#pragma unroll
    for (int sl = 0; sl < 4; ++sl) {
      if (t4 + sl >= tpg) break;              // tpg = 2 for 16-channel heads
      const int i = i0 + t4 + sl;
      const int r0 = sl, r1 = (sl + 1) & 3, r2 = (sl + 2) & 3, r3 = (sl + 3) & 3;
      load_row(i + 3, h[r3]);
      float yv_[4];
#pragma unroll
      for (int jp = 0; jp < 2; ++jp) {
        const f2_t p0 = mul2(w2[jp][0], h[r0][jp]);
        const f2_t p1 = fma2(w2[jp][1], h[r1][jp], p0);
        const f2_t p2 = fma2(w2[jp][2], h[r2][jp], p1);
        const f2_t pre = fma2(w2[jp][3], h[r3][jp], p2);
        // SiLU(pre) = pre / (1 + 2^(-pre log2 e))
        float ea, eb, da, db, s0, s1;
        up2(mul2(pre, neg_log2e), ea, eb);
        up2(add2(one2, pk2(ex2_fast(ea), ex2_fast(eb))), da, db);
        const f2_t sv = mul2(pre, pk2(rcp_fast(da), rcp_fast(db)));
        up2(sv, s0, s1);
        yv_[2 * jp] = s0;
        yv_[2 * jp + 1] = s1;
        if constexpr (kBf16) {
          // half the bound's bracket: 10 |s| + pre s + 0.6 P (pre s = |pre| |s|)
          float a0, a1, b0, b1, c0, c1, e0, e1;
          up2(p0, a0, a1);
          up2(p1, b0, b1);
          up2(p2, c0, c1);
          up2(pre, e0, e1);
          const f2_t P = pk2((fabsf(a0) + fabsf(b0)) + (fabsf(c0) + fabsf(e0)),
                             (fabsf(a1) + fabsf(b1)) + (fabsf(c1) + fabsf(e1)));
          float E0, E1;
          up2(fma2(pre, sv, fma2(P, splat2(0.6f), pk2(10.0f * fabsf(s0), 10.0f * fabsf(s1)))),
              E0, E1);
          if (!bf16_decided_e24(s0, E0 + E0)) m16 |= 1u << (sl * 4 + 2 * jp);
          if (!bf16_decided_e24(s1, E1 + E1)) m16 |= 1u << (sl * 4 + 2 * jp + 1);
        }
      }
      if (i < nt) Vec4<Tio>::store(yt + (long)i * width, yv_);
    }
    umask |= (unsigned long long)m16 << (4 * t4);
  }
  if constexpr (kBf16) {
    if (umask) {                              // into the CTA's list
      int k = atomicAdd(&nlist, __popcll(umask));
      for (unsigned long long m = umask; m; m &= m - 1, ++k) {
        const int bit = __ffsll(m) - 1;
        if (k < kPrologueList) list[k] = (uint16_t)(((i0 + (bit >> 2)) << 8) | (lc * 4 + (bit & 3)));
      }
    }
    __syncthreads();                          // the list is complete, the fast values stored
    const int n = nlist;
    __nv_bfloat16* yb =
        reinterpret_cast<__nv_bfloat16*>(y) + (sp.row0 + t0) * width + (long)head * d;
    const __nv_bfloat16* tb16 = reinterpret_cast<const __nv_bfloat16*>(tile);
    const float* wh = w + (long)head * d * 4;
    if (n <= kPrologueList) {
      for (int e = threadIdx.x; e < n; e += 128) {
        const int i = list[e] >> 8, ch = list[e] & 255;
        if (i < nt)
          yb[(long)i * width + ch] = __double2bfloat16(
              silu_conv_fp64(tb16 + (long)i * d + ch, d, wh + ch * 4));
      }
    } else {                                  // an overfull list (not expected): redo the tile
      for (int e = threadIdx.x; e < nt * d; e += 128) {
        const int i = e / d, ch = e - i * d;
        yb[(long)i * width + ch] = __double2bfloat16(
            silu_conv_fp64(tb16 + (long)i * d + ch, d, wh + ch * 4));
      }
    }
  }
}

// Prologue of the q and k channels (conv, SiLU, then each head row divided by its L2 norm): grid
// (2 Hk, ceil(T / kPrologueTokens), B), q heads then k heads; the thread layout of the v kernel
// (4 channels per thread, so that the fp64 weights and window take 56 registers).
// bf16 outputs: the convolution in fp64 (the weights widened once per thread, each input once, in
// the window), SiLU in fp32 (expf and a Newton-refined reciprocal: within 7 units of roundoff, plus
// the rounded argument's 0.55 |x|), the row's sum of squares in fp32 with its roundoff bound and
// rsqrtf, so that a value's error is a few tens of units of roundoff at most; a row with any value
// whose bf16 rounding that leaves open is redone whole in fp64 afterwards (the row's values share
// the norm).  No step has a data-dependent branch.
template <typename Tio>
__global__ void __launch_bounds__(128, 5)
prologue_qk_kernel(const Tio* __restrict__ xq, const Tio* __restrict__ xk,
                   const Tio* __restrict__ hq, const Tio* __restrict__ hk,
                   const float* __restrict__ wq, const float* __restrict__ wk,
                   Tio* __restrict__ yq, Tio* __restrict__ yk, int T, int Hk, int dk, float eps,
                   const int* __restrict__ cu, int max_len) {
  constexpr int N = 4;                        // channels per thread
  constexpr bool kBf16 = sizeof(Tio) == 2;
  constexpr float u = 5.9604645e-8f;
  extern __shared__ __align__(16) uint8_t pro_smem[];
  Tio* tile = reinterpret_cast<Tio*>(pro_smem);
  __shared__ uint16_t list[kPrologueTokens];  // undecided rows (tokens)
  __shared__ int nlist;
  const bool isq = blockIdx.x < Hk;
  const int head = isq ? blockIdx.x : blockIdx.x - Hk, d = dk, width = Hk * dk;
  const Tio* x = isq ? xq : xk;
  const Tio* hist = isq ? hq : hk;
  const float* w = isq ? wq : wk;
  Tio* y = isq ? yq : yk;
  const long b = blockIdx.z;
  const long t0 = (long)blockIdx.y * kPrologueTokens;
  const RowSpan sp = row_span(cu, (int)b, T, max_len);
  if (t0 >= sp.len) return;                   // past this sequence's end (uniform, no barrier yet)
  const int L = d / N, grp = threadIdx.x / L, lc = threadIdx.x % L, ngrp = 128 / L;
  const int tpg = kPrologueTokens / ngrp, i0 = grp * tpg;
  if (threadIdx.x == 0) nlist = 0;
  prologue_stage(tile, x + sp.row0 * width + (long)head * d,
                 hist ? hist + b * 3 * (long)width + (long)head * d : nullptr, t0, sp.len, width,
                 d);
  const long c0 = (long)head * d + lc * N;
  float wt[N][4];
#pragma unroll
  for (int i = 0; i < N; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) wt[i][j] = w[(c0 + i) * 4 + j];
  __syncthreads();
  const long rem = sp.len - t0;
  const int nt = rem < kPrologueTokens ? (int)rem : kPrologueTokens;
  Tio* const yt = y + (sp.row0 + t0) * width + c0;
  if constexpr (!kBf16) {                     // fp32 outputs: fp32 throughout
    float h0[N], h1[N], h2[N];
    Vec4<Tio>::load(tile + (long)i0 * d + lc * N, h0);
    Vec4<Tio>::load(tile + (long)(i0 + 1) * d + lc * N, h1);
    Vec4<Tio>::load(tile + (long)(i0 + 2) * d + lc * N, h2);
#pragma unroll 2
    for (int tt = 0; tt < tpg; ++tt) {
      const int i = i0 + tt;
      float h3[N], yv_[N], ss = 0.f;
      Vec4<Tio>::load(tile + (long)(i + 3) * d + lc * N, h3);
#pragma unroll
      for (int j = 0; j < N; ++j) {
        const float pre = fmaf(wt[j][3], h3[j], fmaf(wt[j][2], h2[j],
                                                     fmaf(wt[j][1], h1[j], wt[j][0] * h0[j])));
        yv_[j] = pre * rcp_fast(1.0f + ex2_fast(pre * -1.4426950408889634f));
        ss = fmaf(yv_[j], yv_[j], ss);
        h0[j] = h1[j]; h1[j] = h2[j]; h2[j] = h3[j];
      }
      for (int o = L >> 1; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      const float inv = rsqrtf(ss + eps);
#pragma unroll
      for (int j = 0; j < N; ++j) yv_[j] *= inv;
      if (i < nt) Vec4<Tio>::store(yt + (long)i * width, yv_);
    }
  } else {
    double wd[N][4];                          // the weights, widened once
#pragma unroll
    for (int j = 0; j < N; ++j)
#pragma unroll
      for (int k = 0; k < 4; ++k) wd[j][k] = wt[j][k];
    // the window, widened once per input, as a ring of four rows: token i reads rows i .. i + 3
    // at ring slots i .. i + 3 (mod 4), so with the token loop unrolled by four no row is moved
    double dr[4][N];
#pragma unroll
    for (int r = 0; r < 3; ++r) {
      float f[N];
      Vec4<Tio>::load(tile + (long)(i0 + r) * d + lc * N, f);
#pragma unroll
      for (int j = 0; j < N; ++j) dr[r][j] = f[j];
    }
    const int lane = threadIdx.x & 31;
    const unsigned lmask = L == 32 ? 0xffffffffu : (1u << L) - 1u;
#pragma unroll 1
    for (int t4 = 0; t4 < tpg; t4 += 4) {
#pragma unroll
      for (int sl = 0; sl < 4; ++sl) {
        if (t4 + sl >= tpg) break;            // tpg = 2 for 16-channel heads
        const int i = i0 + t4 + sl;
        const int r0 = sl, r1 = (sl + 1) & 3, r2 = (sl + 2) & 3, r3 = (sl + 3) & 3;
        float f[N], s[N], es[N], yv_[N];
        Vec4<Tio>::load(tile + (long)(i + 3) * d + lc * N, f);
        float ss = 0.f, se = 0.f;
#pragma unroll
        for (int j = 0; j < N; ++j) {
          dr[r3][j] = f[j];
          const double acc = fma(wd[j][3], dr[r3][j], fma(wd[j][2], dr[r2][j],
                                                          fma(wd[j][1], dr[r1][j],
                                                              wd[j][0] * dr[r0][j])));
          const float pre = (float)acc;       // within half a unit of the exact sum
          // SiLU = pre / (1 + e^-pre): expf (2 units), the sum (half a unit), 1 / den by
          // rcp.approx and one Newton step (about half a unit; the approximation's own error
          // enters squared) and the product (half a unit): within 7 units of s, plus the
          // rounded argument's 0.55 |pre|
          const float den = 1.0f + expf(-pre);
          const float r0 = rcp_fast(den);
          s[j] = pre * fmaf(r0, fmaf(-den, r0, 1.0f), r0);
          es[j] = u * fmaf(fabsf(pre), 0.6f, 7.0f * fabsf(s[j]));
          ss = fmaf(s[j], s[j], ss);
          se = fmaf(2.0f * fabsf(s[j]), es[j], se);
        }
        for (int o = L >> 1; o > 0; o >>= 1) {
          ss += __shfl_xor_sync(0xffffffffu, ss, o);
          se += __shfl_xor_sync(0xffffffffu, se, o);
        }
        // sum of squares: at most (N + log2 L + 1) units of its own roundoff plus se from the
        // values; inv = rsqrtf (within 2 ulps, 4 units) of the rounded sum: inv's relative error
        // is at most half that of den (1 / den = inv^2 within a few units, 2 % allowed), plus 5
        // units
        const float den = ss + eps;
        const float inv = rsqrtf(den);
        const float dinv = 0.5f * (se + (float)(N + 8) * u * ss) * (inv * inv) * 1.02f + 5.0f * u;
        // y - y* = (s - s*) inv + s* (inv - inv*) + the product's rounding, so |y - y*| is at most
        // es inv + |y| (dinv + u) to first order; the 10 % cover the second-order terms (products
        // of these relative errors, below 1e-12) and |y*| against |y|
        bool need = false;
#pragma unroll
        for (int j = 0; j < N; ++j) {
          yv_[j] = s[j] * inv;
          const float e = 1.1f * (fabsf(yv_[j]) * (dinv + u) + es[j] * inv);
          need = need || !bf16_decided(yv_[j], e);
        }
        // any lane of this row (the L lanes lane & ~(L - 1) ..) undecided
        const unsigned bal = __ballot_sync(0xffffffffu, need);
        if (lc == 0 && ((bal >> (lane & ~(L - 1))) & lmask) != 0)
          list[atomicAdd(&nlist, 1)] = (uint16_t)i;               // at most one per token
        if (i < nt) Vec4<Tio>::store(yt + (long)i * width, yv_);
      }
    }
    __syncthreads();                          // the list is complete, the fast values stored
    const int n = nlist;
    __nv_bfloat16* yb =
        reinterpret_cast<__nv_bfloat16*>(y) + (sp.row0 + t0) * width + (long)head * d;
    const __nv_bfloat16* tb16 = reinterpret_cast<const __nv_bfloat16*>(tile);
    const float* wh = w + (long)head * d * 4;
    // one row per group of L threads (the row's norm by shuffles over those lanes)
    const unsigned rowmask = L == 32 ? 0xffffffffu
                                     : (((1u << L) - 1u) << ((threadIdx.x & 31) & ~(L - 1)));
    for (int e0 = 0; e0 < n; e0 += ngrp) {    // uniform trip count
      const int e = e0 + grp;
      if (e >= n) continue;                   // whole row groups skip together
      const int i = list[e];
      double yd[N], ss = 0.0;
#pragma unroll
      for (int j = 0; j < N; ++j) {
        const int ch = lc * N + j;
        yd[j] = silu_conv_fp64(tb16 + (long)i * d + ch, d, wh + ch * 4);
        ss += yd[j] * yd[j];
      }
      for (int o = L >> 1; o > 0; o >>= 1) ss += __shfl_xor_sync(rowmask, ss, o);
      const double invd = 1.0 / sqrt(ss + (double)eps);
      if (i < nt) {
        uint32_t pk[N / 2];
#pragma unroll
        for (int j = 0; j < N / 2; ++j) pk[j] = bf16_pair_rn(yd[2 * j] * invd, yd[2 * j + 1] * invd);
        *reinterpret_cast<uint2*>(yb + (long)i * width + lc * N) = make_uint2(pk[0], pk[1]);
      }
    }
  }
}

// Shared memory of one prologue CTA for heads of d channels.
inline size_t prologue_smem_bytes(int d, size_t elem) {
  return (size_t)(kPrologueTokens + 3) * d * elem;
}

// The gated norm of one row from the lane's 4 values of o and z (zeros on lanes past dv): the
// row's sum of squares over the warp, then y = o / rms(o) * w * SiLU(z) on the lane's channels.
template <typename Ty>
__device__ __forceinline__ void out_norm_row(const float (&ov)[4], const float (&zv)[4],
                                             const float* __restrict__ w, Ty* yrow, int c,
                                             bool active, int dv, float eps) {
  float ss = (ov[0] * ov[0] + ov[1] * ov[1]) + (ov[2] * ov[2] + ov[3] * ov[3]);
  ss = warp_sum(ss);
  const float inv = rsqrtf(ss / dv + eps);
  if (active) {
    const float ww[4] = {w[c], w[c + 1], w[c + 2], w[c + 3]};
    float yv[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) yv[e] = ov[e] * inv * ww[e] * silu_fast(zv[e]);
    Vec4<Ty>::store(yrow + c, yv);
  }
}

// The gated norm over rows of dv <= 128 values, 4 consecutive channels per lane: each warp takes
// two consecutive rows and loads both before it reduces either (twice the loads in flight of a
// row per warp); blocks of kNormThreads threads cover 8 rows.  `o` may be wider than z / y (the
// layer keeps o in fp32).
constexpr int kNormThreads = 128;
template <typename To, typename Tz, typename Ty = Tz>
__global__ void __launch_bounds__(kNormThreads)
out_norm_kernel(const To* __restrict__ o, const Tz* __restrict__ z, const float* __restrict__ w,
                Ty* __restrict__ y, long long rows, int dv, float eps) {
  const long long row0 = (long long)blockIdx.x * 8 + (threadIdx.x >> 5) * 2;
  if (row0 >= rows) return;
  const int c = 4 * (threadIdx.x & 31);
  const bool active = c < dv;
  const int nr = row0 + 1 < rows ? 2 : 1;    // (uniform over the warp)
  float ov[2][4], zv[2][4];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
#pragma unroll
    for (int e = 0; e < 4; ++e) ov[r][e] = zv[r][e] = 0.f;
    if (active && r < nr) {
      Vec4<To>::load(o + (row0 + r) * dv + c, ov[r]);
      Vec4<Tz>::load(z + (row0 + r) * dv + c, zv[r]);
    }
  }
#pragma unroll
  for (int r = 0; r < 2; ++r)
    if (r < nr) out_norm_row(ov[r], zv[r], w, y + (row0 + r) * dv, c, active, dv, eps);
}

// The conv history after a call: the raw rows of the last three tokens of [history; x] (oldest
// first), per sequence, for `width` channels: with the sequence's length n, row r is token n + r of
// that concatenation, from the incoming history hin while n + r < 3 (zeros when there is none),
// else from x.  Sequences as in row_span.  One thread per 16-byte piece of a row.
template <typename Tio>
__global__ void conv_hist_out_kernel(const Tio* __restrict__ x, const Tio* __restrict__ hin,
                                     Tio* __restrict__ hout, long B, int T, int width,
                                     const int* __restrict__ cu, int max_len) {
  constexpr int N = 16 / sizeof(Tio);
  const int P = width / N;
  const long i = (long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= B * 3 * P) return;
  const long b = i / (3 * P);
  const int r = (int)(i / P % 3), c = (int)(i % P);
  const RowSpan sp = row_span(cu, (int)b, T, max_len);
  const long s = (long)sp.len + r;            // position in [history; x]
  uint4 v = make_uint4(0u, 0u, 0u, 0u);
  if (s >= 3) v = reinterpret_cast<const uint4*>(x + (sp.row0 + s - 3) * (long)width)[c];
  else if (hin) v = reinterpret_cast<const uint4*>(hin + (b * 3 + s) * (long)width)[c];
  reinterpret_cast<uint4*>(hout + (b * 3 + r) * (long)width)[c] = v;
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
