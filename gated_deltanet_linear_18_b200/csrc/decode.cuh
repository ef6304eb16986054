// One decode step of the gated delta rule ("Chapitre 16 - Assembler un système de type Kimi K3",
// 16.3: read the fixed state, compute the output, update the state), bandwidth-bound.
//
// For each (sequence n, value head h), with M = S^T (dk x dv, fp32, in place):
//   r = k^T M,  s = q^T M            (one streaming read of M, reductions over dk)
//   u = beta (v - alpha r)           (= beta (v - S' k) with S' = alpha S)
//   o = alpha s + (q.k) u            (= (alpha M + k u^T)^T q: the output reads the new state)
//   M <- alpha M + k u^T             (one streaming write of M)
// so the 64 KB state of a 128x128 head crosses HBM exactly once each way.
//
// Layout of the CTA over one head: thread t owns 4 consecutive dv columns (one float4) in column
// group t % (DV/4) and the dk rows rg, rg + RG, ... with rg = t / (DV/4).  Each warp therefore reads
// whole 512-byte rows (128-bit coalesced loads), issued all at once before any arithmetic.
#pragma once

#include "common.cuh"

namespace gdn {

template <int DK, int DV>
struct DecodeShape {
  static constexpr int CG = DV / 4;                                   // float4 column groups
  static constexpr int NT = (CG * DK < 256) ? CG * DK : 256;          // threads per CTA
  static constexpr int RG = NT / CG;                                  // row groups
  static constexpr int RPT = DK / RG;                                 // rows per thread
  static_assert(NT % 32 == 0 && DK % RG == 0 && NT >= DV, "decode shape");
};

template <int DK, int DV, typename Tio, typename Tout = Tio>
__global__ void __launch_bounds__(DecodeShape<DK, DV>::NT)
decode_step_kernel(const Tio* __restrict__ q, const Tio* __restrict__ k,
                   const Tio* __restrict__ v, const float* __restrict__ log_alpha,
                   const float* __restrict__ beta, float* __restrict__ S, Tout* __restrict__ o,
                   int Hk, int Hv, float scale) {
  using Sh = DecodeShape<DK, DV>;
  constexpr int CG = Sh::CG, NT = Sh::NT, RG = Sh::RG, RPT = Sh::RPT;
  const long nh = blockIdx.x;                  // n * Hv + h
  const int h = (int)(nh % Hv);
  const long n = nh / Hv;
  const int hk = h / (Hv / Hk);
  const int tid = threadIdx.x;
  const int cg = tid % CG, rg = tid / CG;

  __shared__ __align__(16) float sq[DK];
  __shared__ __align__(16) float sk[DK];
  __shared__ __align__(16) float su[DV];
  __shared__ __align__(16) float red_r[RG][DV + 4];
  __shared__ __align__(16) float red_s[RG][DV + 4];
  __shared__ float s_qk;

  float4* Mh = reinterpret_cast<float4*>(S + nh * (long)DK * DV);
  float4 m[RPT];
#pragma unroll
  for (int r = 0; r < RPT; ++r) m[r] = Mh[(rg + r * RG) * CG + cg];

  for (int i = tid; i < DK; i += NT) {
    const long off = (n * Hk + hk) * (long)DK + i;
    sq[i] = to_f(q[off]) * scale;
    sk[i] = to_f(k[off]);
  }
  const float a = expf(log_alpha[nh]);
  const float bt = beta[nh];
  __syncthreads();
  if (tid < 32) {
    float acc = 0.f;
    for (int i = tid; i < DK; i += 32) acc += sq[i] * sk[i];
    acc = warp_sum(acc);
    if (tid == 0) s_qk = acc;
  }
  float4 r4 = make_float4(0.f, 0.f, 0.f, 0.f), s4 = r4;
#pragma unroll
  for (int r = 0; r < RPT; ++r) {
    const int i = rg + r * RG;
    const float kk = sk[i], qq = sq[i];
    r4.x += kk * m[r].x; r4.y += kk * m[r].y; r4.z += kk * m[r].z; r4.w += kk * m[r].w;
    s4.x += qq * m[r].x; s4.y += qq * m[r].y; s4.z += qq * m[r].z; s4.w += qq * m[r].w;
  }
  *reinterpret_cast<float4*>(&red_r[rg][cg * 4]) = r4;
  *reinterpret_cast<float4*>(&red_s[rg][cg * 4]) = s4;
  __syncthreads();
  if (tid < DV) {
    const int j = tid;
    float rr = 0.f, ss = 0.f;
#pragma unroll
    for (int g = 0; g < RG; ++g) { rr += red_r[g][j]; ss += red_s[g][j]; }
    const float vj = to_f(v[nh * (long)DV + j]);
    const float u = bt * (vj - a * rr);
    su[j] = u;
    o[nh * (long)DV + j] = from_f<Tout>(a * ss + s_qk * u);
  }
  __syncthreads();
  const float4 u4 = *reinterpret_cast<const float4*>(&su[cg * 4]);
#pragma unroll
  for (int r = 0; r < RPT; ++r) {
    const int i = rg + r * RG;
    const float kk = sk[i];
    float4 x = m[r];
    x.x = a * x.x + kk * u4.x; x.y = a * x.y + kk * u4.y;
    x.z = a * x.z + kk * u4.z; x.w = a * x.w + kk * u4.w;
    Mh[i * CG + cg] = x;
  }
}

}  // namespace gdn
