// One decode step of the whole layer ("Chapitre 16 - Assembler un système de type Kimi K3", 16.3:
// read the fixed state, compute the output, update the state) with the layer's prologue and
// epilogue fused around it ("L'attention hybride", "Le décompte": causal conv of 4 taps over the
// q, k, v channels, swish output gate, one 128-wide norm gain; "Les briques d'un réseau de
// neurones", 2. SiLU and 4. RMSNorm).  For each (sequence n, value head h), with M = S^T in place:
//   q^, k^, v^ = SiLU(conv4([history of 3 raw tokens; raw token]))   (q^, k^ of h's key head)
//   q^, k^ /= sqrt(|.|^2 + l2_eps)                                   (per key head, over dk)
//   the recurrence step of the decode kernel on (scale q^, k^, v^)    -> o, M updated
//   y = o / sqrt(mean(o^2) + norm_eps) * w (.) SiLU(z)                (over dv)
// The conv history moves one token on into separate output buffers: the value heads of a key
// head all read its q, k history, so the first value head of the group writes it.  The state
// crosses HBM once each way, as in the plain decode step; the per-token activations never do.
#pragma once

#include "common.cuh"
#include "decode.cuh"
#include "elementwise.cuh"

namespace gdn {

template <int DK, int DV, typename Tio>
__global__ void __launch_bounds__(DecodeShape<DK, DV>::NT)
decode_layer_step_kernel(const Tio* __restrict__ q_raw, const Tio* __restrict__ k_raw,
                         const Tio* __restrict__ v_raw, const Tio* __restrict__ z,
                         const Tio* __restrict__ hq_in, const Tio* __restrict__ hk_in,
                         const Tio* __restrict__ hv_in, Tio* __restrict__ hq_out,
                         Tio* __restrict__ hk_out, Tio* __restrict__ hv_out,
                         const float* __restrict__ wq, const float* __restrict__ wk,
                         const float* __restrict__ wv, const float* __restrict__ log_alpha,
                         const float* __restrict__ beta, float* __restrict__ S,
                         const float* __restrict__ norm_w, Tio* __restrict__ y, int Hk, int Hv,
                         float scale, float l2_eps, float norm_eps) {
  using Sh = DecodeShape<DK, DV>;
  constexpr int CG = Sh::CG, NT = Sh::NT, RG = Sh::RG, RPT = Sh::RPT;
  const long nh = blockIdx.x;                  // n * Hv + h
  const int h = (int)(nh % Hv);
  const long n = nh / Hv;
  const int G = Hv / Hk, hk = h / G;
  const long CQ = (long)Hk * DK, CV = (long)Hv * DV;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int cg = tid % CG, rg = tid / CG;

  __shared__ __align__(16) float sq[DK];
  __shared__ __align__(16) float sk[DK];
  __shared__ __align__(16) float sv[DV];
  __shared__ __align__(16) float su[DV];
  __shared__ __align__(16) float red_r[RG][DV + 4];
  __shared__ __align__(16) float red_s[RG][DV + 4];
  __shared__ float s_part[NT / 32];
  __shared__ float s_qs, s_ks, s_qk, s_rms;

  // the state first: its loads are in flight during the prologue
  float4* Mh = reinterpret_cast<float4*>(S + nh * (long)DK * DV);
  float4 m[RPT];
#pragma unroll
  for (int r = 0; r < RPT; ++r) m[r] = Mh[(rg + r * RG) * CG + cg];

  // conv over [3 history tokens; this token] + SiLU; the history moves on by one token
  auto conv = [&](const Tio* raw, const Tio* hin, Tio* hout, const float* w, long C, long c,
                  bool write) -> float {
    const float x0 = to_f(hin[(n * 3 + 0) * C + c]), x1 = to_f(hin[(n * 3 + 1) * C + c]);
    const float x2 = to_f(hin[(n * 3 + 2) * C + c]);
    const Tio xr = raw[n * C + c];
    const float* ww = w + c * 4;                       // tap 3 on this token
    const float acc = ww[0] * x0 + ww[1] * x1 + ww[2] * x2 + ww[3] * to_f(xr);
    if (write) {
      hout[(n * 3 + 0) * C + c] = hin[(n * 3 + 1) * C + c];
      hout[(n * 3 + 1) * C + c] = hin[(n * 3 + 2) * C + c];
      hout[(n * 3 + 2) * C + c] = xr;
    }
    return silu_fast(acc);
  };
  const bool kv_writer = (h % G) == 0;
  for (int i = tid; i < DK; i += NT) {
    sq[i] = conv(q_raw, hq_in, hq_out, wq, CQ, (long)hk * DK + i, kv_writer);
    sk[i] = conv(k_raw, hk_in, hk_out, wk, CQ, (long)hk * DK + i, kv_writer);
  }
  for (int j = tid; j < DV; j += NT) sv[j] = conv(v_raw, hv_in, hv_out, wv, CV, (long)h * DV + j, true);
  const float a = expf(log_alpha[nh]);
  const float bt = beta[nh];
  __syncthreads();
  // L2 norms of q^ and k^ and their dot product (warp 0)
  if (warp == 0) {
    float qq = 0.f, kk = 0.f, qk = 0.f;
    for (int i = lane; i < DK; i += 32) {
      qq += sq[i] * sq[i];
      kk += sk[i] * sk[i];
      qk += sq[i] * sk[i];
    }
    qq = warp_sum(qq);
    kk = warp_sum(kk);
    qk = warp_sum(qk);
    if (lane == 0) {
      const float iq = 1.0f / sqrtf(qq + l2_eps), ik = 1.0f / sqrtf(kk + l2_eps);
      s_qs = iq * scale;
      s_ks = ik;
      s_qk = qk * iq * ik * scale;
    }
  }
  __syncthreads();
  const float qs = s_qs, ks = s_ks;
  float4 r4 = make_float4(0.f, 0.f, 0.f, 0.f), s4 = r4;
#pragma unroll
  for (int r = 0; r < RPT; ++r) {
    const int i = rg + r * RG;
    const float kk = sk[i] * ks, qq = sq[i] * qs;
    r4.x += kk * m[r].x; r4.y += kk * m[r].y; r4.z += kk * m[r].z; r4.w += kk * m[r].w;
    s4.x += qq * m[r].x; s4.y += qq * m[r].y; s4.z += qq * m[r].z; s4.w += qq * m[r].w;
  }
  *reinterpret_cast<float4*>(&red_r[rg][cg * 4]) = r4;
  *reinterpret_cast<float4*>(&red_s[rg][cg * 4]) = s4;
  __syncthreads();
  float oj = 0.f;
  if (tid < DV) {
    const int j = tid;
    float rr = 0.f, ss = 0.f;
#pragma unroll
    for (int g = 0; g < RG; ++g) { rr += red_r[g][j]; ss += red_s[g][j]; }
    const float u = bt * (sv[j] - a * rr);
    su[j] = u;
    oj = a * ss + s_qk * u;
  }
  // gated RMSNorm over the dv outputs
  float sq_o = warp_sum(oj * oj);                     // threads past dv hold 0
  if (lane == 0) s_part[warp] = sq_o;
  __syncthreads();
  if (tid == 0) {
    float t = 0.f;
#pragma unroll
    for (int w8 = 0; w8 < NT / 32; ++w8) t += s_part[w8];
    s_rms = 1.0f / sqrtf(t / DV + norm_eps);
  }
  __syncthreads();
  if (tid < DV) {
    const int j = tid;
    const float zz = to_f(z[nh * (long)DV + j]);
    y[nh * (long)DV + j] = from_f<Tio>(oj * s_rms * norm_w[j] * silu_fast(zz));
  }
  const float4 u4 = *reinterpret_cast<const float4*>(&su[cg * 4]);
#pragma unroll
  for (int r = 0; r < RPT; ++r) {
    const int i = rg + r * RG;
    const float kk = sk[i] * ks;
    float4 x = m[r];
    x.x = a * x.x + kk * u4.x; x.y = a * x.y + kk * u4.y;
    x.z = a * x.z + kk * u4.z; x.w = a * x.w + kk * u4.w;
    Mh[i * CG + cg] = x;
  }
}

}  // namespace gdn
