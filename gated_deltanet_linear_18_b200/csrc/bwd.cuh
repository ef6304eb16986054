// Backward pass of the gated delta rule: the gradients of L = sum <dO, o> + <dS_T, S_T> with
// respect to q, k, v, log alpha, beta and S0, the exact derivative of the token recurrence
// ("L'attention hybride", "La récurrence": S_t = alpha_t S_{t-1} (I - beta_t k_t k_t^T)
// + beta_t v_t k_t^T, o_t = scale S_t q_t; the pages train their models but give this layer for
// inference only, so the backward is the chain rule through that recurrence).
//
// Per token, with P = S_{t-1}, x = P k, A = P - beta x k^T, S_t = alpha A + beta v k^T, and G the
// gradient reaching S_t (later tokens, plus scale dO_t q_t^T from this token's output):
//   dq = scale S_t^T dO,  dlog_alpha = alpha <G, A>,  Gk = G k,
//   dbeta = (v - alpha x)^T Gk,  dv = beta Gk,  dx = -alpha beta Gk,
//   dk = beta G^T (v - alpha x) + P^T dx,  and the gradient reaching S_{t-1} is alpha G + dx k^T.
// The reverse walk needs every S_{t-1}: a forward pass first stores the state at the start of
// every segment of kSeg tokens (checkpoints in the caller's workspace); the reverse pass then takes
// the segments last to first, holding the segment's first state and its middle state in shared
// memory and recomputing each S_{t-1} from the nearer one (about two token steps per token).
//
// One CTA per (batch, value head), 512 threads.  The state and its gradient live in registers in
// the decode kernel's layout: with M = S^T (dk x dv), thread t owns the 4 value columns of column
// group t % (DV / 4) and the dk rows rg, rg + RG, ... (rg = t / (DV / 4)).  Reductions over dv stay
// inside a warp (shuffles); reductions over dk cross warps (shared memory, one barrier each).
#pragma once

#include "common.cuh"

namespace gdn {
namespace bwd {

constexpr int kSeg = 8;          // tokens per checkpoint segment
constexpr int kHalf = kSeg / 2;  // the segment's middle state is S before token t0 + kHalf

template <int DK, int DV>
struct Shape {
  static constexpr int CG = DV / 4;                                    // float4 column groups
  static constexpr int NT = (CG * DK < 512) ? CG * DK : 512;           // threads per CTA
  static constexpr int RG = NT / CG;                                   // row groups
  static constexpr int RPT = DK / RG;                                  // rows per thread
  static constexpr int NW = NT / 32;                                   // warps
  static_assert(NT % 32 == 0 && DK % RG == 0 && 32 % CG == 0, "bwd shape");
};

// Shared memory of one CTA (floats): the segment's token data, two states, reduction buffers.
template <int DK, int DV>
struct Smem {
  float k[kSeg][DK], q[kSeg][DK], v[kSeg][DV], dO[kSeg][DV];
  float alpha[kSeg], beta[kSeg];
  float state0[DK * DV];      // the state before the segment's first token
  float statem[DK * DV];      // the state before the segment's token t0 + kHalf
  float red[2][2][Shape<DK, DV>::RG][DV];   // [parity][quantity][row group][column]
  float col[2][2][DV];                       // [parity][quantity] the column sums
  float wsum[2][Shape<DK, DV>::NW];         // per-warp partials of <G, A>
};

template <int DK, int DV>
constexpr size_t smem_bytes() { return sizeof(Smem<DK, DV>); }

template <int DK, int DV>
struct Regs {
  float4 m[Shape<DK, DV>::RPT];
};

// Sum over the CG lanes of a warp that share a row group (lanes xor 1 .. CG/2).
template <int CG>
__device__ __forceinline__ float lane_sum(float x) {
#pragma unroll
  for (int o = CG >> 1; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Sums over the CG lanes of a row group of V values per lane, scattered by recursive halving:
// at each step a lane keeps one half of its values (chosen by its lane bit), adds the partner's
// copy of that half and passes the other half on, so V values cost V - 1 shuffles instead of
// V log2(CG).  On return v[0] holds the total of value `idx` (every lane of the row group holds
// the total of one value; lanes that differ only in the bits below `keep_mask` hold the same).
template <int V, int CG>
__device__ __forceinline__ void reduce_scatter(float (&v)[V], int lane, int& idx,
                                               int& keep_mask) {
  static_assert((V & (V - 1)) == 0 && V <= CG, "reduce_scatter");
  idx = 0;
  int n = V;
#pragma unroll
  for (int m = CG >> 1; m > 0; m >>= 1) {
    if (n > 1) {
      const bool up = (lane & m) != 0;
#pragma unroll
      for (int k = 0; k < V / 2; ++k) {
        if (k < n / 2) {
          const float lo = v[k], hi = v[k + n / 2];
          const float keep = up ? hi : lo, send = up ? lo : hi;
          v[k] = keep + __shfl_xor_sync(0xffffffffu, send, m);
        }
      }
      if (up) idx += n / 2;
      n >>= 1;
      keep_mask = m;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], m);
    }
  }
}

// The segment's token data (tokens t0 .. t0 + len - 1) into shared memory, as fp32.
template <int DK, int DV, typename Tin>
__device__ __forceinline__ void load_segment(Smem<DK, DV>& sm, const Tin* __restrict__ q,
                                             const Tin* __restrict__ k, const Tin* __restrict__ v,
                                             const Tin* __restrict__ dO,
                                             const float* __restrict__ la,
                                             const float* __restrict__ be, long b, int h, int hk,
                                             int T, int Hk, int Hv, int t0, int len, bool with_q) {
  constexpr int NT = Shape<DK, DV>::NT;
  for (int e = threadIdx.x; e < len * DK; e += NT) {
    const int j = e / DK, i = e - j * DK;
    const long row = ((b * T + t0 + j) * Hk + hk) * (long)DK + i;
    sm.k[j][i] = to_f(k[row]);
    if (with_q) sm.q[j][i] = to_f(q[row]);
  }
  for (int e = threadIdx.x; e < len * DV; e += NT) {
    const int j = e / DV, i = e - j * DV;
    const long row = ((b * T + t0 + j) * Hv + h) * (long)DV + i;
    sm.v[j][i] = to_f(v[row]);
    if (with_q) sm.dO[j][i] = to_f(dO[row]);
  }
  for (int j = threadIdx.x; j < len; j += NT) {
    const long g = (b * T + t0 + j) * Hv + h;
    sm.alpha[j] = expf(la[g]);
    sm.beta[j] = be[g];
  }
}

__device__ __forceinline__ float4 f4(float a) { return make_float4(a, a, a, a); }
__device__ __forceinline__ float4 add4(float4 a, float4 b) {
  return make_float4(a.x + b.x, a.y + b.y, a.z + b.z, a.w + b.w);
}
__device__ __forceinline__ float4 fma4(float4 a, float4 b, float4 c) {   // a * b + c
  return make_float4(fmaf(a.x, b.x, c.x), fmaf(a.y, b.y, c.y), fmaf(a.z, b.z, c.z),
                     fmaf(a.w, b.w, c.w));
}
__device__ __forceinline__ float4 mul4(float4 a, float4 b) {
  return make_float4(a.x * b.x, a.y * b.y, a.z * b.z, a.w * b.w);
}
__device__ __forceinline__ float dot4(float4 a, float4 b) {
  return fmaf(a.x, b.x, fmaf(a.y, b.y, fmaf(a.z, b.z, a.w * b.w)));
}

// One CTA's state M (its RPT rows of 4 columns) and the shared-memory reductions over dk.
template <int DK, int DV>
struct Ctx {
  using Sh = Shape<DK, DV>;
  Smem<DK, DV>& sm;
  int cg, rg;
  int par = 0;                  // reduction buffer in use (alternates, so one barrier suffices)
  __device__ Ctx(Smem<DK, DV>& s) : sm(s), cg(threadIdx.x % Sh::CG), rg(threadIdx.x / Sh::CG) {}

  // Column sums over dk of NQ per-thread float4 partials (this thread's 4 columns): the row
  // groups' partials go to shared memory, row group q sums quantity q's once, every thread reads
  // the sums back.
  template <int NQ>
  __device__ __forceinline__ void colsum(const float4 (&a)[NQ], float4 (&s)[NQ]) {
    static_assert(NQ <= 2 && NQ <= Sh::RG, "colsum");
#pragma unroll
    for (int qn = 0; qn < NQ; ++qn)
      *reinterpret_cast<float4*>(&sm.red[par][qn][rg][4 * cg]) = a[qn];
    __syncthreads();
    if (rg < NQ) {
      float4 acc = f4(0.f);
#pragma unroll
      for (int g = 0; g < Sh::RG; ++g)
        acc = add4(acc, *reinterpret_cast<const float4*>(&sm.red[par][rg][g][4 * cg]));
      *reinterpret_cast<float4*>(&sm.col[par][rg][4 * cg]) = acc;
    }
    __syncthreads();
#pragma unroll
    for (int qn = 0; qn < NQ; ++qn)
      s[qn] = *reinterpret_cast<const float4*>(&sm.col[par][qn][4 * cg]);
    par ^= 1;
  }

  // One token of the recurrence on M = S^T: x = S k, S <- alpha S + beta (v - alpha x) k^T.
  __device__ __forceinline__ void fwd_step(float4 (&M)[Sh::RPT], int j) {
    const float a = sm.alpha[j], be = sm.beta[j];
    float kk[Sh::RPT];
    float4 x4 = f4(0.f);
#pragma unroll
    for (int r = 0; r < Sh::RPT; ++r) {
      kk[r] = sm.k[j][rg + Sh::RG * r];
      x4 = fma4(M[r], f4(kk[r]), x4);
    }
    float4 xa[1] = {x4}, xs[1];
    colsum<1>(xa, xs);
    const float4 x = xs[0];
    const float4 vv = *reinterpret_cast<const float4*>(&sm.v[j][4 * cg]);
    const float4 w = mul4(f4(be), fma4(f4(-a), x, vv));      // beta (v - alpha x)
#pragma unroll
    for (int r = 0; r < Sh::RPT; ++r) M[r] = fma4(f4(a), M[r], mul4(f4(kk[r]), w));
  }

  __device__ __forceinline__ void put(float* base, const float4 (&M)[Sh::RPT]) const {
#pragma unroll
    for (int r = 0; r < Sh::RPT; ++r)
      *reinterpret_cast<float4*>(base + (long)(rg + Sh::RG * r) * DV + 4 * cg) = M[r];
  }
  __device__ __forceinline__ void get(const float* base, float4 (&M)[Sh::RPT]) const {
#pragma unroll
    for (int r = 0; r < Sh::RPT; ++r)
      M[r] = *reinterpret_cast<const float4*>(base + (long)(rg + Sh::RG * r) * DV + 4 * cg);
  }
};

// grid: B * Hv CTAs (b * Hv + h); block Shape::NT; dynamic shared memory smem_bytes<DK, DV>().
// dq_out, dk_out: [B, T, nqk, DK] with nqk = Hv (one slice per value head, summed afterwards by
// group_sum_kernel) or Hk when each key head has one value head.  ckpt: B * Hv * ceil(T / kSeg)
// states of DK * DV floats.
template <int DK, int DV, typename Tin>
__global__ void __launch_bounds__(Shape<DK, DV>::NT, 1)
bwd_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
           const float* __restrict__ log_alpha, const float* __restrict__ beta,
           const float* __restrict__ S0, const Tin* __restrict__ dO,
           const float* __restrict__ dS_T, float* __restrict__ dq_out,
           float* __restrict__ dk_out, int nqk, float* __restrict__ dv_out,
           float* __restrict__ dla_out, float* __restrict__ dbeta_out, float* __restrict__ dS0,
           float* __restrict__ ckpt, int T, int Hk, int Hv, float scale) {
  using Sh = Shape<DK, DV>;
  constexpr int RPT = Sh::RPT, RG = Sh::RG, CG = Sh::CG;
  extern __shared__ __align__(16) unsigned char bwd_smem[];
  Smem<DK, DV>& sm = *reinterpret_cast<Smem<DK, DV>*>(bwd_smem);
  Ctx<DK, DV> cx(sm);
  const int cg = cx.cg, rg = cx.rg, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const long bh = blockIdx.x;
  const int h = (int)(bh % Hv);
  const long b = bh / Hv;
  const int hk = h / (Hv / Hk);
  const int hq = nqk == Hv ? h : hk;                 // this CTA's slice of dq, dk
  const int nseg = (T + kSeg - 1) / kSeg;
  float* const ck = ckpt + bh * (long)nseg * DK * DV;
  const long sbase = bh * (long)DK * DV;             // [dk][dv] slot of S0, dS_T, dS0

  // pass 1: the recurrence forward, the state before every segment kept
  float4 M[RPT], G[RPT];
  if (S0) cx.get(S0 + sbase, M);
  else
#pragma unroll
    for (int r = 0; r < RPT; ++r) M[r] = f4(0.f);
  for (int sg = 0; sg < nseg; ++sg) {
    const int t0 = sg * kSeg, len = min(kSeg, T - t0);
    __syncthreads();                                 // the previous segment's data is read
    load_segment(sm, q, k, v, dO, log_alpha, beta, b, h, hk, T, Hk, Hv, t0, len, false);
    cx.put(ck + (long)sg * DK * DV, M);
    __syncthreads();
    for (int j = 0; j < len; ++j) cx.fwd_step(M, j);
  }

  // pass 2: segments last to first, tokens last to first
  if (dS_T) cx.get(dS_T + sbase, G);
  else
#pragma unroll
    for (int r = 0; r < RPT; ++r) G[r] = f4(0.f);
  float* const st0 = sm.state0;
  float* const stm = sm.statem;
  for (int sg = nseg - 1; sg >= 0; --sg) {
    const int t0 = sg * kSeg, len = min(kSeg, T - t0);
    __syncthreads();
    load_segment(sm, q, k, v, dO, log_alpha, beta, b, h, hk, T, Hk, Hv, t0, len, true);
    cx.get(ck + (long)sg * DK * DV, M);              // this thread's own elements only
    cx.put(st0, M);
    __syncthreads();
    if (len > kHalf) {
      for (int j = 0; j < kHalf; ++j) cx.fwd_step(M, j);
      cx.put(stm, M);
    }
    for (int j = len - 1; j >= 0; --j) {
      // P = S before token t0 + j, from the nearer kept state
      int j0;
      if (j >= kHalf) { cx.get(stm, M); j0 = kHalf; }
      else { cx.get(st0, M); j0 = 0; }
      for (int u = j0; u < j; ++u) cx.fwd_step(M, u);
      const long t = t0 + j;
      const float a = sm.alpha[j], be = sm.beta[j];
      float kk[RPT], qs[RPT];
#pragma unroll
      for (int r = 0; r < RPT; ++r) {
        kk[r] = sm.k[j][rg + RG * r];
        qs[r] = scale * sm.q[j][rg + RG * r];
      }
      const float4 vv = *reinterpret_cast<const float4*>(&sm.v[j][4 * cg]);
      const float4 dd = *reinterpret_cast<const float4*>(&sm.dO[j][4 * cg]);
      // G += scale dO q^T; partials of x = P k, Gk = G k and <G, P>
      float4 x4 = f4(0.f), g4 = f4(0.f);
      float gp = 0.f;
#pragma unroll
      for (int r = 0; r < RPT; ++r) {
        G[r] = fma4(f4(qs[r]), dd, G[r]);
        x4 = fma4(M[r], f4(kk[r]), x4);
        g4 = fma4(G[r], f4(kk[r]), g4);
        gp += dot4(G[r], M[r]);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) gp += __shfl_xor_sync(0xffffffffu, gp, o);
      if (lane == 0) sm.wsum[cx.par][warp] = gp;
      const int wpar = cx.par;
      float4 pa[2] = {x4, g4}, ps[2];
      cx.colsum<2>(pa, ps);
      const float4 x = ps[0], Gk = ps[1];
      const float4 u = fma4(f4(-a), x, vv);           // v - alpha x
      const float4 w = mul4(f4(be), u);                // S_t = alpha P + k w^T
      const float4 dx = mul4(f4(-a * be), Gk);
      // dq = scale S_t^T dO and dk = beta G^T (v - alpha x) + P^T dx, one value per row
      const float4 bu = mul4(f4(be), u);
      float pv[2 * RPT];                              // dq rows, then dk rows, partial over 4 columns
#pragma unroll
      for (int r = 0; r < RPT; ++r) {
        pv[r] = dot4(fma4(f4(a), M[r], mul4(f4(kk[r]), w)), dd);
        pv[RPT + r] = dot4(G[r], bu) + dot4(M[r], dx);
      }
      {
        int idx, keep_mask = CG;
        reduce_scatter<2 * RPT, CG>(pv, lane, idx, keep_mask);
        if ((lane & (keep_mask - 1)) == 0) {           // one lane per value
          const int r = idx % RPT;
          const long o = ((b * T + t) * nqk + hq) * (long)DK + rg + RG * r;
          if (idx < RPT) dq_out[o] = scale * pv[0];
          else dk_out[o] = pv[0];
        }
      }
      // dv, dbeta and dlog alpha from the row group 0 lanes (they hold every column once); the
      // sums over the columns run in every warp, so that all lanes take part in the shuffles
      const float vg = lane_sum<CG>(dot4(u, Gk)), xg = lane_sum<CG>(dot4(x, Gk));
      if (rg == 0) {
        *reinterpret_cast<float4*>(dv_out + ((b * T + t) * Hv + h) * (long)DV + 4 * cg) =
            mul4(f4(be), Gk);
        if (tid == 0) {
          float gsum = 0.f;
#pragma unroll
          for (int w8 = 0; w8 < Sh::NW; ++w8) gsum += sm.wsum[wpar][w8];
          const long g = (b * T + t) * Hv + h;
          dbeta_out[g] = vg;                         // (v - alpha x)^T Gk
          dla_out[g] = a * (gsum - be * xg);          // alpha <G, P - beta x k^T>
        }
      }
      // the gradient reaching S_{t-1}: alpha G + dx k^T
#pragma unroll
      for (int r = 0; r < RPT; ++r) G[r] = fma4(f4(a), G[r], mul4(f4(kk[r]), dx));
    }
  }
  if (dS0) cx.put(dS0 + sbase, G);
}

// dst [rows, D] = sum over g < G of src [rows * G + g, D] (the value heads of each key head).
__global__ void group_sum_kernel(const float* __restrict__ a_src, float* __restrict__ a_dst,
                                 const float* __restrict__ b_src, float* __restrict__ b_dst,
                                 long rows, int G, int D) {
  const long n = rows * (long)D;
  for (long e = blockIdx.x * (long)blockDim.x + threadIdx.x; e < 2 * n;
       e += (long)gridDim.x * blockDim.x) {
    const bool second = e >= n;
    const long f = second ? e - n : e;
    const long r = f / D, i = f - r * D;
    const float* src = second ? b_src : a_src;
    float acc = 0.f;
    for (int g = 0; g < G; ++g) acc += src[(r * G + g) * D + i];
    (second ? b_dst : a_dst)[f] = acc;
  }
}

}  // namespace bwd
}  // namespace gdn
