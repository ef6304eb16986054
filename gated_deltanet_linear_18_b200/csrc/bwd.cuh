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
// the segments last to first, keeping the segment's first state and its middle state in shared
// memory and recomputing each S_{t-1} from the nearer one (about two token steps per token).
//
// One CTA per (batch, value head).  Layout of the state M = S^T (dk x dv) and of its gradient:
// the lanes of a warp take the dk rows (RL consecutive rows each), the warps the dv columns (CW
// consecutive columns per thread).  So the sums over dk that the recurrence itself needs (S k and
// G k) stay inside a warp (shuffles) and a token step needs no CTA barrier; the sums over dv
// (dq, dk, dbeta, dlog alpha: outputs only) are written per column slice to shared memory and
// added up once every kHalf tokens, in a fixed order.
#pragma once

#include "common.cuh"

namespace gdn {
namespace bwd {

constexpr int kSeg = 8;          // tokens per checkpoint segment
constexpr int kHalf = kSeg / 2;  // the segment's middle state is S before token t0 + kHalf

// A head's dv columns are split over NS CTAs (the recurrence never mixes columns: S k, G k and
// every update act column by column; only the outputs sum over columns, and those partial sums
// are added afterwards), so that small batches still fill the GPU and several CTAs share an SM.
__host__ __device__ constexpr int head_slices(int D) { return D == 128 ? 4 : (D == 64 ? 2 : 1); }

template <int D>
struct Shape {
  static constexpr int NS = head_slices(D);               // CTAs per head
  static constexpr int DC = D / NS;                       // dv columns per CTA
  static constexpr int LR = D < 32 ? D : 32;              // lanes along dk
  static constexpr int RL = D / LR;                       // dk rows per lane
  static constexpr int LC = 32 / LR;                      // column groups per warp
  static constexpr int NT = D == 128 ? 128 : (D == 64 ? 256 : (D == 32 ? 512 : 128));
  static constexpr int NW = NT / 32;
  static constexpr int SL = NW * LC;                      // column slices of the CTA
  static constexpr int CW = DC / SL;                      // dv columns per thread
  static constexpr int VPT = RL * CW;                     // state values per thread
  static constexpr int MINB = D == 128 ? 3 : (D == 64 ? 2 : 1);   // CTAs per SM to fit
  static_assert(CW >= 1 && SL * CW == DC && 2 * CW <= LR && VPT % 2 == 0, "bwd shape");
};

template <int D>
struct Smem {
  static constexpr int DC = Shape<D>::DC;
  float k[kSeg][D], q[kSeg][D], v[kSeg][DC], dO[kSeg][DC];
  float alpha[kSeg], beta[kSeg];
  float state0[D * DC];        // the state before the segment's first token (per-thread layout)
  float statem[D * DC];        // the state before the segment's token t0 + kHalf
  float pdq[kHalf][Shape<D>::SL][D], pdk[kHalf][Shape<D>::SL][D];   // per-slice partials
  float pa[kHalf][Shape<D>::SL], pb[kHalf][Shape<D>::SL];          // of <G, A>, dbeta
};

template <int D>
constexpr size_t smem_bytes() { return sizeof(Smem<D>); }

// All-reduce over the LR lanes of a column group (lanes xor LR/2 .. 1) of V values per lane:
// recursive halving (each step keeps one half, adds the partner's copy of it and passes the other
// half on: V - 1 shuffles), then each total is fetched from the lane that holds it (V shuffles).
template <int V, int LR>
__device__ __forceinline__ void allreduce(float (&v)[V], int lane) {
  static_assert((V & (V - 1)) == 0 && V <= LR, "allreduce");
  int n = V;
#pragma unroll
  for (int m = LR >> 1; m > 0; m >>= 1) {
    if (n > 1) {
      const bool up = (lane & m) != 0;
#pragma unroll
      for (int kk = 0; kk < V / 2; ++kk) {
        if (kk < n / 2) {
          const float lo = v[kk], hi = v[kk + n / 2];
          v[kk] = (up ? hi : lo) + __shfl_xor_sync(0xffffffffu, up ? lo : hi, m);
        }
      }
      n >>= 1;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], m);
    }
  }
  // value c sits in the lanes of this column group whose halving bits spell c
  const float mine = v[0];
  const int group = lane & ~(LR - 1);
#pragma unroll
  for (int c = 0; c < V; ++c) {
    int src = group, half = V >> 1, m = LR >> 1;
#pragma unroll
    for (int s = 0; s < 5; ++s) {
      if (half >= 1) {
        if (c & half) src |= m;
        half >>= 1;
        m >>= 1;
      }
    }
    v[c] = __shfl_sync(0xffffffffu, mine, src);
  }
}

// Sum over the LR lanes of a column group.
template <int LR>
__device__ __forceinline__ float group_sum(float x) {
#pragma unroll
  for (int m = LR >> 1; m > 0; m >>= 1) x += __shfl_xor_sync(0xffffffffu, x, m);
  return x;
}

// The segment's token data (tokens t0 .. t0 + len - 1) into shared memory, as fp32.
template <int D, typename Tin, typename Tdo>
__device__ __forceinline__ void load_segment(Smem<D>& sm, const Tin* __restrict__ q,
                                             const Tin* __restrict__ k, const Tin* __restrict__ v,
                                             const Tdo* __restrict__ dO,
                                             const float* __restrict__ la,
                                             const float* __restrict__ be, long r0, int h,
                                             int hk, int c0, int Hk, int Hv, int t0, int len,
                                             bool with_q) {
  constexpr int NT = Shape<D>::NT, DC = Shape<D>::DC;
  for (int e = threadIdx.x; e < len * D; e += NT) {
    const int j = e / D, i = e - j * D;
    const long rk = ((r0 + t0 + j) * Hk + hk) * (long)D + i;
    sm.k[j][i] = to_f(k[rk]);
    if (with_q) sm.q[j][i] = to_f(q[rk]);
  }
  for (int e = threadIdx.x; e < len * DC; e += NT) {      // this CTA's columns c0 .. c0 + DC - 1
    const int j = e / DC, i = e - j * DC;
    const long rv = ((r0 + t0 + j) * Hv + h) * (long)D + c0 + i;
    sm.v[j][i] = to_f(v[rv]);
    if (with_q) sm.dO[j][i] = to_f(dO[rv]);
  }
  for (int j = threadIdx.x; j < len; j += NT) {
    const long g = (r0 + t0 + j) * Hv + h;
    sm.alpha[j] = expf(la[g]);
    sm.beta[j] = be[g];
  }
}

// One thread's share of a state: rows i0 .. i0 + RL - 1, columns j0 .. j0 + CW - 1, held as
// column pairs (c, c + 1).
template <int D>
struct Tile {
  using Sh = Shape<D>;
  static_assert(Sh::CW % 2 == 0, "column pairs");
  f2_t m[Sh::RL][Sh::CW / 2];
};

// grid: B * Hv * NS CTAs ((b * Hv + h) * NS + column slice); block Shape<D>::NT; dynamic shared
// memory smem_bytes<D>().  Sequences as in row_span: b of [B, T, ...] tensors (cu == nullptr,
// max_len = T), or packed rows cu[b] .. cu[b + 1] - 1 of T in all (none longer than max_len);
// token rows below are rows of those tensors.  direct (one value head per key head and one slice
// per head): dq_out, dk_out are [rows, Hk, D] and dla_out, dbeta_out [rows, Hv]; otherwise they are
// the per-slice partials [rows, Hv * NS, D] and [rows, Hv, NS], summed afterwards by
// group_sum_kernel.  ckpt: B * Hv * NS * ceil(max_len / kSeg) slices of D * DC floats, each in the
// CTA's own per-thread order.
template <int D, typename Tin, typename Tdo = Tin>
__global__ void __launch_bounds__(Shape<D>::NT, Shape<D>::MINB)
bwd_kernel(const Tin* __restrict__ q, const Tin* __restrict__ k, const Tin* __restrict__ v,
           const float* __restrict__ log_alpha, const float* __restrict__ beta,
           const float* __restrict__ S0, const Tdo* __restrict__ dO,
           const float* __restrict__ dS_T, float* __restrict__ dq_out,
           float* __restrict__ dk_out, int direct, float* __restrict__ dv_out,
           float* __restrict__ dla_out, float* __restrict__ dbeta_out, float* __restrict__ dS0,
           float* __restrict__ ckpt, int T, int Hk, int Hv, float scale,
           const int* __restrict__ cu, int max_len) {
  using Sh = Shape<D>;
  constexpr int RL = Sh::RL, CW = Sh::CW, CP = CW / 2, LR = Sh::LR, NT = Sh::NT, SL = Sh::SL;
  constexpr int NS = Sh::NS, DC = Sh::DC, PPT = RL * CP;   // column pairs per thread
  extern __shared__ __align__(16) unsigned char bwd_smem[];
  Smem<D>& sm = *reinterpret_cast<Smem<D>*>(bwd_smem);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int lr = lane % LR, sl = warp * Sh::LC + lane / LR;   // row lane, column slice
  const long bh = blockIdx.x / NS;
  const int ns = blockIdx.x % NS, c0 = ns * DC;      // this CTA's columns c0 .. c0 + DC - 1
  const int i0 = lr * RL, jl = sl * CW, j0 = c0 + jl;   // rows; columns (local, of the head)
  const int h = (int)(bh % Hv);
  const long b = bh / Hv;
  const int hk = h / (Hv / Hk);
  const int nqk = direct ? Hk : Hv * NS, hq = direct ? hk : h * NS + ns;   // dq, dk slot
  const int nab = direct ? 1 : NS, hab = direct ? 0 : ns;                 // dla, dbeta slot
  const RowSpan span = row_span(cu, (int)b, T, max_len);   // this sequence's rows
  const long r0 = span.row0;
  const int Ts = span.len;
  const int nseg = (Ts + kSeg - 1) / kSeg;
  float* const ck = ckpt + (long)blockIdx.x * ((max_len + kSeg - 1) / kSeg) * D * DC;
  const long sbase = bh * (long)D * D;               // [dk][dv] slot of S0, dS_T, dS0

  // a state in the [dk][dv] order of S0 / dS_T / dS0 (8-byte pairs: j0 and CW are even), and in
  // the per-thread order of the checkpoints and the shared-memory copies (pair p of thread t at
  // (p * NT + t) * 2)
  auto get_sq = [&](const float* base, Tile<D>& M) {
#pragma unroll
    for (int r = 0; r < RL; ++r)
#pragma unroll
      for (int c = 0; c < CP; ++c)
        M.m[r][c] = *reinterpret_cast<const f2_t*>(base + (long)(i0 + r) * D + j0 + 2 * c);
  };
  auto put_sq = [&](float* base, const Tile<D>& M) {
#pragma unroll
    for (int r = 0; r < RL; ++r)
#pragma unroll
      for (int c = 0; c < CP; ++c)
        *reinterpret_cast<f2_t*>(base + (long)(i0 + r) * D + j0 + 2 * c) = M.m[r][c];
  };
  auto get_pt = [&](const float* base, Tile<D>& M) {
#pragma unroll
    for (int e = 0; e < PPT; ++e)
      M.m[e / CP][e % CP] = *reinterpret_cast<const f2_t*>(base + ((long)e * NT + tid) * 2);
  };
  auto put_pt = [&](float* base, const Tile<D>& M) {
#pragma unroll
    for (int e = 0; e < PPT; ++e)
      *reinterpret_cast<f2_t*>(base + ((long)e * NT + tid) * 2) = M.m[e / CP][e % CP];
  };
  auto zero = [&](Tile<D>& M) {
#pragma unroll
    for (int e = 0; e < PPT; ++e) M.m[e / CP][e % CP] = 0ull;
  };
  // one token of the recurrence: x = S k (inside the warp), S <- alpha S + k (beta (v - alpha x))^T
  auto fwd_step = [&](Tile<D>& M, int j) {
    const float a = sm.alpha[j], be = sm.beta[j];
    f2_t kk[RL], xp[CP];
#pragma unroll
    for (int r = 0; r < RL; ++r) kk[r] = splat2(sm.k[j][i0 + r]);
#pragma unroll
    for (int c = 0; c < CP; ++c) {
      f2_t acc = 0ull;
#pragma unroll
      for (int r = 0; r < RL; ++r) acc = fma2(M.m[r][c], kk[r], acc);
      xp[c] = acc;
    }
    float x[CW];
#pragma unroll
    for (int c = 0; c < CP; ++c) up2(xp[c], x[2 * c], x[2 * c + 1]);
    allreduce<CW, LR>(x, lane);
    const f2_t a2 = splat2(a);
#pragma unroll
    for (int c = 0; c < CP; ++c) {
      const f2_t w = pk2(be * fmaf(-a, x[2 * c], sm.v[j][jl + 2 * c]),
                         be * fmaf(-a, x[2 * c + 1], sm.v[j][jl + 2 * c + 1]));
#pragma unroll
      for (int r = 0; r < RL; ++r) M.m[r][c] = fma2(a2, M.m[r][c], mul2(kk[r], w));
    }
  };

  // pass 1: the recurrence forward, the state before every segment kept
  Tile<D> M, G;
  if (S0) get_sq(S0 + sbase, M);
  else zero(M);
  for (int sg = 0; sg < nseg; ++sg) {
    const int t0 = sg * kSeg, len = min(kSeg, Ts - t0);
    __syncthreads();                                 // the previous segment's data is read
    load_segment(sm, q, k, v, dO, log_alpha, beta, r0, h, hk, c0, Hk, Hv, t0, len, false);
    put_pt(ck + (long)sg * D * DC, M);
    __syncthreads();
    for (int j = 0; j < len; ++j) fwd_step(M, j);
  }

  // pass 2: segments last to first, tokens last to first
  if (dS_T) get_sq(dS_T + sbase, G);
  else zero(G);
  // the per-slice partials of tokens t0 + jb .. t0 + je - 1, summed into the outputs
  auto flush = [&](int t0, int jb, int je) {
    __syncthreads();
    const int n = je - jb, per = 2 * D + 2;
    for (int e = tid; e < n * per; e += NT) {
      const int jj = e / per, f = e - jj * per, j = jb + jj, hj = j % kHalf;
      const long t = t0 + j;
      float acc = 0.f;
      if (f < 2 * D) {
        const int i = f % D;
#pragma unroll 4
        for (int s2 = 0; s2 < SL; ++s2) acc += f < D ? sm.pdq[hj][s2][i] : sm.pdk[hj][s2][i];
        float* dst = f < D ? dq_out : dk_out;
        dst[((r0 + t) * nqk + hq) * (long)D + i] = acc;
      } else {
        const bool isa = f == 2 * D;
#pragma unroll 4
        for (int s2 = 0; s2 < SL; ++s2) acc += isa ? sm.pa[hj][s2] : sm.pb[hj][s2];
        const long g = ((r0 + t) * Hv + h) * nab + hab;
        if (isa) dla_out[g] = sm.alpha[j] * acc;       // alpha <G, P - beta x k^T>
        else dbeta_out[g] = acc;                       // (v - alpha x)^T Gk
      }
    }
    __syncthreads();
  };
  for (int sg = nseg - 1; sg >= 0; --sg) {
    const int t0 = sg * kSeg, len = min(kSeg, Ts - t0);
    __syncthreads();
    load_segment(sm, q, k, v, dO, log_alpha, beta, r0, h, hk, c0, Hk, Hv, t0, len, true);
    get_pt(ck + (long)sg * D * DC, M);               // this thread's own elements
    put_pt(sm.state0, M);
    __syncthreads();
    if (len > kHalf) {
      for (int j = 0; j < kHalf; ++j) fwd_step(M, j);
      put_pt(sm.statem, M);
    }
    for (int j = len - 1; j >= 0; --j) {
      // P = S before token t0 + j, from the nearer kept state
      int j0s;
      if (j >= kHalf) { get_pt(sm.statem, M); j0s = kHalf; }
      else { get_pt(sm.state0, M); j0s = 0; }
      for (int u = j0s; u < j; ++u) fwd_step(M, u);
      const float a = sm.alpha[j], be = sm.beta[j];
      f2_t kk[RL], qs[RL], dd[CP];
#pragma unroll
      for (int r = 0; r < RL; ++r) {
        kk[r] = splat2(sm.k[j][i0 + r]);
        qs[r] = splat2(scale * sm.q[j][i0 + r]);
      }
#pragma unroll
      for (int c = 0; c < CP; ++c) dd[c] = pk2(sm.dO[j][jl + 2 * c], sm.dO[j][jl + 2 * c + 1]);
      // G += scale dO q^T; x = P k and Gk = G k (sums over dk, in the warp); <G, P> partial
      f2_t gp2 = 0ull;
      float xg[2 * CW];
#pragma unroll
      for (int c = 0; c < CP; ++c) {
        f2_t ax = 0ull, ag = 0ull;
#pragma unroll
        for (int r = 0; r < RL; ++r) {
          G.m[r][c] = fma2(qs[r], dd[c], G.m[r][c]);
          ax = fma2(M.m[r][c], kk[r], ax);
          ag = fma2(G.m[r][c], kk[r], ag);
          gp2 = fma2(G.m[r][c], M.m[r][c], gp2);
        }
        up2(ax, xg[2 * c], xg[2 * c + 1]);
        up2(ag, xg[CW + 2 * c], xg[CW + 2 * c + 1]);
      }
      allreduce<2 * CW, LR>(xg, lane);
      const float gp = group_sum<LR>(hsum2(gp2));
      f2_t w2[CP], dx2[CP];
      float ug = 0.f, xgk = 0.f, gk[CW];
#pragma unroll
      for (int c = 0; c < CW; ++c) {
        gk[c] = xg[CW + c];
        const float uc = fmaf(-a, xg[c], sm.v[j][jl + c]);     // v - alpha x
        ug = fmaf(uc, gk[c], ug);
        xgk = fmaf(xg[c], gk[c], xgk);
      }
#pragma unroll
      for (int c = 0; c < CP; ++c) {
        const float u0 = fmaf(-a, xg[2 * c], sm.v[j][jl + 2 * c]);
        const float u1 = fmaf(-a, xg[2 * c + 1], sm.v[j][jl + 2 * c + 1]);
        w2[c] = pk2(be * u0, be * u1);                  // S_t = alpha P + k w^T
        dx2[c] = pk2(-a * be * gk[2 * c], -a * be * gk[2 * c + 1]);
      }
      // per-slice partials: dq = scale S_t^T dO, dk = beta G^T (v - alpha x) + P^T dx
      const int hj = j % kHalf;
      const f2_t a2 = splat2(a);
#pragma unroll
      for (int r = 0; r < RL; ++r) {
        f2_t pq = 0ull, pkk = 0ull;
#pragma unroll
        for (int c = 0; c < CP; ++c) {
          pq = fma2(fma2(a2, M.m[r][c], mul2(kk[r], w2[c])), dd[c], pq);
          pkk = fma2(G.m[r][c], w2[c], fma2(M.m[r][c], dx2[c], pkk));   // beta G u = G w
        }
        sm.pdq[hj][sl][i0 + r] = scale * hsum2(pq);
        sm.pdk[hj][sl][i0 + r] = hsum2(pkk);
      }
      if (lr == 0) {
        sm.pa[hj][sl] = gp - be * xgk;                // this slice's <G, P - beta x k^T>
        sm.pb[hj][sl] = ug;
#pragma unroll
        for (int c = 0; c < CW; ++c)
          dv_out[((r0 + t0 + j) * Hv + h) * (long)D + j0 + c] = be * gk[c];
      }
      // the gradient reaching S_{t-1}: alpha G + dx k^T
#pragma unroll
      for (int c = 0; c < CP; ++c)
#pragma unroll
        for (int r = 0; r < RL; ++r) G.m[r][c] = fma2(a2, G.m[r][c], mul2(kk[r], dx2[c]));
      if (j == kHalf) flush(t0, kHalf, len);
      if (j == 0) flush(t0, 0, min(len, kHalf));
    }
  }
  if (dS0) put_sq(dS0 + sbase, G);
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
