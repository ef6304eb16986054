// Chunked forward of the gated delta rule on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
// Shapes: d_k = d_v = 128, chunk C = 64, bf16 q/k/v, fp32 gates and state.
//
// Per value head and chunk, with the chunk-start state M = S^T (128 x 128, fp32), the chunk form of
// the recurrence ("Chapitre 16 - Assembler un système de type Kimi K3", 16.2: matrix operations
// inside each block, state handed from block to block) is computed as
//   state-independent part (one per chunk, shared by both halves of the state):
//     G = cumsum(log alpha), gamma = exp(G), S = [Q; K] K^T                (bf16 MMA, 128x64x128)
//     P = lower_incl(exp(G_i - G_j) q_i.k_j) * scale,  A = strict_lower(beta_i exp(G_i - G_j) k_i.k_j)
//     T = (I + A)^-1 (fp32, blocked by 16),  T_b = T diag(beta)
//     A2 = [P T_b; T_b]                     (P T_b: tf32 MMA, 64x64x64)
//   state-dependent chain, for each 64-column half of M independently:
//     X = [Q; K] M                           (bf16 MMA, 128x64x128)
//     R' = V - diag(gamma) (K M)             (rows 64..127 of X)
//     Y = A2 R' = [P Delta; Delta]           (tf32 MMA, 128x64x64), Delta = T_b (V - diag(gamma) K M)
//     o = diag(gamma) scale (Q M) + P Delta  (rows 0..63 of X and Y)
//     M <- gamma_last M + K^T (ktil Delta),  ktil = exp(G_last - G)
//                                            (bf16 MMA on a two-term bf16 split of ktil Delta)
// which is the token recurrence reorganised exactly (Delta's rows are beta_t (v_t - alpha_t
// S_{t-1} k_t)).  Accumulations and the master state are fp32.  The operands that carry the state
// through the chain (A2, R', ktil Delta) use tf32 or a hi+lo bf16 pair: with plain bf16 there the
// state's largest entries drift by a few percent of its RMS.
//
// One CTA per (batch, value head), 512 threads in specialised warps:
//   warp 0        TMA producer (Q, K tiles double-buffered; each V half in its own buffer)
//   warp 1        TMEM owner; issues the state-independent MMAs (S and P T_b)
//   warps 2, 3    issue the chain MMAs of state half 0 / half 1
//   warps 4-7     "pre" warpgroup: gates, A, the triangular solve, P, T_b and A2
//   warps 8-11    chain warpgroup of half 0 (dv columns 0..63); warps 12-15 of half 1
// so the state-independent work of chunk c+1 overlaps the chain of chunk c, and the two halves'
// chains interleave on the tensor pipe.  Every wait is bounded (2 s): on expiry the CTA records
// the library's timeout bit, every role leaves its loop at the next uniform check point, in-flight
// TMA loads and MMAs are drained, TMEM is released and the kernel returns.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "tc_ptx.cuh"

namespace gdn {
namespace tcf {

constexpr int C = 64;
constexpr int kThreads = 512;
constexpr uint64_t kBudgetNs = 4000000000ull;   // wait budget in SM cycles (about 2 s)

// shared memory map (bytes from a 1024-aligned base); every MMA tile is 128-byte swizzled
constexpr uint32_t OFF_QK = 0;          // 2 stages x 32 KB: kb0 [Q 64 rows | K 64 rows], kb1 [...]
constexpr uint32_t QK_STAGE = 32768;
constexpr uint32_t OFF_V = 65536;       // per half 8 KB: V[t][64 dv] bf16
constexpr uint32_t OFF_RD = 81920;      // per half 16 KB: R' tf32 [dv block][64 t][128 B], then
                                        // ktil Delta bf16 hi [64 t][128 B] + lo [64 t][128 B]
constexpr uint32_t OFF_A2 = 114688;     // 32 KB: A2 tf32, [K block][128 rows][128 B]
constexpr uint32_t OFF_MB = 147456;     // per half 16 KB: bf16 M [128 dk rows][128 B]
constexpr uint32_t OFF_W = 180224;      // 32 KB: solve scratch, then P (tf32) and T_b (tf32)
constexpr uint32_t OFF_WT = OFF_W + 16384;   // T_b, [dv block][64 rows][128 B]
constexpr uint32_t SOLVE_T = 12800;     // byte offset of T inside the solve scratch
constexpr uint32_t OFF_GB = 212992;     // 3 slots x 2 KB: G log2(e)[64], gamma[64], ktil[64],
                                        // beta[64], E[4][64] (E[b][j] = exp(G_16b - G_j), j < 16b)
constexpr uint32_t GB_SLOT = 2048;
constexpr uint32_t OFF_BAR = OFF_GB + 3 * GB_SLOT;
constexpr int NBAR = 40;
constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;   // +0 TMEM base, +4 abort flag
constexpr uint32_t SMEM_BYTES = OFF_MISC + 16;
constexpr uint32_t SMEM_ALLOC = SMEM_BYTES + 1024;
static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
static_assert(2 * SOLVE_T <= 32768, "solve scratch");

// TMEM columns (512 allocated, 128 lanes x 32 bit)
constexpr uint32_t TM_S = 0, TM_PT = 64, TM_X = 128, TM_Y = 256, TM_D3 = 384;

// mbarriers
enum : int {
  B_QK_FULL = 0, B_IN_EMPTY = 2, B_S_FULL = 4, B_S_EMPTY = 5, B_PT_READY = 6, B_PT_FULL = 7,
  B_PT_EMPTY = 8, B_PRE_FULL = 9, B_A2_EMPTY = 10, B_GATE = 11, B_HALF = 14, B_DRAIN = 36
};
enum : int {
  H_X_FULL = 0, H_X_EMPTY, H_R_FULL, H_Y_FULL, H_Y_EMPTY, H_D_FULL, H_D3_FULL, H_D3_EMPTY,
  H_M_READY, H_V_FULL, H_V_EMPTY, H_COUNT
};
static_assert(B_HALF + 2 * H_COUNT == B_DRAIN && B_DRAIN + 3 <= NBAR, "barrier map");

constexpr uint32_t ID_S = tc::idesc_bf16(128, 64, false, false);
constexpr uint32_t ID_PT = tc::idesc_tf32(64, 64, false, true);
constexpr uint32_t ID_X = tc::idesc_bf16(128, 64, false, true);
constexpr uint32_t ID_Y = tc::idesc_tf32(128, 64, false, true);
constexpr uint32_t ID_U = tc::idesc_bf16(128, 64, true, true);

// Optional per-chunk timestamps for studying the pipeline (compiled only with GDN_TC_TRACE):
// slot (block, chunk, event) of a caller-provided buffer receives clock64().
#ifdef GDN_TC_TRACE
__device__ unsigned long long* g_tc_trace = nullptr;
#define GDN_TRACE(c, ev)                                                              \
  do {                                                                                \
    if (g_tc_trace) g_tc_trace[((size_t)blockIdx.x * nC + (c)) * 64 + (ev)] = clock64(); \
  } while (0)
#else
#define GDN_TRACE(c, ev) do {} while (0)
#endif

// ------------------------------------------------------------------------------------------
// triangular solve on 16 x 16 blocks stored packed: block (i, k), i >= k, at index
// i(i+1)/2 + k, 16 rows of 20 floats (4 floats of padding against bank conflicts)
// ------------------------------------------------------------------------------------------
constexpr int BLD = 20, BSZ = 16 * BLD;
__device__ __forceinline__ float* blk(float* base, int i, int k) {
  return base + (i * (i + 1) / 2 + k) * BSZ;
}

// acc[0..3] += sum_k X[xr][k] * Y[k][yc .. yc+3], k < 16, X and Y 16 x 16 blocks.
__device__ __forceinline__ void strip16(const float* X, int xr, const float* Y, int yc,
                                        float (&acc)[4]) {
#pragma unroll
  for (int k4 = 0; k4 < 16; k4 += 4) {
    const float4 xa = *reinterpret_cast<const float4*>(&X[xr * BLD + k4]);
    const float xs[4] = {xa.x, xa.y, xa.z, xa.w};
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const float4 y = *reinterpret_cast<const float4*>(&Y[(k4 + kk) * BLD + yc]);
      acc[0] = fmaf(xs[kk], y.x, acc[0]);
      acc[1] = fmaf(xs[kk], y.y, acc[1]);
      acc[2] = fmaf(xs[kk], y.z, acc[2]);
      acc[3] = fmaf(xs[kk], y.w, acc[3]);
    }
  }
}

// T = (I + A)^-1 for a 64 x 64 strictly lower A (128 threads, named barrier 1):
//   D_b = (I + A_bb)^-1 by forward substitution (one column per thread);
//   At_ik = D_i A_ik;  U = (I + At)^-1 by block forward substitution (U_ii = I);  T_ik = U_ik D_k.
// (I + A = blockdiag(I + A_bb) (I + At), so T = U D.)  sA is overwritten with At.
__device__ void solve_unit_lower(float* sA, float* sT, int ptid, int c, int nC) {
  if (ptid < 64) {
    const int b = ptid >> 4, col = ptid & 15;
    const float* Ab = blk(sA, b, b);
    float x[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      float acc = (i == col) ? 1.f : 0.f;
#pragma unroll
      for (int j = 0; j < i; ++j) acc = fmaf(-Ab[i * BLD + j], x[j], acc);
      x[i] = acc;
    }
    float* Tb = blk(sT, b, b);
#pragma unroll
    for (int i = 0; i < 16; ++i) Tb[i * BLD + col] = x[i];
  }
  tc::named_bar(1, 128);
  if (ptid == 0) GDN_TRACE(c, 44);
  // block index bi = 0..5 -> (i, k) = (1,0) (2,0) (2,1) (3,0) (3,1) (3,2)
  auto blk_i = [](int bi) { return bi < 1 ? 1 : (bi < 3 ? 2 : 3); };
  auto blk_k = [](int bi, int i) { return bi - i * (i - 1) / 2; };
  float r1[3][4];
#pragma unroll
  for (int m = 0; m < 3; ++m) {                       // At_ik = D_i A_ik
    const int id = ptid + 128 * m, bi = id >> 6, r = (id >> 2) & 15, cs = id & 3;
    const int i = blk_i(bi), k = blk_k(bi, i);
    r1[m][0] = r1[m][1] = r1[m][2] = r1[m][3] = 0.f;
    strip16(blk(sT, i, i), r, blk(sA, i, k), 4 * cs, r1[m]);
  }
  tc::named_bar(1, 128);
#pragma unroll
  for (int m = 0; m < 3; ++m) {
    const int id = ptid + 128 * m, bi = id >> 6, r = (id >> 2) & 15, cs = id & 3;
    const int i = blk_i(bi), k = blk_k(bi, i);
    *reinterpret_cast<float4*>(&blk(sA, i, k)[r * BLD + 4 * cs]) =
        make_float4(r1[m][0], r1[m][1], r1[m][2], r1[m][3]);
  }
  tc::named_bar(1, 128);
  if (ptid == 0) GDN_TRACE(c, 45);
  // U_20 = -At_20 + At_21 At_10;  U_31 = -At_31 + At_32 At_21;  V_30 = -At_30 + At_31 At_10
  for (int id = ptid; id < 192; id += 128) {
    const int bi = id >> 6, r = (id >> 2) & 15, cs = id & 3;
    const int oi = bi == 0 ? 2 : 3, ok = bi == 1 ? 1 : 0;      // output block (oi, ok)
    const int xk = bi == 1 ? 2 : 1;                             // X = At_(oi, xk), Y = At_(xk, ok)
    const float4 base = *reinterpret_cast<const float4*>(&blk(sA, oi, ok)[r * BLD + 4 * cs]);
    float acc[4] = {-base.x, -base.y, -base.z, -base.w};
    strip16(blk(sA, oi, xk), r, blk(sA, xk, ok), 4 * cs, acc);
    *reinterpret_cast<float4*>(&blk(sT, oi, ok)[r * BLD + 4 * cs]) =
        make_float4(acc[0], acc[1], acc[2], acc[3]);
  }
  tc::named_bar(1, 128);
  if (ptid < 64) {                                    // U_30 = V_30 - At_32 U_20
    const int r = ptid >> 2, cs = ptid & 3;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    strip16(blk(sA, 3, 2), r, blk(sT, 2, 0), 4 * cs, acc);
    float4* dst = reinterpret_cast<float4*>(&blk(sT, 3, 0)[r * BLD + 4 * cs]);
    const float4 v30 = *dst;
    *dst = make_float4(v30.x - acc[0], v30.y - acc[1], v30.z - acc[2], v30.w - acc[3]);
  }
  tc::named_bar(1, 128);
  if (ptid == 0) GDN_TRACE(c, 46);
  float r4[3][4];
#pragma unroll
  for (int m = 0; m < 3; ++m) {                       // T_ik = U_ik D_k (U = -At next to diag)
    const int id = ptid + 128 * m, bi = id >> 6, r = (id >> 2) & 15, cs = id & 3;
    const int i = blk_i(bi), k = blk_k(bi, i);
    const bool sub = (i == k + 1);
    r4[m][0] = r4[m][1] = r4[m][2] = r4[m][3] = 0.f;
    strip16(sub ? blk(sA, i, k) : blk(sT, i, k), r, blk(sT, k, k), 4 * cs, r4[m]);
    if (sub) {
      r4[m][0] = -r4[m][0]; r4[m][1] = -r4[m][1]; r4[m][2] = -r4[m][2]; r4[m][3] = -r4[m][3];
    }
  }
  tc::named_bar(1, 128);
#pragma unroll
  for (int m = 0; m < 3; ++m) {
    const int id = ptid + 128 * m, bi = id >> 6, r = (id >> 2) & 15, cs = id & 3;
    const int i = blk_i(bi), k = blk_k(bi, i);
    *reinterpret_cast<float4*>(&blk(sT, i, k)[r * BLD + 4 * cs]) =
        make_float4(r4[m][0], r4[m][1], r4[m][2], r4[m][3]);
  }
  tc::named_bar(1, 128);
}

__device__ __forceinline__ bool vote_abort(uint32_t id, uint32_t n, volatile int* abort) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %3, 0;\n\t"
      "bar.red.or.pred q, %1, %2, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}\n"
      : "=r"(r)
      : "r"(id), "r"(n), "r"((uint32_t)(*abort != 0))
      : "memory");
  return r != 0;
}

template <typename Tout>
__device__ __forceinline__ void store16(Tout* dst, const float (&v)[16]);
template <>
__device__ __forceinline__ void store16<__nv_bfloat16>(__nv_bfloat16* dst, const float (&v)[16]) {
  uint4 a, b;
  a.x = tc::pack_bf16(v[0], v[1]);   a.y = tc::pack_bf16(v[2], v[3]);
  a.z = tc::pack_bf16(v[4], v[5]);   a.w = tc::pack_bf16(v[6], v[7]);
  b.x = tc::pack_bf16(v[8], v[9]);   b.y = tc::pack_bf16(v[10], v[11]);
  b.z = tc::pack_bf16(v[12], v[13]); b.w = tc::pack_bf16(v[14], v[15]);
  reinterpret_cast<uint4*>(dst)[0] = a;
  reinterpret_cast<uint4*>(dst)[1] = b;
}
template <>
__device__ __forceinline__ void store16<float>(float* dst, const float (&v)[16]) {
#pragma unroll
  for (int i = 0; i < 4; ++i)
    reinterpret_cast<float4*>(dst)[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// Four fp32 values rounded to tf32, stored as one 16-byte chunk.
__device__ __forceinline__ void st_tf32x4(uint32_t addr, float a, float b, float c, float d) {
  tc::st_shared_v4(addr, tc::to_tf32(a), tc::to_tf32(b), tc::to_tf32(c), tc::to_tf32(d));
}

// ------------------------------------------------------------------------------------------
// the kernel
// ------------------------------------------------------------------------------------------
template <typename Tout>
__global__ void __launch_bounds__(kThreads, 1)
chunk_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                    const __grid_constant__ CUtensorMap tmv, const float* __restrict__ log_alpha,
                    const float* __restrict__ beta, const float* __restrict__ S0,
                    Tout* __restrict__ o, float* __restrict__ S_T, int T, int Hk, int Hv,
                    float scale) {
  // Offsetting the __shared__ array itself (not a round trip through an integer) keeps every
  // access below a shared-memory access (ld/st.shared), not a generic one.
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sb = tc::smem_u32(smem);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.x % Hv;
  const int bq = blockIdx.x / Hv;
  const int hk = h / (Hv / Hk);
  const int nC = (T + C - 1) / C;
  auto bar = [&](int i) -> uint32_t { return sb + OFF_BAR + 8u * i; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(bar(B_QK_FULL + s), 1);
      tc::mbar_init(bar(B_IN_EMPTY + s), 5);
    }
    tc::mbar_init(bar(B_S_FULL), 1);
    tc::mbar_init(bar(B_S_EMPTY), 1);
    tc::mbar_init(bar(B_PT_READY), 1);
    tc::mbar_init(bar(B_PT_FULL), 1);
    tc::mbar_init(bar(B_PT_EMPTY), 1);
    tc::mbar_init(bar(B_PRE_FULL), 1);
    tc::mbar_init(bar(B_A2_EMPTY), 2);
    for (int i = 0; i < 3; ++i) tc::mbar_init(bar(B_GATE + i), 1);
    for (int hh = 0; hh < 2; ++hh) {
      const int hb = B_HALF + H_COUNT * hh;
      tc::mbar_init(bar(hb + H_X_FULL), 1);
      tc::mbar_init(bar(hb + H_X_EMPTY), 2);
      tc::mbar_init(bar(hb + H_R_FULL), 1);
      tc::mbar_init(bar(hb + H_Y_FULL), 1);
      tc::mbar_init(bar(hb + H_Y_EMPTY), 2);
      tc::mbar_init(bar(hb + H_D_FULL), 1);
      tc::mbar_init(bar(hb + H_D3_FULL), 1);
      tc::mbar_init(bar(hb + H_D3_EMPTY), 1);
      tc::mbar_init(bar(hb + H_M_READY), 1);
      tc::mbar_init(bar(hb + H_V_FULL), 1);
      tc::mbar_init(bar(hb + H_V_EMPTY), 1);
    }
    for (int i = 0; i < 3; ++i) tc::mbar_init(bar(B_DRAIN + i), 1);
    *abort_flag = 0;
    tc::fence_barrier_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(sb + OFF_MISC, 512);
    tc::tmem_relinquish();
    tc::tc_fence_before();
  }
  if (warp == 0 && lane == 0) {
    tc::tma_prefetch_desc(&tmq);
    tc::tma_prefetch_desc(&tmk);
    tc::tma_prefetch_desc(&tmv);
  }
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + OFF_MISC);

  if (warp == 0) {
    // ------------------------------- TMA producer -------------------------------------------
    if (lane == 0) {
      int armed_qk[2] = {-1, -1}, armed_v[2] = {-1, -1};
      bool ok = true;
      for (int c = 0; c < nC && ok; ++c) {
        const int s = c & 1, t0 = c * C;
        if (c >= 2) ok = tc::mbar_wait(bar(B_IN_EMPTY + s), ((c >> 1) - 1) & 1, abort_flag, kBudgetNs);
        if (!ok) break;
        const uint32_t dst = sb + OFF_QK + s * QK_STAGE;
        tc::mbar_arrive_expect_tx(bar(B_QK_FULL + s), 32768);
        tc::tma_load_4d(dst, &tmq, bar(B_QK_FULL + s), 0, hk, t0, bq);
        tc::tma_load_4d(dst + 8192, &tmk, bar(B_QK_FULL + s), 0, hk, t0, bq);
        tc::tma_load_4d(dst + 16384, &tmq, bar(B_QK_FULL + s), 64, hk, t0, bq);
        tc::tma_load_4d(dst + 24576, &tmk, bar(B_QK_FULL + s), 64, hk, t0, bq);
        armed_qk[s] = c;
        for (int hh = 0; hh < 2 && ok; ++hh) {
          const int hb = B_HALF + H_COUNT * hh;
          if (c >= 1) ok = tc::mbar_wait(bar(hb + H_V_EMPTY), (c - 1) & 1, abort_flag, kBudgetNs);
          if (!ok) break;
          tc::mbar_arrive_expect_tx(bar(hb + H_V_FULL), 8192);
          tc::tma_load_4d(sb + OFF_V + hh * 8192, &tmv, bar(hb + H_V_FULL), 64 * hh, h, t0, bq);
          armed_v[hh] = c;
        }
      }
      if (!ok) {   // let every load already issued land before the CTA can leave
        volatile int never = 0;
        for (int s = 0; s < 2; ++s)
          if (armed_qk[s] >= 0)
            tc::mbar_wait(bar(B_QK_FULL + s), (armed_qk[s] >> 1) & 1, &never, kBudgetNs / 4);
        for (int hh = 0; hh < 2; ++hh)
          if (armed_v[hh] >= 0)
            tc::mbar_wait(bar(B_HALF + H_COUNT * hh + H_V_FULL), armed_v[hh] & 1, &never,
                          kBudgetNs / 4);
      }
    }
  } else if (warp == 1) {
    // -------------------- state-independent MMAs: S = [Q;K] K^T and P T_b --------------------
    if (lane == 0) {
      auto issue_S = [&](int c) -> bool {
        const int s = c & 1;
        if (!tc::mbar_wait(bar(B_QK_FULL + s), (c >> 1) & 1, abort_flag, kBudgetNs)) return false;
        if (c >= 1 && !tc::mbar_wait(bar(B_S_EMPTY), (c - 1) & 1, abort_flag, kBudgetNs))
          return false;
        tc::tc_fence_after();
        const uint32_t qk = sb + OFF_QK + s * QK_STAGE;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
          tc::mma_bf16(tmem + TM_S, tc::sdesc_sw128(qk + off, 16, 1024),
                       tc::sdesc_sw128(qk + off + 8192, 16, 1024), ID_S, ks > 0);
        }
        tc::mma_commit(bar(B_S_FULL));
        tc::mma_commit(bar(B_IN_EMPTY + s));
        return true;
      };
      bool ok = issue_S(0);
      for (int c = 0; c < nC && ok; ++c) {
        ok = tc::mbar_wait(bar(B_PT_READY), c & 1, abort_flag, kBudgetNs) &&
             (c == 0 || tc::mbar_wait(bar(B_PT_EMPTY), (c - 1) & 1, abort_flag, kBudgetNs));
        if (!ok) break;
        tc::tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)   // P (64 x 64, K-major) x T_b (64 x 64, MN-major), tf32
          tc::mma_tf32(tmem + TM_PT,
                       tc::sdesc_sw128(sb + OFF_W + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024),
                       tc::sdesc_sw128_b32(sb + OFF_WT + ks * 1024, 8192), ID_PT, ks > 0);
        tc::mma_commit(bar(B_PT_FULL));
        if (c + 1 < nC) ok = issue_S(c + 1);
      }
      tc::mma_commit(bar(B_DRAIN + 0));
      volatile int never = 0;
      tc::mbar_wait(bar(B_DRAIN + 0), 0, &never, kBudgetNs / 4);
    }
  } else if (warp == 2 || warp == 3) {
    // -------------------------- chain MMAs of one state half ---------------------------------
    if (lane == 0) {
      const int hh = warp - 2, hb = B_HALF + H_COUNT * hh;
      const uint32_t mb = sb + OFF_MB + hh * 16384, rd = sb + OFF_RD + hh * 16384;
      bool ok = true;
      for (int c = 0; c < nC && ok; ++c) {
        const int s = c & 1;
        const uint32_t qk = sb + OFF_QK + s * QK_STAGE;
        // X = [Q; K] M_half                                                      (bf16)
        ok = tc::mbar_wait(bar(B_QK_FULL + s), (c >> 1) & 1, abort_flag, kBudgetNs) &&
             tc::mbar_wait(bar(hb + H_M_READY), c & 1, abort_flag, kBudgetNs) &&
             (c == 0 || tc::mbar_wait(bar(hb + H_X_EMPTY), (c - 1) & 1, abort_flag, kBudgetNs));
        if (!ok) break;
        tc::tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          tc::mma_bf16(tmem + TM_X + 64 * hh,
                       tc::sdesc_sw128(qk + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024),
                       tc::sdesc_sw128(mb + ks * 2048, 16384, 1024), ID_X, ks > 0);
        tc::mma_commit(bar(hb + H_X_FULL));
        tc::mma_commit(bar(B_IN_EMPTY + s));
        GDN_TRACE(c, 10 + 4 * hh);
        // Y = A2 R'                                                              (tf32)
        ok = tc::mbar_wait(bar(hb + H_R_FULL), c & 1, abort_flag, kBudgetNs) &&
             tc::mbar_wait(bar(B_PRE_FULL), c & 1, abort_flag, kBudgetNs) &&
             (c == 0 || tc::mbar_wait(bar(hb + H_Y_EMPTY), (c - 1) & 1, abort_flag, kBudgetNs));
        if (!ok) break;
        tc::tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          tc::mma_tf32(tmem + TM_Y + 64 * hh,
                       tc::sdesc_sw128(sb + OFF_A2 + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024),
                       tc::sdesc_sw128_b32(rd + ks * 1024, 8192), ID_Y, ks > 0);
        tc::mma_commit(bar(hb + H_Y_FULL));
        tc::mma_commit(bar(B_A2_EMPTY));
        GDN_TRACE(c, 11 + 4 * hh);
        // D3 = K^T (ktil Delta)_hi + K^T (ktil Delta)_lo                         (bf16)
        ok = tc::mbar_wait(bar(hb + H_D_FULL), c & 1, abort_flag, kBudgetNs) &&
             (c == 0 || tc::mbar_wait(bar(hb + H_D3_EMPTY), (c - 1) & 1, abort_flag, kBudgetNs));
        if (!ok) break;
        tc::tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          tc::mma_bf16(tmem + TM_D3 + 64 * hh,
                       tc::sdesc_sw128(qk + 8192 + (ks & 3) * 2048, 16384, 1024),
                       tc::sdesc_sw128(rd + (ks >> 2) * 8192 + (ks & 3) * 2048, 8192, 1024), ID_U,
                       ks > 0);
        tc::mma_commit(bar(hb + H_D3_FULL));
        tc::mma_commit(bar(B_IN_EMPTY + s));
        GDN_TRACE(c, 12 + 4 * hh);
      }
      tc::mma_commit(bar(B_DRAIN + 1 + hh));
      volatile int never = 0;
      tc::mbar_wait(bar(B_DRAIN + 1 + hh), 0, &never, kBudgetNs / 4);
    }
  } else if (warp < 8) {
    // ------------------------------- pre warpgroup -------------------------------------------
    const int ptid = threadIdx.x - 128;                 // = TMEM lane of this thread
    const int q = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(32 * q) << 16;
    float* sA = reinterpret_cast<float*>(smem + OFF_W);
    float* sT = reinterpret_cast<float*>(smem + OFF_W + SOLVE_T);
    float pla0 = 0.f, pla1 = 0.f, pbe0 = 0.f, pbe1 = 0.f;   // gates of the next chunk (warp 4)
    auto load_gates = [&](int c) {
      const long ta = (long)c * C + 2 * lane, tb = ta + 1;
      pla0 = pla1 = pbe0 = pbe1 = 0.f;
      if (ta < T) { pla0 = log_alpha[((long)bq * T + ta) * Hv + h]; pbe0 = beta[((long)bq * T + ta) * Hv + h]; }
      if (tb < T) { pla1 = log_alpha[((long)bq * T + tb) * Hv + h]; pbe1 = beta[((long)bq * T + tb) * Hv + h]; }
    };
    if (ptid < 32) load_gates(0);
    for (int c = 0; c < nC; ++c) {
      const int slot = c % 3;
      if (ptid == 0) GDN_TRACE(c, 0);
      float* gG = reinterpret_cast<float*>(smem + OFF_GB + slot * GB_SLOT);
      float* gGam = gG + 64;
      float* gKt = gG + 128;
      float* gBeta = gG + 192;
      float* gE = gG + 256;
      if (ptid < 32) {          // gates of this chunk: lane l holds tokens 2l, 2l+1
        const float la0 = pla0, la1 = pla1, be0 = pbe0, be1 = pbe1;
        if (c + 1 < nC) load_gates(c + 1);
        float incl = la0 + la1;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
          const float n = __shfl_up_sync(0xffffffffu, incl, d);
          if (lane >= d) incl += n;
        }
        const float g1 = incl, g0 = incl - la1;
        const float gl = __shfl_sync(0xffffffffu, incl, 31);
        constexpr float kLog2e = 1.4426950408889634f;
        gG[2 * lane] = g0 * kLog2e;    gG[2 * lane + 1] = g1 * kLog2e;
        gGam[2 * lane] = expf(g0);     gGam[2 * lane + 1] = expf(g1);
        gKt[2 * lane] = expf(gl - g0); gKt[2 * lane + 1] = expf(gl - g1);
        gBeta[2 * lane] = be0;         gBeta[2 * lane + 1] = be1;
        // block factors E[b][j] = exp(G_16b - G_j) for j < 16b (each <= 1: G never increases)
#pragma unroll
        for (int b = 1; b < 4; ++b) {
          const float gb = __shfl_sync(0xffffffffu, g0, 8 * b) * kLog2e;   // G at token 16b
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int j = 2 * lane + e;
            const float gj = (e ? g1 : g0) * kLog2e;
            gE[64 * b + j] = (j < 16 * b) ? tc::ex2(gb - gj) : 0.f;
          }
        }
        __syncwarp();
        __threadfence_block();
        if (lane == 0) tc::mbar_arrive(bar(B_GATE + slot));
      }
      tc::named_bar(1, 128);
      if (ptid == 0) GDN_TRACE(c, 1);
      // Rows of S: threads 0..63 hold (q_t . k_j), threads 64..127 hold (k_t . k_j).  Both
      // halves turn their row into P or A at once; exp(G_t - G_j) = 2^(G'_t - G'_j), G' = G log2 e.
      //   P[t][j] = exp(G_t - G_j) (q_t . k_j) scale, j <= t  (kept in the same TMEM row, as fp32,
      //             until the solve scratch is free for the tf32 copy)
      //   A[t][j] = beta_t exp(G_t - G_j) (k_t . k_j),  j < t  (into the packed solve blocks)
      tc::mbar_wait(bar(B_S_FULL), c & 1, abort_flag, kBudgetNs);
      if (ptid == 0) GDN_TRACE(c, 2);
      tc::tc_fence_after();
      {
        const bool is_p = ptid < 64;
        const int t = is_p ? ptid : ptid - 64, ti = t >> 4, tr = t & 15;
        const float gt = gG[t];
        const float coef = is_p ? scale : gBeta[t];
        // exp(G_t - G_j): inside t's 16-token block directly; across blocks as
        // exp(G_t - G_16ti) * E[ti][j] (both factors <= 1)
        const float et = tc::ex2(gt - gG[16 * ti]);
        const float4* g4 = reinterpret_cast<const float4*>(gG);
        const float4* e4p = reinterpret_cast<const float4*>(gE + 64 * ti);
        const int lim = is_p ? t + 1 : t;            // column j is kept when j < lim
#pragma unroll
        for (int p = 0; p < 2; ++p) {
          float sv[32];
          tc::tmem_ld32(tmem + lane_off + TM_S + 32 * p, sv);
          tc::tmem_wait_ld();
          if (ptid == 64 + 48) GDN_TRACE(c, 53 + 2 * p);
#pragma unroll
          for (int kb2 = 0; kb2 < 2; ++kb2) {
            const int kb = 2 * p + kb2;
            float* v = sv + 16 * kb2;
            if (kb < ti) {
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const float4 e = e4p[4 * kb + i];
                v[4 * i] *= coef * et * e.x;     v[4 * i + 1] *= coef * et * e.y;
                v[4 * i + 2] *= coef * et * e.z; v[4 * i + 3] *= coef * et * e.w;
              }
            } else if (kb == ti) {
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const float4 g = g4[4 * kb + i];
                const float gj[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const int j = 16 * kb + 4 * i + e;
                  v[4 * i + e] = (j < lim) ? coef * tc::ex2(gt - gj[e]) * v[4 * i + e] : 0.f;
                }
              }
            } else {
#pragma unroll
              for (int e = 0; e < 16; ++e) v[e] = 0.f;
            }
          }
          if (is_p) {
            tc::tmem_st32(tmem + lane_off + TM_S + 32 * p, sv);
          } else {
#pragma unroll
            for (int kb2 = 0; kb2 < 2; ++kb2) {
              const int kb = 2 * p + kb2;
              if (kb <= ti) {
                float* dst = blk(sA, ti, kb) + tr * BLD;
#pragma unroll
                for (int e4 = 0; e4 < 16; e4 += 4)
                  *reinterpret_cast<float4*>(dst + e4) =
                      make_float4(sv[16 * kb2 + e4], sv[16 * kb2 + e4 + 1], sv[16 * kb2 + e4 + 2],
                                  sv[16 * kb2 + e4 + 3]);
              }
            }
          }
          if (ptid == 64 + 48) GDN_TRACE(c, 54 + 2 * p);
        }
        if (is_p) tc::tmem_wait_st();
        if (ptid == 48) GDN_TRACE(c, 57);
      }
      tc::tc_fence_before();
      tc::named_bar(1, 128);
      if (ptid == 0) GDN_TRACE(c, 3);
      solve_unit_lower(sA, sT, ptid, c, nC);
      if (ptid == 0) GDN_TRACE(c, 4);
      // T_b = T diag(beta): row k = ptid/2, columns n0..n0+31 (one tf32 column block)
      float tb[32];
      const int kr = ptid >> 1, nb = ptid & 1;
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const int n = 32 * nb + e;
        tb[e] = (n <= kr) ? blk(sT, kr >> 4, n >> 4)[(kr & 15) * BLD + (n & 15)] * gBeta[n] : 0.f;
      }
      if (ptid == 0) GDN_TRACE(c, 48);
      if (c >= 1) tc::mbar_wait(bar(B_A2_EMPTY), (c - 1) & 1, abort_flag, kBudgetNs);
      if (ptid == 0) GDN_TRACE(c, 49);
      tc::named_bar(1, 128);                     // the solve scratch is free from here on
      if (ptid == 0) GDN_TRACE(c, 50);
      {
        // T_b as the MN-major B operand of P T_b (32-byte chunks), and as rows 64..127 of the
        // K-major A2 (16-byte chunks)
        const uint32_t tb_base = sb + OFF_WT + nb * 8192;
        const uint32_t a2_row = sb + OFF_A2 + nb * 16384 + (64 + kr) * 128;
#pragma unroll
        for (int c32 = 0; c32 < 4; ++c32) {
          const uint32_t a = tb_base + tc::sw128_b32(kr, c32);
          st_tf32x4(a, tb[8 * c32], tb[8 * c32 + 1], tb[8 * c32 + 2], tb[8 * c32 + 3]);
          st_tf32x4(a + 16, tb[8 * c32 + 4], tb[8 * c32 + 5], tb[8 * c32 + 6], tb[8 * c32 + 7]);
        }
#pragma unroll
        for (int cc = 0; cc < 8; ++cc)
          st_tf32x4(a2_row + ((cc ^ (kr & 7)) << 4), tb[4 * cc], tb[4 * cc + 1], tb[4 * cc + 2],
                    tb[4 * cc + 3]);
      }
      if (ptid == 0) GDN_TRACE(c, 51);
      // P rows (threads 0..63, warps 4 and 5): back from TMEM, rounded to tf32, into the K-major
      // A operand of P T_b
      if (ptid < 64) {
        const int t = ptid;
#pragma unroll
        for (int p = 0; p < 2; ++p) {
          float pv[32];
          tc::tmem_ld32(tmem + lane_off + TM_S + 32 * p, pv);
          tc::tmem_wait_ld();
          const uint32_t prow = sb + OFF_W + p * 8192 + t * 128;
#pragma unroll
          for (int cc = 0; cc < 8; ++cc)
            st_tf32x4(prow + ((cc ^ (t & 7)) << 4), pv[4 * cc], pv[4 * cc + 1], pv[4 * cc + 2],
                      pv[4 * cc + 3]);
        }
      }
      if (ptid == 0) GDN_TRACE(c, 52);
      tc::tc_fence_before();
      tc::fence_proxy_async_smem();
      tc::named_bar(1, 128);
      if (ptid == 0) {
        tc::mbar_arrive(bar(B_S_EMPTY));
        tc::mbar_arrive(bar(B_PT_READY));
        GDN_TRACE(c, 6);
      }
      // A2 rows 0..63 = P T_b (64-row MMA: row r sits in lane (r % 16) + 32 (r / 16))
      tc::mbar_wait(bar(B_PT_FULL), c & 1, abort_flag, kBudgetNs);
      if (ptid == 0) GDN_TRACE(c, 7);
      tc::tc_fence_after();
      {
        float pv[32];
        const int r = 16 * q + lane;
#pragma unroll
        for (int p = 0; p < 2; ++p) {
          tc::tmem_ld32(tmem + lane_off + TM_PT + 32 * p, pv);
          tc::tmem_wait_ld();
          if (lane < 16) {
            const uint32_t a2_row = sb + OFF_A2 + p * 16384 + r * 128;
#pragma unroll
            for (int cc = 0; cc < 8; ++cc)
              st_tf32x4(a2_row + ((cc ^ (r & 7)) << 4), pv[4 * cc], pv[4 * cc + 1], pv[4 * cc + 2],
                        pv[4 * cc + 3]);
          }
        }
      }
      tc::tc_fence_before();
      tc::fence_proxy_async_smem();
      const bool stop = vote_abort(1, 128, abort_flag);
      if (ptid == 0) {
        tc::mbar_arrive(bar(B_PRE_FULL));
        tc::mbar_arrive(bar(B_PT_EMPTY));
        GDN_TRACE(c, 8);
      }
      if (stop) break;
    }
  } else {
    // ------------------------------- chain warpgroups ----------------------------------------
    const int hh = (warp - 8) >> 2, q = warp & 3, r = 32 * q + lane;
    const int hb = B_HALF + H_COUNT * hh;
    const uint32_t lane_off = static_cast<uint32_t>(32 * q) << 16;
    const uint32_t mb = sb + OFF_MB + hh * 16384, rd = sb + OFF_RD + hh * 16384;
    const uint32_t vb = sb + OFF_V + hh * 8192;
    const uint32_t id_wg = 2 + 3 * hh, id_lo = 3 + 3 * hh, id_hi = 4 + 3 * hh;
    const long head = (long)bq * Hv + h;
    float M[64];
    if (S0) {
      const float4* src = reinterpret_cast<const float4*>(S0 + (head * 128 + r) * 128 + 64 * hh);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float4 v = src[i];
        M[4 * i] = v.x; M[4 * i + 1] = v.y; M[4 * i + 2] = v.z; M[4 * i + 3] = v.w;
      }
    } else {
#pragma unroll
      for (int i = 0; i < 64; ++i) M[i] = 0.f;
    }
#pragma unroll
    for (int cc = 0; cc < 8; ++cc)
      tc::st_shared_v4(mb + tc::sw128(r, cc), tc::pack_bf16(M[8 * cc], M[8 * cc + 1]),
                       tc::pack_bf16(M[8 * cc + 2], M[8 * cc + 3]),
                       tc::pack_bf16(M[8 * cc + 4], M[8 * cc + 5]),
                       tc::pack_bf16(M[8 * cc + 6], M[8 * cc + 7]));
    tc::fence_proxy_async_smem();
    tc::named_bar(id_wg, 128);
    if (q == 0 && lane == 0) tc::mbar_arrive(bar(hb + H_M_READY));

    for (int c = 0; c < nC; ++c) {
      const int slot = c % 3;
      const long t0 = (long)c * C;
      const float* gGam = reinterpret_cast<const float*>(smem + OFF_GB + slot * GB_SLOT) + 64;
      const float* gKt = gGam + 64;
      if (q >= 2) {
        // R' = V - gamma (K M) for token t (tf32), then ktil Delta as bf16 hi + lo
        const int t = r - 64;
        tc::mbar_wait(bar(hb + H_X_FULL), c & 1, abort_flag, kBudgetNs);
        tc::mbar_wait(bar(B_GATE + slot), (c / 3) & 1, abort_flag, kBudgetNs);
        tc::mbar_wait(bar(hb + H_V_FULL), c & 1, abort_flag, kBudgetNs);
        if (q == 2 && lane == 0) GDN_TRACE(c, 20 + 10 * hh);
        tc::tc_fence_after();
        const float g = gGam[t];
#pragma unroll
        for (int p = 0; p < 4; ++p) {          // 16 columns: dv 16p .. 16p+15 of this half
          float x[16];
          tmem_ld16(tmem + lane_off + TM_X + 64 * hh + 16 * p, x);
          tc::tmem_wait_ld();
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            const int cc = 2 * p + half;       // bf16 chunk of V (8 values)
            const uint4 u = tc::ld_shared_v4(vb + tc::sw128(t, cc));
            const float* xx = x + 8 * half;
            const float rv[8] = {tc::bf16lo(u.x) - g * xx[0], tc::bf16hi(u.x) - g * xx[1],
                                 tc::bf16lo(u.y) - g * xx[2], tc::bf16hi(u.y) - g * xx[3],
                                 tc::bf16lo(u.z) - g * xx[4], tc::bf16hi(u.z) - g * xx[5],
                                 tc::bf16lo(u.w) - g * xx[6], tc::bf16hi(u.w) - g * xx[7]};
            // MN-major tf32 layout: dv block nb = col / 32, 32-byte chunk (col % 32) / 8
            const int col = 8 * cc, nb = col >> 5, c32 = (col & 31) >> 3;
            const uint32_t a = rd + nb * 8192 + tc::sw128_b32(t, c32);
            st_tf32x4(a, rv[0], rv[1], rv[2], rv[3]);
            st_tf32x4(a + 16, rv[4], rv[5], rv[6], rv[7]);
          }
        }
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        tc::named_bar(id_hi, 64);
        if (q == 2 && lane == 0) {
          GDN_TRACE(c, 21 + 10 * hh);
          tc::mbar_arrive(bar(hb + H_R_FULL));
          tc::mbar_arrive(bar(hb + H_V_EMPTY));
          tc::mbar_arrive(bar(hb + H_X_EMPTY));
        }
        tc::mbar_wait(bar(hb + H_Y_FULL), c & 1, abort_flag, kBudgetNs);
        if (q == 2 && lane == 0) GDN_TRACE(c, 22 + 10 * hh);
        tc::tc_fence_after();
        const float kt = gKt[t];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          float y[16];
          tmem_ld16(tmem + lane_off + TM_Y + 64 * hh + 16 * p, y);
          tc::tmem_wait_ld();
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            float hi[8], lo[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) tc::split_bf16(kt * y[8 * half + e], hi[e], lo[e]);
            const uint32_t sw = tc::sw128(t, 2 * p + half);
            tc::st_shared_v4(rd + sw, tc::pack_bf16(hi[0], hi[1]), tc::pack_bf16(hi[2], hi[3]),
                             tc::pack_bf16(hi[4], hi[5]), tc::pack_bf16(hi[6], hi[7]));
            tc::st_shared_v4(rd + 8192 + sw, tc::pack_bf16(lo[0], lo[1]), tc::pack_bf16(lo[2], lo[3]),
                             tc::pack_bf16(lo[4], lo[5]), tc::pack_bf16(lo[6], lo[7]));
          }
        }
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        tc::named_bar(id_hi, 64);
        if (q == 2 && lane == 0) {
          GDN_TRACE(c, 23 + 10 * hh);
          tc::mbar_arrive(bar(hb + H_D_FULL));
          tc::mbar_arrive(bar(hb + H_Y_EMPTY));
        }
      } else {
        // o_t = gamma_t scale (Q M)_t + (P Delta)_t
        const int t = r;
        tc::mbar_wait(bar(hb + H_X_FULL), c & 1, abort_flag, kBudgetNs);
        tc::mbar_wait(bar(B_GATE + slot), (c / 3) & 1, abort_flag, kBudgetNs);
        tc::mbar_wait(bar(hb + H_Y_FULL), c & 1, abort_flag, kBudgetNs);
        if (q == 0 && lane == 0) GDN_TRACE(c, 24 + 10 * hh);
        tc::tc_fence_after();
        const float g = gGam[t] * scale;
        const bool valid = t0 + t < T;
        Tout* orow = o + (((long)bq * T + t0 + t) * Hv + h) * 128 + 64 * hh;
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          float x[16], y[16];
          tmem_ld16(tmem + lane_off + TM_X + 64 * hh + 16 * p, x);
          tmem_ld16(tmem + lane_off + TM_Y + 64 * hh + 16 * p, y);
          tc::tmem_wait_ld();
          if (p == 0 && hh == 0 && q == 0 && lane == 0) GDN_TRACE(c, 58);
#pragma unroll
          for (int i = 0; i < 16; ++i) y[i] = fmaf(g, x[i], y[i]);
          if (valid) store16<Tout>(orow + 16 * p, y);
          if (p == 0 && hh == 0 && q == 0 && lane == 0) GDN_TRACE(c, 59);
        }
        if (hh == 0 && q == 0 && lane == 0) GDN_TRACE(c, 60);
        tc::tc_fence_before();
        tc::named_bar(id_lo, 64);
        if (q == 0 && lane == 0) {
          GDN_TRACE(c, 25 + 10 * hh);
          tc::mbar_arrive(bar(hb + H_X_EMPTY));
          tc::mbar_arrive(bar(hb + H_Y_EMPTY));
        }
      }
      // M <- gamma_last M + K^T (ktil Delta)  (row r of this half), and its bf16 copy
      tc::mbar_wait(bar(hb + H_D3_FULL), c & 1, abort_flag, kBudgetNs);
      if (q == 0 && lane == 0) GDN_TRACE(c, 26 + 10 * hh);
      tc::tc_fence_after();
      const float gl = gGam[63];
#pragma unroll
      for (int p = 0; p < 4; ++p) {
        float d[16];
        tmem_ld16(tmem + lane_off + TM_D3 + 64 * hh + 16 * p, d);
        tc::tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) M[16 * p + i] = fmaf(gl, M[16 * p + i], d[i]);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const float* mm = M + 16 * p + 8 * half;
          tc::st_shared_v4(mb + tc::sw128(r, 2 * p + half), tc::pack_bf16(mm[0], mm[1]),
                           tc::pack_bf16(mm[2], mm[3]), tc::pack_bf16(mm[4], mm[5]),
                           tc::pack_bf16(mm[6], mm[7]));
        }
      }
      tc::fence_proxy_async_smem();
      tc::tc_fence_before();
      const bool stop = vote_abort(id_wg, 128, abort_flag);
      if (q == 0 && lane == 0) {
        GDN_TRACE(c, 27 + 10 * hh);
        tc::mbar_arrive(bar(hb + H_D3_EMPTY));
        tc::mbar_arrive(bar(hb + H_M_READY));
      }
      if (stop) break;
    }
    if (S_T && !*abort_flag) {
      float4* dst = reinterpret_cast<float4*>(S_T + (head * 128 + r) * 128 + 64 * hh);
#pragma unroll
      for (int i = 0; i < 16; ++i)
        dst[i] = make_float4(M[4 * i], M[4 * i + 1], M[4 * i + 2], M[4 * i + 3]);
    }
  }

  tc::tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) record_error(kErrTimeout);
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------------------------------
// host side
// ------------------------------------------------------------------------------------------
inline PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult qr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) ==
            cudaSuccess &&
        qr == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// [B, T, H, 128] bf16 tensor, boxes of 64 (head dim) x 64 tokens, 128-byte swizzle, zero fill
// past T (the ragged last chunk reads zeros).
inline bool make_tile_map(CUtensorMap* m, const void* base, int H, int T, int B) {
  auto enc = encode_fn();
  if (!enc) return false;
  cuuint64_t dims[4] = {128, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
  cuuint64_t strides[3] = {256, (cuuint64_t)H * 256, (cuuint64_t)T * H * 256};
  cuuint32_t box[4] = {64, 1, 64, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename Tout>
gdn_status launch(const void* q, const void* k, const void* v, const float* la, const float* be,
                  const float* S0, Tout* o, float* S_T, int B, int T, int Hk, int Hv, float scale,
                  cudaStream_t st) {
  CUtensorMap mq, mk, mv;
  if (!make_tile_map(&mq, q, Hk, T, B) || !make_tile_map(&mk, k, Hk, T, B) ||
      !make_tile_map(&mv, v, Hv, T, B))
    return GDN_ERR_CUDA;
  auto kern = chunk_fwd_tc_kernel<Tout>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_ALLOC) !=
      cudaSuccess)
    return GDN_ERR_CUDA;
  const long grid = (long)B * Hv;
  if (grid > 0x7fffffffL) return GDN_ERR_UNSUPPORTED;
  kern<<<(unsigned)grid, kThreads, SMEM_ALLOC, st>>>(mq, mk, mv, la, be, S0, o, S_T, T, Hk, Hv,
                                                     scale);
  return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

}  // namespace tcf

#ifdef GDN_TC_TRACE
extern "C" GDN_API void gdn_debug_set_trace(void* p) {
  cudaMemcpyToSymbol(tcf::g_tc_trace, &p, sizeof(p));
}
#endif

inline bool tc_chunk_supported(int dk, int dv, int chunk, bool bf16) {
  return bf16 && dk == 128 && dv == 128 && chunk == tcf::C;
}

inline gdn_status tc_chunk_launch(const void* q, const void* k, const void* v, const float* la,
                                  const float* be, const float* S0, void* o, float* S_T, int B,
                                  int T, int Hk, int Hv, float scale, cudaStream_t st) {
  return tcf::launch<__nv_bfloat16>(q, k, v, la, be, S0, static_cast<__nv_bfloat16*>(o), S_T, B,
                                    T, Hk, Hv, scale, st);
}

inline gdn_status tc_chunk_launch_f32out(const void* q, const void* k, const void* v,
                                         const float* la, const float* be, const float* S0,
                                         float* o, float* S_T, int B, int T, int Hk, int Hv,
                                         float scale, cudaStream_t st) {
  return tcf::launch<float>(q, k, v, la, be, S0, o, S_T, B, T, Hk, Hv, scale, st);
}

}  // namespace gdn
