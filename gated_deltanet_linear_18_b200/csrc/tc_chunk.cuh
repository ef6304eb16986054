// Chunked forward of the gated delta rule on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
// Shapes: d_k = d_v = 128, chunk C = 64, bf16 q/k/v, fp32 gates and state.
//
// Per value head and chunk, with the chunk-start state M = S^T (128 x 128, fp32) the chunk form of
// the recurrence ("Chapitre 16 - Assembler un système de type Kimi K3", 16.2: matrix operations
// inside each block, state handed from block to block) is computed as
//   state-independent part (one per chunk, shared by both halves of the state):
//     G = cumsum(log alpha), gamma = exp(G), S = [Q; K] K^T               (MMA, 128 x 64 x 128)
//     P = lower_incl(exp(G_i - G_j) q_i.k_j) * scale,  A = strict_lower(beta_i exp(G_i - G_j) k_i.k_j)
//     T = (I + A)^-1 (fp32, blocked by 16), T_b = T diag(beta)
//     A2 = [P T_b; T_b] = [P; I] T_b                                        (MMA, 128 x 64 x 64)
//     Ktil = diag(exp(G_last - G)) K
//   state-dependent chain, for each 64-column half of M independently:
//     X = [Q; K] M                         (MMA, 128 x 64 x 128)
//     R' = V - diag(gamma) (K M)           (rows 64..127 of X)
//     Y = A2 R' = [P Delta; Delta]         (MMA, 128 x 64 x 64), Delta = T_b (V - diag(gamma) K M)
//     o = diag(gamma) scale (Q M) + P Delta  (rows 0..63 of X and Y)
//     M <- gamma_last M + Ktil^T Delta     (MMA, 128 x 64 x 64; fp32 master copy in registers)
// which is the token recurrence reorganised exactly (Delta's rows are beta_t (v_t - alpha_t
// S_{t-1} k_t)).  MMA operands are bf16, every accumulation and the master state are fp32.
//
// One CTA per (batch, value head), 512 threads in specialised warps:
//   warp 0        TMA producer (Q, K tiles double-buffered, V single-buffered)
//   warp 1        TMEM owner; issues the state-independent MMAs (S and A2)
//   warps 2, 3    issue the chain MMAs of state half 0 / half 1
//   warps 4-7     "pre" warpgroup: gates, P / A, the triangular solve, A2 and Ktil tiles
//   warps 8-11    chain warpgroup of half 0 (dv columns 0..63); warps 12-15 of half 1
// so the state-independent work of chunk c+1 overlaps the chain of chunk c, and the two halves'
// chains interleave on the tensor pipe.  Every wait is bounded (2 s): on expiry the CTA records
// GDN's timeout bit, every role leaves its loop at the next uniform check point, in-flight TMA
// loads and MMAs are drained, TMEM is released and the kernel returns.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "tc_ptx.cuh"

namespace gdn {
namespace tcf {

constexpr int C = 64;
constexpr int kThreads = 512;
constexpr uint64_t kBudgetNs = 2000000000ull;

// shared memory map (bytes from a 1024-aligned base); every MMA tile is 128-byte swizzled
constexpr uint32_t OFF_QK = 0;          // 2 stages x 32 KB: kb0 [Q 64 rows | K 64 rows], kb1 [...]
constexpr uint32_t QK_STAGE = 32768;
constexpr uint32_t OFF_V = 65536;       // 16 KB: dv block 0 [64 rows x 128 B], dv block 1
constexpr uint32_t OFF_A2 = 81920;      // 16 KB: 128 rows x 128 B, K-major
constexpr uint32_t OFF_PI = 98304;      // 16 KB: rows 0..63 P (bf16), rows 64..127 identity
constexpr uint32_t OFF_KT = 114688;     // 16 KB: Ktil, dk block 0 [64 rows x 128 B], dk block 1
constexpr uint32_t OFF_RD = 131072;     // 2 x 8 KB: per half, R' then Delta [64 rows x 128 B]
constexpr uint32_t OFF_MB = 147456;     // 2 x 16 KB: per half, bf16 M [128 rows x 128 B]
constexpr uint32_t OFF_TB = 180224;     // 8 KB: T_b bf16 [64 rows x 128 B]
constexpr int LDA = 68;                 // fp32 row stride of the solve matrices
constexpr uint32_t OFF_SA = 188416;     // 64 x 68 fp32: A, then D A (block rows)
constexpr uint32_t OFF_ST = 205824;     // 64 x 68 fp32: T
constexpr uint32_t OFF_GB = 223232;     // 3 slots x 1 KB: G[64], gamma[64], ktil[64], beta[64]
constexpr uint32_t OFF_BAR = 226304;
constexpr int NBAR = 40;
constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;   // +0 TMEM base, +4 abort flag
constexpr uint32_t SMEM_BYTES = OFF_MISC + 16;
constexpr uint32_t SMEM_ALLOC = SMEM_BYTES + 1024;
static_assert(SMEM_ALLOC <= 232448, "shared memory budget");

// TMEM columns (512 allocated, 128 lanes x 32 bit)
constexpr uint32_t TM_S = 0, TM_PT = 64, TM_X = 128, TM_Y = 256, TM_D3 = 384;

// mbarriers
enum : int {
  B_QK_FULL = 0, B_IN_EMPTY = 2, B_V_FULL = 4, B_V_EMPTY = 5, B_S_FULL = 6, B_S_EMPTY = 7,
  B_PT_READY = 8, B_PT_FULL = 9, B_PT_EMPTY = 10, B_PRE_FULL = 11, B_A2_EMPTY = 12,
  B_KT_EMPTY = 13, B_GATE = 14, B_HALF = 17, B_DRAIN = 35
};
enum : int {
  H_X_FULL = 0, H_X_EMPTY, H_R_FULL, H_Y_FULL, H_Y_EMPTY, H_D_FULL, H_D3_FULL, H_D3_EMPTY,
  H_M_READY, H_COUNT
};
static_assert(B_HALF + 2 * H_COUNT == B_DRAIN && B_DRAIN + 3 <= NBAR, "barrier map");

constexpr uint32_t ID_S = tc::idesc_bf16(128, 64, false, false);
constexpr uint32_t ID_PT = tc::idesc_bf16(128, 64, false, true);
constexpr uint32_t ID_X = tc::idesc_bf16(128, 64, false, true);
constexpr uint32_t ID_Y = tc::idesc_bf16(128, 64, false, true);
constexpr uint32_t ID_U = tc::idesc_bf16(128, 64, true, true);

// ------------------------------------------------------------------------------------------
// pre warpgroup helpers
// ------------------------------------------------------------------------------------------

// out[0..3] += sum_k X[xr][xc + k] * Y[yr + k][yc .. yc+3] for k < 16 (fp32, shared memory).
__device__ __forceinline__ void strip16(const float* X, int xr, int xc, const float* Y, int yr,
                                        int yc, float (&acc)[4]) {
#pragma unroll
  for (int k4 = 0; k4 < 16; k4 += 4) {
    const float4 xa = *reinterpret_cast<const float4*>(&X[xr * LDA + xc + k4]);
    const float xs[4] = {xa.x, xa.y, xa.z, xa.w};
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const float4 y = *reinterpret_cast<const float4*>(&Y[(yr + k4 + kk) * LDA + yc]);
      acc[0] = fmaf(xs[kk], y.x, acc[0]);
      acc[1] = fmaf(xs[kk], y.y, acc[1]);
      acc[2] = fmaf(xs[kk], y.z, acc[2]);
      acc[3] = fmaf(xs[kk], y.w, acc[3]);
    }
  }
}

// T = (I + A)^-1 for a 64 x 64 strictly lower A, by 16 x 16 blocks (128 threads, barrier id 1):
//   D_b = (I + A_bb)^-1 (forward substitution, one column per thread);
//   At_ik = D_i A_ik;  U = (I + At)^-1 by block forward substitution (U_ii = I);  T_ik = U_ik D_k.
// (I + A = blockdiag(I + A_bb) (I + At), so T = U D.)  sA is overwritten by At.
__device__ void solve_unit_lower(float* sA, float* sT, int ptid) {
  if (ptid < 64) {
    const int ob = 16 * (ptid >> 4), c = ptid & 15;
    float x[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      float acc = (i == c) ? 1.f : 0.f;
#pragma unroll
      for (int j = 0; j < i; ++j) acc = fmaf(-sA[(ob + i) * LDA + ob + j], x[j], acc);
      x[i] = acc;
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) sT[(ob + i) * LDA + ob + c] = x[i];
  }
  tc::named_bar(1, 128);
  // At_ik = D_i A_ik for the six blocks below the diagonal
  // block index bi = 0..5 -> (i, k) = (1,0) (2,0) (2,1) (3,0) (3,1) (3,2)
  auto blk_i = [](int bi) { return bi < 1 ? 1 : (bi < 3 ? 2 : 3); };
  auto blk_k = [](int bi, int i) { return bi - i * (i - 1) / 2; };
  float r1[3][4];
#pragma unroll
  for (int m = 0; m < 3; ++m) {
    const int id = ptid + 128 * m, bi = id >> 6, r = (id >> 2) & 15, cs = id & 3;
    const int i = blk_i(bi), k = blk_k(bi, i);
    r1[m][0] = r1[m][1] = r1[m][2] = r1[m][3] = 0.f;
    strip16(sT, 16 * i + r, 16 * i, sA, 16 * i, 16 * k + 4 * cs, r1[m]);
  }
  tc::named_bar(1, 128);
#pragma unroll
  for (int m = 0; m < 3; ++m) {
    const int id = ptid + 128 * m, bi = id >> 6, r = (id >> 2) & 15, cs = id & 3;
    const int i = blk_i(bi), k = blk_k(bi, i);
    *reinterpret_cast<float4*>(&sA[(16 * i + r) * LDA + 16 * k + 4 * cs]) =
        make_float4(r1[m][0], r1[m][1], r1[m][2], r1[m][3]);
  }
  tc::named_bar(1, 128);
  // U_20 = -At_20 + At_21 At_10; U_31 = -At_31 + At_32 At_21; V_30 = -At_30 + At_31 At_10
  // (stored in T's blocks (2,0), (3,1), (3,0), which nothing reads in this round)
  for (int id = ptid; id < 192; id += 128) {
    const int bi = id >> 6, r = (id >> 2) & 15, cs = id & 3;
    const int oi = bi == 0 ? 2 : 3, ok = bi == 1 ? 1 : 0;      // output block (oi, ok)
    const int xi = oi, xk = bi == 0 ? 1 : (bi == 1 ? 2 : 1);    // X = At_(xi, xk)
    const int yi = xk, yk = ok;                                  // Y = At_(yi, yk)
    float acc[4];
    const float4 base = *reinterpret_cast<const float4*>(&sA[(16 * oi + r) * LDA + 16 * ok + 4 * cs]);
    acc[0] = -base.x; acc[1] = -base.y; acc[2] = -base.z; acc[3] = -base.w;
    strip16(sA, 16 * xi + r, 16 * xk, sA, 16 * yi, 16 * yk + 4 * cs, acc);
    *reinterpret_cast<float4*>(&sT[(16 * oi + r) * LDA + 16 * ok + 4 * cs]) =
        make_float4(acc[0], acc[1], acc[2], acc[3]);
  }
  tc::named_bar(1, 128);
  // U_30 = V_30 - At_32 U_20
  if (ptid < 64) {
    const int r = ptid >> 2, cs = ptid & 3;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    strip16(sA, 48 + r, 32, sT, 32, 4 * cs, acc);
    float4* dst = reinterpret_cast<float4*>(&sT[(48 + r) * LDA + 4 * cs]);
    const float4 v30 = *dst;
    *dst = make_float4(v30.x - acc[0], v30.y - acc[1], v30.z - acc[2], v30.w - acc[3]);
  }
  tc::named_bar(1, 128);
  // T_ik = U_ik D_k, with U_10 = -At_10, U_21 = -At_21, U_32 = -At_32
  float r4[3][4];
#pragma unroll
  for (int m = 0; m < 3; ++m) {
    const int id = ptid + 128 * m, bi = id >> 6, r = (id >> 2) & 15, cs = id & 3;
    const int i = blk_i(bi), k = blk_k(bi, i);
    const bool sub = (i == k + 1);                     // U on the first sub-diagonal is -At
    r4[m][0] = r4[m][1] = r4[m][2] = r4[m][3] = 0.f;
    strip16(sub ? sA : sT, 16 * i + r, 16 * k, sT, 16 * k, 16 * k + 4 * cs, r4[m]);
    if (sub) { r4[m][0] = -r4[m][0]; r4[m][1] = -r4[m][1]; r4[m][2] = -r4[m][2]; r4[m][3] = -r4[m][3]; }
  }
  tc::named_bar(1, 128);
#pragma unroll
  for (int m = 0; m < 3; ++m) {
    const int id = ptid + 128 * m, bi = id >> 6, r = (id >> 2) & 15, cs = id & 3;
    const int i = blk_i(bi), k = blk_k(bi, i);
    *reinterpret_cast<float4*>(&sT[(16 * i + r) * LDA + 16 * k + 4 * cs]) =
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
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
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
      tc::mbar_init(bar(B_IN_EMPTY + s), 4);
    }
    tc::mbar_init(bar(B_V_FULL), 1);
    tc::mbar_init(bar(B_V_EMPTY), 2);
    tc::mbar_init(bar(B_S_FULL), 1);
    tc::mbar_init(bar(B_S_EMPTY), 1);
    tc::mbar_init(bar(B_PT_READY), 1);
    tc::mbar_init(bar(B_PT_FULL), 1);
    tc::mbar_init(bar(B_PT_EMPTY), 1);
    tc::mbar_init(bar(B_PRE_FULL), 1);
    tc::mbar_init(bar(B_A2_EMPTY), 2);
    tc::mbar_init(bar(B_KT_EMPTY), 2);
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
      int armed_qk[2] = {-1, -1}, armed_v = -1;
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
        if (c >= 1) ok = tc::mbar_wait(bar(B_V_EMPTY), (c - 1) & 1, abort_flag, kBudgetNs);
        if (!ok) break;
        tc::mbar_arrive_expect_tx(bar(B_V_FULL), 16384);
        tc::tma_load_4d(sb + OFF_V, &tmv, bar(B_V_FULL), 0, h, t0, bq);
        tc::tma_load_4d(sb + OFF_V + 8192, &tmv, bar(B_V_FULL), 64, h, t0, bq);
        armed_v = c;
      }
      if (!ok) {   // let every load already issued land before the CTA can leave
        volatile int never = 0;
        for (int s = 0; s < 2; ++s)
          if (armed_qk[s] >= 0)
            tc::mbar_wait(bar(B_QK_FULL + s), (armed_qk[s] >> 1) & 1, &never, kBudgetNs / 4);
        if (armed_v >= 0) tc::mbar_wait(bar(B_V_FULL), armed_v & 1, &never, kBudgetNs / 4);
      }
    }
  } else if (warp == 1) {
    // -------------------- state-independent MMAs: S = [Q;K] K^T, A2 = [P; I] T_b -------------
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
        for (int ks = 0; ks < 4; ++ks)
          tc::mma_bf16(tmem + TM_PT, tc::sdesc_sw128(sb + OFF_PI + ks * 32, 16, 1024),
                       tc::sdesc_sw128(sb + OFF_TB + ks * 2048, 8192, 1024), ID_PT, ks > 0);
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
      const uint32_t mb = sb + OFF_MB + hh * 16384, rd = sb + OFF_RD + hh * 8192;
      bool ok = true;
      for (int c = 0; c < nC && ok; ++c) {
        const int s = c & 1;
        const uint32_t qk = sb + OFF_QK + s * QK_STAGE;
        // X = [Q; K] M_half
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
        // Y = A2 R'
        ok = tc::mbar_wait(bar(hb + H_R_FULL), c & 1, abort_flag, kBudgetNs) &&
             tc::mbar_wait(bar(B_PRE_FULL), c & 1, abort_flag, kBudgetNs) &&
             (c == 0 || tc::mbar_wait(bar(hb + H_Y_EMPTY), (c - 1) & 1, abort_flag, kBudgetNs));
        if (!ok) break;
        tc::tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          tc::mma_bf16(tmem + TM_Y + 64 * hh, tc::sdesc_sw128(sb + OFF_A2 + ks * 32, 16, 1024),
                       tc::sdesc_sw128(rd + ks * 2048, 8192, 1024), ID_Y, ks > 0);
        tc::mma_commit(bar(hb + H_Y_FULL));
        tc::mma_commit(bar(B_A2_EMPTY));
        // D3 = Ktil^T Delta
        ok = tc::mbar_wait(bar(hb + H_D_FULL), c & 1, abort_flag, kBudgetNs) &&
             (c == 0 || tc::mbar_wait(bar(hb + H_D3_EMPTY), (c - 1) & 1, abort_flag, kBudgetNs));
        if (!ok) break;
        tc::tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          tc::mma_bf16(tmem + TM_D3 + 64 * hh, tc::sdesc_sw128(sb + OFF_KT + ks * 2048, 8192, 1024),
                       tc::sdesc_sw128(rd + ks * 2048, 8192, 1024), ID_U, ks > 0);
        tc::mma_commit(bar(hb + H_D3_FULL));
        tc::mma_commit(bar(B_KT_EMPTY));
      }
      tc::mma_commit(bar(B_DRAIN + 1 + hh));
      volatile int never = 0;
      tc::mbar_wait(bar(B_DRAIN + 1 + hh), 0, &never, kBudgetNs / 4);
    }
  } else if (warp < 8) {
    // ------------------------------- pre warpgroup -------------------------------------------
    const int ptid = threadIdx.x - 128;                 // = TMEM lane of this thread
    const uint32_t lane_off = static_cast<uint32_t>(32 * (warp & 3)) << 16;
    float* sA = reinterpret_cast<float*>(smem + OFF_SA);
    float* sT = reinterpret_cast<float*>(smem + OFF_ST);
    if (ptid >= 64) {   // identity rows of [P; I], written once
      const int r = ptid, j1 = ptid - 64;
#pragma unroll
      for (int cc = 0; cc < 8; ++cc) {
        uint32_t w[4] = {0u, 0u, 0u, 0u};
        if ((j1 >> 3) == cc) w[(j1 & 7) >> 1] = (j1 & 1) ? 0x3F800000u : 0x00003F80u;
        tc::st_shared_v4(sb + OFF_PI + tc::sw128(r, cc), w[0], w[1], w[2], w[3]);
      }
    }
    for (int c = 0; c < nC; ++c) {
      const int s = c & 1, slot = c % 3;
      const long t0 = (long)c * C;
      float* gG = reinterpret_cast<float*>(smem + OFF_GB + slot * 1024);
      float* gGam = gG + 64;
      float* gKt = gG + 128;
      float* gBeta = gG + 192;
      if (ptid < 32) {          // gates of this chunk: lane l holds tokens 2l, 2l+1
        float la0 = 0.f, la1 = 0.f, be0 = 0.f, be1 = 0.f;
        const long ta = t0 + 2 * lane, tb = ta + 1;
        if (ta < T) { la0 = log_alpha[((long)bq * T + ta) * Hv + h]; be0 = beta[((long)bq * T + ta) * Hv + h]; }
        if (tb < T) { la1 = log_alpha[((long)bq * T + tb) * Hv + h]; be1 = beta[((long)bq * T + tb) * Hv + h]; }
        float incl = la0 + la1;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
          const float n = __shfl_up_sync(0xffffffffu, incl, d);
          if (lane >= d) incl += n;
        }
        const float g1 = incl, g0 = incl - la1;
        const float gl = __shfl_sync(0xffffffffu, incl, 31);
        gG[2 * lane] = g0;             gG[2 * lane + 1] = g1;
        gGam[2 * lane] = expf(g0);     gGam[2 * lane + 1] = expf(g1);
        gKt[2 * lane] = expf(gl - g0); gKt[2 * lane + 1] = expf(gl - g1);
        gBeta[2 * lane] = be0;         gBeta[2 * lane + 1] = be1;
        __syncwarp();
        __threadfence_block();
        if (lane == 0) tc::mbar_arrive(bar(B_GATE + slot));
      }
      tc::named_bar(1, 128);
      // S row -> P row (rows 0..63) or A row (rows 64..127)
      tc::mbar_wait(bar(B_S_FULL), c & 1, abort_flag, kBudgetNs);
      tc::tc_fence_after();
      float sv[64];
      {
        float a16[16];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          tmem_ld16(tmem + lane_off + TM_S + 16 * p, a16);
          tc::tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) sv[16 * p + i] = a16[i];
        }
      }
      tc::tc_fence_before();
      tc::named_bar(1, 128);
      if (ptid == 0) tc::mbar_arrive(bar(B_S_EMPTY));
      if (ptid < 64) {
        const int t = ptid;
        const float gt = gG[t];
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) {
          float pv[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int j = 8 * cc + e;
            pv[e] = (j <= t) ? expf(gt - gG[j]) * sv[j] * scale : 0.f;
          }
          tc::st_shared_v4(sb + OFF_PI + tc::sw128(t, cc), tc::pack_bf16(pv[0], pv[1]),
                           tc::pack_bf16(pv[2], pv[3]), tc::pack_bf16(pv[4], pv[5]),
                           tc::pack_bf16(pv[6], pv[7]));
        }
      } else {
        const int t = ptid - 64;
        const float gt = gG[t], bt = gBeta[t];
#pragma unroll
        for (int j4 = 0; j4 < 64; j4 += 4) {
          float4 av;
          av.x = (j4 + 0 < t) ? bt * expf(gt - gG[j4 + 0]) * sv[j4 + 0] : 0.f;
          av.y = (j4 + 1 < t) ? bt * expf(gt - gG[j4 + 1]) * sv[j4 + 1] : 0.f;
          av.z = (j4 + 2 < t) ? bt * expf(gt - gG[j4 + 2]) * sv[j4 + 2] : 0.f;
          av.w = (j4 + 3 < t) ? bt * expf(gt - gG[j4 + 3]) * sv[j4 + 3] : 0.f;
          *reinterpret_cast<float4*>(&sA[t * LDA + j4]) = av;
        }
      }
      tc::named_bar(1, 128);
      solve_unit_lower(sA, sT, ptid);
      {   // T_b = T diag(beta) as the bf16 B operand of [P; I] T_b (row k, 64 columns)
        const int k = ptid >> 1, n0 = (ptid & 1) * 32;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          float tv[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const int n = n0 + 8 * cc + e;
            tv[e] = (n <= k) ? sT[k * LDA + n] * gBeta[n] : 0.f;
          }
          tc::st_shared_v4(sb + OFF_TB + tc::sw128(k, (n0 >> 3) + cc), tc::pack_bf16(tv[0], tv[1]),
                           tc::pack_bf16(tv[2], tv[3]), tc::pack_bf16(tv[4], tv[5]),
                           tc::pack_bf16(tv[6], tv[7]));
        }
      }
      tc::fence_proxy_async_smem();
      tc::named_bar(1, 128);
      if (ptid == 0) tc::mbar_arrive(bar(B_PT_READY));
      // A2 = [P T_b; T_b] from TMEM, Ktil from the K tile
      tc::mbar_wait(bar(B_PT_FULL), c & 1, abort_flag, kBudgetNs);
      tc::tc_fence_after();
      float pt[64];
      {
        float a16[16];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          tmem_ld16(tmem + lane_off + TM_PT + 16 * p, a16);
          tc::tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) pt[16 * p + i] = a16[i];
        }
      }
      tc::tc_fence_before();
      if (c >= 1) tc::mbar_wait(bar(B_A2_EMPTY), (c - 1) & 1, abort_flag, kBudgetNs);
#pragma unroll
      for (int cc = 0; cc < 8; ++cc)
        tc::st_shared_v4(sb + OFF_A2 + tc::sw128(ptid, cc), tc::pack_bf16(pt[8 * cc], pt[8 * cc + 1]),
                         tc::pack_bf16(pt[8 * cc + 2], pt[8 * cc + 3]),
                         tc::pack_bf16(pt[8 * cc + 4], pt[8 * cc + 5]),
                         tc::pack_bf16(pt[8 * cc + 6], pt[8 * cc + 7]));
      tc::mbar_wait(bar(B_QK_FULL + s), (c >> 1) & 1, abort_flag, kBudgetNs);
      if (c >= 1) tc::mbar_wait(bar(B_KT_EMPTY), (c - 1) & 1, abort_flag, kBudgetNs);
      {
        const int t = ptid >> 1, kb = ptid & 1;
        const float f = gKt[t];
        const uint32_t src = sb + OFF_QK + s * QK_STAGE + kb * 16384 + 8192 + t * 128;
        const uint32_t dst = sb + OFF_KT + kb * 8192 + t * 128;
#pragma unroll
        for (int pc = 0; pc < 8; ++pc) {   // same swizzle on both sides: copy chunk positions
          const uint4 u = tc::ld_shared_v4(src + pc * 16);
          tc::st_shared_v4(dst + pc * 16, tc::pack_bf16(tc::bf16lo(u.x) * f, tc::bf16hi(u.x) * f),
                           tc::pack_bf16(tc::bf16lo(u.y) * f, tc::bf16hi(u.y) * f),
                           tc::pack_bf16(tc::bf16lo(u.z) * f, tc::bf16hi(u.z) * f),
                           tc::pack_bf16(tc::bf16lo(u.w) * f, tc::bf16hi(u.w) * f));
        }
      }
      tc::fence_proxy_async_smem();
      const bool stop = vote_abort(1, 128, abort_flag);
      if (ptid == 0) {
        tc::mbar_arrive(bar(B_PRE_FULL));
        tc::mbar_arrive(bar(B_IN_EMPTY + s));
        tc::mbar_arrive(bar(B_PT_EMPTY));
      }
      if (stop) break;
    }
  } else {
    // ------------------------------- chain warpgroups ----------------------------------------
    const int hh = (warp - 8) >> 2, q = warp & 3, r = 32 * q + lane;
    const int hb = B_HALF + H_COUNT * hh;
    const uint32_t lane_off = static_cast<uint32_t>(32 * q) << 16;
    const uint32_t mb = sb + OFF_MB + hh * 16384, rd = sb + OFF_RD + hh * 8192;
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
      const float* gGam = reinterpret_cast<const float*>(smem + OFF_GB + slot * 1024) + 64;
      if (q >= 2) {
        // R' = V - gamma (K M) for token t, then Delta
        const int t = r - 64;
        tc::mbar_wait(bar(hb + H_X_FULL), c & 1, abort_flag, kBudgetNs);
        tc::mbar_wait(bar(B_GATE + slot), (c / 3) & 1, abort_flag, kBudgetNs);
        tc::mbar_wait(bar(B_V_FULL), c & 1, abort_flag, kBudgetNs);
        tc::tc_fence_after();
        const float g = gGam[t];
        const uint32_t vrow = sb + OFF_V + hh * 8192;
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          float x[16];
          tmem_ld16(tmem + lane_off + TM_X + 64 * hh + 16 * p, x);
          tc::tmem_wait_ld();
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            const int cc = 2 * p + half;
            const uint4 u = tc::ld_shared_v4(vrow + tc::sw128(t, cc));
            const float* xx = x + 8 * half;
            tc::st_shared_v4(rd + tc::sw128(t, cc),
                             tc::pack_bf16(tc::bf16lo(u.x) - g * xx[0], tc::bf16hi(u.x) - g * xx[1]),
                             tc::pack_bf16(tc::bf16lo(u.y) - g * xx[2], tc::bf16hi(u.y) - g * xx[3]),
                             tc::pack_bf16(tc::bf16lo(u.z) - g * xx[4], tc::bf16hi(u.z) - g * xx[5]),
                             tc::pack_bf16(tc::bf16lo(u.w) - g * xx[6], tc::bf16hi(u.w) - g * xx[7]));
          }
        }
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        tc::named_bar(id_hi, 64);
        if (q == 2 && lane == 0) {
          tc::mbar_arrive(bar(hb + H_R_FULL));
          tc::mbar_arrive(bar(B_V_EMPTY));
          tc::mbar_arrive(bar(hb + H_X_EMPTY));
        }
        tc::mbar_wait(bar(hb + H_Y_FULL), c & 1, abort_flag, kBudgetNs);
        tc::tc_fence_after();
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          float y[16];
          tmem_ld16(tmem + lane_off + TM_Y + 64 * hh + 16 * p, y);
          tc::tmem_wait_ld();
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            const float* yy = y + 8 * half;
            tc::st_shared_v4(rd + tc::sw128(t, 2 * p + half), tc::pack_bf16(yy[0], yy[1]),
                             tc::pack_bf16(yy[2], yy[3]), tc::pack_bf16(yy[4], yy[5]),
                             tc::pack_bf16(yy[6], yy[7]));
          }
        }
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        tc::named_bar(id_hi, 64);
        if (q == 2 && lane == 0) {
          tc::mbar_arrive(bar(hb + H_D_FULL));
          tc::mbar_arrive(bar(hb + H_Y_EMPTY));
        }
      } else {
        // o_t = gamma_t scale (Q M)_t + (P Delta)_t
        const int t = r;
        tc::mbar_wait(bar(hb + H_X_FULL), c & 1, abort_flag, kBudgetNs);
        tc::mbar_wait(bar(B_GATE + slot), (c / 3) & 1, abort_flag, kBudgetNs);
        tc::mbar_wait(bar(hb + H_Y_FULL), c & 1, abort_flag, kBudgetNs);
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
#pragma unroll
          for (int i = 0; i < 16; ++i) y[i] = fmaf(g, x[i], y[i]);
          if (valid) store16<Tout>(orow + 16 * p, y);
        }
        tc::tc_fence_before();
        tc::named_bar(id_lo, 64);
        if (q == 0 && lane == 0) {
          tc::mbar_arrive(bar(hb + H_X_EMPTY));
          tc::mbar_arrive(bar(hb + H_Y_EMPTY));
        }
      }
      // M <- gamma_last M + Ktil^T Delta  (row r of this half), and its bf16 copy for the MMAs
      tc::mbar_wait(bar(hb + H_D3_FULL), c & 1, abort_flag, kBudgetNs);
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
