// Chunked forward of the gated delta rule on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
// Shapes: d_k = d_v = 128, chunk C = 64, bf16 q/k/v, fp32 gates and state.
//
// Per value head and chunk, with the chunk-start state M = S^T (128 x 128, fp32), the chunk form of
// the recurrence ("Chapitre 16 - Assembler un système de type Kimi K3", 16.2: matrix operations
// inside each block, state handed from block to block) is computed as
//   state-independent part:
//     G = cumsum(log alpha), gamma = exp(G), S = [Q; K] K^T                (bf16 MMA, 128x64x128)
//     P = lower_incl(exp(G_i - G_j) q_i.k_j) * scale,  A = strict_lower(beta_i exp(G_i - G_j) k_i.k_j)
//     T = (I + A)^-1 (fp32, blocked by 16),  T_b = T diag(beta)
//     A2 = [P T_b; T_b]                     (P T_b: tf32 MMA, 64x64x64)
//   state-dependent chain (all 128 value columns at once):
//     X = [Q; K] M                           (bf16 MMA, 128x128x128, M as a two-term bf16 split)
//     R' = V - diag(gamma) (K M)             (rows 64..127 of X)
//     Y = A2 R' = [P Delta; Delta]           (bf16 MMA, 128x128x64, three-term split of both
//                                             operands), Delta = T_b (V - diag(gamma) K M)
//     o = diag(gamma) scale (Q M) + P Delta  (rows 0..63 of X and Y)
//     M <- gamma_last M + K^T (ktil Delta),  ktil = exp(G_last - G)
//                                            (bf16 MMA on a two-term bf16 split of ktil Delta,
//                                             accumulated onto gamma_last M kept in TMEM)
// which is the token recurrence reorganised exactly (Delta's rows are beta_t (v_t - alpha_t
// S_{t-1} k_t)).  Accumulations and the master state are fp32.  The operands that carry the state
// through the chain (M, A2, R', ktil Delta) are split into bf16 pairs hi + lo (|x - hi - lo| <
// 2^-14 |x|) and multiplied term by term (hi.hi + lo.hi + hi.lo where both sides are split): with
// plain bf16, or even tf32, there the state's largest entries drift by a few percent (about one
// percent for tf32) of its RMS.  The splits are integer mask / byte-permute operations (the
// conversion instructions run at a quarter of the ALU rate).
//
// One CTA per (batch, value head), 512 threads in specialised warps:
//   warp 0        TMA producer (Q, K tiles double-buffered; V single-buffered)
//   warp 1        TMEM owner; issues the state-independent MMAs (S and P T_b)
//   warp 2        issues the chain MMAs (X, Y and the state update)
//   warps 4-7     "pre" warpgroup: gates (one chunk ahead), A, P, the triangular solve, T_b
//                 (A2's rows P T_b are written by the chain's O warps once their MMA is done)
//   warps 8-11    chain warpgroup of value columns 0..63; warps 12-15 of columns 64..127
// so the state-independent work of chunk c+1 overlaps the chain of chunk c.  The fp32 master state
// lives in TMEM (the update MMA accumulates onto it); o leaves through shared memory and TMA
// stores.  Every wait is bounded (about 2 s): on expiry the CTA records the library's timeout bit,
// every role leaves its loop at the next uniform check point, in-flight TMA copies and MMAs are
// drained, TMEM is released and the kernel returns.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "tc_ptx.cuh"

namespace gdn {
namespace tcf {

constexpr int C = 64;
constexpr int kThreads = 512;
constexpr uint64_t kBudget = 4000000000ull;   // wait budget in SM cycles (about 2 s)

// shared memory map (bytes from a 1024-aligned base); every MMA tile is 128-byte swizzled
constexpr uint32_t OFF_QK = 0;          // 2 stages x 32 KB: kb0 [Q 64 rows | K 64 rows], kb1 [...]
constexpr uint32_t QK_STAGE = 32768;
constexpr uint32_t OFF_V = 65536;       // 16 KB: V[t][64 dv] bf16, one 8 KB tile per column half
constexpr uint32_t OFF_RD = 81920;      // 32 KB, per column half 16 KB: the bf16 low part of M
                                        // [128 dk][128 B] for X, then R' bf16 hi [64 t][128 B] +
                                        // lo, then ktil Delta bf16 hi [64 t][128 B] + lo
constexpr uint32_t OFF_A2 = 114688;     // 32 KB: A2 bf16 hi [128 rows][128 B] + lo; between the
                                        // Y MMA and the next chunk's A2 it stages the o tile
constexpr uint32_t OFF_MB = 147456;     // 32 KB, per column half 16 KB: bf16 M [128 dk][128 B]
constexpr uint32_t OFF_W = 180224;      // 32 KB: solve scratch, then P (tf32) and T_b (tf32)
constexpr uint32_t OFF_WT = OFF_W + 16384;   // T_b, [dv block][64 rows][128 B]
constexpr uint32_t SOLVE_T = 12800;     // byte offset of T inside the solve scratch
constexpr uint32_t OFF_GB = 212992;     // 3 slots x 2 KB: G log2(e)[64], gamma[64], ktil[64],
                                        // beta[64], E[4][64] (E[b][j] = exp(G_16b - G_j), j < 16b)
constexpr uint32_t GB_SLOT = 2048;
constexpr uint32_t OFF_BAR = OFF_GB + 3 * GB_SLOT;
constexpr int NBAR = 26;
constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;   // +0 TMEM base, +4 abort flag
constexpr uint32_t SMEM_BYTES = OFF_MISC + 16;
constexpr uint32_t SMEM_ALLOC = SMEM_BYTES + 1024;
static_assert(SMEM_ALLOC <= 232448, "shared memory budget");
static_assert(2 * SOLVE_T <= 32768, "solve scratch");

// TMEM columns (512 allocated, 128 lanes x 32 bit)
constexpr uint32_t TM_S = 0, TM_PT = 64, TM_X = 128, TM_Y = 256, TM_M = 384;

// mbarriers
enum : int {
  B_QK_FULL = 0, B_IN_EMPTY = 2, B_S_FULL = 4, B_S_EMPTY, B_PT_READY, B_PT_FULL, B_PT_EMPTY,
  B_PRE_FULL, B_A2_EMPTY, B_GATE, B_X_FULL = B_GATE + 3, B_R_FULL, B_Y_FULL, B_D_FULL, B_D3_FULL,
  B_M_READY, B_V_FULL, B_V_EMPTY, B_O_DONE, B_M_SCALED, B_DRAIN, B_END = B_DRAIN + 2
};
static_assert(B_END <= NBAR, "barrier map");

constexpr uint32_t ID_S = tc::idesc_bf16(128, 64, false, false);
constexpr uint32_t ID_PT = tc::idesc_tf32(128, 64, false, true);   // rows 64..127 unused
constexpr uint32_t ID_X = tc::idesc_bf16(128, 128, false, true);
constexpr uint32_t ID_Y = tc::idesc_bf16(128, 128, false, true);
constexpr uint32_t ID_U = tc::idesc_bf16(128, 128, true, true);

// Optional per-chunk timestamps for studying the pipeline (compiled only with GDN_TC_TRACE):
// slot (block, chunk, event) of a caller-provided buffer receives clock64().
#ifdef GDN_TC_TRACE
__device__ unsigned long long* g_tc_trace = nullptr;
#define GDN_TRACE(c, ev)                                                              \
  do {                                                                                \
    if (g_tc_trace) g_tc_trace[((size_t)blockIdx.x * nC + (c)) * 64 + (ev)] = clock64(); \
  } while (0)
// same with the global nanosecond timer (comparable across SMs)
#define GDN_TRACE_G(c, ev)                                                            \
  do {                                                                                \
    if (g_tc_trace) g_tc_trace[((size_t)blockIdx.x * nC + (c)) * 64 + (ev)] = tc::globaltimer_ns(); \
  } while (0)
#else
#define GDN_TRACE(c, ev) do {} while (0)
#define GDN_TRACE_G(c, ev) do {} while (0)
#endif

// ------------------------------------------------------------------------------------------
// triangular solve on 16 x 16 blocks stored packed: block (i, k), i >= k, at index
// i(i+1)/2 + k, 16 rows of 20 floats (4 floats of padding against bank conflicts)
// ------------------------------------------------------------------------------------------
constexpr int BLD = 20, BSZ = 16 * BLD;
__device__ __forceinline__ uint32_t blk(uint32_t base, int i, int k) {
  return base + (uint32_t)((i * (i + 1) / 2 + k) * BSZ * 4);
}
__device__ __forceinline__ uint32_t at(uint32_t blk_base, int r, int c) {
  return blk_base + (uint32_t)((r * BLD + c) * 4);
}

// block index bi = 0..5 -> (i, k) = (1,0) (2,0) (2,1) (3,0) (3,1) (3,2)
__device__ __forceinline__ int blk_i(int bi) { return bi < 1 ? 1 : (bi < 3 ? 2 : 3); }
__device__ __forceinline__ int blk_k(int bi, int i) { return bi - i * (i - 1) / 2; }

// Warp-level tf32 MMA: d (16 x 8 C fragment) += a (16 x 8) b (8 x 8).  Fragments (lane = 4 g + t):
// a = {A[g][t], A[g+8][t], A[g][t+4], A[g+8][t+4]}, b = {B[t][g], B[t+4][g]},
// d = {D[g][2t], D[g][2t+1], D[g+8][2t], D[g+8][2t+1]}.
__device__ __forceinline__ void mma_m16n8k8_tf32(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                                 uint32_t b1) {
  asm("mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
// x = hi + lo + e with hi, lo tf32 (truncated), |e| < 2^-20 |x|.
__device__ __forceinline__ void split_tf32(float x, uint32_t& hi, uint32_t& lo) {
  hi = __float_as_uint(x) & 0xFFFFE000u;
  lo = __float_as_uint(x - __uint_as_float(hi)) & 0xFFFFE000u;
}
// One 16 x 16 x 16 product X Y[:, n0 .. n0+7] of packed blocks (a 16 x 8 half block of the result).
struct Tile {
  uint32_t X, Y;
  int n0;
};
// acc[m] (C fragments) += X_m Y_m[:, n0_m ..] for N independent tiles, as lo.hi + hi.lo + hi.hi
// tf32 products (fp32-level accuracy), one k half at a time; the MMAs of the tiles interleave.
template <int N>
__device__ __forceinline__ void mma_tiles(const Tile (&tl)[N], int g, int t, float (&acc)[N][4]) {
#pragma unroll
  for (int kk = 0; kk < 16; kk += 8) {
    uint32_t ah[N][4], al[N][4], bh[N][2], bl[N][2];
#pragma unroll
    for (int m = 0; m < N; ++m) {
      const uint32_t X = tl[m].X, Y = tl[m].Y;
      const int n0 = tl[m].n0;
      split_tf32(tc::lds1(at(X, g, kk + t)), ah[m][0], al[m][0]);
      split_tf32(tc::lds1(at(X, g + 8, kk + t)), ah[m][1], al[m][1]);
      split_tf32(tc::lds1(at(X, g, kk + t + 4)), ah[m][2], al[m][2]);
      split_tf32(tc::lds1(at(X, g + 8, kk + t + 4)), ah[m][3], al[m][3]);
      split_tf32(tc::lds1(at(Y, kk + t, n0 + g)), bh[m][0], bl[m][0]);
      split_tf32(tc::lds1(at(Y, kk + t + 4, n0 + g)), bh[m][1], bl[m][1]);
    }
#pragma unroll
    for (int m = 0; m < N; ++m) mma_m16n8k8_tf32(acc[m], al[m], bh[m][0], bh[m][1]);
#pragma unroll
    for (int m = 0; m < N; ++m) mma_m16n8k8_tf32(acc[m], ah[m], bl[m][0], bl[m][1]);
#pragma unroll
    for (int m = 0; m < N; ++m) mma_m16n8k8_tf32(acc[m], ah[m], bh[m][0], bh[m][1]);
  }
}
__device__ __forceinline__ float2 lds2(uint32_t addr) {
  float2 v;
  asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(v.x), "=f"(v.y) : "r"(addr) : "memory");
  return v;
}
__device__ __forceinline__ void sts2(uint32_t addr, float a, float b) {
  asm volatile("st.shared.v2.f32 [%0], {%1, %2};" ::"r"(addr), "f"(a), "f"(b) : "memory");
}
__device__ __forceinline__ void ld_frag(uint32_t B, int n0, int g, int t, float (&c)[4]) {
  const float2 a = lds2(at(B, g, n0 + 2 * t)), b = lds2(at(B, g + 8, n0 + 2 * t));
  c[0] = a.x; c[1] = a.y; c[2] = b.x; c[3] = b.y;
}
__device__ __forceinline__ void st_frag(uint32_t B, int n0, int g, int t, const float (&c)[4]) {
  sts2(at(B, g, n0 + 2 * t), c[0], c[1]);
  sts2(at(B, g + 8, n0 + 2 * t), c[2], c[3]);
}

// T = (I + A)^-1 for a 64 x 64 strictly lower A (128 threads = 4 warps, named barrier 1), blocked
// by 16:  D_b = (I + A_bb)^-1 by forward substitution (one column per thread);  At_ik = D_i A_ik;
// U = (I + At)^-1 (U_ii = I; At is block-nilpotent, so U is closed-form in At's blocks);
// T_ik = U_ik D_k.   (I + A = blockdiag(I + A_bb) (I + At), so T = U D.)  The block products run
// as warp MMAs on 16 x 8 half blocks.  On return the off-diagonal blocks of T are in `tv`: item m
// of warp w is half block hp = w + 4 m (block bi = hp / 2, columns 8 (hp % 2) ..) as a C fragment;
// the diagonal blocks D_b are in sT.  sA's blocks are overwritten.
__device__ __forceinline__ void solve_unit_lower(uint32_t sA, uint32_t sT, int ptid, float (&tv)[3][4],
                                                 [[maybe_unused]] int c, [[maybe_unused]] int nC) {
  if (ptid < 64) {                                    // D_b, column `col` of block b
    const int b = ptid >> 4, col = ptid & 15;
    const uint32_t Ab = blk(sA, b, b);
    float x[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      float a0 = (i == col) ? 1.f : 0.f, a1 = 0.f;
#pragma unroll
      for (int j4 = 0; j4 < i; j4 += 4) {
        const float4 a = tc::lds4(at(Ab, i, j4));
        const float av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (j4 + e < i) {
            if (e & 1) a1 = fmaf(-av[e], x[j4 + e], a1);
            else a0 = fmaf(-av[e], x[j4 + e], a0);
          }
      }
      x[i] = a0 + a1;
    }
    const uint32_t Tb = blk(sT, b, b);
#pragma unroll
    for (int i = 0; i < 16; ++i) tc::sts1(at(Tb, i, col), x[i]);
  }
  tc::named_bar(1, 128);
  if (ptid == 0) GDN_TRACE(c, 9);
  const int w = ptid >> 5, lane = ptid & 31, g = lane >> 2, t = lane & 3;
  {                                                   // At_ik = D_i A_ik, into T's off-diagonal
    Tile tl[3];
    float acc[3][4] = {};
#pragma unroll
    for (int m = 0; m < 3; ++m) {
      const int hp = w + 4 * m, bi = hp >> 1, n0 = (hp & 1) * 8;
      const int i = blk_i(bi), k = blk_k(bi, i);
      tl[m] = Tile{blk(sT, i, i), blk(sA, i, k), n0};
    }
    mma_tiles(tl, g, t, acc);
#pragma unroll
    for (int m = 0; m < 3; ++m) {
      const int bi = (w + 4 * m) >> 1;
      const int i = blk_i(bi), k = blk_k(bi, i);
      st_frag(blk(sT, i, k), tl[m].n0, g, t, acc[m]);
    }
  }
  tc::named_bar(1, 128);
  if (ptid == 0) GDN_TRACE(c, 23);
  // U_20 = -At_20 + At_21 At_10;  U_31 = -At_31 + At_32 At_21;  V_30 = -At_30 + At_31 At_10
  // (into sA's blocks (2,0), (3,1), (3,0); A itself is no longer needed).  Half blocks w, w + 4.
  {
    const int nt = w < 2 ? 2 : 1;                     // warp-uniform
    Tile tl[2];
    float acc[2][4];
#pragma unroll
    for (int m = 0; m < 2; ++m) {
      const int hp = m < nt ? w + 4 * m : w, bi = hp >> 1, n0 = (hp & 1) * 8;
      const int oi = bi == 0 ? 2 : 3, ok = bi == 1 ? 1 : 0;    // output block (oi, ok)
      const int xk = bi == 1 ? 2 : 1;                           // X = At_(oi, xk), Y = At_(xk, ok)
      ld_frag(blk(sT, oi, ok), n0, g, t, acc[m]);
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[m][e] = -acc[m][e];
      tl[m] = Tile{blk(sT, oi, xk), blk(sT, xk, ok), n0};
    }
    mma_tiles(tl, g, t, acc);
#pragma unroll
    for (int m = 0; m < 2; ++m)
      if (m < nt) {
        const int bi = (w + 4 * m) >> 1;
        const int oi = bi == 0 ? 2 : 3, ok = bi == 1 ? 1 : 0;
        st_frag(blk(sA, oi, ok), tl[m].n0, g, t, acc[m]);
      }
  }
  tc::named_bar(1, 128);
  if (ptid == 0) GDN_TRACE(c, 24);
  if (w < 2) {                                        // U_30 = V_30 - At_32 U_20
    const int n0 = 8 * w;
    const Tile tl[1] = {Tile{blk(sT, 3, 2), blk(sA, 2, 0), n0}};
    float acc[1][4] = {}, v[4];
    ld_frag(blk(sA, 3, 0), n0, g, t, v);
    mma_tiles(tl, g, t, acc);
#pragma unroll
    for (int e = 0; e < 4; ++e) v[e] -= acc[0][e];
    st_frag(blk(sA, 3, 0), n0, g, t, v);
  }
  tc::named_bar(1, 128);
  if (ptid == 0) GDN_TRACE(c, 25);
  {                                                   // T_ik = U_ik D_k (U = -At next to diag)
    Tile tl[3];
    float acc[3][4] = {};
#pragma unroll
    for (int m = 0; m < 3; ++m) {
      const int hp = w + 4 * m, bi = hp >> 1, n0 = (hp & 1) * 8;
      const int i = blk_i(bi), k = blk_k(bi, i);
      tl[m] = Tile{(i == k + 1) ? blk(sT, i, k) : blk(sA, i, k), blk(sT, k, k), n0};
    }
    mma_tiles(tl, g, t, acc);
#pragma unroll
    for (int m = 0; m < 3; ++m) {
      const int bi = (w + 4 * m) >> 1;
      const int i = blk_i(bi), k = blk_k(bi, i);
      const float sg = (i == k + 1) ? -1.f : 1.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) tv[m][e] = sg * acc[m][e];
    }
  }
  if (ptid == 0) GDN_TRACE(c, 26);
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

// 16 consecutive fp32 TMEM columns of this thread's lane (no wait).
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
// Store 16 consecutive fp32 TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const float (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"
      "%14,%15,%16};" ::"r"(taddr),
      "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]),
      "f"(v[8]), "f"(v[9]), "f"(v[10]), "f"(v[11]), "f"(v[12]), "f"(v[13]), "f"(v[14]), "f"(v[15])
      : "memory");
}
// 64 consecutive fp32 TMEM columns of this thread's lane (no wait).
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, float (&v)[64]) {
  float (&a)[32] = *reinterpret_cast<float(*)[32]>(&v[0]);
  float (&b)[32] = *reinterpret_cast<float(*)[32]>(&v[32]);
  tc::tmem_ld32(taddr, a);
  tc::tmem_ld32(taddr + 32, b);
}
__device__ __forceinline__ void tmem_st64(uint32_t taddr, const float (&v)[64]) {
  const float (&a)[32] = *reinterpret_cast<const float(*)[32]>(&v[0]);
  const float (&b)[32] = *reinterpret_cast<const float(*)[32]>(&v[32]);
  tc::tmem_st32(taddr, a);
  tc::tmem_st32(taddr + 32, b);
}

// Four fp32 values rounded to tf32, stored as one 16-byte chunk.
__device__ __forceinline__ void st_tf32x4(uint32_t addr, float a, float b, float c, float d) {
  tc::st_shared_v4(addr, tc::to_tf32(a), tc::to_tf32(b), tc::to_tf32(c), tc::to_tf32(d));
}
__device__ __forceinline__ void st_tf32x4(uint32_t addr, float4 v) {
  st_tf32x4(addr, v.x, v.y, v.z, v.w);
}
// Non-finite guard for the tf32 operands.  The tensor cores' tf32 path does not carry a NaN operand
// into the product, while it does carry an infinity; a thread whose tf32 values sum to a non-finite
// value (any NaN or infinity among them; finite values near FLT_MAX can also trip it) rewrites them
// as +infinity, so that a non-finite input still reaches o and the state as a non-finite value.
__device__ __forceinline__ bool nonfinite(float sum) { return !(fabsf(sum) <= 3.402823466e38f); }
constexpr float kInf = __builtin_huge_valf();

// x = hi + lo + e with hi = x truncated to bf16 and lo = (x - hi) truncated to bf16, |e| < 2^-14 |x|;
// returns the packed (low half = first value) bf16 pairs of two values.  NaN and infinities stay
// non-finite in hi or lo.
__device__ __forceinline__ void split2(float a, float b, uint32_t& hi2, uint32_t& lo2) {
  const uint32_t ua = __float_as_uint(a), ub = __float_as_uint(b);
  const float la = a - __uint_as_float(ua & 0xFFFF0000u);
  const float lb = b - __uint_as_float(ub & 0xFFFF0000u);
  hi2 = __byte_perm(ua, ub, 0x7632);
  lo2 = __byte_perm(__float_as_uint(la), __float_as_uint(lb), 0x7632);
}
// Eight values as a hi and a lo 16-byte chunk.
__device__ __forceinline__ void st_split8(uint32_t hi_addr, uint32_t lo_addr, const float* v) {
  uint32_t h[4], l[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) split2(v[2 * i], v[2 * i + 1], h[i], l[i]);
  tc::st_shared_v4(hi_addr, h[0], h[1], h[2], h[3]);
  tc::st_shared_v4(lo_addr, l[0], l[1], l[2], l[3]);
}

// Row `kr` (0..63), columns n..n+3 (n % 4 == 0) of T_b into its two operand layouts: rows 64..127
// of the K-major bf16 hi / lo A2 (8 bytes of a 16-byte chunk each) and the MN-major tf32 B operand
// of P T_b (32-byte chunks).
__device__ __forceinline__ void store_tb(uint32_t sb, int kr, int n, float4 v) {
  uint32_t h0, h1, l0, l1;
  split2(v.x, v.y, h0, l0);
  split2(v.z, v.w, h1, l1);
  const uint32_t a2 = sb + OFF_A2 + (64 + kr) * 128 + (((n >> 3) ^ (kr & 7)) << 4) + (n & 7) * 2;
  asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(a2), "r"(h0), "r"(h1) : "memory");
  asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(a2 + 16384), "r"(l0), "r"(l1) : "memory");
  st_tf32x4(sb + OFF_WT + (n >> 5) * 8192 + kr * 128 + ((((n & 31) >> 3) ^ (kr & 3)) << 5) +
                ((n >> 2) & 1) * 16,
            v);
}

// Same for two values (columns n, n + 1, n even).
__device__ __forceinline__ void store_tb2(uint32_t sb, int kr, int n, float a, float b) {
  uint32_t h, l;
  split2(a, b, h, l);
  const uint32_t a2 = sb + OFF_A2 + (64 + kr) * 128 + (((n >> 3) ^ (kr & 7)) << 4) + (n & 7) * 2;
  asm volatile("st.shared.b32 [%0], %1;" ::"r"(a2), "r"(h) : "memory");
  asm volatile("st.shared.b32 [%0], %1;" ::"r"(a2 + 16384), "r"(l) : "memory");
  const uint32_t wt = sb + OFF_WT + (n >> 5) * 8192 + kr * 128 +
                      ((((n & 31) >> 3) ^ (kr & 3)) << 5) + (n & 7) * 4;
  asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(wt), "r"(tc::to_tf32(a)), "r"(tc::to_tf32(b))
               : "memory");
}

// ------------------------------------------------------------------------------------------
// pre-pass: T_b = (I + A)^-1 diag(beta) of every (batch, value head, chunk), independently
// ------------------------------------------------------------------------------------------
// T_b depends on nothing across chunks, so it is computed ahead of the recurrence by many small
// CTAs at once and handed over through HBM as 10 packed 16 x 16 blocks (block (i, k), i >= k, at
// index i(i+1)/2 + k, rows of 16 floats): 10 KB per chunk.  A = strict_lower(beta_i exp(G_i - G_j)
// k_i . k_j) with k_i . k_j from bf16 warp MMAs (exact products, fp32 sums) and the blocked solve
// above.  A chunk whose A holds a NaN or an infinity gets T_b = +inf everywhere (the solve's
// warp MMAs may drop a NaN operand), so the recurrence still sees a non-finite value.
constexpr int kTbFloats = 10 * 256;                 // floats per chunk
constexpr int PP_THREADS = 128;
constexpr int PP_KROW = 136;                        // K tile row stride in bf16 (272 bytes)
constexpr uint32_t PP_OFF_G = 64 * PP_KROW * 2;     // 17408: G log2(e)[64], beta[64], flag
constexpr uint32_t PP_OFF_A = PP_OFF_G + 1024;      // 18432: solve scratch, A then T
constexpr uint32_t PP_SMEM = PP_OFF_A + 2 * SOLVE_T;   // 44032
static_assert(PP_OFF_A % 16 == 0, "solve scratch alignment");

__device__ __forceinline__ void mma_m16n8k16_bf16(float (&d)[4], const uint32_t (&a)[4],
                                                  uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
      "{%8, %9}, {%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// grid (nC, Hv, B), 128 threads.
__global__ void __launch_bounds__(PP_THREADS)
tb_prepass_kernel(const __nv_bfloat16* __restrict__ k, const float* __restrict__ log_alpha,
                  const float* __restrict__ beta, float* __restrict__ Tb, int T, int Hk, int Hv) {
  extern __shared__ __align__(16) uint8_t pp_smem[];
  const uint32_t sb = tc::smem_u32(pp_smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31, g = lane >> 2, t4 = lane & 3;
  const int c = blockIdx.x, h = blockIdx.y, bq = blockIdx.z, nC = gridDim.x;
  const int hk = h / (Hv / Hk);
  const long t0 = (long)c * C;
  float* gG = reinterpret_cast<float*>(pp_smem + PP_OFF_G);
  float* gB = gG + 64;
  volatile int* flag = reinterpret_cast<volatile int*>(gG + 128);
  const uint32_t sA = sb + PP_OFF_A, sT = sA + SOLVE_T;

  // K tile, rows past T zero
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int idx = tid + PP_THREADS * i, row = idx >> 4, ch = idx & 15;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (t0 + row < T)
      v = *reinterpret_cast<const uint4*>(k + (((long)bq * T + t0 + row) * Hk + hk) * 128 + ch * 8);
    *reinterpret_cast<uint4*>(pp_smem + row * PP_KROW * 2 + ch * 16) = v;
  }
  // gates: G = cumsum(log alpha) over the chunk (log2-scaled), beta; zero past T
  if (tid < 64) {
    const long tt = t0 + tid;
    const float la = tt < T ? log_alpha[((long)bq * T + tt) * Hv + h] : 0.f;
    gB[tid] = tt < T ? beta[((long)bq * T + tt) * Hv + h] : 0.f;
    float incl = la;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const float n = __shfl_up_sync(0xffffffffu, incl, d);
      if (lane >= d) incl += n;
    }
    gG[tid] = incl;
  }
  if (tid == 0) *flag = 0;
  __syncthreads();
  if (tid >= 32 && tid < 64) gG[tid] += gG[31];       // carry of the first 32 tokens
  __syncthreads();
  if (tid < 64) gG[tid] *= 1.4426950408889634f;
  __syncthreads();

  // k_t . k_j for the 20 16 x 8 tiles of the lower block triangle (tile (mi, ni) with
  // 8 ni < 16 (mi + 1)), five per warp, then A = strict_lower(beta_t 2^(G'_t - G'_j) k_t . k_j)
  // into the packed solve blocks
  bool bad = false;
#pragma unroll 1
  for (int m = 0; m < 5; ++m) {
    const int tile = warp + 4 * m;
    // tile -> (mi, ni): mi = 0 holds tiles 0..1, mi = 1 tiles 2..5, mi = 2 tiles 6..11, mi = 3 12..19
    const int mi = tile < 2 ? 0 : (tile < 6 ? 1 : (tile < 12 ? 2 : 3));
    const int ni = tile - (mi == 0 ? 0 : (mi == 1 ? 2 : (mi == 2 ? 6 : 12)));
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    const uint8_t* ra0 = pp_smem + (16 * mi + g) * PP_KROW * 2;
    const uint8_t* ra1 = ra0 + 8 * PP_KROW * 2;
    const uint8_t* rb = pp_smem + (8 * ni + g) * PP_KROW * 2;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const int kc = 16 * ks + 2 * t4;             // bf16 column of this lane's pair
      const uint32_t a[4] = {*reinterpret_cast<const uint32_t*>(ra0 + kc * 2),
                             *reinterpret_cast<const uint32_t*>(ra1 + kc * 2),
                             *reinterpret_cast<const uint32_t*>(ra0 + (kc + 8) * 2),
                             *reinterpret_cast<const uint32_t*>(ra1 + (kc + 8) * 2)};
      mma_m16n8k16_bf16(acc, a, *reinterpret_cast<const uint32_t*>(rb + kc * 2),
                        *reinterpret_cast<const uint32_t*>(rb + (kc + 8) * 2));
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int t = 16 * mi + g + 8 * (e >> 1), j = 8 * ni + 2 * t4 + (e & 1);
      const float a = j < t ? gB[t] * tc::ex2(gG[t] - gG[j]) * acc[e] : 0.f;
      bad |= !(fabsf(a) <= 3.402823466e38f);
      tc::sts1(at(blk(sA, t >> 4, j >> 4), t & 15, j & 15), a);
    }
  }
  if (bad) *flag = 1;
  tc::named_bar(1, PP_THREADS);

  float tv[3][4];
  solve_unit_lower(sA, sT, tid, tv, c, nC);
  const bool poison = *flag != 0;

  // T_b = T diag(beta): off-diagonal half blocks (C fragments of the solve), diagonal blocks
  float* out = Tb + (((long)bq * Hv + h) * nC + c) * kTbFloats;
#pragma unroll
  for (int m = 0; m < 3; ++m) {
    const int hp = warp + 4 * m, bi = hp >> 1, n0 = (hp & 1) * 8;
    const int i = blk_i(bi), kk = blk_k(bi, i);
    const int col = n0 + 2 * t4;
    const float b0 = gB[16 * kk + col], b1 = gB[16 * kk + col + 1];
    float* ob = out + (i * (i + 1) / 2 + kk) * 256;
    const float2 r0 = poison ? make_float2(kInf, kInf) : make_float2(tv[m][0] * b0, tv[m][1] * b1);
    const float2 r1 = poison ? make_float2(kInf, kInf) : make_float2(tv[m][2] * b0, tv[m][3] * b1);
    *reinterpret_cast<float2*>(ob + g * 16 + col) = r0;
    *reinterpret_cast<float2*>(ob + (g + 8) * 16 + col) = r1;
  }
#pragma unroll
  for (int m = 0; m < 2; ++m) {
    const int id = tid + PP_THREADS * m, b = id >> 6, r = (id >> 2) & 15, cs = id & 3;
    const float4 d = tc::lds4(at(blk(sT, b, b), r, 4 * cs));
    const float4 be = *reinterpret_cast<const float4*>(gB + 16 * b + 4 * cs);
    const float4 v = poison ? make_float4(kInf, kInf, kInf, kInf)
                            : make_float4(d.x * be.x, d.y * be.y, d.z * be.z, d.w * be.w);
    *reinterpret_cast<float4*>(out + (b * (b + 1) / 2 + b) * 256 + r * 16 + 4 * cs) = v;
  }
}

// ------------------------------------------------------------------------------------------
// the kernel
// ------------------------------------------------------------------------------------------
template <typename Tout>
__global__ void __launch_bounds__(kThreads, 1)
chunk_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                    const __grid_constant__ CUtensorMap tmv, const __grid_constant__ CUtensorMap tmo,
                    const float* __restrict__ log_alpha, const float* __restrict__ beta,
                    const float* __restrict__ Tb, const float* __restrict__ S0,
                    float* __restrict__ S_T, int T, int Hk, int Hv, float scale) {
  constexpr bool kF32 = sizeof(Tout) == 4;
  // X takes M as a hi + lo bf16 pair when o is fp32 (the layer, whose gated norm magnifies o's
  // error); a bf16 o carries its own rounding, and one round-to-nearest bf16 copy of M suffices.
  constexpr bool kSplitX = kF32;
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
  auto gslot = [&](int c) -> float* {
    return reinterpret_cast<float*>(smem + OFF_GB + (c % 3) * GB_SLOT);
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(bar(B_QK_FULL + s), 1);
      tc::mbar_init(bar(B_IN_EMPTY + s), 3);     // S, X and state-update MMAs read the tile
    }
    const int ones[] = {B_S_FULL, B_S_EMPTY, B_PT_READY, B_PT_FULL, B_A2_EMPTY, B_GATE,
                        B_GATE + 1, B_GATE + 2, B_X_FULL, B_Y_FULL, B_D3_FULL, B_V_FULL, B_DRAIN,
                        B_DRAIN + 1};
    for (int i : ones) tc::mbar_init(bar(i), 1);
    const int twos[] = {B_R_FULL, B_D_FULL, B_M_READY, B_V_EMPTY, B_O_DONE, B_M_SCALED,
                        B_PT_EMPTY};
    for (int i : twos) tc::mbar_init(bar(i), 2);   // one arrive per column half
    tc::mbar_init(bar(B_PRE_FULL), 3);             // T_b rows (pre) + P T_b rows (each half)
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
    tc::tma_prefetch_desc(&tmo);
  }
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + OFF_MISC);
  if (threadIdx.x == 0) GDN_TRACE_G(0, 10);

  if (warp == 0) {
    // ------------------------------- TMA producer -------------------------------------------
    if (lane == 0) {
      int armed_qk[2] = {-1, -1}, armed_v = -1;
      bool ok = true;
      for (int c = 0; c < nC && ok; ++c) {
        const int s = c & 1, t0 = c * C;
        if (c >= 2) ok = tc::mbar_wait(bar(B_IN_EMPTY + s), ((c >> 1) - 1) & 1, abort_flag, kBudget);
        if (!ok) break;
        const uint32_t dst = sb + OFF_QK + s * QK_STAGE;
        tc::mbar_arrive_expect_tx(bar(B_QK_FULL + s), 32768);
        tc::tma_load_4d(dst, &tmq, bar(B_QK_FULL + s), 0, hk, t0, bq);
        tc::tma_load_4d(dst + 8192, &tmk, bar(B_QK_FULL + s), 0, hk, t0, bq);
        tc::tma_load_4d(dst + 16384, &tmq, bar(B_QK_FULL + s), 64, hk, t0, bq);
        tc::tma_load_4d(dst + 24576, &tmk, bar(B_QK_FULL + s), 64, hk, t0, bq);
        armed_qk[s] = c;
        if (c >= 1) ok = tc::mbar_wait(bar(B_V_EMPTY), (c - 1) & 1, abort_flag, kBudget);
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
            tc::mbar_wait(bar(B_QK_FULL + s), (armed_qk[s] >> 1) & 1, &never, kBudget / 4);
        if (armed_v >= 0) tc::mbar_wait(bar(B_V_FULL), armed_v & 1, &never, kBudget / 4);
      }
    }
  } else if (warp == 1) {
    // -------------------- state-independent MMAs: S = [Q;K] K^T and P T_b --------------------
    if (lane == 0) {
      auto issue_S = [&](int c) -> bool {
        const int s = c & 1;
        if (!tc::mbar_wait(bar(B_QK_FULL + s), (c >> 1) & 1, abort_flag, kBudget)) return false;
        if (c >= 1 && !tc::mbar_wait(bar(B_S_EMPTY), (c - 1) & 1, abort_flag, kBudget))
          return false;
        tc::tc_fence_after();
        const uint32_t qk = sb + OFF_QK + s * QK_STAGE;
#pragma unroll 1
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
        ok = tc::mbar_wait(bar(B_PT_READY), c & 1, abort_flag, kBudget) &&
             (c == 0 || tc::mbar_wait(bar(B_PT_EMPTY), (c - 1) & 1, abort_flag, kBudget));
        if (!ok) break;
        tc::tc_fence_after();
#pragma unroll 1
        for (int ks = 0; ks < 8; ++ks)   // P (64 x 64, K-major) x T_b (64 x 64, MN-major), tf32
          tc::mma_tf32(tmem + TM_PT,
                       tc::sdesc_sw128(sb + OFF_W + (ks >> 2) * 8192 + (ks & 3) * 32, 16, 1024),
                       tc::sdesc_sw128_b32(sb + OFF_WT + ks * 1024, 8192), ID_PT, ks > 0);
        tc::mma_commit(bar(B_PT_FULL));
        if (c + 1 < nC) ok = issue_S(c + 1);
      }
      tc::mma_commit(bar(B_DRAIN + 0));
      volatile int never = 0;
      tc::mbar_wait(bar(B_DRAIN + 0), 0, &never, kBudget / 4);
    }
  } else if (warp == 2) {
    // -------------------------------- chain MMAs ---------------------------------------------
    if (lane == 0) {
      bool ok = true;
      for (int c = 0; c < nC && ok; ++c) {
        const int s = c & 1;
        const uint32_t qk = sb + OFF_QK + s * QK_STAGE;
        // X = [Q; K] M_hi + [Q; K] M_lo  (M = M_hi + M_lo, two bf16 terms)      (bf16)
        ok = tc::mbar_wait(bar(B_QK_FULL + s), (c >> 1) & 1, abort_flag, kBudget) &&
             tc::mbar_wait(bar(B_M_READY), c & 1, abort_flag, kBudget);
        if (!ok) break;
        tc::tc_fence_after();
#pragma unroll 1
        for (int ks = 0; ks < (kSplitX ? 16 : 8); ++ks)
          tc::mma_bf16(tmem + TM_X,
                       tc::sdesc_sw128(qk + ((ks >> 2) & 1) * 16384 + (ks & 3) * 32, 16, 1024),
                       tc::sdesc_sw128(sb + (ks < 8 ? OFF_MB : OFF_RD) + (ks & 7) * 2048, 16384, 1024),
                       ID_X, ks > 0);
        tc::mma_commit(bar(B_X_FULL));
        tc::mma_commit(bar(B_IN_EMPTY + s));
        GDN_TRACE(c, 20);
        // Y = A2_hi R'_hi + A2_lo R'_hi + A2_hi R'_lo                           (bf16)
        ok = tc::mbar_wait(bar(B_R_FULL), c & 1, abort_flag, kBudget) &&
             tc::mbar_wait(bar(B_PRE_FULL), c & 1, abort_flag, kBudget);
        if (!ok) break;
        tc::tc_fence_after();
#pragma unroll 1
        for (int i = 0; i < 12; ++i) {
          const int ks = i / 3, term = i - 3 * ks;
          tc::mma_bf16(tmem + TM_Y,
                       tc::sdesc_sw128(sb + OFF_A2 + (term == 1 ? 16384 : 0) + ks * 32, 16, 1024),
                       tc::sdesc_sw128(sb + OFF_RD + (term == 2 ? 8192 : 0) + ks * 2048, 16384, 1024),
                       ID_Y, i > 0);
        }
        tc::mma_commit(bar(B_Y_FULL));
        tc::mma_commit(bar(B_A2_EMPTY));
        GDN_TRACE(c, 21);
        // M += K^T (ktil Delta)_hi + K^T (ktil Delta)_lo  (TMEM holds gamma_last M)  (bf16)
        ok = tc::mbar_wait(bar(B_D_FULL), c & 1, abort_flag, kBudget) &&
             tc::mbar_wait(bar(B_M_SCALED), c & 1, abort_flag, kBudget);
        if (!ok) break;
        tc::tc_fence_after();
#pragma unroll 1
        for (int ks = 0; ks < 8; ++ks)
          tc::mma_bf16(tmem + TM_M, tc::sdesc_sw128(qk + 8192 + (ks & 3) * 2048, 16384, 1024),
                       tc::sdesc_sw128(sb + OFF_RD + (ks >> 2) * 8192 + (ks & 3) * 2048, 16384, 1024),
                       ID_U, 1);
        tc::mma_commit(bar(B_D3_FULL));
        tc::mma_commit(bar(B_IN_EMPTY + s));
        GDN_TRACE(c, 22);
      }
      tc::mma_commit(bar(B_DRAIN + 1));
      volatile int never = 0;
      tc::mbar_wait(bar(B_DRAIN + 1), 0, &never, kBudget / 4);
    }
  } else if (warp == 3) {
    // idle
  } else if (warp < 8) {
    // ------------------------------- pre warpgroup -------------------------------------------
    const int ptid = threadIdx.x - 128;                 // = TMEM lane of this thread
    const int q = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(32 * q) << 16;
    // gates, computed by warp 4 one chunk ahead: lane l holds tokens 2l, 2l+1 of the next chunk
    float pla0 = 0.f, pla1 = 0.f, pbe0 = 0.f, pbe1 = 0.f;
    auto load_gates = [&](int c) {
      const long ta = (long)c * C + 2 * lane, tb = ta + 1;
      pla0 = pla1 = pbe0 = pbe1 = 0.f;
      if (ta < T) { pla0 = log_alpha[((long)bq * T + ta) * Hv + h]; pbe0 = beta[((long)bq * T + ta) * Hv + h]; }
      if (tb < T) { pla1 = log_alpha[((long)bq * T + tb) * Hv + h]; pbe1 = beta[((long)bq * T + tb) * Hv + h]; }
    };
    auto publish_gates = [&](int c) {
      float* gG = gslot(c);
      float* gGam = gG + 64;
      float* gKt = gG + 128;
      float* gBeta = gG + 192;
      float* gE = gG + 256;
      const float la0 = pla0, la1 = pla1, be0 = pbe0, be1 = pbe1;
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
      gGam[2 * lane] = tc::ex2(g0 * kLog2e);     gGam[2 * lane + 1] = tc::ex2(g1 * kLog2e);
      gKt[2 * lane] = tc::ex2((gl - g0) * kLog2e); gKt[2 * lane + 1] = tc::ex2((gl - g1) * kLog2e);
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
      if (lane == 0) tc::mbar_arrive(bar(B_GATE + c % 3));   // release: orders the stores above
      if (c + 1 < nC) load_gates(c + 1);                      // after the arrive, never before it
    };
    // T_b of a chunk from the pre-pass: this thread's items id = ptid + 128 m (m < 5) of the 640
    // float4 of the 10 packed blocks (block id / 64, row (id / 4) % 16, columns 4 (id % 4) ..),
    // loaded one chunk ahead
    float4 tbv[5];
    auto load_tb = [&](int cc) {
      const float4* src =
          reinterpret_cast<const float4*>(Tb + (((long)bq * Hv + h) * nC + cc) * kTbFloats);
#pragma unroll
      for (int m = 0; m < 5; ++m) tbv[m] = src[ptid + 128 * m];
    };
    load_tb(0);
    if (ptid < 32) {
      load_gates(0);
      publish_gates(0);
    }
    bool stop = false;
    for (int c = 0; c < nC && !stop; ++c) {
      if (ptid == 0) GDN_TRACE(c, 0);
      const float* gG = gslot(c);
      const float* gE = gG + 256;
      tc::mbar_wait(bar(B_GATE + c % 3), (c / 3) & 1, abort_flag, kBudget);
      tc::mbar_wait(bar(B_S_FULL), c & 1, abort_flag, kBudget);
      if (ptid == 0) GDN_TRACE(c, 1);
      tc::tc_fence_after();
      // Rows 0..63 of S hold (q_t . k_j): P[t][j] = exp(G_t - G_j) (q_t . k_j) scale for j <= t,
      // kept in the same TMEM row as fp32 until it goes out as the tf32 A operand of P T_b;
      // exp(G_t - G_j) = 2^(G'_t - G'_j), G' = G log2 e, inside t's 16-token block directly and
      // across blocks as 2^(G'_t - G'_16ti) E[ti][j] (both factors <= 1)
      if (ptid < 64) {
        const int t = ptid, ti = t >> 4;
        const float gt = gG[t];
        const float rowf = scale * tc::ex2(gt - gG[16 * ti]);
        const float4* g4 = reinterpret_cast<const float4*>(gG);
        const float4* e4p = reinterpret_cast<const float4*>(gE + 64 * ti);
#pragma unroll 1
        for (int p = 0; p < 2; ++p) {                // columns 32p .. 32p+31
          float sv[32];
          tc::tmem_ld32(tmem + lane_off + TM_S + 32 * p, sv);
          tc::tmem_wait_ld();
#pragma unroll
          for (int kb2 = 0; kb2 < 2; ++kb2) {
            const int kb = 2 * p + kb2;
            float* v = sv + 16 * kb2;
            if (kb < ti) {
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const float4 e = e4p[4 * kb + i];
                v[4 * i] *= rowf * e.x;     v[4 * i + 1] *= rowf * e.y;
                v[4 * i + 2] *= rowf * e.z; v[4 * i + 3] *= rowf * e.w;
              }
            } else if (kb == ti) {
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                const float4 g = g4[4 * kb + i];
                const float gj[4] = {g.x, g.y, g.z, g.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const int j = 16 * kb + 4 * i + e;
                  v[4 * i + e] = (j <= t) ? scale * tc::ex2(gt - gj[e]) * v[4 * i + e] : 0.f;
                }
              }
            } else {
#pragma unroll
              for (int e = 0; e < 16; ++e) v[e] = 0.f;
            }
          }
          tc::tmem_st32(tmem + lane_off + TM_S + 32 * p, sv);
        }
        tc::tmem_wait_st();
      }
      if (ptid == 0) GDN_TRACE(c, 2);
      float4 cur[5];
#pragma unroll
      for (int m = 0; m < 5; ++m) cur[m] = tbv[m];
      if (c + 1 < nC) load_tb(c + 1);
      if (c >= 1) {   // A2 (and the o tile staged in it) is free once Y and the o stores are done
        tc::mbar_wait(bar(B_A2_EMPTY), (c - 1) & 1, abort_flag, kBudget);
        tc::mbar_wait(bar(B_O_DONE), (c - 1) & 1, abort_flag, kBudget);
      }
      if (ptid == 0) GDN_TRACE(c, 4);
      // T_b into A2's rows 64..127 (bf16 hi / lo) and into the B operand of P T_b (tf32), zero
      // above the diagonal; the P T_b operands of the previous chunk are free (S of this chunk
      // was issued after, and completed after, that MMA)
      {
        float sum = 0.f;
#pragma unroll
        for (int m = 0; m < 5; ++m) sum += (cur[m].x + cur[m].y) + (cur[m].z + cur[m].w);
        const bool bad = nonfinite(sum);
        const float4 inf4 = make_float4(kInf, kInf, kInf, kInf);
#pragma unroll
        for (int m = 0; m < 5; ++m) {
          const int id = ptid + 128 * m, bb = id >> 6, r = (id >> 2) & 15, cs = id & 3;
          const int i = bb >= 6 ? 3 : (bb >= 3 ? 2 : (bb >= 1 ? 1 : 0));
          const int k = bb - i * (i + 1) / 2;
          store_tb(sb, 16 * i + r, 16 * k + 4 * cs, bad ? inf4 : cur[m]);
          if (i > k) store_tb(sb, 16 * k + r, 16 * i + 4 * cs, make_float4(0.f, 0.f, 0.f, 0.f));
        }
      }
      if (ptid == 0) GDN_TRACE(c, 5);
      // P rows (threads 0..63, warps 4 and 5): back from TMEM, rounded to tf32, into the K-major
      // A operand of P T_b
      if (ptid < 64) {
        const int t = ptid;
        float sum = 0.f;
#pragma unroll 1
        for (int p = 0; p < 2; ++p) {
          float pv[32];
          tc::tmem_ld32(tmem + lane_off + TM_S + 32 * p, pv);
          tc::tmem_wait_ld();
          const uint32_t prow = sb + OFF_W + p * 8192 + t * 128;
#pragma unroll
          for (int cc = 0; cc < 8; ++cc) {
            const float* v = pv + 4 * cc;
            sum += (v[0] + v[1]) + (v[2] + v[3]);
            st_tf32x4(prow + ((cc ^ (t & 7)) << 4), v[0], v[1], v[2], v[3]);
          }
        }
        if (nonfinite(sum)) {
#pragma unroll 1
          for (int p = 0; p < 2; ++p)
#pragma unroll
            for (int cc = 0; cc < 8; ++cc)
              st_tf32x4(sb + OFF_W + p * 8192 + t * 128 + ((cc ^ (t & 7)) << 4), kInf, kInf, kInf, kInf);
        }
      }
      tc::tc_fence_before();
      tc::fence_proxy_async_smem();
      tc::named_bar(1, 128);
      if (ptid == 0) {
        tc::mbar_arrive(bar(B_S_EMPTY));
        tc::mbar_arrive(bar(B_PT_READY));
        GDN_TRACE(c, 6);
      }
      if (ptid < 32 && c + 1 < nC) publish_gates(c + 1);
      // A2 rows 0..63 = P T_b are written by the chain's O warps once the MMA is done
      stop = vote_abort(1, 128, abort_flag);
      if (ptid == 0) {
        tc::mbar_arrive(bar(B_PRE_FULL));
        GDN_TRACE(c, 8);
      }
    }
  } else {
    // ------------------------------- chain warpgroups ----------------------------------------
    const int hh = (warp - 8) >> 2, q = warp & 3, r = 32 * q + lane;
    const uint32_t lane_off = static_cast<uint32_t>(32 * q) << 16;
    const uint32_t tcol = 64 * hh;                       // this half's TMEM / value columns
    const uint32_t mb = sb + OFF_MB + hh * 16384, rd = sb + OFF_RD + hh * 16384;
    const uint32_t vb = sb + OFF_V + hh * 8192;
    const uint32_t id_wg = 2 + 3 * hh, id_lo = 3 + 3 * hh, id_hi = 4 + 3 * hh;
    const long head = (long)bq * Hv + h;
    const bool leader = (q == 0 && lane == 0);
    [[maybe_unused]] const int ev = 10 * hh;
    // 32 columns (32p ..) of M row r (this half) for the X MMA: one round-to-nearest bf16 copy in Mb,
    // or (kSplitX) a hi + lo pair, hi into Mb and lo into the R' buffer
    auto store_m32 = [&](const float (&m)[32], int p) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t sw = tc::sw128(r, 4 * p + j);
        if constexpr (kSplitX) {
          st_split8(mb + sw, rd + sw, m + 8 * j);
        } else {
          const float* v = m + 8 * j;
          tc::st_shared_v4(mb + sw, tc::pack_bf16(v[0], v[1]), tc::pack_bf16(v[2], v[3]),
                           tc::pack_bf16(v[4], v[5]), tc::pack_bf16(v[6], v[7]));
        }
      }
    };
    // A2 rows 0..63 = P T_b of chunk cn (O warps, q < 2): row r = TMEM lane r, this half takes
    // columns 32 hh .. 32 hh + 31 of the 64
    auto a2_top = [&](int cn) {
      tc::mbar_wait(bar(B_PT_FULL), cn & 1, abort_flag, kBudget);
      if (cn >= 1) tc::mbar_wait(bar(B_O_DONE), (cn - 1) & 1, abort_flag, kBudget);
      if (leader && hh == 0) GDN_TRACE(cn, 16);
      tc::tc_fence_after();
      float pv[32];
      tc::tmem_ld32(tmem + lane_off + TM_PT + 32 * hh, pv);
      tc::tmem_wait_ld();
      const uint32_t a2_row = sb + OFF_A2 + r * 128;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t sw = ((4 * hh + j) ^ (r & 7)) << 4;
        st_split8(a2_row + sw, a2_row + 16384 + sw, pv + 8 * j);
      }
      tc::fence_proxy_async_smem();
      tc::tc_fence_before();
      tc::named_bar(id_lo, 64);
      if (leader) {
        if (hh == 0) GDN_TRACE(cn, 17);
        tc::mbar_arrive(bar(B_PT_EMPTY));
        tc::mbar_arrive(bar(B_PRE_FULL));
      }
    };
    bool stop = false;
    {
      float m[64];
      if (S0) {
        const float4* src = reinterpret_cast<const float4*>(S0 + (head * 128 + r) * 128 + tcol);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float4 v = src[i];
          m[4 * i] = v.x; m[4 * i + 1] = v.y; m[4 * i + 2] = v.z; m[4 * i + 3] = v.w;
        }
      } else {
#pragma unroll
        for (int i = 0; i < 64; ++i) m[i] = 0.f;
      }
      store_m32(*reinterpret_cast<const float(*)[32]>(&m[0]), 0);
      store_m32(*reinterpret_cast<const float(*)[32]>(&m[32]), 1);
      tc::mbar_wait(bar(B_GATE + 0), 0, abort_flag, kBudget);
      const float gl = gslot(0)[64 + 63];
#pragma unroll
      for (int i = 0; i < 64; ++i) m[i] *= gl;
      tmem_st64(tmem + lane_off + TM_M + tcol, m);
      tc::tmem_wait_st();
      tc::fence_proxy_async_smem();
      tc::tc_fence_before();
      stop = vote_abort(id_wg, 128, abort_flag);
      if (leader) {
        tc::mbar_arrive(bar(B_M_READY));
        tc::mbar_arrive(bar(B_M_SCALED));
      }
      if (!stop && q < 2) a2_top(0);
    }

    for (int c = 0; c < nC && !stop; ++c) {
      const float* gGam = gslot(c) + 64;
      const float* gKt = gGam + 64;
      if (q >= 2) {
        // R' = V - gamma (K M) for token t (tf32), then ktil Delta as bf16 hi + lo
        const int t = r - 64;
        tc::mbar_wait(bar(B_X_FULL), c & 1, abort_flag, kBudget);
        tc::mbar_wait(bar(B_GATE + c % 3), (c / 3) & 1, abort_flag, kBudget);
        tc::mbar_wait(bar(B_V_FULL), c & 1, abort_flag, kBudget);
        if (q == 2 && lane == 0) GDN_TRACE(c, 30 + ev);
        tc::tc_fence_after();
        const float g = gGam[t];
#pragma unroll 1
        for (int p = 0; p < 2; ++p) {            // value columns 32p .. 32p+31 of this half
          float x[32];
          tc::tmem_ld32(tmem + lane_off + TM_X + tcol + 32 * p, x);
          uint4 u[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) u[j] = tc::ld_shared_v4(vb + tc::sw128(t, 4 * p + j));
          tc::tmem_wait_ld();
          if (p == 0 && hh == 0 && q == 2 && lane == 0) GDN_TRACE(c, 55);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float* xx = x + 8 * j;
            const uint32_t w4[4] = {u[j].x, u[j].y, u[j].z, u[j].w};
            float rv[8];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              rv[2 * e] = fmaf(-g, xx[2 * e], tc::bf16lo(w4[e]));
              rv[2 * e + 1] = fmaf(-g, xx[2 * e + 1], tc::bf16hi(w4[e]));
            }
            // MN-major bf16 B operand of Y: row t (K), 16-byte chunk 4p + j of this half's columns
            const uint32_t sw = tc::sw128(t, 4 * p + j);
            st_split8(rd + sw, rd + 8192 + sw, rv);
          }
          if (hh == 0 && q == 2 && lane == 0) GDN_TRACE(c, 56 + p);
        }
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        if (hh == 0 && q == 2 && lane == 0) GDN_TRACE(c, 58);
        tc::named_bar(id_hi, 64);
        if (q == 2 && lane == 0) {
          GDN_TRACE(c, 31 + ev);
          tc::mbar_arrive(bar(B_R_FULL));
          tc::mbar_arrive(bar(B_V_EMPTY));
        }
        tc::mbar_wait(bar(B_Y_FULL), c & 1, abort_flag, kBudget);
        if (q == 2 && lane == 0) GDN_TRACE(c, 32 + ev);
        tc::tc_fence_after();
        const float kt = gKt[t];
#pragma unroll 1
        for (int p = 0; p < 2; ++p) {
          float y[32];
          tc::tmem_ld32(tmem + lane_off + TM_Y + tcol + 32 * p, y);
          tc::tmem_wait_ld();
          if (p == 0 && hh == 0 && q == 2 && lane == 0) GDN_TRACE(c, 59);
#pragma unroll
          for (int i = 0; i < 32; ++i) y[i] *= kt;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint32_t sw = tc::sw128(t, 4 * p + j);
            st_split8(rd + sw, rd + 8192 + sw, y + 8 * j);
          }
        }
        if (hh == 0 && q == 2 && lane == 0) GDN_TRACE(c, 60);
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        if (hh == 0 && q == 2 && lane == 0) GDN_TRACE(c, 61);
        tc::named_bar(id_hi, 64);
        if (q == 2 && lane == 0) {
          GDN_TRACE(c, 33 + ev);
          tc::mbar_arrive(bar(B_D_FULL));
        }
      } else {
        // o_t = gamma_t scale (Q M)_t + (P Delta)_t, staged in shared memory for a TMA store
        const int t = r;
        tc::mbar_wait(bar(B_X_FULL), c & 1, abort_flag, kBudget);
        tc::mbar_wait(bar(B_GATE + c % 3), (c / 3) & 1, abort_flag, kBudget);
        tc::mbar_wait(bar(B_Y_FULL), c & 1, abort_flag, kBudget);
        if (leader) GDN_TRACE(c, 34 + ev);
        tc::tc_fence_after();
        const float g = gGam[t] * scale;
        // bf16: one [64 t][64 dv] tile per half; fp32: two [64 t][32 dv] tiles per half
        const uint32_t stage = sb + OFF_A2 + hh * (kF32 ? 16384 : 8192);
#pragma unroll 1
        for (int p = 0; p < 4; ++p) {            // value columns 16p .. 16p+15 of this half
          float x[16], y[16];
          tmem_ld16(tmem + lane_off + TM_X + tcol + 16 * p, x);
          tmem_ld16(tmem + lane_off + TM_Y + tcol + 16 * p, y);
          tc::tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) y[i] = fmaf(g, x[i], y[i]);
          if constexpr (kF32) {                  // tile p / 2, 16-byte chunks 4 (p % 2) ..
#pragma unroll
            for (int j = 0; j < 4; ++j)
              tc::st_shared_v4(stage + (p >> 1) * 8192 + tc::sw128(t, 4 * (p & 1) + j),
                               __float_as_uint(y[4 * j]), __float_as_uint(y[4 * j + 1]),
                               __float_as_uint(y[4 * j + 2]), __float_as_uint(y[4 * j + 3]));
          } else {                               // 16-byte chunks 2p, 2p + 1
#pragma unroll
            for (int j = 0; j < 2; ++j)
              tc::st_shared_v4(stage + tc::sw128(t, 2 * p + j), tc::pack_bf16(y[8 * j], y[8 * j + 1]),
                               tc::pack_bf16(y[8 * j + 2], y[8 * j + 3]),
                               tc::pack_bf16(y[8 * j + 4], y[8 * j + 5]),
                               tc::pack_bf16(y[8 * j + 6], y[8 * j + 7]));
          }
        }
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        tc::named_bar(id_lo, 64);
        if (leader) {
          GDN_TRACE(c, 35 + ev);
          if constexpr (kF32) {
            tc::tma_store_4d(&tmo, stage, 64 * hh, h, c * C, bq);
            tc::tma_store_4d(&tmo, stage + 8192, 64 * hh + 32, h, c * C, bq);
          } else {
            tc::tma_store_4d(&tmo, stage, 64 * hh, h, c * C, bq);
          }
          tc::bulk_commit();
          tc::bulk_wait_read_all();
          tc::mbar_arrive(bar(B_O_DONE));
          GDN_TRACE(c, 36 + ev);
        }
      }
      // M <- gamma_last M + K^T (ktil Delta) is now in TMEM (row r of this half).  Its bf16 pair
      // goes out first (the next X needs it); then TMEM is scaled by the next chunk's
      // gamma_last for the next update, which waits for that separately.
      tc::mbar_wait(bar(B_D3_FULL), c & 1, abort_flag, kBudget);
      if (leader) GDN_TRACE(c, 37 + ev);
      tc::tc_fence_after();
      if (c + 1 < nC) {
        float m[64];
        tmem_ld64(tmem + lane_off + TM_M + tcol, m);
        tc::mbar_wait(bar(B_GATE + (c + 1) % 3), ((c + 1) / 3) & 1, abort_flag, kBudget);
        const float gl = gslot(c + 1)[64 + 63];
        tc::tmem_wait_ld();
        if (leader && hh == 0) GDN_TRACE(c, 50);
        store_m32(*reinterpret_cast<const float(*)[32]>(&m[0]), 0);
        store_m32(*reinterpret_cast<const float(*)[32]>(&m[32]), 1);
        tc::fence_proxy_async_smem();
        tc::named_bar(id_wg, 128);
        if (leader) {
          GDN_TRACE(c, 38 + ev);
          tc::mbar_arrive(bar(B_M_READY));
        }
#pragma unroll
        for (int i = 0; i < 64; ++i) m[i] *= gl;
        tmem_st64(tmem + lane_off + TM_M + tcol, m);
        tc::tmem_wait_st();
        if (leader && hh == 0) GDN_TRACE(c, 51);
      } else if (S_T && !*abort_flag) {
        float m[64];
        tmem_ld64(tmem + lane_off + TM_M + tcol, m);
        tc::tmem_wait_ld();
        float4* dst = reinterpret_cast<float4*>(S_T + (head * 128 + r) * 128 + tcol);
#pragma unroll
        for (int i = 0; i < 16; ++i)
          dst[i] = make_float4(m[4 * i], m[4 * i + 1], m[4 * i + 2], m[4 * i + 3]);
      }
      tc::tc_fence_before();
      stop = vote_abort(id_wg, 128, abort_flag);
      if (leader) {
        if (hh == 0) GDN_TRACE(c, 52);
        tc::mbar_arrive(bar(B_M_SCALED));
      }
      if (!stop && q < 2 && c + 1 < nC) a2_top(c + 1);
    }
    if (leader) tc::bulk_wait_all();               // every o tile has reached global memory
  }

  tc::tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) GDN_TRACE_G(nC - 1, 11);
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

// [B, T, H, 128] tensor of 2- or 4-byte elements, boxes of 128 bytes (head dim) x 64 tokens,
// 128-byte swizzle.  Loads past T read zeros (the ragged last chunk); stores past T are clipped.
inline bool make_tile_map(CUtensorMap* m, const void* base, int H, int T, int B, bool f32) {
  auto enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t es = f32 ? 4 : 2;
  cuuint64_t dims[4] = {128, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
  cuuint64_t strides[3] = {128 * es, (cuuint64_t)H * 128 * es, (cuuint64_t)T * H * 128 * es};
  cuuint32_t box[4] = {f32 ? 32u : 64u, 1, 64, 1};
  cuuint32_t estr[4] = {1, 1, 1, 1};
  return enc(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4,
             const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Bytes of the T_b hand-over buffer between the pre-pass and the recurrence.
inline size_t scratch_bytes(int B, int T, int Hv) {
  const size_t nC = (size_t)(T + C - 1) / C;
  return (size_t)B * Hv * nC * kTbFloats * sizeof(float);
}

template <typename Tout>
gdn_status launch(const void* q, const void* k, const void* v, const float* la, const float* be,
                  const float* S0, Tout* o, float* S_T, int B, int T, int Hk, int Hv, float scale,
                  float* tb, cudaStream_t st) {
  CUtensorMap mq, mk, mv, mo;
  if (!make_tile_map(&mq, q, Hk, T, B, false) || !make_tile_map(&mk, k, Hk, T, B, false) ||
      !make_tile_map(&mv, v, Hv, T, B, false) ||
      !make_tile_map(&mo, o, Hv, T, B, sizeof(Tout) == 4))
    return GDN_ERR_CUDA;
  auto kern = chunk_fwd_tc_kernel<Tout>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_ALLOC) !=
      cudaSuccess)
    return GDN_ERR_CUDA;
  if (cudaFuncSetAttribute(tb_prepass_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           PP_SMEM) != cudaSuccess)
    return GDN_ERR_CUDA;
  const long grid = (long)B * Hv;
  const int nC = (T + C - 1) / C;
  if (grid > 0x7fffffffL || Hv > 65535 || B > 65535) return GDN_ERR_UNSUPPORTED;
  tb_prepass_kernel<<<dim3(nC, Hv, B), PP_THREADS, PP_SMEM, st>>>(
      static_cast<const __nv_bfloat16*>(k), la, be, tb, T, Hk, Hv);
  if (cudaGetLastError() != cudaSuccess) return GDN_ERR_CUDA;
  kern<<<(unsigned)grid, kThreads, SMEM_ALLOC, st>>>(mq, mk, mv, mo, la, be, tb, S0, S_T, T, Hk,
                                                     Hv, scale);
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

// Scratch bytes of the tensor-core forward (the T_b hand-over buffer), 256-byte aligned.
inline size_t tc_chunk_scratch_bytes(int B, int T, int Hv) { return tcf::scratch_bytes(B, T, Hv); }

inline gdn_status tc_chunk_launch(const void* q, const void* k, const void* v, const float* la,
                                  const float* be, const float* S0, void* o, float* S_T, int B,
                                  int T, int Hk, int Hv, float scale, void* scratch,
                                  cudaStream_t st) {
  return tcf::launch<__nv_bfloat16>(q, k, v, la, be, S0, static_cast<__nv_bfloat16*>(o), S_T, B,
                                    T, Hk, Hv, scale, static_cast<float*>(scratch), st);
}

inline gdn_status tc_chunk_launch_f32out(const void* q, const void* k, const void* v,
                                         const float* la, const float* be, const float* S0,
                                         float* o, float* S_T, int B, int T, int Hk, int Hv,
                                         float scale, void* scratch, cudaStream_t st) {
  return tcf::launch<float>(q, k, v, la, be, S0, o, S_T, B, T, Hk, Hv, scale,
                            static_cast<float*>(scratch), st);
}

}  // namespace gdn
