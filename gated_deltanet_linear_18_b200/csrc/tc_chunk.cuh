// Chunked forward of the gated delta rule on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
// Shapes: d_k = d_v = 128, chunk C = 64, bf16 q/k/v, fp32 gates and state.
//
// Per value head and chunk, with the chunk-start state M = S^T (128 x 128, fp32), the chunk form of
// the recurrence ("Chapitre 16 - Assembler un système de type Kimi K3", 16.2: matrix operations
// inside each block, state handed from block to block) splits into
//   a state-independent part, for every chunk at once in a pre-pass (many small CTAs):
//     G = cumsum(log alpha), gamma = exp(G), ktil_t = exp(G_last - G_t)
//     P = lower_incl(exp(G_i - G_j) q_i.k_j) * scale,  A = strict_lower(beta_i exp(G_i - G_j) k_i.k_j)
//     T_b = (I + A)^-1 diag(beta)                     (fp32, blocked by 16)
//     PT = P T_b,  W = (diag(ktil) K)^T T_b           (64 x 64 and 128 x 64)
//   and the state-dependent chain, one CTA per (batch, value head), all 128 value columns at once:
//     X = [Q; K] M                           (bf16 MMA, 128x128x128, M as one bf16 copy or a pair)
//     R' = V - diag(gamma) (K M)             (rows 64..127 of X)
//     o = diag(gamma) scale (Q M) + PT R'    (rows 0..63 of X;  Y = PT R', bf16 MMA 128x128x64)
//     M <- gamma_last M + W R'               (bf16 MMA accumulating onto gamma_last M in TMEM)
// which is the token recurrence reorganised exactly: Delta = T_b R' has rows beta_t (v_t - alpha_t
// S_{t-1} k_t), and M's update K^T diag(ktil) Delta is W R'.  Accumulations and the master state are
// fp32.  The operands that carry the state through the chain (PT, W, R') are bf16 pairs hi + lo
// (|x - hi - lo| < 2^-14 |x|) multiplied term by term (hi.hi + lo.hi + hi.lo): with plain bf16, or
// even tf32, the state's largest entries drift by a few percent (about one percent for tf32) of its
// RMS.  The splits are integer mask / byte-permute operations (the conversion instructions run at a
// quarter of the ALU rate).
//
// The pre-pass hands each chunk to the recurrence as its MMA operands themselves (48 KB of
// swizzled tiles plus gamma), so the recurrence's critical path holds only X, R', the state
// update and the state's bf16 copy.  Recurrence CTA, 384 threads in specialised warps:
//   warp 0        TMA producer (the Q, K tile of the next chunk as soon as X has read the last;
//                 the chunks' operand tiles double-buffered)
//   warp 1        TMEM owner; issues every MMA: X of chunk c, Y of chunk c - 1 (from the other
//                 of two R' buffers, while R' of chunk c is formed), the state update of c
//   warps 4-7     value columns 0..63; warps 8-11 columns 64..127.  Lanes 0..63 of each group
//                 make o, lanes 64..127 make R' (V comes straight into registers one chunk
//                 ahead); all four warps copy the updated state out of TMEM.
// The fp32 master state lives in TMEM (the update MMA accumulates onto it); o leaves through
// shared memory (staged in the chunk's PT tiles once Y has read them) and TMA stores.  Every
// wait is bounded (about 2 s): on expiry the CTA records the library's timeout bit, every role
// leaves its loop at the next uniform check point, in-flight TMA copies and MMAs are drained,
// TMEM is released and the kernel returns.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "common.cuh"
#include "tc_ptx.cuh"

namespace gdn {
namespace tcf {

constexpr int C = 64;
constexpr int kThreads = 384;
constexpr uint64_t kBudget = 4000000000ull;   // wait budget in SM cycles (about 2 s)

// shared memory map (bytes from a 1024-aligned base); every MMA tile is 128-byte swizzled
constexpr uint32_t OFF_QK = 0;          // 32 KB: kb0 [Q 64 rows | K 64 rows], kb1 [...]
constexpr uint32_t OFF_RD = 32768;      // 2 buffers (chunk parity) x 32 KB, per column half 16 KB:
constexpr uint32_t RD_BUF = 32768;      // R' bf16 hi [64 t][128 B] + lo; with a split X, before
                                        // R' of a chunk, the bf16 low part of M for its X
constexpr uint32_t OFF_MB = 98304;      // 32 KB, per column half 16 KB: bf16 M [128 dk][128 B]
constexpr uint32_t OFF_PW = 131072;     // 2 slots x 48 KB: a chunk's PT hi, PT lo, W hi, W lo
constexpr uint32_t PW_SLOT = 49152;     // after Y (and the update) the o tile is staged there
constexpr uint32_t OFF_BAR = OFF_PW + 2 * PW_SLOT;
constexpr int NBAR = 22;
constexpr uint32_t OFF_MISC = OFF_BAR + NBAR * 8;   // +0 TMEM base, +4 abort flag
constexpr uint32_t OFF_GAM = OFF_MISC + 16;         // 2 slots (chunk parity) x gamma_t, 64 fp32
constexpr uint32_t SMEM_BYTES = OFF_GAM + 2 * 256;
constexpr uint32_t SMEM_ALLOC = SMEM_BYTES + 1024;
static_assert(SMEM_ALLOC <= 232448, "shared memory budget");

// TMEM columns (512 allocated, 128 lanes x 32 bit): X double-buffered by chunk parity
constexpr uint32_t TM_X = 0, TM_Y = 256, TM_M = 384;

// mbarriers
// The chunk's operand slot arrives in two parts with their own barriers: W (for the state update,
// on the critical path) is reloaded as soon as the update has read it; PT (for o) once o has
// left the slot.
enum : int {
  B_QK_FULL = 0, B_QK_EMPTY, B_W_FULL = 2, B_W_EMPTY = 4, B_P_FULL = 6, B_P_EMPTY = 8,
  B_X_FULL = 10, B_R_FULL, B_D3_FULL, B_Y_FULL, B_Y_EMPTY, B_M_READY, B_M_SCALED, B_DRAIN,
  B_G_FULL = 18, B_G_EMPTY = 20, B_END = 22
};
static_assert(B_END <= NBAR, "barrier map");

constexpr uint32_t ID_X = tc::idesc_bf16(128, 128, false, true);
constexpr uint32_t ID_Y = tc::idesc_bf16(128, 128, false, true);

// Optional per-chunk timestamps for studying the pipeline (compiled only with GDN_TC_TRACE):
// slot (block, chunk, event) of a caller-provided buffer receives clock64().
#ifdef GDN_TC_TRACE
__device__ unsigned long long* g_tc_trace = nullptr;
// the buffer pointer is read once per kernel (GDN_TRACE_INIT), so a timestamp costs one store
#define GDN_TRACE_INIT unsigned long long* const tr_buf_ = g_tc_trace
#define GDN_TRACE(c, ev)                                                              \
  do {                                                                                \
    if (tr_buf_) tr_buf_[((size_t)blockIdx.x * nC + (c)) * 64 + (ev)] = clock64();    \
  } while (0)
// same with the global nanosecond timer (comparable across SMs)
#define GDN_TRACE_G(c, ev)                                                            \
  do {                                                                                \
    if (tr_buf_) tr_buf_[((size_t)blockIdx.x * nC + (c)) * 64 + (ev)] = tc::globaltimer_ns(); \
  } while (0)
#define GDN_TRACE_PP(ev)                                                               \
  do {                                                                                 \
    if (tr_buf_ && threadIdx.x == 0)                                                   \
      tr_buf_[(((size_t)blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x) * 64 + (ev)] = clock64(); \
  } while (0)
// the pre-pass's slot receives a value (the SM, the global time) instead of clock64()
#define GDN_TRACE_PPV(ev, val)                                                         \
  do {                                                                                 \
    if (tr_buf_ && threadIdx.x == 0)                                                   \
      tr_buf_[(((size_t)blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x) * 64 + (ev)] = (val); \
  } while (0)
// clock64() as seen by thread t
#define GDN_TRACE_PPT(ev, t)                                                           \
  do {                                                                                 \
    if (tr_buf_ && threadIdx.x == (t))                                                 \
      tr_buf_[(((size_t)blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x) * 64 + (ev)] = clock64(); \
  } while (0)
// inside the solve (a device function: the buffer pointer is read where it is used)
#define GDN_TRACE_SOLVE(ev)                                                            \
  do {                                                                                 \
    if (g_tc_trace && threadIdx.x == 0)                                                \
      g_tc_trace[(((size_t)blockIdx.z * gridDim.y + blockIdx.y) * gridDim.x + blockIdx.x) * 64 + (ev)] = clock64(); \
  } while (0)
#else
#define GDN_TRACE_SOLVE(ev) do {} while (0)
#define GDN_TRACE_INIT do {} while (0)
#define GDN_TRACE_PPT(ev, t) do {} while (0)
#define GDN_TRACE_PPV(ev, val) do {} while (0)
#define GDN_TRACE_PP(ev) do {} while (0)
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
// The solve's scratch: A's ten blocks, then the six off-diagonal blocks of T; T's diagonal blocks
// take the place of A's.
constexpr uint32_t SOLVE_BYTES = 16 * BSZ * 4;
__device__ __forceinline__ uint32_t blkT(uint32_t base, int i, int k) {
  return i == k ? blk(base, i, i)
                : base + (uint32_t)((10 + i * (i - 1) / 2 + k) * BSZ * 4);
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

// T = (I + A)^-1 for a 64 x 64 strictly lower A (128 threads = 4 warps, named barriers 1 and 3),
// blocked by 16:  D_b = (I + A_bb)^-1 by forward substitution (one column per thread);  At_ik = D_i A_ik;
// U = (I + At)^-1 (U_ii = I; At is block-nilpotent, so U is closed-form in At's blocks);
// T_ik = U_ik D_k.   (I + A = blockdiag(I + A_bb) (I + At), so T = U D.)  The block products run
// as warp MMAs on 16 x 8 half blocks.  On return the off-diagonal blocks of T are in `tv`: item m
// of warp w is half block hp = w + 4 m (block bi = hp / 2, columns 8 (hp % 2) ..) as a C fragment;
// the diagonal blocks D_b are in blkT(s, b, b), over A_bb.  A's other blocks are overwritten.
__device__ __forceinline__ void solve_unit_lower(uint32_t s, int ptid, float (&tv)[3][4]) {
  const uint32_t sA = s;
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
    GDN_TRACE_SOLVE(23);
    tc::named_bar(3, 64);                             // every row of A_bb read: D_b replaces it
    const uint32_t Tb = blkT(s, b, b);
#pragma unroll
    for (int i = 0; i < 16; ++i) tc::sts1(at(Tb, i, col), x[i]);
  }
  tc::named_bar(1, 128);
  GDN_TRACE_SOLVE(24);
  const int w = ptid >> 5, lane = ptid & 31, g = lane >> 2, t = lane & 3;
  {                                                   // At_ik = D_i A_ik, into T's off-diagonal
    Tile tl[3];
    float acc[3][4] = {};
#pragma unroll
    for (int m = 0; m < 3; ++m) {
      const int hp = w + 4 * m, bi = hp >> 1, n0 = (hp & 1) * 8;
      const int i = blk_i(bi), k = blk_k(bi, i);
      tl[m] = Tile{blkT(s, i, i), blk(sA, i, k), n0};
    }
    mma_tiles(tl, g, t, acc);
#pragma unroll
    for (int m = 0; m < 3; ++m) {
      const int bi = (w + 4 * m) >> 1;
      const int i = blk_i(bi), k = blk_k(bi, i);
      st_frag(blkT(s, i, k), tl[m].n0, g, t, acc[m]);
    }
  }
  tc::named_bar(1, 128);
  GDN_TRACE_SOLVE(25);
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
      ld_frag(blkT(s, oi, ok), n0, g, t, acc[m]);
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[m][e] = -acc[m][e];
      tl[m] = Tile{blkT(s, oi, xk), blkT(s, xk, ok), n0};
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
  GDN_TRACE_SOLVE(26);
  if (w < 2) {                                        // U_30 = V_30 - At_32 U_20
    const int n0 = 8 * w;
    const Tile tl[1] = {Tile{blkT(s, 3, 2), blk(sA, 2, 0), n0}};
    float acc[1][4] = {}, v[4];
    ld_frag(blk(sA, 3, 0), n0, g, t, v);
    mma_tiles(tl, g, t, acc);
#pragma unroll
    for (int e = 0; e < 4; ++e) v[e] -= acc[0][e];
    st_frag(blk(sA, 3, 0), n0, g, t, v);
  }
  tc::named_bar(1, 128);
  GDN_TRACE_SOLVE(27);
  {                                                   // T_ik = U_ik D_k (U = -At next to diag)
    Tile tl[3];
    float acc[3][4] = {};
#pragma unroll
    for (int m = 0; m < 3; ++m) {
      const int hp = w + 4 * m, bi = hp >> 1, n0 = (hp & 1) * 8;
      const int i = blk_i(bi), k = blk_k(bi, i);
      tl[m] = Tile{(i == k + 1) ? blkT(s, i, k) : blk(sA, i, k), blkT(s, k, k), n0};
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

// +infinity, written over the operands of a chunk whose P or A is not finite.
constexpr float kInf = __builtin_huge_valf();

// x = hi + lo + e with hi = x truncated to bf16 and lo = (x - hi) truncated to bf16, |e| < 2^-14 |x|;
// returns the packed (low half = first value) bf16 pairs of two values.  NaN and infinities stay
// non-finite in hi or lo.
__device__ __forceinline__ void split2(float a, float b, uint32_t& hi2, uint32_t& lo2) {
  const uint32_t ua = __float_as_uint(a), ub = __float_as_uint(b);
  float la, lb;
  tc::f2_get(tc::sub2(tc::f2(a, b), tc::f2(__uint_as_float(ua & 0xFFFF0000u),
                                           __uint_as_float(ub & 0xFFFF0000u))), la, lb);
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

// ------------------------------------------------------------------------------------------
// Where sequence s lives.  Fixed length (cu == nullptr): batch s of [B, T, ...] tensors.  Packed
// (cu != nullptr): tokens cu[s] .. cu[s + 1] - 1 of [1, T, ...] tensors (T = total tokens); the
// offsets come from device memory, so they are clamped to the tensor and the length to max_len,
// which keeps every access in bounds whatever they hold.
// ------------------------------------------------------------------------------------------
struct SeqSpan {
  int tok0;      // first token in the tensor map's token dimension
  int len;       // tokens of the sequence
  int bcoord;    // tensor map batch coordinate
  long row0;     // row of the first token in [rows, heads, d] tensors and [rows, heads] gates
};
__device__ __forceinline__ SeqSpan seq_span(const int* __restrict__ cu, int s, int T, int max_len) {
  if (!cu) return SeqSpan{0, T, s, (long)s * T};
  const int a = min(max(cu[s], 0), T);
  const int b = min(max(cu[s + 1], a), min(T, a + max_len));
  return SeqSpan{a, b - a, 0, (long)a};
}

// ------------------------------------------------------------------------------------------
// pre-pass: the state-independent operands of every (batch, value head, chunk), independently
// ------------------------------------------------------------------------------------------
// With T_b = (I + A)^-1 diag(beta), P = lower_incl(exp(G_i - G_j) q_i.k_j) scale and
// ktil_t = exp(G_last - G_t), the chunk needs from outside the state only
//   PT = P T_b      (64 x 64: o = gamma scale Q M + PT R')
//   W  = K^T diag(ktil) T_b   (128 x 64: M <- gamma_last M + W R')
// since Delta = T_b R'.  Neither depends on the state, so one small CTA per chunk computes them
// ahead of the recurrence, on the tensor cores: S = [Q; K] K^T (bf16 MMA into TMEM), P and A from
// S with the gates (one TMEM row per thread), the blocked solve, then PT = P T_b and, through the
// same pair of operand tiles once PT has read them, W = K^T (ktil T_b), as bf16 MMAs on hi + lo
// splits (hi.hi + lo.hi + hi.lo for PT; K is exact, so two terms for W).  The result goes to HBM
// as the recurrence's MMA operands themselves: per chunk 48 KB of 128-byte-swizzled K-major bf16
// tiles, PT hi [64 rows][128 B], PT lo, W hi [128 rows][128 B], W lo, followed by
// gamma_t = exp(G_t) (64 fp32).  A chunk whose P or A holds a NaN or an infinity gets +inf in
// every tile, so the recurrence still sees a non-finite value.
constexpr int kPwTiles = 49152;              // the four operand tiles of a chunk
constexpr int kPwBytes = kPwTiles + 256;     // + gamma_t = exp(G_t), 64 fp32
constexpr int PP_THREADS = 256;   // warps w and w + 4 share TMEM lane quadrant w, one column half each
constexpr uint32_t PP_QK = 0;        // 32 KB: Q cols 0..63 | K cols 0..63 | Q 64..127 | K 64..127;
                                     // P hi over the first Q box, P lo over the second
constexpr uint32_t PP_TB = 32768;    // solve scratch, then 2 x 8 KB MN-major B tiles [64 rows][128 B]:
                                     // T_b hi, T_b lo, later ktil T_b hi, ktil T_b lo
constexpr uint32_t PP_G = PP_TB + SOLVE_BYTES;   // G'[64], beta[64], ktil[64], flag, abort, then
                                                 // at float 256 E[4][64]; barriers at +2048
constexpr uint32_t PP_BAR = PP_G + 2048;
constexpr uint32_t PP_SMEM = PP_BAR + 64 + 1024;   // + alignment slack (four CTAs per SM)
static_assert(SOLVE_BYTES >= 16384, "the B tile pair fits the solve scratch's space");
static_assert(4 * (PP_SMEM + 1024) <= 233472, "four pre-pass CTAs per SM");
constexpr uint32_t ID_S = tc::idesc_bf16(128, 64, false, false);   // [Q; K] K^T
constexpr uint32_t ID_PT = tc::idesc_bf16(128, 64, false, true);   // P T_b (rows 64..127 unused)
constexpr uint32_t ID_W = tc::idesc_bf16(128, 64, true, true);     // K^T (ktil T_b)

// Byte offset of element (r, j), j < 64, of a [rows][128 B] bf16 tile, 128-byte swizzle.
__device__ __forceinline__ uint32_t sw_elem(int r, int j) {
  return (uint32_t)(r * 128 + ((((j >> 3) ^ (r & 7))) << 4) + (j & 7) * 2);
}
// Values (row, n), (row, n + 1) (n even) into the B tile pair (hi at tb, lo at tb + 8192).
__device__ __forceinline__ void store_b_pair(uint32_t tb, int row, int n, float a, float b) {
  uint32_t h, l;
  split2(a, b, h, l);
  const uint32_t o = tb + sw_elem(row, n);
  tc::sts1(o, __uint_as_float(h));
  tc::sts1(o + 8192, __uint_as_float(l));
}

// grid (Hv, nCmax, sequences), 256 threads; thread r owns TMEM lane r % 128 and column half r / 128
// of that lane's row (the solve runs on the first 128).  CTAs past the end of their sequence
// return at once.
__global__ void __launch_bounds__(PP_THREADS, 4)
pw_prepass_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                  const float* __restrict__ log_alpha, const float* __restrict__ beta,
                  uint8_t* __restrict__ pw, int T, int Hk, int Hv, float scale,
                  const int* __restrict__ cu, int max_len, const __nv_bfloat16* __restrict__ ba) {
  GDN_TRACE_INIT;
  GDN_TRACE_PP(63);
  extern __shared__ __align__(1024) uint8_t pp_raw[];
  uint8_t* smem = pp_raw + ((1024u - (tc::smem_u32(pp_raw) & 1023u)) & 1023u);
  const uint32_t sb = tc::smem_u32(smem);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.x, c = blockIdx.y, sq = blockIdx.z, nC = gridDim.y;
  const SeqSpan sp = seq_span(cu, sq, T, max_len);
  if (c * C >= sp.len) return;                        // (uniform: before any barrier)
  const int vrows = min(C, sp.len - c * C);           // tokens of this chunk in the sequence
  const int hk = h / (Hv / Hk);
  const long t0 = (long)c * C;
  float* gG = reinterpret_cast<float*>(smem + PP_G);
  float* gB = gG + 64;
  float* gKt = gG + 128;
  volatile int* flag = reinterpret_cast<volatile int*>(gG + 192);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(gG + 193);
  const uint32_t tma_bar = sb + PP_BAR, mma_bar = sb + PP_BAR + 8, pt_bar = sb + PP_BAR + 24;
  const uint32_t qk = sb + PP_QK, tb = sb + PP_TB;
  uint8_t* rec = pw + (((long)sq * Hv + h) * nC + c) * (long)kPwBytes;

  // The chunk's gates are loaded first, by warps 2-3 (token t0 + gi), so that the loads are in
  // flight during the setup and the tile load; thread 0 issues the tile load before the TMEM
  // allocation and the S MMA as soon as the tile is in.
  const int gi = tid - 64;
  const bool gw = gi >= 0 && gi < 64;                 // a gate thread
  float la = 0.f, bt = 0.f;
  if (gw && t0 + gi < sp.len) {
    const long r = sp.row0 + t0 + gi;
    if (ba) {
      bt = __bfloat162float(ba[r * 2 * Hv + h]);      // b, a: converted below
      la = __bfloat162float(ba[r * 2 * Hv + Hv + h]);
    } else {
      la = log_alpha[r * Hv + h];
      bt = beta[r * Hv + h];
    }
  }
  if (tid == 0) {
    tc::mbar_init(tma_bar, 1);
    tc::mbar_init(mma_bar, 1);
    tc::mbar_init(pt_bar, 1);
    *flag = 0;
    *abort_flag = 0;
    tc::fence_barrier_init();
    tc::fence_proxy_async_smem();                     // the barriers, for the tile load below
    tc::mbar_arrive_expect_tx(tma_bar, 32768);
    const int tc0 = sp.tok0 + (int)t0;
    tc::tma_load_4d(qk, &tmq, tma_bar, 0, hk, tc0, sp.bcoord);
    tc::tma_load_4d(qk + 8192, &tmk, tma_bar, 0, hk, tc0, sp.bcoord);
    tc::tma_load_4d(qk + 16384, &tmq, tma_bar, 64, hk, tc0, sp.bcoord);
    tc::tma_load_4d(qk + 24576, &tmk, tma_bar, 64, hk, tc0, sp.bcoord);
  }
  if (warp == 0) {
    tc::tmem_alloc(sb + PP_BAR + 16, 128);
    tc::tmem_relinquish();
    tc::tc_fence_before();
  }
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + PP_BAR + 16);
  const uint32_t lane_off = static_cast<uint32_t>(32 * (warp & 3)) << 16;
  const int row = tid & 127, half = tid >> 7;         // TMEM lane and column half of this thread
  GDN_TRACE_PP(1);
  GDN_TRACE_PPV(55, tc::globaltimer_ns());
  GDN_TRACE_PPV(57, tc::smid());
  // S = [Q; K] K^T into TMEM columns 0..63.  Rows of the tile past the sequence's end (the next
  // packed sequence's tokens) are zeroed first, so they reach no product.
  bool tile_ok = true;
  if (vrows < C) {                                    // (uniform)
    tile_ok = tc::mbar_wait(tma_bar, 0, abort_flag, kBudget);
    for (int i = tid; i < 4 * (C - vrows) * 8; i += PP_THREADS) {
      const int box = i / ((C - vrows) * 8), rem = i - box * (C - vrows) * 8;
      tc::st_shared_v4(qk + box * 8192 + (vrows + (rem >> 3)) * 128 + (rem & 7) * 16, 0u, 0u, 0u,
                       0u);
    }
    tc::fence_proxy_async_smem();
    __syncthreads();
  }
  if (tid == 0) {
    if (vrows == C) tile_ok = tc::mbar_wait(tma_bar, 0, abort_flag, kBudget);
    GDN_TRACE_PP(62);
    if (tile_ok) {
      GDN_TRACE_PP(2);
      tc::tc_fence_after();
      const uint64_t dq = tc::sdesc_sw128(qk, 16, 1024);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
        tc::mma_bf16(tmem, tc::desc_adv(dq, off), tc::desc_adv(dq, off + 8192), ID_S, ks > 0);
      }
    }
    tc::mma_commit(mma_bar);
  }
  // gates (warps 2-3, meanwhile): G' = cumsum(log alpha) log2(e) over the chunk, beta, ktil,
  // gamma (zero / flat past the sequence's end)
  float* gE = gG + 256;
  if (gw) {
    if (ba && t0 + gi < sp.len) {   // from the in_proj_ba outputs: beta = sigmoid(b),
      const float b = bt, a = la;   // log alpha = -softplus(-a)
      bt = 1.0f / (1.0f + expf(-b));
      la = a >= 0.f ? -log1pf(expf(-a)) : a - log1pf(expf(a));
    }
    gB[gi] = bt;
    float incl = la;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const float n = __shfl_up_sync(0xffffffffu, incl, d);
      if (lane >= d) incl += n;
    }
    if (gi == 31) gG[31] = incl;
    tc::named_bar(5, 64);
    if (gi >= 32) incl += gG[31];                     // carry of the first 32 tokens
    const float g2 = incl * 1.4426950408889634f;
    tc::named_bar(5, 64);                             // gG[31] read before it is rescaled
    gG[gi] = g2;
    tc::named_bar(5, 64);
    gKt[gi] = tc::ex2(gG[63] - g2);
    reinterpret_cast<float*>(rec + kPwTiles)[gi] = tc::ex2(g2);
    // block factors E[b][j] = exp(G_16b - G_j) for j < 16b (each <= 1: G never increases)
#pragma unroll
    for (int b = 1; b < 4; ++b) gE[64 * b + gi] = gi < 16 * b ? tc::ex2(gG[16 * b] - g2) : 0.f;
  }
  GDN_TRACE_PPT(61, 64);
  __syncthreads();                                    // gates visible
  tc::mbar_wait(mma_bar, 0, abort_flag, kBudget);
  GDN_TRACE_PP(3);
  tc::tc_fence_after();
  {
    // row r of S: r < 64 is (q_t . k_j), r >= 64 is (k_t . k_j), t = r mod 64; this thread takes
    // columns j = 32 half .. 32 half + 31
    float s[32];
    tc::tmem_ld32(tmem + lane_off + 32 * half, s);
    tc::tmem_wait_ld();
    // exp(G_t - G_j) = 2^(G'_t - G'_j) inside t's 16-token block directly, across blocks as
    // 2^(G'_t - G'_16ti) E[ti][j] (both factors <= 1, so strong decay underflows to 0 instead of
    // overflowing); P takes scale and j <= t, A takes beta_t and j < t
    const int t = row & 63, ti = t >> 4;
    const bool isP = row < 64;
    const float gt = gG[t];
    const float rowf = (isP ? scale : gB[t]) * tc::ex2(gt - gG[16 * ti]);
    const float diagf = isP ? scale : gB[t];
    const int jmax = isP ? t : t - 1;                 // last j kept
    float sum = 0.f;
#pragma unroll
    for (int kk = 0; kk < 2; ++kk) {
      const int kb = 2 * half + kk;                   // 16-column block of this thread
      float f[16];
      if (kb < ti) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float4 e = *reinterpret_cast<const float4*>(gE + 64 * ti + 16 * kb + 4 * i);
          tc::f2_get(tc::mul2(tc::f2(rowf, rowf), tc::f2(e.x, e.y)), f[4 * i], f[4 * i + 1]);
          tc::f2_get(tc::mul2(tc::f2(rowf, rowf), tc::f2(e.z, e.w)), f[4 * i + 2], f[4 * i + 3]);
        }
      } else if (kb == ti) {
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int j = 16 * kb + e;
          f[e] = j <= jmax ? diagf * tc::ex2(gt - gG[j]) : 0.f;
        }
      } else {
#pragma unroll
        for (int e = 0; e < 16; ++e) f[e] = 0.f;
      }
#pragma unroll
      for (int e = 0; e < 16; e += 2)
        tc::f2_get(tc::mul2(tc::f2(f[e], f[e + 1]), tc::f2(s[16 * kk + e], s[16 * kk + e + 1])),
                   f[e], f[e + 1]);
#pragma unroll
      for (int e = 0; e < 16; ++e) sum += f[e];
      if (isP) {                // P row t: K-major bf16 hi over the first Q box, lo over the second
#pragma unroll
        for (int h8 = 0; h8 < 2; ++h8) {
          const int j8 = 2 * kb + h8;
          const uint32_t o = qk + (uint32_t)(t * 128 + ((j8 ^ (t & 7)) << 4));
          st_split8(o, o + 16384, f + 8 * h8);
        }
      } else if (kb <= ti) {    // A row t into the solve's packed 16 x 16 blocks
#pragma unroll
        for (int i = 0; i < 4; ++i)
          tc::sts4(at(blk(tb, ti, kb), t & 15, 4 * i),
                   make_float4(f[4 * i], f[4 * i + 1], f[4 * i + 2], f[4 * i + 3]));
      }
    }
    if (!(fabsf(sum) <= 3.402823466e38f)) *flag = 1;
  }
  tc::tc_fence_before();
  __syncthreads();

  GDN_TRACE_PP(4);
  float tv[3][4];
  if (tid < 128) solve_unit_lower(tb, tid, tv);       // (warps 0-3; named barriers of 128, 64)
  __syncthreads();                                    // T's diagonal blocks are in place
  GDN_TRACE_PP(5);
  // one (diagonal block, row, 4-column group) per thread: 4 x 16 x 4 = 256
  const float4 dg = tc::lds4(at(blkT(tb, tid >> 6, tid >> 6), (tid >> 2) & 15, 4 * (tid & 3)));
  __syncthreads();                                    // the solve scratch is dead
  // T_b (kt false) or ktil T_b (kt true) into the B tile pair; the zeros above the diagonal
  // blocks are written once and serve both
  auto put_b = [&](bool kt) {
    const int g = lane >> 2, t4 = lane & 3;
#pragma unroll
    for (int m = 0; m < 3 && tid < 128; ++m) {        // off-diagonal blocks and their zero mirrors
                                                      // (from the solve's fragments, warps 0-3)
      const int hp = warp + 4 * m, bi = hp >> 1, n0 = (hp & 1) * 8;
      const int i = blk_i(bi), kk = blk_k(bi, i);
      const int col = 16 * kk + n0 + 2 * t4, row = 16 * i + g;
      const float f0 = kt ? gKt[row] : 1.f, f1 = kt ? gKt[row + 8] : 1.f;
      store_b_pair(tb, row, col, f0 * (tv[m][0] * gB[col]), f0 * (tv[m][1] * gB[col + 1]));
      store_b_pair(tb, row + 8, col, f1 * (tv[m][2] * gB[col]), f1 * (tv[m][3] * gB[col + 1]));
      if (!kt) {
        const int urow = 16 * kk + g, ucol = 16 * i + n0 + 2 * t4;
        store_b_pair(tb, urow, ucol, 0.f, 0.f);
        store_b_pair(tb, urow + 8, ucol, 0.f, 0.f);
      }
    }
    {                                                 // diagonal blocks (zero above the diagonal)
      const int b = tid >> 6, r = (tid >> 2) & 15, cs = tid & 3;
      const int brow = 16 * b + r, col = 16 * b + 4 * cs;
      const float f = kt ? gKt[brow] : 1.f;
      store_b_pair(tb, brow, col, f * (dg.x * gB[col]), f * (dg.y * gB[col + 1]));
      store_b_pair(tb, brow, col + 2, f * (dg.z * gB[col + 2]), f * (dg.w * gB[col + 3]));
    }
    tc::fence_proxy_async_smem();
    tc::tc_fence_before();
    __syncthreads();
  };
  const uint64_t dt = tc::sdesc_sw128(tb, 8192, 1024);
  put_b(false);
  // PT = P T_b into columns 64..127
  GDN_TRACE_PP(6);
  if (tid == 0) {
    tc::tc_fence_after();
    const uint64_t dp = tc::sdesc_sw128(qk, 16, 1024);
#pragma unroll
    for (int i = 0; i < 12; ++i) {
      const int ks = i / 3, term = i - 3 * ks;
      tc::mma_bf16(tmem + 64, tc::desc_adv(dp, (term == 1 ? 16384 : 0) + ks * 32),
                   tc::desc_adv(dt, (term == 2 ? 8192 : 0) + ks * 2048), ID_PT, i > 0);
    }
    tc::mma_commit(pt_bar);
  }
  tc::mbar_wait(pt_bar, 0, abort_flag, kBudget);
  tc::tc_fence_after();
  // W = K^T (ktil T_b) into columns 0..63 (S is consumed) from the same tiles, now free
  put_b(true);
  if (tid == 0) {
    tc::tc_fence_after();
    const uint64_t dk = tc::sdesc_sw128(qk + 8192, 16384, 1024);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int ks = i >> 1, term = i & 1;
      tc::mma_bf16(tmem, tc::desc_adv(dk, ks * 2048), tc::desc_adv(dt, term * 8192 + ks * 2048),
                   ID_W, i > 0);
    }
    tc::mma_commit(mma_bar);
  }
  GDN_TRACE_PP(7);
  const bool poison = *flag != 0;
  // Rows from TMEM are split and staged (swizzled, in the record's tile layout) in shared memory
  // the MMAs no longer read, then leave by bulk copies: PT's while W is still being multiplied
  // (hi over P hi, lo over P lo), W's once it is done (hi over the B tile pair, lo rows 0..63 /
  // 64..127 over the two K boxes).
  // 32 values (this thread's column half) of row r, split and staged in the record's tile layout
  auto stage_half = [&](uint32_t hi_base, uint32_t lo_base, int r, const float* w) {
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      const int j8 = 4 * half + jj;
      const uint32_t o = (uint32_t)(r * 128 + ((j8 ^ (r & 7)) << 4));
      st_split8(hi_base + o, lo_base + o, w + 8 * jj);
    }
  };
  {
    float w[32];
    if (row < 64) {             // PT rows: warps 0, 1 (columns 0..31) and 4, 5 (32..63)
      tc::tmem_ld32(tmem + lane_off + 64 + 32 * half, w);
      tc::tmem_wait_ld();
      if (poison) {
#pragma unroll
        for (int j = 0; j < 32; ++j) w[j] = kInf;
      }
      stage_half(qk, qk + 16384, row, w);
      tc::fence_proxy_async_smem();
      tc::named_bar(2, 128);
      if (tid == 0) {
        tc::bulk_store(rec, qk, 8192);
        tc::bulk_store(rec + 8192, qk + 16384, 8192);
        tc::bulk_commit();
      }
    }
    GDN_TRACE_PP(58);
    tc::mbar_wait(mma_bar, 1, abort_flag, kBudget);
    GDN_TRACE_PP(59);
    tc::tc_fence_after();
    tc::tmem_ld32(tmem + lane_off + 32 * half, w);
    tc::tmem_wait_ld();
    if (poison) {
#pragma unroll
      for (int j = 0; j < 32; ++j) w[j] = kInf;
    }
    // W row r: hi at tb + r * 128, lo at qk + 8192 (r < 64) or qk + 24576 (r >= 64)
    stage_half(tb, qk + (row < 64 ? 8192 : 24576 - 64 * 128), row, w);
    tc::fence_proxy_async_smem();
    tc::named_bar(4, PP_THREADS);
    if (tid == 0) {
      tc::bulk_store(rec + 16384, tb, 16384);
      tc::bulk_store(rec + 32768, qk + 8192, 8192);
      tc::bulk_store(rec + 40960, qk + 24576, 8192);
      tc::bulk_commit();
      tc::bulk_wait_read_all();                       // every source read; the writes complete
    }                                                 // on their own
  }
  GDN_TRACE_PP(8);
  GDN_TRACE_PPV(56, tc::globaltimer_ns());
  if (tid == 0 && *abort_flag) record_error(kErrTimeout);
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 128);
  }
}

// ------------------------------------------------------------------------------------------
// the recurrence
// ------------------------------------------------------------------------------------------
template <typename Tout>
__global__ void __launch_bounds__(kThreads, 1)
chunk_fwd_tc_kernel(const __grid_constant__ CUtensorMap tmq, const __grid_constant__ CUtensorMap tmk,
                    const __grid_constant__ CUtensorMap tmo, const __nv_bfloat16* __restrict__ v,
                    const uint8_t* __restrict__ pw, const float* __restrict__ S0,
                    float* __restrict__ S_T, int T, int Hk, int Hv, float scale,
                    const int* __restrict__ cu, int max_len, int nCmax, Tout* __restrict__ o) {
  constexpr bool kF32 = sizeof(Tout) == 4;
  // X takes M as a hi + lo bf16 pair when o is fp32 (the layer, whose gated norm magnifies o's
  // error); a bf16 o carries its own rounding, and one round-to-nearest bf16 copy of M suffices.
  constexpr bool kSplitX = kF32;
  GDN_TRACE_INIT;
  // Offsetting the __shared__ array itself (not a round trip through an integer) keeps every
  // access below a shared-memory access (ld/st.shared), not a generic one.
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (tc::smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t sb = tc::smem_u32(smem);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.x % Hv;
  const int bq = blockIdx.x / Hv;                    // the sequence
  const int hk = h / (Hv / Hk);
  const SeqSpan sp = seq_span(cu, bq, T, max_len);
  const int nC = (sp.len + C - 1) / C;
  const bool packed = cu != nullptr;
  const long head = (long)bq * Hv + h;
  const uint8_t* pw_head = pw + head * nCmax * (long)kPwBytes;
  if (nC == 0) {   // an empty sequence: the state passes through (uniform, before any barrier)
    if (S_T)
      for (int i = threadIdx.x; i < 128 * 128 / 4; i += blockDim.x)
        reinterpret_cast<float4*>(S_T + head * 128 * 128)[i] =
            S0 ? reinterpret_cast<const float4*>(S0 + head * 128 * 128)[i]
               : make_float4(0.f, 0.f, 0.f, 0.f);
    return;
  }
  auto bar = [&](int i) -> uint32_t { return sb + OFF_BAR + 8u * i; };

  if (threadIdx.x == 0) {
    const int ones[] = {B_QK_FULL, B_QK_EMPTY, B_W_FULL, B_W_FULL + 1, B_P_FULL, B_P_FULL + 1,
                        B_X_FULL, B_D3_FULL, B_Y_FULL, B_DRAIN};
    for (int i : ones) tc::mbar_init(bar(i), 1);
    const int twos[] = {B_R_FULL, B_Y_EMPTY, B_M_READY, B_M_SCALED};
    for (int i : twos) tc::mbar_init(bar(i), 2);   // one arrive per column half
    // the MMAs that read a part, and the o stores of both halves staged in it (an fp32 o tile
    // spills into W's part)
    for (int s = 0; s < 2; ++s) {
      tc::mbar_init(bar(B_P_EMPTY + s), 3);
      tc::mbar_init(bar(B_W_EMPTY + s), kF32 ? 3 : 1);
      tc::mbar_init(bar(B_G_FULL + s), 1);
      tc::mbar_init(bar(B_G_EMPTY + s), 8);           // one arrive per chain warp
    }
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
    tc::tma_prefetch_desc(&tmo);
  }
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(smem + OFF_MISC);
  if (threadIdx.x == 0) GDN_TRACE_G(0, 10);

  if (warp == 0) {
    // ------------------------------- loads ----------------------------------------------------
    if (lane == 0) {
      int armed_qk = -1, armed_w[2] = {-1, -1}, armed_p[2] = {-1, -1};
      bool ok = true;
      for (int c = 0; c < nC && ok; ++c) {
        const int s = c & 1, t0 = sp.tok0 + c * C;
        // one Q/K stage: chunk c's tile is loaded as soon as X of chunk c - 1 has read the last
        if (c >= 1) ok = tc::mbar_wait(bar(B_QK_EMPTY), (c - 1) & 1, abort_flag, kBudget);
        if (!ok) break;
        const uint32_t dst = sb + OFF_QK;
        tc::mbar_arrive_expect_tx(bar(B_QK_FULL), 32768);
        tc::tma_load_4d(dst, &tmq, bar(B_QK_FULL), 0, hk, t0, sp.bcoord);
        tc::tma_load_4d(dst + 8192, &tmk, bar(B_QK_FULL), 0, hk, t0, sp.bcoord);
        tc::tma_load_4d(dst + 16384, &tmq, bar(B_QK_FULL), 64, hk, t0, sp.bcoord);
        tc::tma_load_4d(dst + 24576, &tmk, bar(B_QK_FULL), 64, hk, t0, sp.bcoord);
        armed_qk = c;
        const uint8_t* src = pw_head + (long)c * kPwBytes;
        const uint32_t slot = sb + OFF_PW + s * PW_SLOT;
        if (c >= 2) ok = tc::mbar_wait(bar(B_W_EMPTY + s), ((c >> 1) - 1) & 1, abort_flag, kBudget);
        if (!ok) break;
        tc::mbar_arrive_expect_tx(bar(B_W_FULL + s), 32768);
        tc::bulk_load(slot + 16384, src + 16384, 32768, bar(B_W_FULL + s));
        GDN_TRACE(c, 17);
        armed_w[s] = c;
        if (c >= 2) ok = tc::mbar_wait(bar(B_P_EMPTY + s), ((c >> 1) - 1) & 1, abort_flag, kBudget);
        if (!ok) break;
        tc::mbar_arrive_expect_tx(bar(B_P_FULL + s), 16384);
        tc::bulk_load(slot, src, 16384, bar(B_P_FULL + s));
        GDN_TRACE(c, 18);
        armed_p[s] = c;
      }
      // every load issued lands before the CTA can leave (at once unless a consumer gave up)
      volatile int never = 0;
      if (armed_qk >= 0) tc::mbar_wait(bar(B_QK_FULL), armed_qk & 1, &never, kBudget / 4);
      for (int s = 0; s < 2; ++s) {
        if (armed_w[s] >= 0)
          tc::mbar_wait(bar(B_W_FULL + s), (armed_w[s] >> 1) & 1, &never, kBudget / 4);
        if (armed_p[s] >= 0)
          tc::mbar_wait(bar(B_P_FULL + s), (armed_p[s] >> 1) & 1, &never, kBudget / 4);
      }
    }
  } else if (warp == 1) {
    // -------------------------------- MMAs -----------------------------------------------------
    // Per chunk c: X(c), then Y(c - 1) (it reads the other R' buffer and runs while R'(c) is
    // being formed, off the state chain), then the state update of chunk c; Y of the last chunk
    // follows the loop.
    if (lane == 0) {
      const uint64_t dq = tc::sdesc_sw128(sb + OFF_QK, 16, 1024);
      const uint64_t dm = tc::sdesc_sw128(sb + OFF_MB, 16384, 1024);
      // Y = PT R' (rows 0..63 used), as hi.hi + lo.hi + hi.lo bf16 products             (bf16)
      auto issue_Y = [&](int cy) -> bool {
        const int sy = cy & 1;
        if (cy >= 1 && !tc::mbar_wait_spin(bar(B_Y_EMPTY), (cy - 1) & 1, abort_flag, kBudget)) return false;
        if (!tc::mbar_wait_spin(bar(B_P_FULL + sy), (cy >> 1) & 1, abort_flag, kBudget)) return false;
        tc::tc_fence_after();
        const uint64_t dpw = tc::sdesc_sw128(sb + OFF_PW + sy * PW_SLOT, 16, 1024);
        const uint64_t drd = tc::sdesc_sw128(sb + OFF_RD + sy * RD_BUF, 16384, 1024);
#pragma unroll
        for (int i = 0; i < 12; ++i) {
          const int ks = i / 3, term = i - 3 * ks;
          tc::mma_bf16(tmem + TM_Y, tc::desc_adv(dpw, (term == 1 ? 8192 : 0) + ks * 32),
                       tc::desc_adv(drd, (term == 2 ? 8192 : 0) + ks * 2048), ID_Y, i > 0);
        }
        tc::mma_commit(bar(B_Y_FULL));
        tc::mma_commit(bar(B_P_EMPTY + sy));
        GDN_TRACE(cy, 22);
        return true;
      };
      bool ok = true;
      for (int c = 0; c < nC && ok; ++c) {
        const int s = c & 1;
        // X = [Q; K] M  (M as one bf16 copy, or a hi + lo pair)                     (bf16)
        // X(c) goes to the TMEM buffer of X(c - 2), whose o rows the o path of chunk c - 2 reads:
        // it signals Y_EMPTY once its TMEM reads are done
        ok = tc::mbar_wait_spin(bar(B_QK_FULL), c & 1, abort_flag, kBudget) &&
             tc::mbar_wait_spin(bar(B_M_READY), c & 1, abort_flag, kBudget) &&
             (c < 2 || tc::mbar_wait_spin(bar(B_Y_EMPTY), c & 1, abort_flag, kBudget));
        if (!ok) break;
        GDN_TRACE(c, 12);
        tc::tc_fence_after();
        {
          const uint64_t dml = tc::sdesc_sw128(sb + OFF_RD + s * RD_BUF, 16384, 1024);
#pragma unroll
          for (int ks = 0; ks < (kSplitX ? 16 : 8); ++ks)
            tc::mma_bf16(tmem + TM_X + 128 * s, tc::desc_adv(dq, ((ks >> 2) & 1) * 16384 + (ks & 3) * 32),
                         tc::desc_adv(ks < 8 ? dm : dml, (ks & 7) * 2048), ID_X, ks > 0);
        }
        tc::mma_commit(bar(B_X_FULL));
        tc::mma_commit(bar(B_QK_EMPTY));
        GDN_TRACE(c, 20);
        if (c >= 1 && !(ok = issue_Y(c - 1))) break;
        // M += W R' (TMEM holds gamma_last M), hi.hi + lo.hi + hi.lo bf16 products     (bf16)
        ok = tc::mbar_wait_spin(bar(B_R_FULL), c & 1, abort_flag, kBudget);
        GDN_TRACE(c, 14);
        ok = ok && tc::mbar_wait_spin(bar(B_M_SCALED), c & 1, abort_flag, kBudget);
        GDN_TRACE(c, 15);
        ok = ok && tc::mbar_wait_spin(bar(B_W_FULL + s), (c >> 1) & 1, abort_flag, kBudget);
        if (!ok) break;
        GDN_TRACE(c, 13);
        tc::tc_fence_after();
        {
          const uint64_t dpw = tc::sdesc_sw128(sb + OFF_PW + s * PW_SLOT, 16, 1024);
          const uint64_t drd = tc::sdesc_sw128(sb + OFF_RD + s * RD_BUF, 16384, 1024);
#pragma unroll
          for (int i = 0; i < 12; ++i) {
            const int ks = i / 3, term = i - 3 * ks;
            tc::mma_bf16(tmem + TM_M, tc::desc_adv(dpw, 16384 + (term == 1 ? 16384 : 0) + ks * 32),
                         tc::desc_adv(drd, (term == 2 ? 8192 : 0) + ks * 2048), ID_Y, 1);
          }
        }
        tc::mma_commit(bar(B_D3_FULL));
        tc::mma_commit(bar(B_W_EMPTY + s));
        GDN_TRACE(c, 21);
      }
      if (ok && nC >= 1) issue_Y(nC - 1);
      tc::mma_commit(bar(B_DRAIN));
      volatile int never = 0;
      tc::mbar_wait(bar(B_DRAIN), 0, &never, kBudget / 4);
    }
  } else if (warp == 2) {
    // ------------------------------- gamma ---------------------------------------------------
    // gamma_t of chunk c into ring slot c & 1, so that the chain reads it from shared memory
    // (off the chain's critical path) instead of global memory
    const float* gsrc = reinterpret_cast<const float*>(pw_head + kPwTiles);
    for (int c = 0; c < nC; ++c) {
      const int s = c & 1;
      int ok = 1;
      if (lane == 0 && c >= 2)
        ok = tc::mbar_wait(bar(B_G_EMPTY + s), ((c >> 1) - 1) & 1, abort_flag, kBudget);
      __syncwarp();                                    // the slot's readers before its writers
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      const float2 g = reinterpret_cast<const float2*>(gsrc + (long)c * (kPwBytes / 4))[lane];
      *reinterpret_cast<float2*>(smem + OFF_GAM + s * 256 + 8 * lane) = g;
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(bar(B_G_FULL + s));
    }
  } else if (warp >= 4) {
    // ------------------------------- chain warpgroups ----------------------------------------
    // warps 4-7: value columns 0..63, warps 8-11: 64..127.  Lanes 0..63 (q < 2) make o of token
    // t = r, lanes 64..127 make R' of token t = r - 64; all take M's row r.
    const int hh = (warp - 4) >> 2, q = warp & 3, r = 32 * q + lane, t = r & 63;
    const uint32_t lane_off = static_cast<uint32_t>(32 * q) << 16;
    const uint32_t tcol = 64 * hh;                       // this half's TMEM / value columns
    const uint32_t mb = sb + OFF_MB + hh * 16384, rd0 = sb + OFF_RD + hh * 16384;
    const uint32_t id_wg = 1 + 3 * hh, id_lo = 2 + 3 * hh, id_hi = 3 + 3 * hh;
    const bool leader = (q == 0 && lane == 0);
    [[maybe_unused]] const int ev = 10 * hh;
    // gamma_t (t) and gamma_last of chunk c from the ring; the slot is handed back at once
    auto gam_get = [&](int c, float& gt, float& gl) {
      tc::mbar_wait(bar(B_G_FULL + (c & 1)), (c >> 1) & 1, abort_flag, kBudget);
      const float* g = reinterpret_cast<const float*>(smem + OFF_GAM + (c & 1) * 256);
      gt = g[t];
      gl = g[63];
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(bar(B_G_EMPTY + (c & 1)));
    };
    // 32 columns (32p ..) of M row r (this half) for the X MMA: one round-to-nearest bf16 copy in Mb,
    // or (kSplitX) a hi + lo pair, hi into Mb and lo into the R' buffer
    auto store_m32 = [&](const float (&m)[32], int p, uint32_t rd) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const uint32_t sw = tc::sw128(r, 4 * p + j);
        if constexpr (kSplitX) {
          st_split8(mb + sw, rd + sw, m + 8 * j);
        } else {
          const float* w = m + 8 * j;
          tc::st_shared_v4(mb + sw, tc::pack_bf16(w[0], w[1]), tc::pack_bf16(w[2], w[3]),
                           tc::pack_bf16(w[4], w[5]), tc::pack_bf16(w[6], w[7]));
        }
      }
    };
    // row t of V for this half's columns (R' lanes), loaded one chunk ahead into registers
    uint4 vr[8];
    auto load_v = [&](int c) {
      const long tok = (long)c * C + t;
      if (tok < sp.len) {
        const uint4* src = reinterpret_cast<const uint4*>(v + ((sp.row0 + tok) * Hv + h) * 128 + tcol);
#pragma unroll
        for (int i = 0; i < 8; ++i) vr[i] = src[i];
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) vr[i] = make_uint4(0u, 0u, 0u, 0u);
      }
    };
    if (q >= 2) load_v(0);
    float g_t, g_l0;
    gam_get(0, g_t, g_l0);
    bool stop = false;
    {
      float m[64];
      if (S0) {
        const float4* src = reinterpret_cast<const float4*>(S0 + (head * 128 + r) * 128 + tcol);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float4 w = src[i];
          m[4 * i] = w.x; m[4 * i + 1] = w.y; m[4 * i + 2] = w.z; m[4 * i + 3] = w.w;
        }
      } else {
#pragma unroll
        for (int i = 0; i < 64; ++i) m[i] = 0.f;
      }
      store_m32(*reinterpret_cast<const float(*)[32]>(&m[0]), 0, rd0);
      store_m32(*reinterpret_cast<const float(*)[32]>(&m[32]), 1, rd0);
#pragma unroll
      for (int i = 0; i < 64; ++i) m[i] *= g_l0;
      tmem_st64(tmem + lane_off + TM_M + tcol, m);
      tc::tmem_wait_st();
      tc::fence_proxy_async_smem();
      tc::tc_fence_before();
      stop = vote_abort(id_wg, 128, abort_flag);
      if (leader) {
        tc::mbar_arrive(bar(B_M_READY));
        tc::mbar_arrive(bar(B_M_SCALED));
      }
    }

    for (int c = 0; c < nC && !stop; ++c) {
      const int s = c & 1;
      const uint32_t tx = tmem + lane_off + TM_X + 128 * s + tcol;
      // the next chunk's gates: gamma_last for the state below, gamma_t for the next chunk
      float g_nt = 0.f, g_nl = 0.f;
      if (c + 1 < nC) gam_get(c + 1, g_nt, g_nl);
      if (q >= 2) {
        // R' = V - gamma (K M) for token t, as a bf16 hi + lo pair (the B operand of Y and of
        // the state update)
        tc::mbar_wait(bar(B_X_FULL), c & 1, abort_flag, kBudget);
        if (q == 2 && lane == 0) GDN_TRACE(c, 30 + ev);
        tc::tc_fence_after();
        const bool t_out = (long)c * C + t >= sp.len;
        // this half's 64 columns of the row in one TMEM round trip
        float x[64];
        tc::tmem_ld32(tx, *reinterpret_cast<float(*)[32]>(&x[0]));
        tc::tmem_ld32(tx + 32, *reinterpret_cast<float(*)[32]>(&x[32]));
        tc::tmem_wait_ld();
#pragma unroll
        for (int p = 0; p < 2; ++p) {            // value columns 32p .. 32p+31 of this half
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const float* xx = x + 32 * p + 8 * j;
            const uint4 u = p ? vr[4 + j] : vr[j];   // (no dynamic register indexing)
            const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
            float rv[8];
#pragma unroll
            for (int e = 0; e < 4; ++e)
              tc::f2_get(tc::fma2(tc::f2(-g_t, -g_t), tc::f2(xx[2 * e], xx[2 * e + 1]),
                                  tc::f2(tc::bf16lo(w4[e]), tc::bf16hi(w4[e]))),
                         rv[2 * e], rv[2 * e + 1]);
            if (t_out) {                         // past the sequence's end: no contribution
#pragma unroll
              for (int e = 0; e < 8; ++e) rv[e] = 0.f;
            }
            // MN-major bf16 B operand: row t (K), 16-byte chunk 4p + j of this half's columns
            const uint32_t sw = tc::sw128(t, 4 * p + j);
            st_split8(rd0 + s * RD_BUF + sw, rd0 + s * RD_BUF + 8192 + sw, rv);
          }
        }
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        tc::named_bar(id_hi, 64);
        if (q == 2 && lane == 0) {
          GDN_TRACE(c, 31 + ev);
          tc::mbar_arrive(bar(B_R_FULL));
        }
        if (c + 1 < nC) load_v(c + 1);
      }
      // M <- gamma_last M + W R' is now in TMEM (row r of this half).  Its bf16 copy goes out
      // first (the next X needs it); then TMEM is scaled by the next chunk's gamma_last for the
      // next update, which waits for that separately.
      tc::mbar_wait(bar(B_D3_FULL), c & 1, abort_flag, kBudget);
      if (leader) GDN_TRACE(c, 37 + ev);
      tc::tc_fence_after();
      if (c + 1 < nC) {
        float m[64];
        tmem_ld64(tmem + lane_off + TM_M + tcol, m);
        tc::tmem_wait_ld();
        // the next chunk's X reads the low part from the other R' buffer (whose Y is done:
        // this update was issued after it)
        store_m32(*reinterpret_cast<const float(*)[32]>(&m[0]), 0, rd0 + ((c + 1) & 1) * RD_BUF);
        store_m32(*reinterpret_cast<const float(*)[32]>(&m[32]), 1, rd0 + ((c + 1) & 1) * RD_BUF);
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        tc::named_bar(id_wg, 128);
        if (leader) {
          GDN_TRACE(c, 38 + ev);
          tc::mbar_arrive(bar(B_M_READY));
        }
#pragma unroll
        for (int i = 0; i < 64; i += 2)
          tc::f2_get(tc::mul2(tc::f2(m[i], m[i + 1]), tc::f2(g_nl, g_nl)), m[i], m[i + 1]);
        tmem_st64(tmem + lane_off + TM_M + tcol, m);
        tc::tmem_wait_st();
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
      if (q < 2 && !stop) {
        // o_t = gamma_t scale (Q M)_t + (PT R')_t, staged in the chunk's operand slot (the PT
        // tiles, which Y has finished reading; fp32 also takes W's, after the update) for a TMA
        // store
        const bool t_valid = (long)c * C + t < sp.len;
        tc::mbar_wait(bar(B_Y_FULL), c & 1, abort_flag, kBudget);
        if (leader) GDN_TRACE(c, 34 + ev);
        tc::tc_fence_after();
        const float g = g_t * scale;
        // bf16: one [64 t][64 dv] tile per half; fp32: two [64 t][32 dv] tiles per half
        const uint32_t stage = sb + OFF_PW + s * PW_SLOT + hh * (kF32 ? 16384 : 8192);
        // the last chunk of a packed sequence ends inside the tile: its valid rows go straight to
        // global memory (a box store would write into the next sequence)
        const bool ragged = packed && (c + 1) * C > sp.len;
        Tout* orow = o + ((sp.row0 + (long)c * C + t) * Hv + h) * 128 + tcol;
        // value columns 16p .. 16p+15 of this half (y[16]) to global memory or the staged tile
        auto put16 = [&](int p, const float* y) {
          if (ragged) {
            if (t_valid) {
              if constexpr (kF32) {
#pragma unroll
                for (int j = 0; j < 4; ++j)
                  reinterpret_cast<float4*>(orow + 16 * p)[j] =
                      make_float4(y[4 * j], y[4 * j + 1], y[4 * j + 2], y[4 * j + 3]);
              } else {
#pragma unroll
                for (int j = 0; j < 2; ++j)
                  reinterpret_cast<uint4*>(orow + 16 * p)[j] =
                      make_uint4(tc::pack_bf16(y[8 * j], y[8 * j + 1]),
                                 tc::pack_bf16(y[8 * j + 2], y[8 * j + 3]),
                                 tc::pack_bf16(y[8 * j + 4], y[8 * j + 5]),
                                 tc::pack_bf16(y[8 * j + 6], y[8 * j + 7]));
              }
            }
          } else if constexpr (kF32) {           // tile p / 2, 16-byte chunks 4 (p % 2) ..
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
        };
#pragma unroll 1
        for (int p = 0; p < 4; p += 2) {         // value columns 16p .. 16p+31 of this half
          float x[32], y[32];
          tc::tmem_ld32(tx + 16 * p, x);
          tc::tmem_ld32(tmem + lane_off + TM_Y + tcol + 16 * p, y);
          tc::tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; i += 2)
            tc::f2_get(tc::fma2(tc::f2(g, g), tc::f2(x[i], x[i + 1]), tc::f2(y[i], y[i + 1])),
                       y[i], y[i + 1]);
          put16(p, y);
          put16(p + 1, y + 16);
        }
        tc::fence_proxy_async_smem();
        tc::tc_fence_before();
        tc::named_bar(id_lo, 64);
        if (leader) {
          tc::mbar_arrive(bar(B_Y_EMPTY));
          GDN_TRACE(c, 35 + ev);
          if (!ragged) {
            const int oc = sp.tok0 + c * C;
            if constexpr (kF32) {
              tc::tma_store_4d(&tmo, stage, 64 * hh, h, oc, sp.bcoord);
              tc::tma_store_4d(&tmo, stage + 8192, 64 * hh + 32, h, oc, sp.bcoord);
            } else {
              tc::tma_store_4d(&tmo, stage, 64 * hh, h, oc, sp.bcoord);
            }
            tc::bulk_commit();
            tc::bulk_wait_read_all();
          }
          tc::mbar_arrive(bar(B_P_EMPTY + s));
          if constexpr (kF32) tc::mbar_arrive(bar(B_W_EMPTY + s));
          GDN_TRACE(c, 36 + ev);
        }
      }
      g_t = g_nt;
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

// A single sequence of at least 2 * kRangeChunks chunks whose recurrences leave at least half of
// the SMs idle runs in ranges of kRangeChunks chunks (see launch()).
constexpr int kRangeChunks = 128;
inline bool ranged(int nseq, int T, int Hv, int sms) {
  return nseq == 1 && 2L * Hv <= sms && (T + C - 1) / C >= 2 * kRangeChunks;
}

// How launch() runs a call: in one part (pre-pass + recurrence), in ranges of a long single
// sequence, or split into leading and tail batches.  launch() and launch_count() both decide here.
enum class Plan { kOne, kRanges, kSplit };
inline Plan plan(int nseq, int T, int Hv, int sms, bool packed) {
  if (!packed && ranged(nseq, T, Hv, sms)) return Plan::kRanges;
  const int head_b = sms / (Hv > 0 ? Hv : 1);        // batches that fill at most one wave
  if (packed || nseq < 2 || (long)nseq * Hv <= sms || head_b < 1 || head_b >= nseq)
    return Plan::kOne;
  return Plan::kSplit;
}
// Kernel launches of one call (two per part: pre-pass and recurrence).
inline int launch_count(int nseq, int T, int Hv, int sms, bool packed) {
  if (nseq <= 0 || T <= 0) return 0;
  switch (plan(nseq, T, Hv, sms, packed)) {
    case Plan::kRanges: {
      const int nC = (T + C - 1) / C;
      return 2 * ((nC + kRangeChunks - 1) / kRangeChunks);
    }
    case Plan::kSplit: return 4;
    default: return 2;
  }
}
// Bytes of the operand hand-over buffer between the pre-pass and the recurrence; for sequences
// long enough to run in ranges, two fp32 states follow the records (the state between ranges).
inline size_t scratch_bytes(int B, int T, int Hv) {
  const size_t nC = (size_t)(T + C - 1) / C;
  const size_t states = nC >= 2 * (size_t)kRangeChunks ? 2 * (size_t)B * Hv * 128 * 128 * 4 : 0;
  return (size_t)B * Hv * nC * kPwBytes + states;
}

// Per device: a high- and a low-priority stream and two events for the split launch below, and
// the SM count; calls enqueue under the mutex, so they never share the events.
struct Split {
  cudaStream_t s_hi = nullptr, s_lo = nullptr;
  cudaEvent_t ev_fork = nullptr, ev_pre = nullptr, ev_hi = nullptr, ev_lo = nullptr;
  int sms = 0;
  bool ready = false;
};
inline std::mutex& split_mutex() {
  static std::mutex mu;
  return mu;
}
inline Split* split_for_device() {   // call with split_mutex() held
  static Split splits[64];
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  Split& p = splits[dev];
  if (!p.ready) {
    int least = 0, greatest = 0;
    if (cudaDeviceGetStreamPriorityRange(&least, &greatest) != cudaSuccess ||
        cudaDeviceGetAttribute(&p.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaStreamCreateWithPriority(&p.s_hi, cudaStreamNonBlocking, greatest) != cudaSuccess ||
        cudaStreamCreateWithPriority(&p.s_lo, cudaStreamNonBlocking, least) != cudaSuccess)
      return nullptr;
    for (cudaEvent_t* e : {&p.ev_fork, &p.ev_pre, &p.ev_hi, &p.ev_lo})
      if (cudaEventCreateWithFlags(e, cudaEventDisableTiming) != cudaSuccess) return nullptr;
    p.ready = true;
  }
  return &p;
}

// The two kernels of one call on `st`.  `nseq` sequences.  Fixed length (cu == nullptr): [nseq, T,
// ...] tensors, max_len = T.  Packed: [T, ...] tensors of T tokens in all, sequence s at cu[s] ..
// cu[s + 1] - 1 (device offsets), none longer than max_len.  `pw`: nseq * Hv * ceil(max_len / 64)
// records.  The recurrence reads the pre-pass's records only after it in stream order.  `parts`:
// kPre, kRec or both; a recurrence launched alone must follow its pre-pass on `st` by an event.
constexpr int kPre = 1, kRec = 2;
// Gates taken from the in_proj_ba outputs (ba [tokens, 2 Hv] bf16) instead of log_alpha / beta
// (ba == nullptr: the gates are given).  at(): the same for the part of the call starting
// `tokens` tokens in.
struct GateSrc {
  const __nv_bfloat16* ba = nullptr;
  int Hv = 0;
  GateSrc at(size_t tokens) const { return GateSrc{ba ? ba + tokens * 2 * Hv : nullptr, Hv}; }
};
template <typename Tout>
gdn_status launch_one(const void* q, const void* k, const void* v, const float* la,
                      const float* be, const float* S0, Tout* o, float* S_T, int nseq, int T,
                      int Hk, int Hv, float scale, uint8_t* pw, const int* cu, int max_len,
                      const GateSrc& nrm, cudaStream_t st, cudaEvent_t ev_after_pre,
                      int parts = kPre | kRec) {
  const int mapB = cu ? 1 : nseq;
  CUtensorMap mq, mk, mo;
  if (!make_tile_map(&mq, q, Hk, T, mapB, false) || !make_tile_map(&mk, k, Hk, T, mapB, false) ||
      !make_tile_map(&mo, o, Hv, T, mapB, sizeof(Tout) == 4))
    return GDN_ERR_CUDA;
  auto kern = chunk_fwd_tc_kernel<Tout>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_ALLOC) !=
      cudaSuccess)
    return GDN_ERR_CUDA;
  if (cudaFuncSetAttribute(pw_prepass_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           PP_SMEM) != cudaSuccess)
    return GDN_ERR_CUDA;
  const long grid = (long)nseq * Hv;
  const int nCmax = (max_len + C - 1) / C;
  if (grid > 0x7fffffffL || nCmax > 65535 || nseq > 65535) return GDN_ERR_UNSUPPORTED;
  if (nCmax == 0) return GDN_OK;
  if (parts & kPre) {
    // head-fastest: the value heads that share a key head's Q/K tiles run side by side
    pw_prepass_kernel<<<dim3(Hv, nCmax, nseq), PP_THREADS, PP_SMEM, st>>>(
        mq, mk, la, be, pw, T, Hk, Hv, scale, cu, max_len, nrm.ba);
    if (cudaGetLastError() != cudaSuccess) return GDN_ERR_CUDA;
  }
  if (ev_after_pre && cudaEventRecord(ev_after_pre, st) != cudaSuccess) return GDN_ERR_CUDA;
  if (parts & kRec) {
    kern<<<(unsigned)grid, kThreads, SMEM_ALLOC, st>>>(
        mq, mk, mo, static_cast<const __nv_bfloat16*>(v), pw, S0, S_T, T, Hk, Hv, scale, cu,
        max_len, nCmax, o);
    if (cudaGetLastError() != cudaSuccess) return GDN_ERR_CUDA;
  }
  return GDN_OK;
}

// One call.  When a batched call has more (batch, head) recurrences than SMs, its recurrence would
// run in two waves with most SMs idle in the second.  The call is then split by batches: the tail
// batches go first (their pre-pass, then their recurrence on a high-priority stream), and the
// pre-pass of the leading batches runs on the SMs the tail's recurrence leaves free, after which
// their recurrence fills the GPU in one wave.  Results are those of one launch (the recurrences
// are independent); the caller's stream waits for both parts.
template <typename Tout>
gdn_status launch(const void* q, const void* k, const void* v, const float* la, const float* be,
                  const float* S0, Tout* o, float* S_T, int nseq, int T, int Hk, int Hv,
                  float scale, uint8_t* pw, const int* cu, int max_len, cudaStream_t st,
                  const GateSrc& nrm = GateSrc{}) {
  if ((max_len + C - 1) / C > 65535) return GDN_ERR_UNSUPPORTED;   // chunks index a grid's y
  std::unique_lock<std::mutex> lock(split_mutex());
  Split* sp = split_for_device();
  if (!sp) return GDN_ERR_CUDA;
  const Plan pl = plan(nseq, T, Hv, sp->sms, cu != nullptr);
  if (pl == Plan::kRanges) {
    // Ranges of kRangeChunks chunks: every pre-pass on the low-priority stream, one after the
    // other; the recurrence of range r on the high-priority stream once pre-pass r is done and
    // after recurrence r - 1, starting from its final state.  Pre-pass r + 1 thus runs on the
    // SMs recurrence r leaves idle.  Splitting at chunk boundaries gives the one-launch result.
    const int nC = (T + C - 1) / C, nR = (nC + kRangeChunks - 1) / kRangeChunks;
    float* mid[2];
    mid[0] = reinterpret_cast<float*>(pw + (size_t)Hv * nC * kPwBytes);
    mid[1] = mid[0] + (size_t)Hv * 128 * 128;
    bool ok = cudaEventRecord(sp->ev_fork, st) == cudaSuccess &&
              cudaStreamWaitEvent(sp->s_hi, sp->ev_fork, 0) == cudaSuccess &&
              cudaStreamWaitEvent(sp->s_lo, sp->ev_fork, 0) == cudaSuccess;
    gdn_status s = ok ? GDN_OK : GDN_ERR_CUDA;
    for (int r = 0; r < nR && s == GDN_OK; ++r) {
      const long t0 = (long)r * kRangeChunks * C;
      const int Tr = (int)std::min<long>(T - t0, (long)kRangeChunks * C);
      const auto* bq = static_cast<const __nv_bfloat16*>(q) + t0 * Hk * 128;
      const auto* bk = static_cast<const __nv_bfloat16*>(k) + t0 * Hk * 128;
      const auto* bv = static_cast<const __nv_bfloat16*>(v) + t0 * Hv * 128;
      const float* S0r = r == 0 ? S0 : mid[(r - 1) & 1];
      float* STr = r == nR - 1 ? S_T : mid[r & 1];
      uint8_t* pwr = pw + (size_t)Hv * r * kRangeChunks * kPwBytes;
      const GateSrc nr = nrm.at((size_t)t0);
      const float* lar = la ? la + t0 * Hv : nullptr;
      const float* ber = be ? be + t0 * Hv : nullptr;
      s = launch_one<Tout>(bq, bk, bv, lar, ber, S0r, o + t0 * Hv * 128, STr, 1,
                           Tr, Hk, Hv, scale, pwr, nullptr, Tr, nr, sp->s_lo, sp->ev_pre, kPre);
      if (s == GDN_OK && cudaStreamWaitEvent(sp->s_hi, sp->ev_pre, 0) != cudaSuccess)
        s = GDN_ERR_CUDA;
      if (s == GDN_OK)
        s = launch_one<Tout>(bq, bk, bv, lar, ber, S0r, o + t0 * Hv * 128, STr,
                             1, Tr, Hk, Hv, scale, pwr, nullptr, Tr, nr, sp->s_hi, nullptr, kRec);
    }
    const bool joined = cudaEventRecord(sp->ev_hi, sp->s_hi) == cudaSuccess &&
                        cudaEventRecord(sp->ev_lo, sp->s_lo) == cudaSuccess &&
                        cudaStreamWaitEvent(st, sp->ev_hi, 0) == cudaSuccess &&
                        cudaStreamWaitEvent(st, sp->ev_lo, 0) == cudaSuccess;
    return s != GDN_OK ? s : (joined ? GDN_OK : GDN_ERR_CUDA);
  }
  const int head_b = sp->sms / (Hv > 0 ? Hv : 1);        // batches that fill at most one wave
  if (pl == Plan::kOne) {
    lock.unlock();
    return launch_one<Tout>(q, k, v, la, be, S0, o, S_T, nseq, T, Hk, Hv, scale, pw, cu, max_len,
                            nrm, st, nullptr);
  }
  const int tail_b = nseq - head_b;
  const size_t tq = (size_t)T * Hk * 128, tv = (size_t)T * Hv * 128, tg = (size_t)T * Hv;
  const size_t ts = (size_t)Hv * 128 * 128;
  const size_t tpw = (size_t)Hv * ((T + C - 1) / C) * kPwBytes;
  auto at_b = [&](const void* p, size_t per_batch, int b, size_t esize) -> const void* {
    return p ? static_cast<const char*>(p) + (size_t)b * per_batch * esize : nullptr;
  };
  const void* qt = at_b(q, tq, head_b, 2);
  const void* kt = at_b(k, tq, head_b, 2);
  const void* vt = at_b(v, tv, head_b, 2);
  const float* lat = static_cast<const float*>(at_b(la, tg, head_b, 4));
  const float* bet = static_cast<const float*>(at_b(be, tg, head_b, 4));
  const float* S0t = static_cast<const float*>(at_b(S0, ts, head_b, 4));
  Tout* ot = const_cast<Tout*>(static_cast<const Tout*>(at_b(o, tv, head_b, sizeof(Tout))));
  float* STt = const_cast<float*>(static_cast<const float*>(at_b(S_T, ts, head_b, 4)));
  uint8_t* pwt = pw + (size_t)head_b * tpw;
  bool ok = cudaEventRecord(sp->ev_fork, st) == cudaSuccess &&
            cudaStreamWaitEvent(sp->s_hi, sp->ev_fork, 0) == cudaSuccess &&
            cudaStreamWaitEvent(sp->s_lo, sp->ev_fork, 0) == cudaSuccess;
  gdn_status s = ok ? GDN_OK : GDN_ERR_CUDA;
  if (s == GDN_OK)   // the tail: pre-pass, then its recurrence, both on the high-priority stream
    s = launch_one<Tout>(qt, kt, vt, lat, bet, S0t, ot, STt, tail_b, T, Hk, Hv, scale, pwt,
                         nullptr, T, nrm.at((size_t)head_b * T), sp->s_hi, sp->ev_pre);
  // the leading batches start once the tail's pre-pass is done
  if (s == GDN_OK && cudaStreamWaitEvent(sp->s_lo, sp->ev_pre, 0) != cudaSuccess)
    s = GDN_ERR_CUDA;
  if (s == GDN_OK)
    s = launch_one<Tout>(q, k, v, la, be, S0, o, S_T, head_b, T, Hk, Hv, scale, pw, nullptr, T,
                         nrm, sp->s_lo, nullptr);
  // the caller's stream waits for both parts, also after a failure, so no work outlives it
  const bool joined = cudaEventRecord(sp->ev_hi, sp->s_hi) == cudaSuccess &&
                      cudaEventRecord(sp->ev_lo, sp->s_lo) == cudaSuccess &&
                      cudaStreamWaitEvent(st, sp->ev_hi, 0) == cudaSuccess &&
                      cudaStreamWaitEvent(st, sp->ev_lo, 0) == cudaSuccess;
  return s != GDN_OK ? s : (joined ? GDN_OK : GDN_ERR_CUDA);
}

}  // namespace tcf

#ifdef GDN_TC_TRACE
extern "C" GDN_API void gdn_debug_set_trace(void* p) {
  cudaMemcpyToSymbol(tcf::g_tc_trace, &p, sizeof(p));
}
#endif

// Kernel launches of one tensor-core call on a device of `sms` SMs, or on the current device when
// sms is 0 (-1 if that query fails).
inline int tc_chunk_launches(int nseq, int T, int Hv, bool packed, int sms) {
  if (sms == 0) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return -1;
  }
  return tcf::launch_count(nseq, T, Hv, sms, packed);
}

inline bool tc_chunk_supported(int dk, int dv, int chunk, bool bf16) {
  return bf16 && dk == 128 && dv == 128 && chunk == tcf::C;
}

// Sequences of up to 65535 chunks (the pre-pass's grid holds the chunk index in y).
inline bool tc_chunk_length_ok(long max_len) { return (max_len + tcf::C - 1) / tcf::C <= 65535; }

// Scratch bytes of the tensor-core forward (the pre-pass's operand hand-over buffer).
inline size_t tc_chunk_scratch_bytes(int B, int T, int Hv) { return tcf::scratch_bytes(B, T, Hv); }

// o in bf16, or in fp32 when f32out (o's box stores then carry fp32 and the X product takes the
// state as a hi + lo pair).
// `ba` (optional, [B, T, 2 Hv] bf16): gates from the in_proj_ba outputs instead of la / be.
inline gdn_status tc_chunk_launch(const void* q, const void* k, const void* v, const float* la,
                                  const float* be, const float* S0, void* o, float* S_T, int B,
                                  int T, int Hk, int Hv, float scale, bool f32out, void* scratch,
                                  cudaStream_t st, const void* ba = nullptr) {
  uint8_t* pw = static_cast<uint8_t*>(scratch);
  const tcf::GateSrc ex{static_cast<const __nv_bfloat16*>(ba), Hv};
  if (f32out)
    return tcf::launch<float>(q, k, v, la, be, S0, static_cast<float*>(o), S_T, B, T, Hk, Hv,
                              scale, pw, nullptr, T, st, ex);
  return tcf::launch<__nv_bfloat16>(q, k, v, la, be, S0, static_cast<__nv_bfloat16*>(o), S_T, B,
                                    T, Hk, Hv, scale, pw, nullptr, T, st, ex);
}

// Packed sequences: q, k [total, Hk, 128], v, o [total, Hv, 128], gates [total, Hv]; sequence s is
// tokens cu[s] .. cu[s + 1] - 1 (device int32 offsets), none longer than max_len; S0, S_T
// [nseq, Hv, 128, 128].  `scratch`: tc_chunk_varlen_scratch_bytes(nseq, max_len, Hv).
inline size_t tc_chunk_varlen_scratch_bytes(int nseq, int max_len, int Hv) {
  return tcf::scratch_bytes(nseq, max_len, Hv);
}
inline gdn_status tc_chunk_launch_varlen(const void* q, const void* k, const void* v,
                                         const float* la, const float* be, const int* cu,
                                         int nseq, int max_len, const float* S0, void* o,
                                         float* S_T, int total, int Hk, int Hv, float scale,
                                         bool f32out, void* scratch, cudaStream_t st) {
  uint8_t* pw = static_cast<uint8_t*>(scratch);
  if (f32out)
    return tcf::launch<float>(q, k, v, la, be, S0, static_cast<float*>(o), S_T, nseq, total, Hk,
                              Hv, scale, pw, cu, max_len, st);
  return tcf::launch<__nv_bfloat16>(q, k, v, la, be, S0, static_cast<__nv_bfloat16*>(o), S_T,
                                    nseq, total, Hk, Hv, scale, pw, cu, max_len, st);
}

}  // namespace gdn
