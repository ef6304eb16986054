// Chunked forward of the gated delta rule on CUDA cores, fp32 arithmetic (any supported shape).
//
// Chunk algebra ("Chapitre 16 - Assembler un système de type Kimi K3", 16.2: blocks of tokens are
// processed with matrix operations and the state is handed from block to block).  For one value
// head and one block of C tokens with block-start state M (= S^T, dk x dv):
//   G_i   = sum_{s<=i} log alpha_s,  gamma_i = exp(G_i),  Gam_ij = exp(G_i - G_j)  (i >= j, <= 1)
//   A     = strict_lower(beta_i Gam_ij k_i.k_j),  T = (I + A)^-1   (forward substitution)
//   W     = T diag(beta gamma) K,  U = T diag(beta) V,  Delta = U - W M
//   O     = diag(gamma) Q M + P Delta,  P = lower_incl(Gam_ij q_i.k_j)
//   M'    = gamma_last M + Ktil^T Delta,  Ktil_j = exp(G_last - G_j) k_j
// which is the token recurrence M_t = alpha_t (I - beta_t k_t k_t^T) M_{t-1} + beta_t k_t v_t^T,
// o_t = M_t^T q_t reorganised exactly (row i of Delta is beta_i (v_i - alpha_i M_{i-1}^T k_i)).
// Rows past T in the last block act as alpha = 1, beta = 0, k = 0 (identity update), unstored.
//
// One CTA per (dv tile of DVT columns, value head, batch); the dv columns of M evolve
// independently, so tiles need no communication.  Everything lives in shared memory in fp32.
#pragma once

#include "common.cuh"

namespace gdn {

constexpr int kSimtThreads = 256;

template <int DK, int DVT, int C>
constexpr size_t simt_chunk_smem_floats() {
  return 3 * C * DK + DK * DVT + 2 * C * DVT + 3 * C * C + 4 * C;
}

template <int DK, int DVT, int C, typename Tio, typename Tout>
__global__ void __launch_bounds__(kSimtThreads)
chunk_fwd_simt_kernel(const Tio* __restrict__ q, const Tio* __restrict__ k,
                      const Tio* __restrict__ v, const float* __restrict__ log_alpha,
                      const float* __restrict__ beta, const float* __restrict__ S0,
                      Tout* __restrict__ o, float* __restrict__ S_T, int T, int Hk, int Hv,
                      int dv, float scale) {
  constexpr int NT = kSimtThreads;
  const int j0 = blockIdx.x * DVT;
  const int h = blockIdx.y;
  const long b = blockIdx.z;
  const int hk = h / (Hv / Hk);
  const int tid = threadIdx.x;

  extern __shared__ float smem[];
  float* sQ = smem;               // [C][DK]  q * scale
  float* sK = sQ + C * DK;        // [C][DK]
  float* sW = sK + C * DK;        // [C][DK]
  float* sM = sW + C * DK;        // [DK][DVT] state tile
  float* sV = sM + DK * DVT;      // [C][DVT] v, then Delta
  float* sU = sV + C * DVT;       // [C][DVT]
  float* sA = sU + C * DVT;       // [C][C]
  float* sT = sA + C * C;         // [C][C]   (I + A)^-1, then times diag(beta)
  float* sP = sT + C * C;         // [C][C]
  float* sG = sP + C * C;         // [C] cumulative log decay
  float* sB = sG + C;             // [C] beta
  float* sGam = sB + C;           // [C] gamma_j = exp(G_j)
  float* sKt = sGam + C;          // [C] exp(G_last - G_j)

  for (int idx = tid; idx < DK * DVT; idx += NT) {
    const int i = idx / DVT, j = idx % DVT;
    sM[idx] = S0 ? S0[((b * Hv + h) * DK + i) * (long)dv + j0 + j] : 0.f;
  }
  const int nchunks = (T + C - 1) / C;
  for (int c = 0; c < nchunks; ++c) {
    const long t0 = (long)c * C;
    const int len = min((long)C, (long)T - t0);
    __syncthreads();
    for (int idx = tid; idx < C * DK; idx += NT) {
      const int i = idx / DK, d = idx % DK;
      float qq = 0.f, kk = 0.f;
      if (i < len) {
        const long off = ((b * T + t0 + i) * Hk + hk) * (long)DK + d;
        qq = to_f(q[off]) * scale;
        kk = to_f(k[off]);
      }
      sQ[idx] = qq;
      sK[idx] = kk;
    }
    for (int idx = tid; idx < C * DVT; idx += NT) {
      const int i = idx / DVT, j = idx % DVT;
      sV[idx] = (i < len) ? to_f(v[((b * T + t0 + i) * Hv + h) * (long)dv + j0 + j]) : 0.f;
    }
    if (tid < C) {
      float la = 0.f, bt = 0.f;
      if (tid < len) {
        const long g = (b * T + t0 + tid) * Hv + h;
        la = log_alpha[g];
        bt = beta[g];
      }
      sG[tid] = la;
      sB[tid] = bt;
    }
    __syncthreads();
    if (tid == 0) {
      float acc = 0.f;
      for (int i = 0; i < C; ++i) { acc += sG[i]; sG[i] = acc; }
    }
    __syncthreads();
    if (tid < C) {
      sGam[tid] = expf(sG[tid]);
      sKt[tid] = expf(sG[C - 1] - sG[tid]);
    }
    // A (strictly lower) and P (lower, diagonal included)
    for (int idx = tid; idx < C * C; idx += NT) {
      const int i = idx / C, j = idx % C;
      float a = 0.f, p = 0.f;
      if (j <= i) {
        float kk = 0.f, qk = 0.f;
        for (int d = 0; d < DK; ++d) {
          const float kj = sK[j * DK + d];
          kk += sK[i * DK + d] * kj;
          qk += sQ[i * DK + d] * kj;
        }
        const float gam = expf(sG[i] - sG[j]);
        p = gam * qk;
        if (j < i) a = sB[i] * gam * kk;
      }
      sA[idx] = a;
      sP[idx] = p;
    }
    __syncthreads();
    // T = (I + A)^-1: column `col` solves (I + A) x = e_col by forward substitution
    if (tid < C) {
      const int col = tid;
      for (int i = 0; i < C; ++i) {
        float val = (i == col) ? 1.f : 0.f;
        if (i > col) {
          float acc = 0.f;
          for (int j = col; j < i; ++j) acc += sA[i * C + j] * sT[j * C + col];
          val = -acc;
        }
        sT[i * C + col] = val;
      }
    }
    __syncthreads();
    for (int idx = tid; idx < C * C; idx += NT) sT[idx] *= sB[idx % C];
    __syncthreads();
    for (int idx = tid; idx < C * DK; idx += NT) {
      const int i = idx / DK, d = idx % DK;
      float acc = 0.f;
      for (int j = 0; j <= i; ++j) acc += sT[i * C + j] * sGam[j] * sK[j * DK + d];
      sW[idx] = acc;
    }
    for (int idx = tid; idx < C * DVT; idx += NT) {
      const int i = idx / DVT, n = idx % DVT;
      float acc = 0.f;
      for (int j = 0; j <= i; ++j) acc += sT[i * C + j] * sV[j * DVT + n];
      sU[idx] = acc;
    }
    __syncthreads();
    for (int idx = tid; idx < C * DVT; idx += NT) {          // Delta = U - W M  (into sV)
      const int i = idx / DVT, n = idx % DVT;
      float acc = 0.f;
      for (int d = 0; d < DK; ++d) acc += sW[i * DK + d] * sM[d * DVT + n];
      sV[idx] = sU[idx] - acc;
    }
    __syncthreads();
    for (int idx = tid; idx < C * DVT; idx += NT) {          // O = diag(gamma) Q M + P Delta
      const int i = idx / DVT, n = idx % DVT;
      if (i < len) {
        float qm = 0.f;
        for (int d = 0; d < DK; ++d) qm += sQ[i * DK + d] * sM[d * DVT + n];
        float pd = 0.f;
        for (int j = 0; j <= i; ++j) pd += sP[i * C + j] * sV[j * DVT + n];
        o[((b * T + t0 + i) * Hv + h) * (long)dv + j0 + n] = from_f<Tout>(sGam[i] * qm + pd);
      }
    }
    __syncthreads();
    const float decay = sGam[C - 1];
    for (int idx = tid; idx < DK * DVT; idx += NT) {          // M' = gamma_last M + Ktil^T Delta
      const int d = idx / DVT, n = idx % DVT;
      float acc = 0.f;
      for (int j = 0; j < C; ++j) acc += sKt[j] * sK[j * DK + d] * sV[j * DVT + n];
      sM[idx] = decay * sM[idx] + acc;
    }
  }
  __syncthreads();
  if (S_T) {
    for (int idx = tid; idx < DK * DVT; idx += NT) {
      const int i = idx / DVT, j = idx % DVT;
      S_T[((b * Hv + h) * DK + i) * (long)dv + j0 + j] = sM[idx];
    }
  }
}

}  // namespace gdn
