// C ABI of the gated delta rule library (declared in include/gdn.h): argument validation,
// kernel selection and launches.  All kernels of the library are compiled in this one unit.
#include <stdint.h>
#include <string.h>

#include <mutex>

#include "gdn.h"
#include "common.cuh"
#include "decode.cuh"
#include "bwd.cuh"
#include "decode_layer.cuh"
#include "elementwise.cuh"
#include "layer_bwd.cuh"
#include "simt_chunk.cuh"
#include "tc_chunk.cuh"

using namespace gdn;

namespace {

constexpr int kVersion = 10000;   // 1.0.0

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool opt_aligned16(const void* p) { return p == nullptr || aligned16(p); }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
bool opt_aligned4(const void* p) { return p == nullptr || aligned4(p); }
bool supported_dim(int d) { return d == 16 || d == 32 || d == 64 || d == 128; }
bool supported_chunk(int c) { return c == 16 || c == 32 || c == 64; }
bool valid_dtype(gdn_dtype t) { return t == GDN_F32 || t == GDN_BF16; }

gdn_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}

// ---------------------------------------------------------------------------------------------
// SIMT chunked forward dispatch: DK in {16,32,64,128} x C in {16,32,64}, dv tiles of 16 columns.
// ---------------------------------------------------------------------------------------------
template <int DK, int C, typename Tio, typename Tout>
gdn_status simt_launch(const void* q, const void* k, const void* v, const float* la,
                       const float* be, const float* S0, void* o, float* S_T, int B, int T,
                       int Hk, int Hv, int dv, float scale, cudaStream_t st) {
  constexpr int DVT = 16;
  auto kern = chunk_fwd_simt_kernel<DK, DVT, C, Tio, Tout>;
  const size_t smem = simt_chunk_smem_floats<DK, DVT, C>() * sizeof(float);
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return GDN_ERR_CUDA;
  dim3 grid(dv / DVT, Hv, B);
  kern<<<grid, kSimtThreads, smem, st>>>(
      static_cast<const Tio*>(q), static_cast<const Tio*>(k), static_cast<const Tio*>(v), la,
      be, S0, static_cast<Tout*>(o), S_T, T, Hk, Hv, dv, scale);
  return launch_status();
}

template <typename Tio, typename Tout = Tio>
gdn_status simt_dispatch(int dk, int chunk, const void* q, const void* k, const void* v,
                         const float* la, const float* be, const float* S0, void* o, float* S_T,
                         int B, int T, int Hk, int Hv, int dv, float scale, cudaStream_t st) {
#define GDN_SIMT_CASE(DK_, C_)                                                             \
  if (dk == DK_ && chunk == C_)                                                            \
    return simt_launch<DK_, C_, Tio, Tout>(q, k, v, la, be, S0, o, S_T, B, T, Hk, Hv, dv, scale, \
                                           st);
  GDN_SIMT_CASE(16, 16) GDN_SIMT_CASE(16, 32) GDN_SIMT_CASE(16, 64)
  GDN_SIMT_CASE(32, 16) GDN_SIMT_CASE(32, 32) GDN_SIMT_CASE(32, 64)
  GDN_SIMT_CASE(64, 16) GDN_SIMT_CASE(64, 32) GDN_SIMT_CASE(64, 64)
  GDN_SIMT_CASE(128, 16) GDN_SIMT_CASE(128, 32) GDN_SIMT_CASE(128, 64)
#undef GDN_SIMT_CASE
  return GDN_ERR_UNSUPPORTED;
}

// ---------------------------------------------------------------------------------------------
// Decode dispatch over (dk, dv)
// ---------------------------------------------------------------------------------------------
template <int DK, int DV, typename Tio, typename Tout>
gdn_status decode_launch(const void* q, const void* k, const void* v, const float* la,
                         const float* be, float* S, void* o, int N, int Hk, int Hv, float scale,
                         cudaStream_t st) {
  using Sh = DecodeShape<DK, DV>;
  decode_step_kernel<DK, DV, Tio, Tout><<<(unsigned)((long)N * Hv), Sh::NT, 0, st>>>(
      static_cast<const Tio*>(q), static_cast<const Tio*>(k), static_cast<const Tio*>(v), la,
      be, S, static_cast<Tout*>(o), Hk, Hv, scale);
  return launch_status();
}

template <typename Tio, typename Tout, int DK>
gdn_status decode_dispatch_dv(int dv, const void* q, const void* k, const void* v,
                              const float* la, const float* be, float* S, void* o, int N, int Hk,
                              int Hv, float scale, cudaStream_t st) {
  switch (dv) {
    case 16: return decode_launch<DK, 16, Tio, Tout>(q, k, v, la, be, S, o, N, Hk, Hv, scale, st);
    case 32: return decode_launch<DK, 32, Tio, Tout>(q, k, v, la, be, S, o, N, Hk, Hv, scale, st);
    case 64: return decode_launch<DK, 64, Tio, Tout>(q, k, v, la, be, S, o, N, Hk, Hv, scale, st);
    case 128:
      return decode_launch<DK, 128, Tio, Tout>(q, k, v, la, be, S, o, N, Hk, Hv, scale, st);
  }
  return GDN_ERR_UNSUPPORTED;
}

template <typename Tio, typename Tout>
gdn_status decode_dispatch(int dk, int dv, const void* q, const void* k, const void* v,
                           const float* la, const float* be, float* S, void* o, int N, int Hk,
                           int Hv, float scale, cudaStream_t st) {
  switch (dk) {
    case 16:
      return decode_dispatch_dv<Tio, Tout, 16>(dv, q, k, v, la, be, S, o, N, Hk, Hv, scale, st);
    case 32:
      return decode_dispatch_dv<Tio, Tout, 32>(dv, q, k, v, la, be, S, o, N, Hk, Hv, scale, st);
    case 64:
      return decode_dispatch_dv<Tio, Tout, 64>(dv, q, k, v, la, be, S, o, N, Hk, Hv, scale, st);
    case 128:
      return decode_dispatch_dv<Tio, Tout, 128>(dv, q, k, v, la, be, S, o, N, Hk, Hv, scale, st);
  }
  return GDN_ERR_UNSUPPORTED;
}

// ---------------------------------------------------------------------------------------------
// Failure-detection self-test: one thread waits on a barrier that nothing completes
// ---------------------------------------------------------------------------------------------
__global__ void wait_timeout_selftest_kernel(unsigned long long budget) {
  __shared__ __align__(8) unsigned long long bar;
  __shared__ int abort_word;
  if (threadIdx.x == 0) {
    const uint32_t b = tc::smem_u32(&bar);
    tc::mbar_init(b, 1);                  // phase 0 needs one arrive; none comes
    tc::fence_barrier_init();
    abort_word = 0;
    volatile int* abort_flag = &abort_word;
    if (!tc::mbar_wait(b, 0, abort_flag, budget)) record_error(kErrTimeout);
  }
}

// ---------------------------------------------------------------------------------------------
// Full-layer decode step dispatch over (dk, dv)
// ---------------------------------------------------------------------------------------------
struct DecodeLayerArgs {
  const void *q_raw, *k_raw, *v_raw, *z, *hq_in, *hk_in, *hv_in;
  void *hq_out, *hk_out, *hv_out;
  const float *wq, *wk, *wv, *la, *be;
  float* S;
  const float* norm_w;
  void* y;
  int N, Hk, Hv;
  float scale, l2_eps, norm_eps;
};

template <int DK, int DV, typename Tio>
gdn_status decode_layer_launch(const DecodeLayerArgs& a, cudaStream_t st) {
  using Sh = DecodeShape<DK, DV>;
  decode_layer_step_kernel<DK, DV, Tio><<<(unsigned)((long)a.N * a.Hv), Sh::NT, 0, st>>>(
      static_cast<const Tio*>(a.q_raw), static_cast<const Tio*>(a.k_raw),
      static_cast<const Tio*>(a.v_raw), static_cast<const Tio*>(a.z),
      static_cast<const Tio*>(a.hq_in), static_cast<const Tio*>(a.hk_in),
      static_cast<const Tio*>(a.hv_in), static_cast<Tio*>(a.hq_out), static_cast<Tio*>(a.hk_out),
      static_cast<Tio*>(a.hv_out), a.wq, a.wk, a.wv, a.la, a.be, a.S, a.norm_w,
      static_cast<Tio*>(a.y), a.Hk, a.Hv, a.scale, a.l2_eps, a.norm_eps);
  return launch_status();
}

template <typename Tio, int DK>
gdn_status decode_layer_dispatch_dv(int dv, const DecodeLayerArgs& a, cudaStream_t st) {
  switch (dv) {
    case 16: return decode_layer_launch<DK, 16, Tio>(a, st);
    case 32: return decode_layer_launch<DK, 32, Tio>(a, st);
    case 64: return decode_layer_launch<DK, 64, Tio>(a, st);
    case 128: return decode_layer_launch<DK, 128, Tio>(a, st);
  }
  return GDN_ERR_UNSUPPORTED;
}

template <typename Tio>
gdn_status decode_layer_dispatch(int dk, int dv, const DecodeLayerArgs& a, cudaStream_t st) {
  switch (dk) {
    case 16: return decode_layer_dispatch_dv<Tio, 16>(dv, a, st);
    case 32: return decode_layer_dispatch_dv<Tio, 32>(dv, a, st);
    case 64: return decode_layer_dispatch_dv<Tio, 64>(dv, a, st);
    case 128: return decode_layer_dispatch_dv<Tio, 128>(dv, a, st);
  }
  return GDN_ERR_UNSUPPORTED;
}

// The recurrence inside gdn_layer_fwd: inputs in `dtype`, output o in fp32 (for the separate
// gated norm); `scratch` is the tensor-core forward's hand-over buffer (part of the layer
// workspace).
gdn_status layer_chunk_fwd(const void* q, const void* k, const void* v, const float* la,
                           const float* be, const float* S0, float* o, float* S_T, int B, int T,
                           int Hk, int Hv, int dk, int dv, int chunk, float scale,
                           gdn_dtype dtype, void* scratch, cudaStream_t st) {
  if (tc_chunk_supported(dk, dv, chunk, dtype == GDN_BF16))
    return tc_chunk_launch(q, k, v, la, be, S0, o, S_T, B, T, Hk, Hv, scale, true, scratch, st);
  if (dtype == GDN_F32)
    return simt_dispatch<float, float>(dk, chunk, q, k, v, la, be, S0, o, S_T, B, T, Hk, Hv, dv,
                                       scale, st);
  return simt_dispatch<__nv_bfloat16, float>(dk, chunk, q, k, v, la, be, S0, o, S_T, B, T, Hk,
                                             Hv, dv, scale, st);
}

// A caller workspace: present, 256-byte aligned and large enough for `need` bytes.
bool workspace_ok(const void* ws, size_t bytes, size_t need) {
  if (need == 0) return true;
  return ws != nullptr && bytes >= need && (reinterpret_cast<uintptr_t>(ws) & 255u) == 0;
}

// Input/output dtype pairs with a kernel: fp32 -> fp32, bf16 -> bf16, bf16 -> fp32.
bool io_pair_ok(gdn_dtype in, gdn_dtype out) { return !(in == GDN_F32 && out == GDN_BF16); }

gdn_status validate_heads(int Hk, int Hv, int dk, int dv) {
  if (Hk <= 0 || Hv <= 0 || dk <= 0 || dv <= 0 || Hv % Hk != 0) return GDN_ERR_INVALID_ARG;
  if (Hv > 65535) return GDN_ERR_UNSUPPORTED;
  if (!supported_dim(dk) || !supported_dim(dv)) return GDN_ERR_UNSUPPORTED;
  return GDN_OK;
}

// ---------------------------------------------------------------------------------------------
// Backward pass: checkpoints every bwd::kSeg tokens; per-slice dq, dk (when key heads are shared
// or heads are split over CTAs) and dlog alpha, dbeta (when heads are split), summed afterwards.
// Workspace sections 256-aligned.
// ---------------------------------------------------------------------------------------------
size_t align256(size_t n) { return (n + 255) & ~(size_t)255; }
struct BwdLayout {
  size_t dqh = 0, dkh = 0, dah = 0, dbh = 0, total = 0;   // section offsets; total bytes
};
// nseq sequences of at most max_len tokens, `rows` token rows in all: checkpoints per (sequence,
// head) for max_len tokens, per-token partials for every row.
BwdLayout bwd_layout_rows(int nseq, int max_len, size_t rows, int Hk, int Hv, int dk, int dv) {
  BwdLayout L;
  const size_t ns = (size_t)bwd::head_slices(dk);
  const size_t nseg = ((size_t)max_len + bwd::kSeg - 1) / bwd::kSeg;
  const size_t ck = align256((size_t)nseq * Hv * nseg * dk * dv * sizeof(float));
  const bool direct = Hv == Hk && ns == 1;
  const size_t per = direct ? 0 : align256(rows * Hv * ns * dk * sizeof(float));
  const size_t gate = ns > 1 ? align256(rows * Hv * ns * sizeof(float)) : 0;
  L.dqh = ck;
  L.dkh = ck + per;
  L.dah = ck + 2 * per;
  L.dbh = ck + 2 * per + gate;
  L.total = ck + 2 * per + 2 * gate;
  return L;
}
BwdLayout bwd_layout(int B, int T, int Hk, int Hv, int dk, int dv) {
  return bwd_layout_rows(B, T, (size_t)B * T, Hk, Hv, dk, dv);
}

template <int D, typename Tin, typename Tdo = Tin>
gdn_status bwd_launch(const void* q, const void* k, const void* v, const float* la,
                      const float* be, const float* S0, const void* dO, const float* dST,
                      float* dq, float* dk, float* dv, float* dla, float* dbeta, float* dS0,
                      void* ws, int B, int T, int Hk, int Hv, float scale, cudaStream_t st,
                      const int* cu = nullptr, int max_len = -1) {
  // B sequences: [B, T] rows, or (cu) packed rows of T in all, none longer than max_len
  if (!cu) max_len = T;
  const long rows = cu ? (long)T : (long)B * T;
  constexpr int NS = bwd::Shape<D>::NS;
  auto kern = bwd::bwd_kernel<D, Tin, Tdo>;
  const size_t smem = bwd::smem_bytes<D>();
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) !=
      cudaSuccess)
    return GDN_ERR_CUDA;
  const BwdLayout L = bwd_layout_rows(B, max_len, (size_t)rows, Hk, Hv, D, D);
  uint8_t* w = static_cast<uint8_t*>(ws);
  const bool direct = Hv == Hk && NS == 1;
  float* dqo = direct ? dq : reinterpret_cast<float*>(w + L.dqh);
  float* dko = direct ? dk : reinterpret_cast<float*>(w + L.dkh);
  float* dao = NS > 1 ? reinterpret_cast<float*>(w + L.dah) : dla;
  float* dbo = NS > 1 ? reinterpret_cast<float*>(w + L.dbh) : dbeta;
  const long ctas = (long)B * Hv * NS;
  if (ctas > 0x7fffffffL) return GDN_ERR_UNSUPPORTED;
  kern<<<(unsigned)ctas, bwd::Shape<D>::NT, smem, st>>>(
      static_cast<const Tin*>(q), static_cast<const Tin*>(k), static_cast<const Tin*>(v), la, be,
      S0, static_cast<const Tdo*>(dO), dST, dqo, dko, direct ? 1 : 0, dv, dao, dbo, dS0,
      reinterpret_cast<float*>(w), T, Hk, Hv, scale, cu, max_len);
  if (cudaGetLastError() != cudaSuccess) return GDN_ERR_CUDA;
  auto sum = [&](const float* a_src, float* a_dst, const float* b_src, float* b_dst, long rows,
                 int G, int Dd) {
    const long n = 2 * rows * Dd;
    const unsigned blocks = (unsigned)std::min<long>((n + 255) / 256, 148L * 16);
    if (blocks > 0) bwd::group_sum_kernel<<<blocks, 256, 0, st>>>(a_src, a_dst, b_src, b_dst, rows, G, Dd);
  };
  if (!direct && rows > 0) sum(dqo, dq, dko, dk, rows * Hk, (Hv / Hk) * NS, D);
  if (NS > 1 && rows > 0) sum(dao, dla, dbo, dbeta, rows * Hv, NS, 1);
  return launch_status();
}

template <typename Tin, typename Tdo = Tin>
gdn_status bwd_dispatch(int d, const void* q, const void* k, const void* v, const float* la,
                        const float* be, const float* S0, const void* dO, const float* dST,
                        float* dq, float* dk, float* dv, float* dla, float* dbeta, float* dS0,
                        void* ws, int B, int T, int Hk, int Hv, float scale, cudaStream_t st,
                        const int* cu = nullptr, int max_len = -1) {
#define GDN_BWD(D)                                                                              \
  case D:                                                                                       \
    return bwd_launch<D, Tin, Tdo>(q, k, v, la, be, S0, dO, dST, dq, dk, dv, dla, dbeta, dS0, ws, \
                                   B, T, Hk, Hv, scale, st, cu, max_len);
  switch (d) {
    GDN_BWD(16)
    GDN_BWD(32)
    GDN_BWD(64)
    GDN_BWD(128)
    default: return GDN_ERR_UNSUPPORTED;
  }
#undef GDN_BWD
}

}  // namespace

extern "C" {

int gdn_bwd_launches(int B, int T, int Hk, int Hv, int dk, int dv) {
  if (B < 0 || T < 0 || validate_heads(Hk, Hv, dk, dv) != GDN_OK || dk != dv) return -1;
  if (B == 0) return 0;
  const int ns = bwd::head_slices(dk);
  if (T == 0) return 1;                       // the kernel alone hands dS_T to dS0
  return 1 + ((Hv == Hk && ns == 1) ? 0 : 1) + (ns > 1 ? 1 : 0);
}

size_t gdn_bwd_workspace_bytes(int B, int T, int Hk, int Hv, int dk, int dv) {
  if (B < 0 || T < 0 || validate_heads(Hk, Hv, dk, dv) != GDN_OK || dk != dv) return 0;
  if ((long)B * T == 0) return 0;
  return bwd_layout(B, T, Hk, Hv, dk, dv).total;
}

gdn_status gdn_bwd(const void* q, const void* k, const void* v, const float* log_alpha,
                   const float* beta, const float* S0, const void* dO, const float* dS_T,
                   float* dq, float* dk, float* dv, float* dlog_alpha, float* dbeta, float* dS0,
                   void* workspace, size_t workspace_bytes, int B, int T, int Hk, int Hv,
                   int dk_, int dv_, float scale, gdn_dtype dtype, gdn_stream_t stream) {
  if (B < 0 || T < 0 || !valid_dtype(dtype)) return GDN_ERR_INVALID_ARG;
  gdn_status s = validate_heads(Hk, Hv, dk_, dv_);
  if (s != GDN_OK) return s;
  if (dk_ != dv_) return GDN_ERR_UNSUPPORTED;
  if ((long)B * Hv > 0x7fffffffL) return GDN_ERR_UNSUPPORTED;
  const bool work = (long)B * T > 0;
  if (work && (!q || !k || !v || !log_alpha || !beta || !dO || !dq || !dk || !dv ||
               !dlog_alpha || !dbeta))
    return GDN_ERR_INVALID_ARG;
  if (!opt_aligned4(q) || !opt_aligned4(k) || !opt_aligned4(v) || !opt_aligned4(dO) ||
      !opt_aligned4(log_alpha) || !opt_aligned4(beta) || !opt_aligned4(dq) ||
      !opt_aligned4(dk) || !opt_aligned4(dlog_alpha) || !opt_aligned4(dbeta) ||
      !opt_aligned16(dv) || !opt_aligned16(S0) || !opt_aligned16(dS_T) || !opt_aligned16(dS0))
    return GDN_ERR_INVALID_ARG;
  if (work && !workspace_ok(workspace, workspace_bytes, bwd_layout(B, T, Hk, Hv, dk_, dv_).total))
    return GDN_ERR_INVALID_ARG;
  if (B == 0) return GDN_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == GDN_F32)
    return bwd_dispatch<float>(dk_, q, k, v, log_alpha, beta, S0, dO, dS_T, dq, dk, dv,
                               dlog_alpha, dbeta, dS0, workspace, B, T, Hk, Hv, scale, st);
  return bwd_dispatch<__nv_bfloat16>(dk_, q, k, v, log_alpha, beta, S0, dO, dS_T, dq, dk, dv,
                                     dlog_alpha, dbeta, dS0, workspace, B, T, Hk, Hv, scale, st);
}

size_t gdn_bwd_varlen_workspace_bytes(int nseq, int max_seqlen, int total_T, int Hk, int Hv,
                                      int dk, int dv) {
  if (nseq <= 0 || max_seqlen < 0 || total_T < 0 || validate_heads(Hk, Hv, dk, dv) != GDN_OK ||
      dk != dv)
    return 0;
  return bwd_layout_rows(nseq, max_seqlen, (size_t)total_T, Hk, Hv, dk, dv).total;
}

gdn_status gdn_bwd_varlen(const void* q, const void* k, const void* v, const float* log_alpha,
                          const float* beta, const int* cu_seqlens, int nseq, int max_seqlen,
                          const float* S0, const void* dO, const float* dS_T, float* dq,
                          float* dk, float* dv, float* dlog_alpha, float* dbeta, float* dS0,
                          void* workspace, size_t workspace_bytes, int total_T, int Hk, int Hv,
                          int dk_, int dv_, float scale, gdn_dtype dtype, gdn_stream_t stream) {
  if (nseq < 0 || max_seqlen < 0 || total_T < 0 || !valid_dtype(dtype)) return GDN_ERR_INVALID_ARG;
  gdn_status s = validate_heads(Hk, Hv, dk_, dv_);
  if (s != GDN_OK) return s;
  if (dk_ != dv_) return GDN_ERR_UNSUPPORTED;
  if ((long)nseq * Hv * bwd::head_slices(dk_) > 0x7fffffffL) return GDN_ERR_UNSUPPORTED;
  if (nseq == 0) return GDN_OK;
  if (!cu_seqlens || !aligned4(cu_seqlens)) return GDN_ERR_INVALID_ARG;
  const bool work = total_T > 0 && max_seqlen > 0;
  if (work && (!q || !k || !v || !log_alpha || !beta || !dO || !dq || !dk || !dv ||
               !dlog_alpha || !dbeta))
    return GDN_ERR_INVALID_ARG;
  if (!opt_aligned4(q) || !opt_aligned4(k) || !opt_aligned4(v) || !opt_aligned4(dO) ||
      !opt_aligned4(log_alpha) || !opt_aligned4(beta) || !opt_aligned4(dq) ||
      !opt_aligned4(dk) || !opt_aligned4(dlog_alpha) || !opt_aligned4(dbeta) ||
      !opt_aligned16(dv) || !opt_aligned16(S0) || !opt_aligned16(dS_T) || !opt_aligned16(dS0))
    return GDN_ERR_INVALID_ARG;
  const int ml = work ? max_seqlen : 0;
  if (!workspace_ok(workspace, workspace_bytes,
                    bwd_layout_rows(nseq, ml, (size_t)total_T, Hk, Hv, dk_, dv_).total))
    return GDN_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == GDN_F32)
    return bwd_dispatch<float>(dk_, q, k, v, log_alpha, beta, S0, dO, dS_T, dq, dk, dv,
                               dlog_alpha, dbeta, dS0, workspace, nseq, total_T, Hk, Hv, scale,
                               st, cu_seqlens, ml);
  return bwd_dispatch<__nv_bfloat16>(dk_, q, k, v, log_alpha, beta, S0, dO, dS_T, dq, dk, dv,
                                     dlog_alpha, dbeta, dS0, workspace, nseq, total_T, Hk, Hv,
                                     scale, st, cu_seqlens, ml);
}

const char* gdn_status_string(gdn_status s) {
  switch (s) {
    case GDN_OK: return "GDN_OK";
    case GDN_ERR_INVALID_ARG: return "GDN_ERR_INVALID_ARG";
    case GDN_ERR_UNSUPPORTED: return "GDN_ERR_UNSUPPORTED";
    case GDN_ERR_CUDA: return "GDN_ERR_CUDA";
    case GDN_ERR_TIMEOUT: return "GDN_ERR_TIMEOUT";
  }
  return "GDN_ERR_UNKNOWN";
}

int gdn_version(void) { return kVersion; }

gdn_status gdn_check_error(gdn_stream_t stream) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return GDN_ERR_CUDA;
  unsigned int word = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&word, g_error_word, sizeof(word)) != cudaSuccess) return GDN_ERR_CUDA;
  if (word != 0 && cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero)) != cudaSuccess)
    return GDN_ERR_CUDA;
  return (word & kErrTimeout) ? GDN_ERR_TIMEOUT : GDN_OK;
}

size_t gdn_chunk_fwd_varlen_workspace_bytes(int nseq, int max_seqlen, int Hk, int Hv, int dk,
                                            int dv, int chunk, gdn_dtype dtype) {
  (void)Hk;
  if (nseq <= 0 || max_seqlen <= 0 || Hv <= 0) return 0;
  if (!tc_chunk_supported(dk, dv, chunk, dtype == GDN_BF16)) return 0;
  return tc_chunk_varlen_scratch_bytes(nseq, max_seqlen, Hv);
}

gdn_status gdn_chunk_fwd_varlen(const void* q, const void* k, const void* v,
                                const float* log_alpha, const float* beta, const int* cu_seqlens,
                                int nseq, int max_seqlen, const float* S0, void* o, float* S_T,
                                void* workspace, size_t workspace_bytes, int total_T, int Hk,
                                int Hv, int dk, int dv, int chunk, float scale, gdn_dtype dtype,
                                gdn_dtype o_dtype, gdn_stream_t stream) {
  if (nseq < 0 || max_seqlen < 0 || total_T < 0 || !valid_dtype(dtype) || !valid_dtype(o_dtype))
    return GDN_ERR_INVALID_ARG;
  gdn_status s = validate_heads(Hk, Hv, dk, dv);
  if (s != GDN_OK) return s;
  if (chunk <= 0) return GDN_ERR_INVALID_ARG;
  if (!tc_chunk_supported(dk, dv, chunk, dtype == GDN_BF16)) return GDN_ERR_UNSUPPORTED;
  if (nseq > 65535) return GDN_ERR_UNSUPPORTED;
  if (nseq == 0) return GDN_OK;
  if (!cu_seqlens || !aligned4(cu_seqlens) || !opt_aligned16(S0) || !opt_aligned16(S_T))
    return GDN_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (total_T == 0 || max_seqlen == 0) {   // every sequence is empty: the states pass through
    if (!S_T) return GDN_OK;
    const size_t bytes = (size_t)nseq * Hv * dk * dv * sizeof(float);
    cudaError_t e = S0 ? cudaMemcpyAsync(S_T, S0, bytes, cudaMemcpyDeviceToDevice, st)
                       : cudaMemsetAsync(S_T, 0, bytes, st);
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
  }
  if (!q || !k || !v || !log_alpha || !beta || !o) return GDN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned4(log_alpha) ||
      !aligned4(beta))
    return GDN_ERR_INVALID_ARG;
  if (!tc_chunk_length_ok(max_seqlen)) return GDN_ERR_UNSUPPORTED;
  const size_t need = tc_chunk_varlen_scratch_bytes(nseq, max_seqlen, Hv);
  if (!workspace_ok(workspace, workspace_bytes, need)) return GDN_ERR_INVALID_ARG;
  return tc_chunk_launch_varlen(q, k, v, log_alpha, beta, cu_seqlens, nseq, max_seqlen, S0, o,
                                S_T, total_T, Hk, Hv, scale, o_dtype == GDN_F32, workspace, st);
}

gdn_status gdn_gates(const void* ba, float* log_alpha, float* beta, long long rows, int Hv,
                     gdn_dtype dtype, gdn_stream_t stream) {
  if (rows < 0 || Hv <= 0 || !valid_dtype(dtype)) return GDN_ERR_INVALID_ARG;
  if (rows == 0) return GDN_OK;
  if (!ba || !log_alpha || !beta || !aligned16(ba) || !aligned4(log_alpha) || !aligned4(beta))
    return GDN_ERR_INVALID_ARG;
  const long long n = rows * Hv;
  if (n / Hv != rows || (n + 255) / 256 > 0x7fffffffLL) return GDN_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const unsigned grid = (unsigned)((n + 255) / 256);
  if (dtype == GDN_F32)
    gates_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float*>(ba), log_alpha, beta,
                                              rows, Hv);
  else
    gates_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(ba),
                                                      log_alpha, beta, rows, Hv);
  return launch_status();
}

gdn_status gdn_wait_timeout_selftest(long long budget_cycles, gdn_stream_t stream) {
  if (budget_cycles < 1 || budget_cycles > 4000000000LL) return GDN_ERR_INVALID_ARG;
  wait_timeout_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      (unsigned long long)budget_cycles);
  return launch_status();
}

gdn_variant gdn_chunk_fwd_variant(int dk, int dv, int chunk, gdn_dtype dtype) {
  if (tc_chunk_supported(dk, dv, chunk, dtype == GDN_BF16)) return GDN_VARIANT_TCGEN05;
  return GDN_VARIANT_SIMT;
}

size_t gdn_chunk_fwd_workspace_bytes(int B, int T, int Hk, int Hv, int dk, int dv, int chunk,
                                     gdn_dtype dtype) {
  (void)Hk;
  if (B <= 0 || T <= 0 || Hv <= 0) return 0;
  if (!tc_chunk_supported(dk, dv, chunk, dtype == GDN_BF16)) return 0;
  return tc_chunk_scratch_bytes(B, T, Hv);
}

// Arguments of gdn_chunk_fwd_ex that decide the kernel family, checked without any CUDA call.
// On success *tc says whether the tensor-core family runs.
static gdn_status chunk_fwd_check(int B, int T, int Hk, int Hv, int dk, int dv, int chunk,
                                  gdn_dtype dtype, gdn_dtype o_dtype, gdn_variant variant,
                                  bool* tc) {
  if (B < 0 || T < 0 || !valid_dtype(dtype) || !valid_dtype(o_dtype)) return GDN_ERR_INVALID_ARG;
  if (variant != GDN_VARIANT_AUTO && variant != GDN_VARIANT_SIMT &&
      variant != GDN_VARIANT_TCGEN05)
    return GDN_ERR_INVALID_ARG;
  gdn_status s = validate_heads(Hk, Hv, dk, dv);
  if (s != GDN_OK) return s;
  if (chunk <= 0) return GDN_ERR_INVALID_ARG;
  if (!supported_chunk(chunk)) return GDN_ERR_UNSUPPORTED;
  if (!io_pair_ok(dtype, o_dtype)) return GDN_ERR_UNSUPPORTED;
  if (B > 65535) return GDN_ERR_UNSUPPORTED;
  const bool tc_ok = tc_chunk_supported(dk, dv, chunk, dtype == GDN_BF16);
  if (variant == GDN_VARIANT_TCGEN05 && !tc_ok) return GDN_ERR_UNSUPPORTED;
  *tc = tc_ok && variant != GDN_VARIANT_SIMT;
  if (*tc && !tc_chunk_length_ok(T)) return GDN_ERR_UNSUPPORTED;
  return GDN_OK;
}

int gdn_chunk_fwd_launches(int B, int T, int Hk, int Hv, int dk, int dv, int chunk,
                           gdn_dtype dtype, gdn_variant variant, int sms) {
  bool tc = false;
  if (chunk_fwd_check(B, T, Hk, Hv, dk, dv, chunk, dtype, dtype == GDN_BF16 ? GDN_BF16 : GDN_F32,
                      variant, &tc) != GDN_OK)
    return -1;
  if ((long)B * T == 0) return 0;
  if (sms < 0) return -1;
  return tc ? tc_chunk_launches(B, T, Hv, false, sms) : 1;
}

gdn_status gdn_chunk_fwd_ex(const void* q, const void* k, const void* v, const float* log_alpha,
                            const float* beta, const float* S0, void* o, float* S_T,
                            void* workspace, size_t workspace_bytes, int B, int T, int Hk,
                            int Hv, int dk, int dv, int chunk, float scale, gdn_dtype dtype,
                            gdn_dtype o_dtype, gdn_variant variant, gdn_stream_t stream) {
  bool tc = false;
  gdn_status s = chunk_fwd_check(B, T, Hk, Hv, dk, dv, chunk, dtype, o_dtype, variant, &tc);
  if (s != GDN_OK) return s;
  const bool work = (long)B * T > 0;
  if (work && (!q || !k || !v || !log_alpha || !beta || !o)) return GDN_ERR_INVALID_ARG;
  if (!opt_aligned16(q) || !opt_aligned16(k) || !opt_aligned16(v) || !opt_aligned16(o) ||
      !opt_aligned4(log_alpha) || !opt_aligned4(beta) || !opt_aligned16(S0) ||
      !opt_aligned16(S_T))
    return GDN_ERR_INVALID_ARG;
  if (work && tc && !workspace_ok(workspace, workspace_bytes, tc_chunk_scratch_bytes(B, T, Hv)))
    return GDN_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (B == 0) return GDN_OK;
  if (T == 0) {     // no token: the state is handed through unchanged (or is the zero state)
    if (!S_T) return GDN_OK;
    const size_t bytes = (size_t)B * Hv * dk * dv * sizeof(float);
    cudaError_t e = S0 ? cudaMemcpyAsync(S_T, S0, bytes, cudaMemcpyDeviceToDevice, st)
                       : cudaMemsetAsync(S_T, 0, bytes, st);
    return e == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
  }
  if (tc)
    return tc_chunk_launch(q, k, v, log_alpha, beta, S0, o, S_T, B, T, Hk, Hv, scale,
                           o_dtype == GDN_F32, workspace, st);
  if (dtype == GDN_F32)
    return simt_dispatch<float>(dk, chunk, q, k, v, log_alpha, beta, S0, o, S_T, B, T, Hk, Hv,
                                dv, scale, st);
  if (o_dtype == GDN_F32)
    return simt_dispatch<__nv_bfloat16, float>(dk, chunk, q, k, v, log_alpha, beta, S0, o, S_T, B,
                                                T, Hk, Hv, dv, scale, st);
  return simt_dispatch<__nv_bfloat16>(dk, chunk, q, k, v, log_alpha, beta, S0, o, S_T, B, T, Hk,
                                      Hv, dv, scale, st);
}

gdn_status gdn_chunk_fwd_ba(const void* q, const void* k, const void* v, const void* ba,
                            const float* S0, void* o, float* S_T, void* workspace,
                            size_t workspace_bytes, int B, int T, int Hk, int Hv, int dk, int dv,
                            int chunk, float scale, gdn_dtype dtype, gdn_dtype o_dtype,
                            gdn_stream_t stream) {
  bool tc = false;
  gdn_status s = chunk_fwd_check(B, T, Hk, Hv, dk, dv, chunk, dtype, o_dtype,
                                 GDN_VARIANT_AUTO, &tc);
  if (s != GDN_OK) return s;
  if (!tc) return GDN_ERR_UNSUPPORTED;
  const bool work = (long)B * T > 0;
  if (work && (!q || !k || !v || !ba || !o)) return GDN_ERR_INVALID_ARG;
  if (!opt_aligned16(q) || !opt_aligned16(k) || !opt_aligned16(v) || !opt_aligned16(o) ||
      !opt_aligned4(ba) || !opt_aligned16(S0) || !opt_aligned16(S_T))
    return GDN_ERR_INVALID_ARG;
  if (work && !workspace_ok(workspace, workspace_bytes, tc_chunk_scratch_bytes(B, T, Hv)))
    return GDN_ERR_INVALID_ARG;
  if (!work)
    return gdn_chunk_fwd(nullptr, nullptr, nullptr, nullptr, nullptr, S0, nullptr, S_T, nullptr, 0,
                         B, T, Hk, Hv, dk, dv, chunk, scale, dtype, o_dtype, stream);
  return tc_chunk_launch(q, k, v, nullptr, nullptr, S0, o, S_T, B, T, Hk, Hv, scale,
                         o_dtype == GDN_F32, workspace, reinterpret_cast<cudaStream_t>(stream),
                         ba);
}

gdn_status gdn_chunk_fwd(const void* q, const void* k, const void* v, const float* log_alpha,
                         const float* beta, const float* S0, void* o, float* S_T, void* workspace,
                         size_t workspace_bytes, int B, int T, int Hk, int Hv, int dk, int dv,
                         int chunk, float scale, gdn_dtype dtype, gdn_dtype o_dtype,
                         gdn_stream_t stream) {
  return gdn_chunk_fwd_ex(q, k, v, log_alpha, beta, S0, o, S_T, workspace, workspace_bytes, B, T,
                          Hk, Hv, dk, dv, chunk, scale, dtype, o_dtype, GDN_VARIANT_AUTO,
                          stream);
}

gdn_status gdn_decode_layer_step(const void* q_raw, const void* k_raw, const void* v_raw,
                                 const void* z, const void* hq_in, const void* hk_in,
                                 const void* hv_in, void* hq_out, void* hk_out, void* hv_out,
                                 const float* wq, const float* wk, const float* wv,
                                 const float* log_alpha, const float* beta, float* S,
                                 const float* norm_w, void* y, int N, int Hk, int Hv, int dk,
                                 int dv, float scale, float l2_eps, float norm_eps,
                                 gdn_dtype dtype, gdn_stream_t stream) {
  if (N < 0 || !valid_dtype(dtype)) return GDN_ERR_INVALID_ARG;
  gdn_status s = validate_heads(Hk, Hv, dk, dv);
  if (s != GDN_OK) return s;
  if (!(l2_eps >= 0.f) || !(norm_eps >= 0.f)) return GDN_ERR_INVALID_ARG;
  if (N == 0) return GDN_OK;
  const void* tensors[] = {q_raw, k_raw, v_raw, z, hq_in, hk_in, hv_in, hq_out, hk_out, hv_out,
                           S, y};
  for (const void* p : tensors)
    if (!p || !aligned16(p)) return GDN_ERR_INVALID_ARG;
  const float* weights[] = {wq, wk, wv, log_alpha, beta, norm_w};
  for (const float* p : weights)
    if (!p || !aligned4(p)) return GDN_ERR_INVALID_ARG;
  if ((long)N * Hv > 0x7fffffffL) return GDN_ERR_UNSUPPORTED;
  const DecodeLayerArgs a{q_raw, k_raw, v_raw, z, hq_in, hk_in, hv_in, hq_out, hk_out, hv_out,
                          wq, wk, wv, log_alpha, beta, S, norm_w, y, N, Hk, Hv, scale,
                          l2_eps, norm_eps};
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == GDN_F32) return decode_layer_dispatch<float>(dk, dv, a, st);
  return decode_layer_dispatch<__nv_bfloat16>(dk, dv, a, st);
}

gdn_status gdn_decode_step(const void* q, const void* k, const void* v, const float* log_alpha,
                           const float* beta, float* S, void* o, int N, int Hk, int Hv, int dk,
                           int dv, float scale, gdn_dtype dtype, gdn_dtype o_dtype,
                           gdn_stream_t stream) {
  if (N < 0 || !valid_dtype(dtype) || !valid_dtype(o_dtype)) return GDN_ERR_INVALID_ARG;
  gdn_status s = validate_heads(Hk, Hv, dk, dv);
  if (s != GDN_OK) return s;
  if (!io_pair_ok(dtype, o_dtype)) return GDN_ERR_UNSUPPORTED;
  if (N == 0) return GDN_OK;
  if (!q || !k || !v || !log_alpha || !beta || !S || !o) return GDN_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned4(log_alpha) ||
      !aligned4(beta) || !aligned16(S) || !aligned16(o))
    return GDN_ERR_INVALID_ARG;
  if ((long)N * Hv > 0x7fffffffL) return GDN_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == GDN_F32)
    return decode_dispatch<float, float>(dk, dv, q, k, v, log_alpha, beta, S, o, N, Hk, Hv, scale,
                                         st);
  if (o_dtype == GDN_F32)
    return decode_dispatch<__nv_bfloat16, float>(dk, dv, q, k, v, log_alpha, beta, S, o, N, Hk,
                                                 Hv, scale, st);
  return decode_dispatch<__nv_bfloat16, __nv_bfloat16>(dk, dv, q, k, v, log_alpha, beta, S, o, N,
                                                       Hk, Hv, scale, st);
}

// The two prologue kernels for `nseq` sequences (cu == nullptr: [nseq, T] rows; else packed rows
// cu[s] .. cu[s + 1] - 1 of T in all, none longer than max_len), arguments already checked.  The q
// and k heads (normalised rows) run on the library's high-priority stream, forked from and joined
// back into `stream`, beside the v heads on `stream`: the two kernels share the SMs (both are
// bound by instruction issue and latency, not by HBM); head slots fastest in each grid.
static gdn_status prologue_launch(const void* q_raw, const void* k_raw, const void* v_raw,
                                  const void* hq_in, const void* hk_in, const void* hv_in,
                                  const float* wq, const float* wk, const float* wv, void* q,
                                  void* k, void* v, int nseq, int T, int Hk, int Hv, int dk,
                                  int dv, float l2_eps, gdn_dtype dtype, const int* cu,
                                  int max_len, cudaStream_t st) {
  const unsigned tb = (unsigned)((max_len + kPrologueTokens - 1) / kPrologueTokens);
  const dim3 gqk(2 * Hk, tb, nseq), gv(Hv, tb, nseq);
  std::lock_guard<std::mutex> lock(tcf::split_mutex());
  tcf::Split* sp = tcf::split_for_device();
  if (!sp || cudaEventRecord(sp->ev_fork, st) != cudaSuccess ||
      cudaStreamWaitEvent(sp->s_hi, sp->ev_fork, 0) != cudaSuccess)
    return GDN_ERR_CUDA;
  if (dtype == GDN_F32) {
    prologue_qk_kernel<float><<<gqk, 128, prologue_smem_bytes(dk, 4), sp->s_hi>>>(
        (const float*)q_raw, (const float*)k_raw, (const float*)hq_in, (const float*)hk_in, wq,
        wk, (float*)q, (float*)k, T, Hk, dk, l2_eps, cu, max_len);
    prologue_v_kernel<float><<<gv, 128, prologue_smem_bytes(dv, 4), st>>>(
        (const float*)v_raw, (const float*)hv_in, wv, (float*)v, T, Hv, dv, cu, max_len);
  } else {
    using bf = __nv_bfloat16;
    prologue_qk_kernel<bf><<<gqk, 128, prologue_smem_bytes(dk, 2), sp->s_hi>>>(
        (const bf*)q_raw, (const bf*)k_raw, (const bf*)hq_in, (const bf*)hk_in, wq, wk, (bf*)q,
        (bf*)k, T, Hk, dk, l2_eps, cu, max_len);
    prologue_v_kernel<bf><<<gv, 128, prologue_smem_bytes(dv, 2), st>>>(
        (const bf*)v_raw, (const bf*)hv_in, wv, (bf*)v, T, Hv, dv, cu, max_len);
  }
  const gdn_status ls = launch_status();
  // the caller's stream waits for the q/k kernel, also after a failed launch
  if (cudaEventRecord(sp->ev_hi, sp->s_hi) != cudaSuccess ||
      cudaStreamWaitEvent(st, sp->ev_hi, 0) != cudaSuccess)
    return GDN_ERR_CUDA;
  return ls;
}

gdn_status gdn_prologue_ex(const void* q_raw, const void* k_raw, const void* v_raw,
                           const void* hq_in, const void* hk_in, const void* hv_in,
                           const float* wq, const float* wk, const float* wv, void* q, void* k,
                           void* v, int B, int T, int Hk, int Hv, int dk, int dv, float l2_eps,
                           gdn_dtype dtype, gdn_stream_t stream) {
  if (B < 0 || T < 0 || !valid_dtype(dtype) || !(l2_eps >= 0.f)) return GDN_ERR_INVALID_ARG;
  gdn_status s = validate_heads(Hk, Hv, dk, dv);
  if (s != GDN_OK) return s;
  const void* hist[] = {hq_in, hk_in, hv_in};
  for (const void* p : hist)
    if (p && !aligned16(p)) return GDN_ERR_INVALID_ARG;
  if ((long)B * T == 0) return GDN_OK;
  if (B > 65535 || 2L * Hk + Hv > 65535) return GDN_ERR_UNSUPPORTED;
  const void* ptrs[] = {q_raw, k_raw, v_raw, q, k, v};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return GDN_ERR_INVALID_ARG;
  if (!wq || !wk || !wv || !aligned4(wq) || !aligned4(wk) || !aligned4(wv))
    return GDN_ERR_INVALID_ARG;
  if ((T + kPrologueTokens - 1) / kPrologueTokens > 65535) return GDN_ERR_UNSUPPORTED;
  return prologue_launch(q_raw, k_raw, v_raw, hq_in, hk_in, hv_in, wq, wk, wv, q, k, v, B, T, Hk,
                         Hv, dk, dv, l2_eps, dtype, nullptr, T,
                         reinterpret_cast<cudaStream_t>(stream));
}

gdn_status gdn_prologue(const void* q_raw, const void* k_raw, const void* v_raw, const float* wq,
                        const float* wk, const float* wv, void* q, void* k, void* v, int B, int T,
                        int Hk, int Hv, int dk, int dv, float l2_eps, gdn_dtype dtype,
                        gdn_stream_t stream) {
  return gdn_prologue_ex(q_raw, k_raw, v_raw, nullptr, nullptr, nullptr, wq, wk, wv, q, k, v, B,
                         T, Hk, Hv, dk, dv, l2_eps, dtype, stream);
}

gdn_status gdn_out_norm(const void* o, const void* z, const float* w, void* y, long long rows,
                        int dv, float eps, gdn_dtype dtype, gdn_stream_t stream) {
  if (rows < 0 || !valid_dtype(dtype) || dv <= 0 || !(eps >= 0.f)) return GDN_ERR_INVALID_ARG;
  if (!supported_dim(dv)) return GDN_ERR_UNSUPPORTED;
  if (rows == 0) return GDN_OK;
  if (!o || !z || !w || !y || !aligned16(o) || !aligned16(z) || !aligned4(w) || !aligned16(y))
    return GDN_ERR_INVALID_ARG;
  const long long blocks = (rows + 7) / 8;
  if (blocks > 0x7fffffffLL) return GDN_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == GDN_F32)
    out_norm_kernel<float, float><<<(unsigned)blocks, kNormThreads, 0, st>>>(
        (const float*)o, (const float*)z, w, (float*)y, rows, dv, eps);
  else
    out_norm_kernel<__nv_bfloat16, __nv_bfloat16><<<(unsigned)blocks, kNormThreads, 0, st>>>(
        (const __nv_bfloat16*)o, (const __nv_bfloat16*)z, w, (__nv_bfloat16*)y, rows, dv, eps);
  return launch_status();
}

size_t gdn_layer_workspace_bytes(int B, int T, int Hk, int Hv, int dk, int dv, int chunk,
                                 gdn_dtype dtype) {
  if (B <= 0 || T <= 0 || Hk <= 0 || Hv <= 0 || dk <= 0 || dv <= 0) return 0;
  const size_t el = dtype == GDN_F32 ? 4 : 2;
  const size_t tok = (size_t)B * T;
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  // normalised q, k and convolved v in the storage dtype; the pre-norm output o in fp32; the
  // tensor-core forward's hand-over buffer when that forward runs
  const size_t qkv = 2 * up(tok * Hk * dk * el) + up(tok * Hv * dv * el);
  const size_t tc = tc_chunk_supported(dk, dv, chunk, dtype == GDN_BF16)
                        ? up(tc_chunk_scratch_bytes(B, T, Hv)) : 0;
  return qkv + up(tok * Hv * dv * 4) + tc;
}

// The conv history after a layer call: the last three raw rows of [history; x] for the q, k and
// v channels (see conv_hist_out_kernel).
static gdn_status layer_hist_out(const void* q_raw, const void* k_raw, const void* v_raw,
                                 const void* hq_in, const void* hk_in, const void* hv_in,
                                 void* hq_out, void* hk_out, void* hv_out, int B, int T, int Hk,
                                 int Hv, int dk, int dv, gdn_dtype dtype, cudaStream_t st,
                                 const int* cu = nullptr, int max_len = 0) {
  const void* x[] = {q_raw, k_raw, v_raw};
  const void* hin[] = {hq_in, hk_in, hv_in};
  void* hout[] = {hq_out, hk_out, hv_out};
  const int width[] = {Hk * dk, Hk * dk, Hv * dv};
  for (int i = 0; i < 3; ++i) {
    if (!hout[i]) continue;
    const long pieces = (long)B * 3 * width[i] / (dtype == GDN_F32 ? 4 : 8);
    const unsigned blocks = (unsigned)((pieces + 255) / 256);
    if (blocks == 0) continue;
    if (dtype == GDN_F32)
      conv_hist_out_kernel<float><<<blocks, 256, 0, st>>>(
          (const float*)x[i], (const float*)hin[i], (float*)hout[i], B, T, width[i], cu, max_len);
    else
      conv_hist_out_kernel<__nv_bfloat16><<<blocks, 256, 0, st>>>(
          (const __nv_bfloat16*)x[i], (const __nv_bfloat16*)hin[i], (__nv_bfloat16*)hout[i], B,
          T, width[i], cu, max_len);
  }
  return launch_status();
}

gdn_status gdn_layer_fwd_ex(const void* q_raw, const void* k_raw, const void* v_raw,
                            const void* z, const void* hq_in, const void* hk_in,
                            const void* hv_in, const float* wq, const float* wk, const float* wv,
                            const float* log_alpha, const float* beta, const float* S0,
                            const float* norm_w, void* y, float* S_T, void* hq_out,
                            void* hk_out, void* hv_out, void* workspace, size_t workspace_bytes,
                            int B, int T, int Hk, int Hv, int dk, int dv, int chunk, float scale,
                            float l2_eps, float norm_eps, gdn_dtype dtype, gdn_dtype y_dtype,
                            gdn_stream_t stream) {
  if (B < 0 || T < 0 || !valid_dtype(dtype) || !valid_dtype(y_dtype)) return GDN_ERR_INVALID_ARG;
  if (!io_pair_ok(dtype, y_dtype)) return GDN_ERR_UNSUPPORTED;
  gdn_status s = validate_heads(Hk, Hv, dk, dv);
  if (s != GDN_OK) return s;
  if (chunk <= 0 || !(norm_eps >= 0.f)) return GDN_ERR_INVALID_ARG;
  if (!supported_chunk(chunk)) return GDN_ERR_UNSUPPORTED;
  const void* hs[] = {hq_in, hk_in, hv_in, hq_out, hk_out, hv_out};
  for (const void* p : hs)
    if (p && !aligned16(p)) return GDN_ERR_INVALID_ARG;
  if ((hq_out && hq_out == hq_in) || (hk_out && hk_out == hk_in) ||
      (hv_out && hv_out == hv_in))
    return GDN_ERR_INVALID_ARG;
  if ((long)B * T > 0 && (hq_out || hk_out || hv_out) && (!q_raw || !k_raw || !v_raw))
    return GDN_ERR_INVALID_ARG;
  const bool tc = tc_chunk_supported(dk, dv, chunk, dtype == GDN_BF16);
  if (tc && !tc_chunk_length_ok(T)) return GDN_ERR_UNSUPPORTED;
  const size_t need = gdn_layer_workspace_bytes(B, T, Hk, Hv, dk, dv, chunk, dtype);
  if ((long)B * T > 0) {
    if (!z || !norm_w || !y || !aligned16(z) || !aligned4(norm_w) || !aligned16(y))
      return GDN_ERR_INVALID_ARG;
    if (!workspace_ok(workspace, workspace_bytes, need)) return GDN_ERR_INVALID_ARG;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if ((long)B * T == 0) {
    s = gdn_chunk_fwd(nullptr, nullptr, nullptr, nullptr, nullptr, S0, nullptr, S_T, nullptr, 0,
                      B, T, Hk, Hv, dk, dv, chunk, scale, dtype, dtype, stream);
    if (s != GDN_OK) return s;
    return layer_hist_out(q_raw, k_raw, v_raw, hq_in, hk_in, hv_in, hq_out, hk_out, hv_out, B, T,
                          Hk, Hv, dk, dv, dtype, st);
  }
  const size_t el = dtype == GDN_F32 ? 4 : 2;
  const size_t tok = (size_t)B * T;
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  char* ws = static_cast<char*>(workspace);
  void* qn = ws;
  void* kn = ws + up(tok * Hk * dk * el);
  void* vc = ws + 2 * up(tok * Hk * dk * el);
  char* rest = ws + 2 * up(tok * Hk * dk * el) + up(tok * Hv * dv * el);
  s = gdn_prologue_ex(q_raw, k_raw, v_raw, hq_in, hk_in, hv_in, wq, wk, wv, qn, kn, vc, B, T, Hk,
                      Hv, dk, dv, l2_eps, dtype, stream);
  if (s != GDN_OK) return s;
  // the recurrence writes o in fp32 so that the gated norm reads it unrounded
  float* o = reinterpret_cast<float*>(rest);
  void* tc_scratch = rest + up(tok * Hv * dv * 4);
  s = layer_chunk_fwd(qn, kn, vc, log_alpha, beta, S0, o, S_T, B, T, Hk, Hv, dk, dv, chunk, scale,
                      dtype, tc_scratch, st);
  if (s != GDN_OK) return s;
  const long long rows = (long long)tok * Hv;
  const long long blocks = (rows + 7) / 8;
  if (blocks > 0x7fffffffLL) return GDN_ERR_UNSUPPORTED;
  if (dtype == GDN_F32)
    out_norm_kernel<float, float><<<(unsigned)blocks, kNormThreads, 0, st>>>(
        (const float*)o, (const float*)z, norm_w, (float*)y, rows, dv, norm_eps);
  else if (y_dtype == GDN_F32)
    out_norm_kernel<float, __nv_bfloat16, float><<<(unsigned)blocks, kNormThreads, 0, st>>>(
        (const float*)o, (const __nv_bfloat16*)z, norm_w, (float*)y, rows, dv, norm_eps);
  else
    out_norm_kernel<float, __nv_bfloat16><<<(unsigned)blocks, kNormThreads, 0, st>>>(
        (const float*)o, (const __nv_bfloat16*)z, norm_w, (__nv_bfloat16*)y, rows, dv, norm_eps);
  s = launch_status();
  if (s != GDN_OK) return s;
  return layer_hist_out(q_raw, k_raw, v_raw, hq_in, hk_in, hv_in, hq_out, hk_out, hv_out, B, T,
                        Hk, Hv, dk, dv, dtype, st);
}

gdn_status gdn_layer_fwd(const void* q_raw, const void* k_raw, const void* v_raw, const void* z,
                         const float* wq, const float* wk, const float* wv,
                         const float* log_alpha, const float* beta, const float* S0,
                         const float* norm_w, void* y, float* S_T, void* workspace,
                         size_t workspace_bytes, int B, int T, int Hk, int Hv, int dk, int dv,
                         int chunk, float scale, float l2_eps, float norm_eps, gdn_dtype dtype,
                         gdn_dtype y_dtype, gdn_stream_t stream) {
  return gdn_layer_fwd_ex(q_raw, k_raw, v_raw, z, nullptr, nullptr, nullptr, wq, wk, wv,
                          log_alpha, beta, S0, norm_w, y, S_T, nullptr, nullptr, nullptr,
                          workspace, workspace_bytes, B, T, Hk, Hv, dk, dv, chunk, scale, l2_eps,
                          norm_eps, dtype, y_dtype, stream);
}


size_t gdn_layer_fwd_varlen_workspace_bytes(int nseq, int max_seqlen, int total_T, int Hk, int Hv,
                                            int dk, int dv, int chunk, gdn_dtype dtype) {
  if (nseq <= 0 || max_seqlen <= 0 || total_T <= 0 || !valid_dtype(dtype) ||
      validate_heads(Hk, Hv, dk, dv) != GDN_OK ||
      !tc_chunk_supported(dk, dv, chunk, dtype == GDN_BF16))
    return 0;
  const size_t tok = (size_t)total_T;
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  // normalised q, k and convolved v (bf16), the recurrence's fp32 o, the hand-over buffer
  return 2 * up(tok * Hk * dk * 2) + up(tok * Hv * dv * 2) + up(tok * Hv * dv * 4) +
         up(tc_chunk_varlen_scratch_bytes(nseq, max_seqlen, Hv));
}

gdn_status gdn_layer_fwd_varlen(const void* q_raw, const void* k_raw, const void* v_raw,
                                const void* z, const int* cu_seqlens, int nseq, int max_seqlen,
                                const void* hq_in, const void* hk_in, const void* hv_in,
                                const float* wq, const float* wk, const float* wv,
                                const float* log_alpha, const float* beta, const float* S0,
                                const float* norm_w, void* y, float* S_T, void* hq_out,
                                void* hk_out, void* hv_out, void* workspace,
                                size_t workspace_bytes, int total_T, int Hk, int Hv, int dk,
                                int dv, int chunk, float scale, float l2_eps, float norm_eps,
                                gdn_dtype dtype, gdn_dtype y_dtype, gdn_stream_t stream) {
  if (nseq < 0 || max_seqlen < 0 || total_T < 0 || !valid_dtype(dtype) || !valid_dtype(y_dtype))
    return GDN_ERR_INVALID_ARG;
  if (!io_pair_ok(dtype, y_dtype)) return GDN_ERR_UNSUPPORTED;
  gdn_status s = validate_heads(Hk, Hv, dk, dv);
  if (s != GDN_OK) return s;
  if (chunk <= 0 || !(norm_eps >= 0.f) || !(l2_eps >= 0.f)) return GDN_ERR_INVALID_ARG;
  if (!tc_chunk_supported(dk, dv, chunk, dtype == GDN_BF16)) return GDN_ERR_UNSUPPORTED;
  if (nseq > 65535 || 2L * Hk + Hv > 65535) return GDN_ERR_UNSUPPORTED;
  if (nseq == 0) return GDN_OK;
  const void* hs[] = {hq_in, hk_in, hv_in, hq_out, hk_out, hv_out};
  for (const void* p : hs)
    if (p && !aligned16(p)) return GDN_ERR_INVALID_ARG;
  if ((hq_out && hq_out == hq_in) || (hk_out && hk_out == hk_in) ||
      (hv_out && hv_out == hv_in))
    return GDN_ERR_INVALID_ARG;
  if (!cu_seqlens || !aligned4(cu_seqlens) || !opt_aligned16(S0) || !opt_aligned16(S_T))
    return GDN_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (total_T == 0 || max_seqlen == 0) {   // every sequence is empty: state and history pass on
    s = gdn_chunk_fwd_varlen(nullptr, nullptr, nullptr, nullptr, nullptr, cu_seqlens, nseq, 0, S0,
                             nullptr, S_T, nullptr, 0, 0, Hk, Hv, dk, dv, chunk, scale, dtype,
                             dtype, stream);
    if (s != GDN_OK) return s;
    return layer_hist_out(q_raw, k_raw, v_raw, hq_in, hk_in, hv_in, hq_out, hk_out, hv_out, nseq,
                          0, Hk, Hv, dk, dv, dtype, st, cu_seqlens, 0);
  }
  const void* ptrs[] = {q_raw, k_raw, v_raw, z, y};
  for (const void* p : ptrs)
    if (!p || !aligned16(p)) return GDN_ERR_INVALID_ARG;
  if (!wq || !wk || !wv || !norm_w || !log_alpha || !beta || !aligned4(wq) || !aligned4(wk) ||
      !aligned4(wv) || !aligned4(norm_w) || !aligned4(log_alpha) || !aligned4(beta))
    return GDN_ERR_INVALID_ARG;
  if (!tc_chunk_length_ok(max_seqlen) ||
      (max_seqlen + kPrologueTokens - 1) / kPrologueTokens > 65535)
    return GDN_ERR_UNSUPPORTED;
  const size_t need = gdn_layer_fwd_varlen_workspace_bytes(nseq, max_seqlen, total_T, Hk, Hv, dk,
                                                           dv, chunk, dtype);
  if (!workspace_ok(workspace, workspace_bytes, need)) return GDN_ERR_INVALID_ARG;
  const size_t tok = (size_t)total_T;
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  char* ws = static_cast<char*>(workspace);
  void* qn = ws;
  void* kn = ws + up(tok * Hk * dk * 2);
  void* vc = ws + 2 * up(tok * Hk * dk * 2);
  float* o = reinterpret_cast<float*>(ws + 2 * up(tok * Hk * dk * 2) + up(tok * Hv * dv * 2));
  void* tc_scratch = reinterpret_cast<char*>(o) + up(tok * Hv * dv * 4);
  s = prologue_launch(q_raw, k_raw, v_raw, hq_in, hk_in, hv_in, wq, wk, wv, qn, kn, vc, nseq,
                      total_T, Hk, Hv, dk, dv, l2_eps, dtype, cu_seqlens, max_seqlen, st);
  if (s != GDN_OK) return s;
  s = tc_chunk_launch_varlen(qn, kn, vc, log_alpha, beta, cu_seqlens, nseq, max_seqlen, S0, o,
                             S_T, total_T, Hk, Hv, scale, true, tc_scratch, st);
  if (s != GDN_OK) return s;
  const long long rows = (long long)tok * Hv;
  const long long blocks = (rows + 7) / 8;
  if (blocks > 0x7fffffffLL) return GDN_ERR_UNSUPPORTED;
  if (y_dtype == GDN_F32)
    out_norm_kernel<float, __nv_bfloat16, float><<<(unsigned)blocks, kNormThreads, 0, st>>>(
        o, (const __nv_bfloat16*)z, norm_w, (float*)y, rows, dv, norm_eps);
  else
    out_norm_kernel<float, __nv_bfloat16><<<(unsigned)blocks, kNormThreads, 0, st>>>(
        o, (const __nv_bfloat16*)z, norm_w, (__nv_bfloat16*)y, rows, dv, norm_eps);
  s = launch_status();
  if (s != GDN_OK) return s;
  return layer_hist_out(q_raw, k_raw, v_raw, hq_in, hk_in, hv_in, hq_out, hk_out, hv_out, nseq,
                        total_T, Hk, Hv, dk, dv, dtype, st, cu_seqlens, max_seqlen);
}

}  // extern "C"

// ---------------------------------------------------------------------------------------------
// Layer backward: the forward recomputed (prologue, recurrence with fp32 o), then the gated norm's
// backward (dO in fp32), the recurrence's (gdn_bwd with an fp32 dO), the prologue's.
// ---------------------------------------------------------------------------------------------
namespace {
constexpr unsigned kNormBwdCtas = 592;   // fixed grid of the norm backward (its dw partial sums)
struct LayerBwdLayout {
  size_t fwd = 0, d_o = 0, dq = 0, dk = 0, dv = 0, bwd = 0, dpre = 0, nw = 0, cw = 0, total = 0;
};
// The layer backward's workspace for B sequences of T tokens, or (packed) nseq = B sequences of
// at most max_len tokens, T rows in all: the forward's buffers (q, k, v, fp32 o, hand-over), then
// the backward's.
LayerBwdLayout layer_bwd_layout(int B, int T, int Hk, int Hv, int dk, int dv, int chunk,
                                gdn_dtype dtype, bool packed = false, int max_len = 0) {
  LayerBwdLayout L;
  if (!packed) max_len = T;
  const size_t tok = packed ? (size_t)T : (size_t)B * T;
  const size_t C = std::max((size_t)Hk * dk, (size_t)Hv * dv);
  const size_t tiles = (size_t)B * ((max_len + lbwd::kConvTok - 1) / lbwd::kConvTok);
  size_t o = align256(packed ? gdn_layer_fwd_varlen_workspace_bytes(B, max_len, T, Hk, Hv, dk, dv,
                                                                    chunk, dtype)
                             : gdn_layer_workspace_bytes(B, T, Hk, Hv, dk, dv, chunk, dtype));
  L.fwd = 0;
  L.d_o = o;  o += align256(tok * Hv * dv * 4);
  L.dq = o;   o += align256(tok * Hk * dk * 4);
  L.dk = o;   o += align256(tok * Hk * dk * 4);
  L.dv = o;   o += align256(tok * Hv * dv * 4);
  L.bwd = o;  o += align256(bwd_layout_rows(B, max_len, tok, Hk, Hv, dk, dv).total);
  L.dpre = o; o += align256(tok * C * 4);
  L.nw = o;   o += align256((size_t)kNormBwdCtas * dv * 4);
  L.cw = o;   o += align256(tiles * C * 4 * 4);
  L.total = o;
  return L;
}

template <typename Tin>
gdn_status prologue_bwd_one(const void* x_raw, const float* w, const float* dy, float* dx_raw,
                            float* dw, float* dpre, float* dw_part, int B, int T, int heads,
                            int d, bool normalize, float eps, cudaStream_t st,
                            const int* cu = nullptr, int max_len = -1) {
  if (!cu) max_len = T;                       // B sequences of T rows, or packed (T rows in all)
  const dim3 gd(heads, (max_len + lbwd::kDpreTok - 1) / lbwd::kDpreTok, B);
  const Tin* xr = static_cast<const Tin*>(x_raw);
  const int nz = normalize ? 1 : 0;
  if (d == 128)
    lbwd::conv_dpre_kernel<Tin, 4><<<gd, 128, 0, st>>>(xr, w, dy, dpre, T, heads, d, nz, eps, cu,
                                                       max_len);
  else if (d == 64)
    lbwd::conv_dpre_kernel<Tin, 2><<<gd, 128, 0, st>>>(xr, w, dy, dpre, T, heads, d, nz, eps, cu,
                                                       max_len);
  else
    lbwd::conv_dpre_kernel<Tin, 1><<<gd, 128, 0, st>>>(xr, w, dy, dpre, T, heads, d, nz, eps, cu,
                                                       max_len);
  const int C = heads * d;
  const dim3 grid((C + 127) / 128, (max_len + lbwd::kConvTok - 1) / lbwd::kConvTok, B);
  lbwd::conv_bwd_kernel<Tin><<<grid, 128, 0, st>>>(static_cast<const Tin*>(x_raw), w, dpre,
                                                   dx_raw, dw_part, T, C, cu, max_len);
  lbwd::col_sum_kernel<<<(C * 4 + 255) / 256, 256, 0, st>>>(dw_part, dw, (int)(grid.y * grid.z),
                                                            C * 4);
  return launch_status();
}

template <typename Tin, typename Tdy>
gdn_status layer_bwd_run(const void* q_raw, const void* k_raw, const void* v_raw, const void* z,
                         const float* wq, const float* wk, const float* wv, const float* la,
                         const float* be, const float* S0, const float* norm_w, const void* dy,
                         const float* dS_T, float* dq_raw, float* dk_raw, float* dv_raw,
                         float* dz, float* dwq, float* dwk, float* dwv, float* dla, float* dbeta,
                         float* dS0, float* dnorm_w, char* ws, const LayerBwdLayout& L, int B,
                         int T, int Hk, int Hv, int dk, int dv, int chunk, float scale,
                         float l2_eps, float norm_eps, gdn_dtype dtype, gdn_stream_t stream,
                         const int* cu = nullptr, int max_len = -1) {
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t el = dtype == GDN_F32 ? 4 : 2;
  const size_t tok = cu ? (size_t)T : (size_t)B * T;   // packed: B sequences, T rows in all
  void* qn = ws;
  void* kn = ws + align256(tok * Hk * dk * el);
  void* vc = ws + 2 * align256(tok * Hk * dk * el);
  char* rest = ws + 2 * align256(tok * Hk * dk * el) + align256(tok * Hv * dv * el);
  float* o = reinterpret_cast<float*>(rest);
  void* tc_scratch = rest + align256(tok * Hv * dv * 4);
  gdn_status s;
  if (cu) {   // packed rows: the tensor-core recurrence over the sequences' spans
    // o of rows in no sequence stays zero, so the norm's backward adds nothing from them
    if (cudaMemsetAsync(o, 0, tok * Hv * dv * 4, st) != cudaSuccess) return GDN_ERR_CUDA;
    s = prologue_launch(q_raw, k_raw, v_raw, nullptr, nullptr, nullptr, wq, wk, wv, qn, kn, vc, B,
                        T, Hk, Hv, dk, dv, l2_eps, dtype, cu, max_len, st);
    if (s != GDN_OK) return s;
    s = tc_chunk_launch_varlen(qn, kn, vc, la, be, cu, B, max_len, S0, o, nullptr, T, Hk, Hv,
                               scale, true, tc_scratch, st);
  } else {
    s = gdn_prologue(q_raw, k_raw, v_raw, wq, wk, wv, qn, kn, vc, B, T, Hk, Hv, dk, dv, l2_eps,
                     dtype, stream);
    if (s != GDN_OK) return s;
    s = layer_chunk_fwd(qn, kn, vc, la, be, S0, o, nullptr, B, T, Hk, Hv, dk, dv, chunk, scale,
                        dtype, tc_scratch, st);
  }
  if (s != GDN_OK) return s;
  float* d_o = reinterpret_cast<float*>(ws + L.d_o);
  float* nw = reinterpret_cast<float*>(ws + L.nw);
  const long long rows = (long long)tok * Hv;
  lbwd::out_norm_bwd_kernel<Tin, Tdy><<<kNormBwdCtas, 32 * lbwd::kNormWarps, 0, st>>>(
      o, static_cast<const Tin*>(z), norm_w, static_cast<const Tdy*>(dy), d_o, dz, nw, rows, dv,
      norm_eps, aligned16(dz) ? 1 : 0);
  lbwd::col_sum_kernel<<<(dv + 255) / 256, 256, 0, st>>>(nw, dnorm_w, (int)kNormBwdCtas, dv);
  if (launch_status() != GDN_OK) return GDN_ERR_CUDA;
  float* dqg = reinterpret_cast<float*>(ws + L.dq);
  float* dkg = reinterpret_cast<float*>(ws + L.dk);
  float* dvg = reinterpret_cast<float*>(ws + L.dv);
  s = bwd_dispatch<Tin, float>(dk, qn, kn, vc, la, be, S0, d_o, dS_T, dqg, dkg, dvg, dla, dbeta,
                               dS0, ws + L.bwd, B, T, Hk, Hv, scale, st, cu, max_len);
  if (s != GDN_OK) return s;
  float* dpre = reinterpret_cast<float*>(ws + L.dpre);
  float* cw = reinterpret_cast<float*>(ws + L.cw);
  s = prologue_bwd_one<Tin>(q_raw, wq, dqg, dq_raw, dwq, dpre, cw, B, T, Hk, dk, true, l2_eps, st,
                            cu, max_len);
  if (s == GDN_OK)
    s = prologue_bwd_one<Tin>(k_raw, wk, dkg, dk_raw, dwk, dpre, cw, B, T, Hk, dk, true, l2_eps,
                              st, cu, max_len);
  if (s == GDN_OK)
    s = prologue_bwd_one<Tin>(v_raw, wv, dvg, dv_raw, dwv, dpre, cw, B, T, Hv, dv, false, 0.f, st,
                              cu, max_len);
  return s;
}
}  // namespace

extern "C" {

size_t gdn_layer_bwd_workspace_bytes(int B, int T, int Hk, int Hv, int dk, int dv, int chunk,
                                     gdn_dtype dtype) {
  if (B <= 0 || T <= 0 || validate_heads(Hk, Hv, dk, dv) != GDN_OK || dk != dv ||
      !valid_dtype(dtype) || !supported_chunk(chunk))
    return 0;
  return layer_bwd_layout(B, T, Hk, Hv, dk, dv, chunk, dtype).total;
}

gdn_status gdn_layer_bwd(const void* q_raw, const void* k_raw, const void* v_raw, const void* z,
                         const float* wq, const float* wk, const float* wv,
                         const float* log_alpha, const float* beta, const float* S0,
                         const float* norm_w, const void* dy, const float* dS_T, float* dq_raw,
                         float* dk_raw, float* dv_raw, float* dz, float* dwq, float* dwk,
                         float* dwv, float* dlog_alpha, float* dbeta, float* dS0, float* dnorm_w,
                         void* workspace, size_t workspace_bytes, int B, int T, int Hk, int Hv,
                         int dk, int dv, int chunk, float scale, float l2_eps, float norm_eps,
                         gdn_dtype dtype, gdn_dtype dy_dtype, gdn_stream_t stream) {
  if (B < 0 || T < 0 || !valid_dtype(dtype) || !valid_dtype(dy_dtype)) return GDN_ERR_INVALID_ARG;
  if (!io_pair_ok(dtype, dy_dtype)) return GDN_ERR_UNSUPPORTED;
  gdn_status s = validate_heads(Hk, Hv, dk, dv);
  if (s != GDN_OK) return s;
  if (dk != dv) return GDN_ERR_UNSUPPORTED;
  if (chunk <= 0 || !(norm_eps >= 0.f) || !(l2_eps >= 0.f)) return GDN_ERR_INVALID_ARG;
  if (!supported_chunk(chunk)) return GDN_ERR_UNSUPPORTED;
  const bool tc = tc_chunk_supported(dk, dv, chunk, dtype == GDN_BF16);
  if (tc && !tc_chunk_length_ok(T)) return GDN_ERR_UNSUPPORTED;
  if ((long)B * T == 0) return GDN_OK;
  if (B > 65535 || (long)B * T * Hv > 0x7fffffffL * 8L) return GDN_ERR_UNSUPPORTED;
  const void* in16[] = {q_raw, k_raw, v_raw, z, dy};
  for (const void* p : in16)
    if (!p || !aligned16(p)) return GDN_ERR_INVALID_ARG;
  const void* in4[] = {wq, wk, wv, log_alpha, beta, norm_w, dq_raw, dk_raw, dv_raw, dz, dwq, dwk,
                       dwv, dlog_alpha, dbeta, dnorm_w};
  for (const void* p : in4)
    if (!p || !aligned4(p)) return GDN_ERR_INVALID_ARG;
  if (!opt_aligned16(S0) || !opt_aligned16(dS_T) || !opt_aligned16(dS0)) return GDN_ERR_INVALID_ARG;
  const LayerBwdLayout L = layer_bwd_layout(B, T, Hk, Hv, dk, dv, chunk, dtype);
  if (!workspace_ok(workspace, workspace_bytes, L.total)) return GDN_ERR_INVALID_ARG;
  char* ws = static_cast<char*>(workspace);
  if (dtype == GDN_F32)
    return layer_bwd_run<float, float>(q_raw, k_raw, v_raw, z, wq, wk, wv, log_alpha, beta, S0,
                                       norm_w, dy, dS_T, dq_raw, dk_raw, dv_raw, dz, dwq, dwk, dwv,
                                       dlog_alpha, dbeta, dS0, dnorm_w, ws, L, B, T, Hk, Hv, dk,
                                       dv, chunk, scale, l2_eps, norm_eps, dtype, stream);
  if (dy_dtype == GDN_F32)
    return layer_bwd_run<__nv_bfloat16, float>(
        q_raw, k_raw, v_raw, z, wq, wk, wv, log_alpha, beta, S0, norm_w, dy, dS_T, dq_raw, dk_raw,
        dv_raw, dz, dwq, dwk, dwv, dlog_alpha, dbeta, dS0, dnorm_w, ws, L, B, T, Hk, Hv, dk, dv,
        chunk, scale, l2_eps, norm_eps, dtype, stream);
  return layer_bwd_run<__nv_bfloat16, __nv_bfloat16>(
      q_raw, k_raw, v_raw, z, wq, wk, wv, log_alpha, beta, S0, norm_w, dy, dS_T, dq_raw, dk_raw,
      dv_raw, dz, dwq, dwk, dwv, dlog_alpha, dbeta, dS0, dnorm_w, ws, L, B, T, Hk, Hv, dk, dv,
      chunk, scale, l2_eps, norm_eps, dtype, stream);
}

size_t gdn_layer_bwd_varlen_workspace_bytes(int nseq, int max_seqlen, int total_T, int Hk, int Hv,
                                            int dk, int dv, int chunk, gdn_dtype dtype) {
  if (nseq <= 0 || max_seqlen <= 0 || total_T <= 0 || validate_heads(Hk, Hv, dk, dv) != GDN_OK ||
      dk != dv || !valid_dtype(dtype) || !tc_chunk_supported(dk, dv, chunk, dtype == GDN_BF16))
    return 0;
  return layer_bwd_layout(nseq, total_T, Hk, Hv, dk, dv, chunk, dtype, true, max_seqlen).total;
}

gdn_status gdn_layer_bwd_varlen(const void* q_raw, const void* k_raw, const void* v_raw,
                                const void* z, const int* cu_seqlens, int nseq, int max_seqlen,
                                const float* wq, const float* wk, const float* wv,
                                const float* log_alpha, const float* beta, const float* S0,
                                const float* norm_w, const void* dy, const float* dS_T,
                                float* dq_raw, float* dk_raw, float* dv_raw, float* dz,
                                float* dwq, float* dwk, float* dwv, float* dlog_alpha,
                                float* dbeta, float* dS0, float* dnorm_w, void* workspace,
                                size_t workspace_bytes, int total_T, int Hk, int Hv, int dk,
                                int dv, int chunk, float scale, float l2_eps, float norm_eps,
                                gdn_dtype dtype, gdn_dtype dy_dtype, gdn_stream_t stream) {
  if (nseq < 0 || max_seqlen < 0 || total_T < 0 || !valid_dtype(dtype) || !valid_dtype(dy_dtype))
    return GDN_ERR_INVALID_ARG;
  if (!io_pair_ok(dtype, dy_dtype)) return GDN_ERR_UNSUPPORTED;
  gdn_status s = validate_heads(Hk, Hv, dk, dv);
  if (s != GDN_OK) return s;
  if (chunk <= 0 || !(norm_eps >= 0.f) || !(l2_eps >= 0.f)) return GDN_ERR_INVALID_ARG;
  if (dk != dv || !tc_chunk_supported(dk, dv, chunk, dtype == GDN_BF16)) return GDN_ERR_UNSUPPORTED;
  if (nseq > 65535 || (long)nseq * Hv * bwd::head_slices(dk) > 0x7fffffffL ||
      (long)total_T * Hv > 0x7fffffffL * 8L)
    return GDN_ERR_UNSUPPORTED;
  if (nseq == 0) return GDN_OK;
  if (!cu_seqlens || !aligned4(cu_seqlens)) return GDN_ERR_INVALID_ARG;
  const float* w4[] = {wq, wk, wv, norm_w};
  float* dw4[] = {dwq, dwk, dwv, dnorm_w};
  for (int i = 0; i < 4; ++i)
    if (!w4[i] || !dw4[i] || !aligned4(w4[i]) || !aligned4(dw4[i])) return GDN_ERR_INVALID_ARG;
  if (!opt_aligned16(S0) || !opt_aligned16(dS_T) || !opt_aligned16(dS0)) return GDN_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (total_T == 0 || max_seqlen == 0) {   // every sequence is empty: dS0 = dS_T, no weight grads
    const size_t wb[] = {(size_t)Hk * dk * 16, (size_t)Hk * dk * 16, (size_t)Hv * dv * 16,
                         (size_t)dv * 4};
    for (int i = 0; i < 4; ++i)
      if (cudaMemsetAsync(dw4[i], 0, wb[i], st) != cudaSuccess) return GDN_ERR_CUDA;
    return gdn_bwd_varlen(nullptr, nullptr, nullptr, nullptr, nullptr, cu_seqlens, nseq, 0, S0,
                          nullptr, dS_T, nullptr, nullptr, nullptr, nullptr, nullptr, dS0,
                          nullptr, 0, 0, Hk, Hv, dk, dv, scale, dtype, stream);
  }
  const void* in16[] = {q_raw, k_raw, v_raw, z, dy};
  for (const void* p : in16)
    if (!p || !aligned16(p)) return GDN_ERR_INVALID_ARG;
  const void* in4[] = {log_alpha, beta, dq_raw, dk_raw, dv_raw, dz, dlog_alpha, dbeta};
  for (const void* p : in4)
    if (!p || !aligned4(p)) return GDN_ERR_INVALID_ARG;
  if (!tc_chunk_length_ok(max_seqlen) ||
      (max_seqlen + kPrologueTokens - 1) / kPrologueTokens > 65535)
    return GDN_ERR_UNSUPPORTED;
  const LayerBwdLayout L =
      layer_bwd_layout(nseq, total_T, Hk, Hv, dk, dv, chunk, dtype, true, max_seqlen);
  if (!workspace_ok(workspace, workspace_bytes, L.total)) return GDN_ERR_INVALID_ARG;
  char* ws = static_cast<char*>(workspace);
  if (dy_dtype == GDN_F32)
    return layer_bwd_run<__nv_bfloat16, float>(
        q_raw, k_raw, v_raw, z, wq, wk, wv, log_alpha, beta, S0, norm_w, dy, dS_T, dq_raw, dk_raw,
        dv_raw, dz, dwq, dwk, dwv, dlog_alpha, dbeta, dS0, dnorm_w, ws, L, nseq, total_T, Hk, Hv,
        dk, dv, chunk, scale, l2_eps, norm_eps, dtype, stream, cu_seqlens, max_seqlen);
  return layer_bwd_run<__nv_bfloat16, __nv_bfloat16>(
      q_raw, k_raw, v_raw, z, wq, wk, wv, log_alpha, beta, S0, norm_w, dy, dS_T, dq_raw, dk_raw,
      dv_raw, dz, dwq, dwk, dwv, dlog_alpha, dbeta, dS0, dnorm_w, ws, L, nseq, total_T, Hk, Hv, dk,
      dv, chunk, scale, l2_eps, norm_eps, dtype, stream, cu_seqlens, max_seqlen);
}

gdn_status gdn_gates_bwd(const void* ba, const float* dlog_alpha, const float* dbeta, float* dba,
                         long long rows, int Hv, gdn_dtype dtype, gdn_stream_t stream) {
  if (rows < 0 || Hv <= 0 || !valid_dtype(dtype)) return GDN_ERR_INVALID_ARG;
  if (rows == 0) return GDN_OK;
  if (!ba || !dlog_alpha || !dbeta || !dba || !aligned4(ba) || !aligned4(dlog_alpha) ||
      !aligned4(dbeta) || !aligned4(dba))
    return GDN_ERR_INVALID_ARG;
  const long long n = rows * Hv, blocks = (n + 255) / 256;
  if (blocks > 0x7fffffffLL) return GDN_ERR_UNSUPPORTED;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (dtype == GDN_F32)
    lbwd::gates_bwd_kernel<float><<<(unsigned)blocks, 256, 0, st>>>(
        (const float*)ba, dlog_alpha, dbeta, dba, rows, Hv);
  else
    lbwd::gates_bwd_kernel<__nv_bfloat16><<<(unsigned)blocks, 256, 0, st>>>(
        (const __nv_bfloat16*)ba, dlog_alpha, dbeta, dba, rows, Hv);
  return launch_status();
}

}  // extern "C"

// ---------------------------------------------------------------------------------------------
// gdn_layer_fwd_static: the whole layer with its scratch in the library's own device memory.
// ---------------------------------------------------------------------------------------------

// The scratch is part of the library's device image: it exists on a device once the library's
// device code is loaded there, and no call allocates or frees it.  Every byte the layer reads
// from it is written earlier in the same call, so nothing in it has to start at zero.
static __device__ __align__(256) unsigned char gdn_layer_scratch[GDN_LAYER_STATIC_SCRATCH_BYTES];

namespace {
constexpr int kScratchDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_addr[kScratchDevices] = {};

// Device address of gdn_layer_scratch on the current device; looked up on the first call per
// device (a runtime query; it allocates nothing) and kept for later calls.
gdn_status layer_scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kScratchDevices) return GDN_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_scratch_mu);
  if (!g_scratch_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, gdn_layer_scratch) != cudaSuccess || p == nullptr)
      return GDN_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return GDN_OK;
}
}  // namespace

extern "C" gdn_status gdn_layer_fwd_static(
    const void* q_raw, const void* k_raw, const void* v_raw, const void* z, const float* wq,
    const float* wk, const float* wv, const float* log_alpha, const float* beta, const float* S0,
    const float* norm_w, void* y, float* S_T, int B, int T, int Hk, int Hv, int dk, int dv,
    int chunk, float scale, float l2_eps, float norm_eps, gdn_dtype dtype, gdn_dtype y_dtype,
    gdn_stream_t stream) {
  if (B < 0 || T < 0 || !valid_dtype(dtype)) return GDN_ERR_INVALID_ARG;
  const size_t need = gdn_layer_workspace_bytes(B, T, Hk, Hv, dk, dv, chunk, dtype);
  if (need > (size_t)GDN_LAYER_STATIC_SCRATCH_BYTES) return GDN_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  if (need > 0) {
    const gdn_status s = layer_scratch_address(&scratch);
    if (s != GDN_OK) return s;
  }
  return gdn_layer_fwd(q_raw, k_raw, v_raw, z, wq, wk, wv, log_alpha, beta, S0, norm_w, y, S_T,
                       scratch, need > 0 ? (size_t)GDN_LAYER_STATIC_SCRATCH_BYTES : 0, B, T, Hk,
                       Hv, dk, dv, chunk, scale, l2_eps, norm_eps, dtype, y_dtype, stream);
}
