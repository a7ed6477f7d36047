// common.cuh -- internal declarations shared by the CUDA translation units of
// libqwm.so (device helpers, problem dimensions, kernel launchers).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "qwm.h"

namespace qwm {

// Problem dimensions derived from a validated qwm_config.
struct Dims {
  int H, d, C, G, M, r, ng;
  int64_t tcap;
  int idx_bytes;  // 1 if C <= 256 else 2
  int qsac_full;  // QSAC stage 2 by the full quadratic form e^T A e
  int max_queries;  // query rows the WORKSPACE holds attention partials for
};

// ---------------------------------------------------------------- host-side validation
constexpr int32_t kCacheMagic = 0x51574d31;  // "QWM1"

inline bool config_ok(const qwm_config* c) {
  if (!c) return false;
  if (c->heads < 1 || c->heads > 4096) return false;
  if (c->head_dim != 64 && c->head_dim != 128) return false;
  if (c->group != 16 && c->group != 32) return false;
  if (c->head_dim % c->group) return false;
  if (c->n_centroids < 1 || c->n_centroids > 512) return false;
  if (c->n_cand < 1 || c->n_cand > 8 || c->n_cand > c->n_centroids) return false;
  if (c->rank < 0 || c->rank > 16) return false;
  if (c->max_versions < 1 || c->max_versions > 65535) return false;
  if (c->max_cent_versions < 1 || c->max_cent_versions > 65535) return false;
  if (c->max_queries < 0 || c->max_queries > (1 << 24)) return false;
  if ((c->flags & ~QWM_FLAG_QSAC_FULL) != 0) return false;
  if (c->max_tokens < 1 || c->max_tokens > (int64_t(1) << 40)) return false;
  return true;
}

inline bool cache_ok(const qwm_cache* c) {
  return c && c->magic == kCacheMagic && config_ok(&c->cfg);
}

inline Dims dims_of(const qwm_config* c) {
  Dims D;
  D.H = c->heads;
  D.d = c->head_dim;
  D.C = c->n_centroids;
  D.G = c->group;
  D.M = c->n_cand;
  D.r = c->rank;
  D.ng = c->head_dim / c->group;
  D.tcap = (c->max_tokens + 127) / 128 * 128;
  D.idx_bytes = c->n_centroids <= 256 ? 1 : 2;
  D.qsac_full = (c->flags & QWM_FLAG_QSAC_FULL) ? 1 : 0;
  D.max_queries = c->max_queries;
  return D;
}

// Common checks of a centroid build (either entry point) and the table slot it
// writes: version 0 first; then, once tokens are cached, the next free slot
// (they keep decoding with the tables they were encoded with); on an empty
// cache the slot in force is rewritten, since no token references it.
inline qwm_status centroid_build_slot(const qwm_cache* c, const void* K, const void* V, int64_t n,
                                      int32_t iters, int* slot) {
  if (!cache_ok(c) || !K || !V) return QWM_ERR_INVALID_ARG;
  if (((uintptr_t)K % 16) || ((uintptr_t)V % 16)) return QWM_ERR_ALIGNMENT;
  const Dims D = dims_of(&c->cfg);
  if (n < D.C || n > D.tcap || iters < 1 || iters > 1000) return QWM_ERR_INVALID_ARG;
  if (!c->has_centroids) {
    *slot = 0;
  } else if (c->len == 0) {
    *slot = c->cur_cent_version;
  } else {
    if (c->n_cent_versions >= c->cfg.max_cent_versions) return QWM_ERR_CAPACITY;
    *slot = c->n_cent_versions;
  }
  return QWM_OK;
}

// Host state after the tables of `slot` have been enqueued.
inline void centroid_build_commit(qwm_cache* c, int slot) {
  c->has_centroids = 1;
  c->cur_cent_version = slot;
  if (slot + 1 > c->n_cent_versions) c->n_cent_versions = slot + 1;
}

// fp32 snapshot A = M / n of head h kept with the refresh state (after the
// first 32 Ritz-vector columns of the head's d x d fp64 block).
__host__ __device__ inline float* qsnap_of(double* eigvec, int d, int h) {
  return reinterpret_cast<float*>(eigvec + (size_t)h * d * d + 32 * (size_t)d);
}

// Views of the cache buffers (device pointers).
struct CacheView {
  uint8_t* k_codes;
  uint16_t* k_params;
  void* k_idx;
  int8_t* k_coef;
  uint16_t* k_cscale;
  uint8_t* v_codes;
  uint16_t* v_params;
  void* v_idx;
  uint16_t* cent_k;
  uint16_t* cent_v;
  double* qstats;
  float* sens;
  float* wgroup;
  float* basis;
  uint16_t* tokver;
  uint16_t* centver;
  double* eigvec;
  void* workspace;
};

inline CacheView view_of(const qwm_cache* c) {
  CacheView v;
  v.k_codes = (uint8_t*)c->buf.ptr[QWM_BUF_K_CODES];
  v.k_params = (uint16_t*)c->buf.ptr[QWM_BUF_K_PARAMS];
  v.k_idx = c->buf.ptr[QWM_BUF_K_IDX];
  v.k_coef = (int8_t*)c->buf.ptr[QWM_BUF_K_COEF];
  v.k_cscale = (uint16_t*)c->buf.ptr[QWM_BUF_K_CSCALE];
  v.v_codes = (uint8_t*)c->buf.ptr[QWM_BUF_V_CODES];
  v.v_params = (uint16_t*)c->buf.ptr[QWM_BUF_V_PARAMS];
  v.v_idx = c->buf.ptr[QWM_BUF_V_IDX];
  v.cent_k = (uint16_t*)c->buf.ptr[QWM_BUF_CENT_K];
  v.cent_v = (uint16_t*)c->buf.ptr[QWM_BUF_CENT_V];
  v.qstats = (double*)c->buf.ptr[QWM_BUF_QSTATS];
  v.sens = (float*)c->buf.ptr[QWM_BUF_SENS];
  v.wgroup = (float*)c->buf.ptr[QWM_BUF_WGROUP];
  v.basis = (float*)c->buf.ptr[QWM_BUF_BASIS];
  v.tokver = (uint16_t*)c->buf.ptr[QWM_BUF_TOKVER];
  v.centver = (uint16_t*)c->buf.ptr[QWM_BUF_CENTVER];
  v.eigvec = (double*)c->buf.ptr[QWM_BUF_EIGVEC];
  v.workspace = c->buf.ptr[QWM_BUF_WORKSPACE];
  return v;
}

// Attention partials of a split key range: per range, [nq][H][d] fp32 outputs
// (each normalized by its own softmax sum) then [nq][H] fp32 log-sum-exps.
inline size_t attn_partial_bytes(const Dims& D, int64_t nq, int nsplit) {
  return (size_t)nsplit * (size_t)nq * D.H * (D.d + 1) * 4;
}

// The centroid tables of one version: [H][C][d] bf16 starting at the slot.
__host__ __device__ inline size_t cent_slot_elems(const Dims& D) { return (size_t)D.H * D.C * D.d; }

// ---------------------------------------------------------------- device helpers
__device__ __forceinline__ float bf2f(uint16_t b) { return __uint_as_float((uint32_t)b << 16); }
__device__ __forceinline__ uint16_t f2bf(float x) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}
__device__ __forceinline__ float h2f(uint16_t h) { return __half2float(__ushort_as_half(h)); }
__device__ __forceinline__ uint16_t f2h_rd(float x) { return __half_as_ushort(__float2half_rd(x)); }
__device__ __forceinline__ uint16_t f2h_ru(float x) { return __half_as_ushort(__float2half_ru(x)); }

// Canonical INT2 group parameters from the fp32 residual range [lo, hi]:
// mn = fp16 round-down(lo), sc = fp16 round-up((hi - mn) / 3); zeros as +0.
__device__ __forceinline__ void int2_params(float lo, float hi, uint16_t& mnh, uint16_t& sch,
                                            float& mn, float& sc) {
  if (lo == 0.0f) lo = 0.0f;
  if (hi == 0.0f) hi = 0.0f;
  mnh = f2h_rd(lo);
  mn = h2f(mnh);
  sch = f2h_ru(__fdiv_rn(__fsub_rn(hi, mn), 3.0f));
  sc = h2f(sch);
}

// code = #{k in 0..2 : rho >= mn + (k + 0.5) sc}, 0 when sc == 0.
__device__ __forceinline__ int int2_code(float rho, float mn, float sc) {
  if (sc == 0.0f) return 0;
  int c = 0;
  c += rho >= __fadd_rn(mn, __fmul_rn(0.5f, sc));
  c += rho >= __fadd_rn(mn, __fmul_rn(1.5f, sc));
  c += rho >= __fadd_rn(mn, __fmul_rn(2.5f, sc));
  return c;
}

// Keys and values attended after the packed cache: a bf16 segment
// [n][H][d] (token-major, like K and V), and an optional [nq][H] fp32 output of
// the natural-log softmax denominators.
struct Segment {
  const uint16_t* K = nullptr;
  const uint16_t* V = nullptr;
  int64_t n = 0;
  float* lse = nullptr;
};

// ---------------------------------------------------------------- launchers
cudaError_t launch_init_state(const Dims& D, const CacheView& v, cudaStream_t s);
cudaError_t launch_kmeans(const Dims& D, const uint16_t* X, int64_t n, int iters, uint16_t* cent_out,
                          void* workspace, cudaStream_t s);
cudaError_t launch_stats_accumulate(const Dims& D, const uint16_t* Q, int64_t n, double* qstats,
                                    cudaStream_t s);
cudaError_t launch_refresh(const Dims& D, const CacheView& v, int64_t n_total, int version,
                           int warm, cudaStream_t s);
cudaError_t launch_append(const Dims& D, const CacheView& v, const uint16_t* K, const uint16_t* V,
                          int64_t n, int64_t t0, int version, int cent_version, cudaStream_t s);
cudaError_t launch_attention(const Dims& D, const CacheView& v, int64_t T, const uint16_t* Q,
                             int64_t nq, float scale, uint16_t* O, const Segment& sg,
                             cudaStream_t s);
cudaError_t launch_reconstruct(const Dims& D, const CacheView& v, int64_t t0, int64_t n,
                               uint16_t* Kp, uint16_t* Vp, cudaStream_t s);
cudaError_t launch_top1(const Dims& D, const CacheView& v, int64_t T, const uint16_t* Q,
                        int64_t nq, const uint16_t* Kexact, int32_t* idx_exact,
                        int32_t* idx_quant, cudaStream_t s);

size_t kmeans_workspace_bytes(const Dims& D);
bool attention_tc_supported(const Dims& D);
cudaError_t launch_attention_tc(const Dims& D, const CacheView& v, int64_t T, const uint16_t* Q,
                                int64_t nq, float scale, uint16_t* O, const Segment& sg,
                                cudaStream_t s);
cudaError_t launch_attention_simt(const Dims& D, const CacheView& v, int64_t T, const uint16_t* Q,
                                  int64_t nq, float scale, uint16_t* O, const Segment& sg,
                                  cudaStream_t s);
int read_and_clear_tc_timeout();
int read_and_clear_append_timeout();
bool append_tc_supported(const Dims& D);
cudaError_t launch_append_tc(const Dims& D, const CacheView& v, const uint16_t* K,
                             const uint16_t* V, int64_t n, int64_t t0, int version,
                             int cent_version, cudaStream_t s);

}  // namespace qwm
