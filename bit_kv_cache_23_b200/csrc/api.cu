// api.cu -- the extern "C" entry points of libqwm.so: argument validation,
// buffer sizing, host-side cache bookkeeping and kernel dispatch.
#include <string.h>

#include "common.cuh"

using namespace qwm;

namespace {

bool aligned(const void* p, uintptr_t a) { return ((uintptr_t)p % a) == 0; }

qwm_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return QWM_OK;
  return QWM_ERR_CUDA;
}

}  // namespace

extern "C" {

int32_t qwm_abi_version(void) { return QWM_ABI_VERSION; }

const char* qwm_status_string(qwm_status s) {
  switch (s) {
    case QWM_OK: return "ok";
    case QWM_ERR_INVALID_ARG: return "invalid argument";
    case QWM_ERR_ALIGNMENT: return "misaligned pointer";
    case QWM_ERR_CAPACITY: return "capacity exceeded";
    case QWM_ERR_STATE: return "invalid cache state for this call";
    case QWM_ERR_CUDA: return "CUDA error";
    case QWM_ERR_TIMEOUT: return "device wait timed out";
    case QWM_ERR_UNSUPPORTED: return "unsupported device or configuration";
  }
  return "unknown status";
}

qwm_status qwm_cache_sizes(const qwm_config* cfg, qwm_sizes* out) {
  if (!cfg || !out || !config_ok(cfg)) return QWM_ERR_INVALID_ARG;
  Dims D = dims_of(cfg);
  memset(out, 0, sizeof(*out));
  const uint64_t HT = (uint64_t)D.H * D.tcap;
  out->tcap = D.tcap;
  out->bytes[QWM_BUF_K_CODES] = HT * (D.d / 4);
  out->bytes[QWM_BUF_K_PARAMS] = HT * D.ng * 4;
  out->bytes[QWM_BUF_K_IDX] = HT * D.idx_bytes;
  out->bytes[QWM_BUF_K_COEF] = HT * D.r;
  out->bytes[QWM_BUF_K_CSCALE] = HT * 2;
  out->bytes[QWM_BUF_V_CODES] = HT * (D.d / 4);
  out->bytes[QWM_BUF_V_PARAMS] = HT * D.ng * 4;
  out->bytes[QWM_BUF_V_IDX] = HT * D.idx_bytes;
  out->bytes[QWM_BUF_CENT_K] = (uint64_t)cfg->max_cent_versions * cent_slot_elems(D) * 2;
  out->bytes[QWM_BUF_CENT_V] = (uint64_t)cfg->max_cent_versions * cent_slot_elems(D) * 2;
  out->bytes[QWM_BUF_QSTATS] = (uint64_t)D.H * D.d * D.d * 8;
  out->bytes[QWM_BUF_SENS] = (uint64_t)D.H * D.d * 4;
  out->bytes[QWM_BUF_WGROUP] = (uint64_t)D.H * D.ng * 4;
  out->bytes[QWM_BUF_BASIS] = (uint64_t)cfg->max_versions * D.H * D.d * (D.r > 0 ? D.r : 1) * 4;
  out->bytes[QWM_BUF_TOKVER] = (uint64_t)D.tcap * 2;
  out->bytes[QWM_BUF_CENTVER] = (uint64_t)D.tcap * 2;
  out->bytes[QWM_BUF_EIGVEC] = (uint64_t)D.H * D.d * D.d * 8 + (uint64_t)D.H * 8;
  const size_t ws_attn = attn_partial_bytes(D, cfg->max_queries, QWM_ATTN_MAX_SPLIT);
  const size_t ws_km = kmeans_workspace_bytes(D);
  out->bytes[QWM_BUF_WORKSPACE] = ws_km > ws_attn ? ws_km : ws_attn;
  out->bytes_per_token_head = 2 * (D.d / 4 + 4 * D.ng + D.idx_bytes) + D.r + 2;
  return QWM_OK;
}

qwm_status qwm_cache_init(qwm_cache* c, const qwm_config* cfg, const qwm_buffers* bufs,
                          void* stream) {
  if (!c || !cfg || !bufs || !config_ok(cfg)) return QWM_ERR_INVALID_ARG;
  for (int i = 0; i < QWM_NBUF; ++i) {
    if (i == QWM_BUF_K_COEF && cfg->rank == 0) continue;
    if (!bufs->ptr[i]) return QWM_ERR_INVALID_ARG;
  }
  for (int i = 0; i < QWM_NBUF; ++i)
    if (bufs->ptr[i] && !aligned(bufs->ptr[i], 256)) return QWM_ERR_ALIGNMENT;
  Dims D = dims_of(cfg);
  qwm_cache tmp;
  memset(&tmp, 0, sizeof(tmp));
  tmp.cfg = *cfg;
  tmp.buf = *bufs;
  tmp.tcap = D.tcap;
  tmp.n_versions = 1;
  tmp.cur_version = 0;
  tmp.n_cent_versions = 0;
  tmp.cur_cent_version = 0;
  tmp.magic = kCacheMagic;
  CacheView v = view_of(&tmp);
  cudaError_t e = launch_init_state(D, v, (cudaStream_t)stream);
  if (e != cudaSuccess) return QWM_ERR_CUDA;
  *c = tmp;
  return QWM_OK;
}

qwm_status qwm_build_centroids(qwm_cache* c, const void* K, const void* V, int64_t n,
                               int32_t iters, void* stream) {
  int slot = 0;
  const qwm_status st = centroid_build_slot(c, K, V, n, iters, &slot);
  if (st != QWM_OK) return st;
  Dims D = dims_of(&c->cfg);
  CacheView v = view_of(c);
  cudaStream_t s = (cudaStream_t)stream;
  const size_t off = (size_t)slot * cent_slot_elems(D);
  cudaError_t e = launch_kmeans(D, (const uint16_t*)K, n, iters, v.cent_k + off, v.workspace, s);
  if (e == cudaSuccess)
    e = launch_kmeans(D, (const uint16_t*)V, n, iters, v.cent_v + off, v.workspace, s);
  if (e != cudaSuccess) return QWM_ERR_CUDA;
  centroid_build_commit(c, slot);
  return QWM_OK;
}

qwm_status qwm_update_query_stats(qwm_cache* c, const void* Q, int64_t n_q, int32_t refresh_basis,
                                  void* stream) {
  if (!cache_ok(c) || n_q < 0 || (n_q > 0 && !Q)) return QWM_ERR_INVALID_ARG;
  if (Q && !aligned(Q, 16)) return QWM_ERR_ALIGNMENT;
  if (refresh_basis && c->n_versions >= c->cfg.max_versions) return QWM_ERR_CAPACITY;
  Dims D = dims_of(&c->cfg);
  CacheView v = view_of(c);
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e = cudaSuccess;
  if (n_q > 0) e = launch_stats_accumulate(D, (const uint16_t*)Q, n_q, v.qstats, s);
  if (e != cudaSuccess) return QWM_ERR_CUDA;
  c->n_queries += n_q;
  if (refresh_basis) {
    int ver = c->n_versions;
    e = launch_refresh(D, v, c->n_queries, ver, c->has_eigvec, s);
    if (e != cudaSuccess) return QWM_ERR_CUDA;
    c->n_versions += 1;
    c->cur_version = ver;
    if (c->n_queries > 0) c->has_eigvec = 1;
  }
  return QWM_OK;
}

qwm_status qwm_append_kv(qwm_cache* c, const void* K, const void* V, int64_t n, void* stream) {
  if (!cache_ok(c) || n < 0 || (n > 0 && (!K || !V))) return QWM_ERR_INVALID_ARG;
  if ((K && !aligned(K, 16)) || (V && !aligned(V, 16))) return QWM_ERR_ALIGNMENT;
  if (!c->has_centroids) return QWM_ERR_STATE;
  if (c->len + n > c->tcap) return QWM_ERR_CAPACITY;
  if (n == 0) return QWM_OK;
  Dims D = dims_of(&c->cfg);
  CacheView v = view_of(c);
  cudaError_t e = launch_append(D, v, (const uint16_t*)K, (const uint16_t*)V, n, c->len,
                                c->cur_version, c->cur_cent_version, (cudaStream_t)stream);
  if (e != cudaSuccess) return QWM_ERR_CUDA;
  c->len += n;
  c->frames += 1;
  return QWM_OK;
}

qwm_status qwm_attention(const qwm_cache* c, const void* Q, int64_t n_q, float scale, void* O,
                         void* stream) {
  if (!cache_ok(c) || n_q < 0 || (n_q > 0 && (!Q || !O))) return QWM_ERR_INVALID_ARG;
  if ((Q && !aligned(Q, 16)) || (O && !aligned(O, 16))) return QWM_ERR_ALIGNMENT;
  if (c->len <= 0 || !c->has_centroids) return QWM_ERR_STATE;
  if (n_q == 0) return QWM_OK;
  Dims D = dims_of(&c->cfg);
  if (!(scale > 0.0f)) scale = 1.0f / sqrtf((float)D.d);
  CacheView v = view_of(c);
  return cuda_status(launch_attention(D, v, c->len, (const uint16_t*)Q, n_q, scale, (uint16_t*)O,
                                      Segment{}, (cudaStream_t)stream));
}

qwm_status qwm_attention_ext(const qwm_cache* c, const void* Q, int64_t n_q, const void* K_seg,
                             const void* V_seg, int64_t n_seg, float scale, void* O, float* lse,
                             void* stream) {
  if (!cache_ok(c) || n_q < 0 || n_seg < 0 || (n_q > 0 && (!Q || !O)) ||
      (n_seg > 0 && (!K_seg || !V_seg)))
    return QWM_ERR_INVALID_ARG;
  if ((Q && !aligned(Q, 16)) || (O && !aligned(O, 16)) || (K_seg && !aligned(K_seg, 16)) ||
      (V_seg && !aligned(V_seg, 16)) || (lse && !aligned(lse, 4)))
    return QWM_ERR_ALIGNMENT;
  if (c->len + n_seg <= 0 || (c->len > 0 && !c->has_centroids)) return QWM_ERR_STATE;
  if (n_q == 0) return QWM_OK;
  Dims D = dims_of(&c->cfg);
  if (!(scale > 0.0f)) scale = 1.0f / sqrtf((float)D.d);
  CacheView v = view_of(c);
  Segment sg;
  sg.K = (const uint16_t*)K_seg;
  sg.V = (const uint16_t*)V_seg;
  sg.n = n_seg;
  sg.lse = lse;
  return cuda_status(launch_attention(D, v, c->len, (const uint16_t*)Q, n_q, scale, (uint16_t*)O,
                                      sg, (cudaStream_t)stream));
}

qwm_status qwm_reconstruct(const qwm_cache* c, int64_t t0, int64_t n, void* Kp, void* Vp,
                           void* stream) {
  if (!cache_ok(c) || t0 < 0 || n < 0 || t0 + n > c->len || (n > 0 && (!Kp || !Vp)))
    return QWM_ERR_INVALID_ARG;
  if ((Kp && !aligned(Kp, 16)) || (Vp && !aligned(Vp, 16))) return QWM_ERR_ALIGNMENT;
  if (n == 0) return QWM_OK;
  Dims D = dims_of(&c->cfg);
  CacheView v = view_of(c);
  return cuda_status(
      launch_reconstruct(D, v, t0, n, (uint16_t*)Kp, (uint16_t*)Vp, (cudaStream_t)stream));
}

qwm_status qwm_top1_shift(const qwm_cache* c, const void* Q, int64_t n_q, const void* K_exact,
                          int32_t* idx_exact, int32_t* idx_quant, void* stream) {
  if (!cache_ok(c) || n_q < 0 || (n_q > 0 && (!Q || !K_exact || !idx_exact || !idx_quant)))
    return QWM_ERR_INVALID_ARG;
  if ((Q && !aligned(Q, 16)) || (K_exact && !aligned(K_exact, 16)) ||
      (idx_exact && !aligned(idx_exact, 4)) || (idx_quant && !aligned(idx_quant, 4)))
    return QWM_ERR_ALIGNMENT;
  if (c->len <= 0) return QWM_ERR_STATE;
  if (n_q == 0) return QWM_OK;
  Dims D = dims_of(&c->cfg);
  CacheView v = view_of(c);
  return cuda_status(launch_top1(D, v, c->len, (const uint16_t*)Q, n_q, (const uint16_t*)K_exact,
                                 idx_exact, idx_quant, (cudaStream_t)stream));
}

qwm_status qwm_device_status(int32_t* flags) {
  if (!flags) return QWM_ERR_INVALID_ARG;
  if (cudaDeviceSynchronize() != cudaSuccess) return QWM_ERR_CUDA;
  int v = read_and_clear_tc_timeout();
  int v2 = read_and_clear_append_timeout();
  if (v < 0 || v2 < 0) return QWM_ERR_CUDA;
  v = v | v2;
  *flags = v;
  return v ? QWM_ERR_TIMEOUT : QWM_OK;
}

}  // extern "C"
