/*
 * qwm.h -- C ABI of the B200 QuantWM 2-bit KV-cache library (libqwm.so).
 *
 * What the library computes (QuantWM: Temporally Consistent 2-Bit KV Cache
 * Quantization for Video World Models):
 *   - Keys are stored as a centroid (bf16) plus an INT2 residual; the centroid
 *     is chosen by QSAC (quantization-sensitivity-aware clustering): shortlist
 *     by Query-sensitivity-weighted distance, then the expected squared
 *     logit-perturbation of the INT2 residual decides.
 *     ["Flickering after quantization?" (SynthePulse en-US), QSAC paragraph;
 *      evolve.pub review, Summary and Strengths, Eq. 7]
 *   - PSAC (principal-subspace attention compensation) stores the remaining Key
 *     error projected on the top-r principal Query directions as INT8, added
 *     back when the cache is reconstructed.
 *     [same SynthePulse page, PSAC paragraph; review Summary, Fig. 4, Table 9]
 *   - Values: nearest centroid plus INT2 residual (the centroid-residual scheme
 *     QuantWM builds on; review Summary).
 *   - Attention of new queries over the packed cache with the reconstruction
 *     K' = C[a] + deq(R) + U deq8(c), V' = C_V[b] + deq(R_V) fused in.
 *
 * Conventions
 *   - Every device buffer is allocated and owned by the caller, at the sizes
 *     qwm_cache_sizes() reports, 256-byte aligned.  The library never allocates
 *     device memory.  qwm_cache is a small host struct the caller owns.
 *   - `stream` is a cudaStream_t passed as void*.  Calls enqueue kernels on it
 *     and return without synchronizing.  Calls on one cache must be ordered on
 *     one stream.  The host fields of qwm_cache change at enqueue time.
 *   - Tensors Q, K, V, O are token-major [n][heads][head_dim] bf16 (uint16 bit
 *     patterns), contiguous, device pointers, 16-byte aligned.
 *   - Errors: every argument is validated before anything is enqueued; on error
 *     nothing is enqueued and the cache is unchanged.  QWM_ERR_CUDA reports a
 *     launch failure (cudaGetLastError).  Nothing aborts or throws across the ABI.
 *   - Inputs must be finite.  Residuals beyond the fp16 range (|k - c| > 65504)
 *     are outside the supported domain.
 */
#ifndef QWM_H
#define QWM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define QWM_ABI_VERSION 2

#if defined(__GNUC__)
#define QWM_API __attribute__((visibility("default")))
#else
#define QWM_API
#endif

typedef enum qwm_status {
  QWM_OK = 0,
  QWM_ERR_INVALID_ARG = 1, /* null pointer, bad size, unsupported combination */
  QWM_ERR_ALIGNMENT = 2,   /* pointer not aligned as documented             */
  QWM_ERR_CAPACITY = 3,    /* tokens or basis versions beyond the capacity  */
  QWM_ERR_STATE = 4,       /* e.g. append before centroids were built       */
  QWM_ERR_CUDA = 5,        /* a CUDA launch or runtime call failed          */
  QWM_ERR_TIMEOUT = 6,     /* a bounded device wait gave up                  */
  QWM_ERR_UNSUPPORTED = 7  /* no kernel for this device / configuration     */
} qwm_status;

/* Quantizer and capacity.  Supported: head_dim 64 or 128; group 16 or 32 and
 * dividing head_dim; 1 <= n_centroids <= 512; 1 <= n_cand <= min(8, C);
 * 0 <= rank <= 16; 1 <= max_versions <= 65535; 1 <= max_cent_versions <= 65535;
 * 0 <= max_queries <= 2^24; max_tokens >= 1; flags a combination of the
 * QWM_FLAG_* bits. */

/* Split of the key range across CTA pairs in qwm_attention: at most this many
 * key ranges, each giving an fp32 partial result per query row and head that a
 * final pass merges through the log-sum-exp.  The WORKSPACE buffer holds the
 * partials for up to max_queries query rows; calls with more rows (or
 * max_queries == 0) attend over the whole key range in one pass. */
#define QWM_ATTN_MAX_SPLIT 6

/* QSAC stage 2 with the full quadratic form: each shortlisted centroid c is
 * scored by e^T A e, where e = k - (c + deq(INT2(k - c))) is the Key error
 * that c would leave and A = fp32(M / n) is the Query second moment in force
 * (Eq. 7 E[(q^T e)^2] = e^T M e with all of M; evolve.pub review, Strengths:
 * "full quadratic form gives no consistent gain at higher latency", Table 10).
 * Folds: y_i = sum_j A_ij e_j over j in order, then sum_i e_i y_i over i in
 * order, fp32 fused multiply-adds.  Without the flag the diagonal score
 * sum_g w_g R_g^2 is used.  Appends with the flag run on the CUDA cores. */
#define QWM_FLAG_QSAC_FULL 1

typedef struct qwm_config {
  int32_t heads;        /* H                                             */
  int32_t head_dim;     /* d                                             */
  int32_t n_centroids;  /* C (per head, same count for K and V)          */
  int32_t group;        /* G: channels per INT2 group                    */
  int32_t n_cand;       /* M: QSAC shortlist size                        */
  int32_t rank;         /* r: PSAC rank                                  */
  int32_t max_versions; /* slots for successive bases U (one per refresh) */
  int32_t flags;        /* QWM_FLAG_* bits (0: the method as described)   */
  int32_t max_cent_versions; /* slots for successive centroid tables      */
  int32_t max_queries;  /* query rows per attention call the WORKSPACE
                           holds split-key partials for (0: none)         */
  int64_t max_tokens;   /* cache capacity per head                       */
} qwm_config;

/* Device buffers, indexed by qwm_buffer_id.  Layout (Tcap = max_tokens rounded
 * up to a multiple of 128, ng = d / G, idx = uint8 if C <= 256 else uint16):
 *   K_CODES   [H][Tcap][d/4]   uint8   4 INT2 codes per byte, channel j in bits 2(j%4)
 *   K_PARAMS  [H][Tcap][ng][2] fp16    per group {mn, sc}: deq = mn + code * sc
 *   K_IDX     [H][Tcap]        idx     centroid of each key
 *   K_COEF    [H][Tcap][r]     int8    PSAC coefficients
 *   K_CSCALE  [H][Tcap]        fp16    PSAC per-token scale
 *   V_CODES, V_PARAMS, V_IDX   as for K
 *   CENT_K, CENT_V [max_cent_versions][H][C][d] bf16  centroid tables, slot =
 *                                      centroid-table version
 *   QSTATS    [H][d][d]        fp64    running sum of q q^T
 *   SENS      [H][d]           fp32    s_j = E[q_j^2] in force
 *   WGROUP    [H][ng]          fp32    w_g = sum of s_j over group g
 *   BASIS     [max_versions][H][d][r] fp32  PSAC bases, slot = version
 *   TOKVER    [Tcap]           uint16  basis version of each cached token
 *   CENTVER   [Tcap]           uint16  centroid-table version of each cached token
 *   EIGVEC    [H][d][d] + [H]  fp64    refresh state: per head the Ritz vectors
 *                                      of the last refresh (first 32 columns of d),
 *                                      then, with QWM_FLAG_QSAC_FULL, A = fp32(M/n)
 *                                      in force ([d][d] fp32 from double offset
 *                                      32 d); after all heads one warm-start flag
 *                                      per head
 *   WORKSPACE                  bytes   scratch for centroid building, basis refresh
 *                                      and attention partials: at least
 *                                      QWM_ATTN_MAX_SPLIT x max_queries x H x
 *                                      (d + 1) fp32 */
typedef enum qwm_buffer_id {
  QWM_BUF_K_CODES = 0, QWM_BUF_K_PARAMS, QWM_BUF_K_IDX, QWM_BUF_K_COEF, QWM_BUF_K_CSCALE,
  QWM_BUF_V_CODES, QWM_BUF_V_PARAMS, QWM_BUF_V_IDX, QWM_BUF_CENT_K, QWM_BUF_CENT_V,
  QWM_BUF_QSTATS, QWM_BUF_SENS, QWM_BUF_WGROUP, QWM_BUF_BASIS, QWM_BUF_TOKVER,
  QWM_BUF_CENTVER, QWM_BUF_EIGVEC, QWM_BUF_WORKSPACE, QWM_NBUF
} qwm_buffer_id;

typedef struct qwm_sizes {
  uint64_t bytes[QWM_NBUF]; /* size of each buffer                       */
  int64_t tcap;             /* token capacity per head after rounding    */
  int64_t bytes_per_token_head; /* packed bytes per cached token and head */
} qwm_sizes;

typedef struct qwm_buffers {
  void* ptr[QWM_NBUF];
} qwm_buffers;

/* Host-side cache state; owned by the caller, filled by qwm_cache_init. */
typedef struct qwm_cache {
  qwm_config cfg;
  qwm_buffers buf;
  int64_t tcap;
  int64_t len;          /* tokens cached (per head)                 */
  int64_t n_queries;    /* query rows accumulated into QSTATS       */
  int32_t frames;       /* qwm_append_kv calls so far               */
  int32_t n_versions;   /* basis versions written (>= 1 after init) */
  int32_t cur_version;  /* version used by the next append          */
  int32_t has_centroids;
  int32_t has_eigvec;   /* EIGVEC holds a previous decomposition    */
  int32_t magic;
  int32_t n_cent_versions;  /* centroid-table versions written      */
  int32_t cur_cent_version; /* table version used by the next append */
} qwm_cache;

QWM_API int32_t qwm_abi_version(void);
QWM_API const char* qwm_status_string(qwm_status s);

/* Buffer sizes for `cfg` (host only, no device work).
 * Errors: QWM_ERR_INVALID_ARG for a null pointer or an unsupported config. */
QWM_API qwm_status qwm_cache_sizes(const qwm_config* cfg, qwm_sizes* out);

/* Fill `c` and enqueue the initial device state: QSTATS = 0, SENS = 1,
 * WGROUP = G, BASIS version 0 = 0 (no history: PSAC adds nothing).
 * Every pointer in `bufs` must be non-null (K_COEF may be null when rank is 0)
 * and 256-byte aligned.  Errors: INVALID_ARG, ALIGNMENT, CUDA. */
QWM_API qwm_status qwm_cache_init(qwm_cache* c, const qwm_config* cfg, const qwm_buffers* bufs,
                          void* stream);

/* Centroid tables (k-means, per head, separately for K and V) from n tokens,
 * usually the newest frame.  The pages say only that each Key is assigned to a
 * cluster centre kept at higher precision (SynthePulse, QSAC paragraph).
 * Here: centroid i starts at token floor(i n / C); `iters` Lloyd rounds with
 * fp32 squared distances (ties to the lower index) and fp64 means taken in
 * token order; an empty cluster keeps its centroid; the result is rounded to
 * bf16.
 * Versions: the first call writes table version 0.  A later call on a cache
 * that already holds tokens writes the next version (a centroid refresh under
 * Key drift; the pages are silent on refreshing the centres): later appends
 * encode against it, while every cached token keeps decoding with the version
 * it was encoded with (CENTVER).  A later call on an empty cache rewrites the
 * version in force, which no token references.
 * K, V: [n][H][d] bf16 device.  Requires n >= C, n <= tcap and
 * 1 <= iters <= 1000.  Errors: INVALID_ARG, ALIGNMENT, CAPACITY (all
 * max_cent_versions slots used), CUDA. */
QWM_API qwm_status qwm_build_centroids(qwm_cache* c, const void* K, const void* V, int64_t n,
                               int32_t iters, void* stream);

/* Historical Query statistics [review, Summary: "historical Query
 * second-moment statistics"; Eq. 7 M = E[q q^T]]: QSTATS[h] += sum_t q_t q_t^T,
 * n_queries += n_q.  Each fp64 entry is summed in token order, so QSTATS is
 * the sequential fp64 sum bit for bit (the products of bf16 values are exact).
 * With refresh_basis != 0 it then refreshes what QSAC and PSAC read:
 * s_j = fp32(M_jj / n), w_g = the fp32 sum of s_j over group g in channel
 * order, U = top-r eigenvectors of M / n (fp64 block subspace iteration with
 * a Rayleigh-Ritz step, warm-started from the last refresh; columns signed so
 * that the largest-magnitude entry is positive), stored as a new basis version
 * used by later appends.  Q: [n_q][H][d] bf16 device, n_q >= 0.
 * Errors: INVALID_ARG, ALIGNMENT, CAPACITY (no free basis slot), CUDA. */
QWM_API qwm_status qwm_update_query_stats(qwm_cache* c, const void* Q, int64_t n_q,
                                  int32_t refresh_basis, void* stream);

/* Quantize and append n tokens at position len (QSAC + INT2 + PSAC for Keys,
 * nearest centroid + INT2 for Values) with the statistics, basis and centroid
 * tables in force; TOKVER and CENTVER of the new tokens record the basis and
 * table versions.
 * Codes, indices and INT8 coefficients are bit-identical to the canonical
 * fp32 definition the CPU oracle implements.  K, V: [n][H][d] bf16 device.
 * Errors: INVALID_ARG, ALIGNMENT, CAPACITY (len + n > tcap), STATE (no
 * centroids), CUDA. */
QWM_API qwm_status qwm_append_kv(qwm_cache* c, const void* K, const void* V, int64_t n, void* stream);

/* O = softmax(scale Q K'^T) V' over all `len` cached tokens, with K', V'
 * reconstructed on the fly from the packed cache (each key with the basis and
 * centroid-table versions in force when it was appended):
 *   K'_j = bf16(C_K[a]_j + (mn + code_j sc) + sum_i U_ji (c8_i cs)),
 *   V'_j = bf16(C_V[b]_j + (mn + code_j sc)),
 * each element rounded once, so the attention reads exactly the bf16 cache
 * that qwm_reconstruct returns (up to the order of the fp32 sum).  No mask.  Q, O: [n_q][H][d] bf16
 * device (O written, fp32 accumulation).  scale <= 0 selects 1/sqrt(d).
 * Errors: INVALID_ARG, ALIGNMENT, STATE (empty cache), CUDA. */
QWM_API qwm_status qwm_attention(const qwm_cache* c, const void* Q, int64_t n_q, float scale, void* O,
                         void* stream);

/* Attention over the packed history followed by a bf16 segment: keys
 * 0 .. len-1 reconstructed from the packed cache as in qwm_attention, then
 * keys len .. len+n_seg-1 taken exactly from K_seg / V_seg.  In an
 * autoregressive world model the cache holds the finished frames while the
 * frame being generated attends to them and to its own, not yet quantized,
 * keys and values at every denoising step ("Flickering after quantization?",
 * opening paragraphs: the KV cache stores the historical frames); the pages do
 * not describe this step, and this is its plainest reading.  With len == 0 it
 * is plain bf16 attention over the segment.
 * Q, O: [n_q][H][d] bf16 device; K_seg, V_seg: [n_seg][H][d] bf16 device
 * (may be null when n_seg == 0); lse: null, or [n_q][H] fp32 device receiving
 * ln sum_t exp(scale q . k_t) over all len + n_seg keys, for merging with
 * attention over other keys.  scale <= 0 selects 1/sqrt(d).  Nothing is
 * stored in the cache.  Errors: INVALID_ARG, ALIGNMENT, STATE (no keys at all,
 * or a non-empty cache without centroids), CUDA. */
QWM_API qwm_status qwm_attention_ext(const qwm_cache* c, const void* Q, int64_t n_q,
                                     const void* K_seg, const void* V_seg, int64_t n_seg,
                                     float scale, void* O, float* lse, void* stream);

/* Reconstructed cache, for inspection: K', V' of tokens [t0, t0+n) as
 * [H][n][d] bf16 device arrays.  Errors: INVALID_ARG, ALIGNMENT, CUDA. */
QWM_API qwm_status qwm_reconstruct(const qwm_cache* c, int64_t t0, int64_t n, void* Kp, void* Vp,
                           void* stream);

/* Top-1 key selection of each query row (argmax_t q . k_t, fp32 dot, ties to
 * the lower t) over the exact keys `K_exact` ([len][H][d] bf16, the keys as
 * they were appended) and over the reconstructed cache; the fraction that
 * differ is the selection shift the pages report ("Flickering after
 * quantization?", attention-analysis paragraph).  idx_exact, idx_quant:
 * [n_q][H] int32 device.  Errors: INVALID_ARG, ALIGNMENT, STATE, CUDA. */
QWM_API qwm_status qwm_top1_shift(const qwm_cache* c, const void* Q, int64_t n_q, const void* K_exact,
                          int32_t* idx_exact, int32_t* idx_quant, void* stream);

/* Size of the fixed device scratch array used by
 * qwm_build_centroids_noalloc (16 MiB per GPU that loads the library). */
#define QWM_NOALLOC_SCRATCH_BYTES (16u << 20)

/* qwm_build_centroids for callers that cannot allocate device memory -- no
 * counterpart in the paper.  Hosts such as inference servers or engine plugin
 * frameworks own the GPU memory budget and hand out fixed buffers; code running
 * inside them may not call cudaMalloc/cudaFree (these synchronize the device
 * and fragment the host's pool).  This variant writes the same centroid tables
 * as qwm_build_centroids (with the same version rules) but takes its scratch
 * from one fixed device array inside the library instead of the cache's
 * WORKSPACE buffer, and allocates nothing.  The array is
 * QWM_NOALLOC_SCRATCH_BYTES long and stays allocated on every GPU that loads
 * the library until the process exits; the call needs
 * 4*H*C*d bytes (rounded up to 256) + 4*H*n bytes of it and returns
 * QWM_ERR_CAPACITY when that exceeds the array.  The first call on each device
 * looks up the array's device address (cudaGetSymbolAddress, with that device
 * current), so make that first call before any stream capture.  No scratch
 * entry needs to start at zero (each is written before it is read).  All calls
 * share the one array and it keeps the last call's contents: calls whose
 * kernels can overlap on the GPU (several streams of one device) race, and the
 * caller must order them.  Arguments and other errors as for
 * qwm_build_centroids: INVALID_ARG, ALIGNMENT, CAPACITY (also when every
 * table slot is used), CUDA. */
QWM_API qwm_status qwm_build_centroids_noalloc(qwm_cache* c, const void* K, const void* V,
                                               int64_t n, int32_t iters, void* stream);

/* Device-side health check: synchronizes the current device, then reads and
 * clears the flag that the tensor-core kernels set when one of their bounded
 * waits gave up (about one second per wait) instead of hanging.  *flags = 1 and
 * QWM_ERR_TIMEOUT if any wait timed out since the last call, else 0 and QWM_OK.
 * Errors: INVALID_ARG (null), CUDA. */
QWM_API qwm_status qwm_device_status(int32_t* flags);

#ifdef __cplusplus
}
#endif
#endif /* QWM_H */
