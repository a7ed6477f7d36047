/* abi_probe.c -- compiled with gcc against include/qwm.h and linked to
 * libqwm.so by tests/test_abi.py: prints the header's struct layouts, enum
 * values and the results of host-only calls, one "key value" pair per line,
 * so that the test can compare them with the Python binding's ctypes
 * declarations and with the documented sizes.  Makes no CUDA call. */
#include <stddef.h>
#include <stdio.h>

#include "qwm.h"

#define FIELD(T, f) printf("off %s.%s %zu\n", #T, #f, offsetof(T, f))

int main(void) {
  printf("abi_macro %d\n", QWM_ABI_VERSION);
  printf("abi_lib %d\n", (int)qwm_abi_version());
  printf("nbuf %d\n", (int)QWM_NBUF);
  printf("noalloc_bytes %u\n", (unsigned)QWM_NOALLOC_SCRATCH_BYTES);
  printf("flag_qsac_full %d\n", (int)QWM_FLAG_QSAC_FULL);
  printf("attn_max_split %d\n", (int)QWM_ATTN_MAX_SPLIT);
  printf("size qwm_config %zu\n", sizeof(qwm_config));
  printf("size qwm_sizes %zu\n", sizeof(qwm_sizes));
  printf("size qwm_buffers %zu\n", sizeof(qwm_buffers));
  printf("size qwm_cache %zu\n", sizeof(qwm_cache));
  FIELD(qwm_config, heads); FIELD(qwm_config, head_dim); FIELD(qwm_config, n_centroids);
  FIELD(qwm_config, group); FIELD(qwm_config, n_cand); FIELD(qwm_config, rank);
  FIELD(qwm_config, max_versions); FIELD(qwm_config, flags);
  FIELD(qwm_config, max_cent_versions); FIELD(qwm_config, max_queries);
  FIELD(qwm_config, max_tokens);
  FIELD(qwm_sizes, bytes); FIELD(qwm_sizes, tcap); FIELD(qwm_sizes, bytes_per_token_head);
  FIELD(qwm_cache, cfg); FIELD(qwm_cache, buf); FIELD(qwm_cache, tcap); FIELD(qwm_cache, len);
  FIELD(qwm_cache, n_queries); FIELD(qwm_cache, frames); FIELD(qwm_cache, n_versions);
  FIELD(qwm_cache, cur_version); FIELD(qwm_cache, has_centroids); FIELD(qwm_cache, has_eigvec);
  FIELD(qwm_cache, magic); FIELD(qwm_cache, n_cent_versions); FIELD(qwm_cache, cur_cent_version);
  printf("enum QWM_BUF_K_CODES %d\n", (int)QWM_BUF_K_CODES);
  printf("enum QWM_BUF_CENT_K %d\n", (int)QWM_BUF_CENT_K);
  printf("enum QWM_BUF_TOKVER %d\n", (int)QWM_BUF_TOKVER);
  printf("enum QWM_BUF_CENTVER %d\n", (int)QWM_BUF_CENTVER);
  printf("enum QWM_BUF_WORKSPACE %d\n", (int)QWM_BUF_WORKSPACE);
  /* the 480p layer's configuration, two centroid-table slots */
  qwm_config cfg = {.heads = 40, .head_dim = 128, .n_centroids = 256, .group = 32,
                    .n_cand = 4, .rank = 8, .max_versions = 64, .flags = 0,
                    .max_cent_versions = 2, .max_queries = 1560, .max_tokens = 37440};
  qwm_sizes s;
  qwm_status st = qwm_cache_sizes(&cfg, &s);
  printf("sizes_status %d\n", (int)st);
  printf("sizes_tcap %lld\n", (long long)s.tcap);
  printf("sizes_bpth %lld\n", (long long)s.bytes_per_token_head);
  for (int i = 0; i < QWM_NBUF; ++i) printf("sizes_bytes_%d %llu\n", i, (unsigned long long)s.bytes[i]);
  cfg.max_cent_versions = 0;
  printf("sizes_bad_status %d\n", (int)qwm_cache_sizes(&cfg, &s));
  printf("status_capacity %s\n", qwm_status_string(QWM_ERR_CAPACITY));
  return 0;
}
