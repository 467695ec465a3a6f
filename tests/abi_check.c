/* A plain C caller of include/confkv.h, compiled and run by
 * tests/test_library_abi.py on a machine without a GPU. It prints the layout
 * of the header's structs as the C compiler sees it (for comparison with the
 * Python binding's mirror) and exercises the entry points that need no
 * device: default parameters, status strings, the version, and argument
 * checks that fail before anything touches the device. */
#include <stddef.h>
#include <stdio.h>
#include <string.h>

#include "confkv.h"

#define FIELD(type, f) printf("%s.%s %zu %zu\n", #type, #f, offsetof(type, f), sizeof(((type*)0)->f))

int main(void) {
  printf("sizeof confkv_params %zu\n", sizeof(confkv_params));
  FIELD(confkv_params, mode);
  FIELD(confkv_params, n_low);
  FIELD(confkv_params, n_high);
  FIELD(confkv_params, tau);
  FIELD(confkv_params, alpha);
  FIELD(confkv_params, ema_decay);
  FIELD(confkv_params, protect_last);
  FIELD(confkv_params, fp16_window);
  FIELD(confkv_params, n_sink);
  FIELD(confkv_params, fixed_budget);
  FIELD(confkv_params, pyramidal);
  FIELD(confkv_params, gate);
  FIELD(confkv_params, int8_enable);
  FIELD(confkv_params, compact);
  FIELD(confkv_params, max_batch);
  FIELD(confkv_params, max_prefill);
  FIELD(confkv_params, score_source);
  FIELD(confkv_params, seed);
  FIELD(confkv_params, single_stream);
  printf("sizeof confkv_stats %zu\n", sizeof(confkv_stats));
  FIELD(confkv_stats, tokens_int8);
  FIELD(confkv_stats, tokens_fp16);
  FIELD(confkv_stats, bytes_payload);
  FIELD(confkv_stats, bytes_meta);
  FIELD(confkv_stats, bytes_capacity);
  FIELD(confkv_stats, min_len);
  FIELD(confkv_stats, max_len);
  FIELD(confkv_stats, attn_tokens_int8);
  FIELD(confkv_stats, attn_tokens_fp16);
  FIELD(confkv_stats, evict_tokens);
  FIELD(confkv_stats, moved_rows);
  FIELD(confkv_stats, requant_rows);
  FIELD(confkv_stats, kernel_launches);
  FIELD(confkv_stats, evict_block_segments);
  FIELD(confkv_stats, moved_window_rows);
  printf("sizeof confkv_profile %zu\n", sizeof(confkv_profile));
  FIELD(confkv_profile, launches);
  FIELD(confkv_profile, ms);

  confkv_params p;
  memset(&p, 0xff, sizeof p);
  if (confkv_default_params(&p) != CONFKV_OK) return 10;
  printf("default %d %d %d %d %d %.7g %.7g %.7g\n", p.n_low, p.n_high, p.protect_last, p.fp16_window,
         p.max_prefill, p.tau, p.alpha, p.ema_decay);
  if (confkv_default_params(NULL) != CONFKV_ERR_ARG) return 11;
  for (int s = CONFKV_OK; s <= CONFKV_ERR_DEVICE; ++s) printf("status %d %s\n", s, confkv_status_string((confkv_status)s));
  printf("version %d\n", confkv_version());

  /* rejected before any device work: a head_dim the kernels do not serve,
     and a budget gate that does not exist */
  confkv_handle* h = (confkv_handle*)&p;
  if (confkv_create(2, 4, 8, 96, &p, &h) != CONFKV_ERR_ARG || h != NULL) return 12;
  p.gate = 5;
  h = (confkv_handle*)&p;
  if (confkv_create(2, 4, 8, 128, &p, &h) != CONFKV_ERR_ARG || h != NULL) return 13;
  if (confkv_create(2, 4, 8, 128, NULL, &h) != CONFKV_ERR_ARG) return 14;
  /* the allocation-free confidence entry rejects missing buffers and a
     batch beyond its fixed scratch before it looks for a device */
  confkv_default_params(&p);
  if (confkv_confidence_noalloc(&p, 1, NULL, 1, 16, NULL, NULL, NULL) != CONFKV_ERR_ARG) return 15;
  float dummy[4];
  int32_t bud[4];
  if (confkv_confidence_noalloc(&p, 1, dummy, 257, 16, dummy, bud, NULL) != CONFKV_ERR_CAPACITY) return 16;
  if (confkv_destroy(NULL) != CONFKV_OK) return 17;
  printf("ok\n");
  return 0;
}
