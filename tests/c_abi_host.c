/*
 * A plain C99 caller of the library: every public header compiled as C, the
 * shared object linked by a C toolchain, and the calls that need no device run
 * (argument errors that return before any CUDA call, status strings, the
 * shard planner). Built and run by tests/test_c_abi.py; prints one line per
 * check and exits non-zero when one fails.
 */
#include <stdio.h>
#include <string.h>

#include "enc.h"
#include "enc_cache.h"
#include "enc_frontend.h"
#include "enc_kernels.h"
#include "enc_profile.h"
#include "enc_shard.h"

static int failures = 0;

static void check(int ok, const char *what) {
  printf("%s %s\n", ok ? "ok" : "FAIL", what);
  if (!ok) ++failures;
}

static enc_config tiny(int max_batch) {
  enc_config c;
  memset(&c, 0, sizeof c);
  c.n_mels = 8;
  c.d_model = 128;
  c.n_layers = 1;
  c.n_heads = 2;
  c.head_dim = 64;
  c.ffn_dim = 128;
  c.max_frames = 40;
  c.max_batch = max_batch;
  c.pool_step = 1;
  c.ln_eps = 1e-5f;
  c.dtype = ENC_DTYPE_BF16;
  return c;
}

int main(void) {
  enc_config cfg = tiny(4);
  enc_weights w;
  enc_handle *h = (enc_handle *)&cfg;   /* must be reset to NULL on failure */
  int32_t rank_of[10], index_of[10], count[3], b;
  double flops = 0.0, rank_flops[3];

  check(strcmp(enc_status_string(ENC_OK), "ok") == 0, "status string of ENC_OK");
  check(strcmp(enc_status_string((enc_status)99), "unknown status") == 0, "status string of an unknown code");

  memset(&w, 0, sizeof w);
  check(enc_create(&cfg, NULL, &h) == ENC_ERR_INVALID_ARG && h == NULL, "enc_create without weights");
  h = (enc_handle *)&cfg;
  check(enc_create(NULL, &w, &h) == ENC_ERR_INVALID_ARG && h == NULL, "enc_create without a config");
  cfg.head_dim = 32;
  cfg.n_heads = 4;
  check(enc_create(&cfg, &w, &h) == ENC_ERR_UNSUPPORTED && h == NULL, "enc_create with head_dim 32");
  cfg = tiny(4);
  check(enc_create(&cfg, &w, NULL) == ENC_ERR_INVALID_ARG, "enc_create without an output pointer");
  check(enc_forward(NULL, NULL, NULL, 1, NULL, NULL) == ENC_ERR_INVALID_ARG, "enc_forward without a handle");
  check(enc_selftest_timeout(NULL, 1000000, NULL) == ENC_ERR_INVALID_ARG, "enc_selftest_timeout without a handle");
  enc_destroy(NULL);
  enc_cache_destroy(NULL);
  enc_frontend_destroy(NULL);
  check(1, "destroy calls accept NULL");

  /* len 3 -> 2 positions: conv1 24,576 + conv2 196,608 + QKV 196,608 + attention 2,048
     + out-proj 65,536 + FFN 131,072 FLOPs */
  check(enc_clip_flops(&cfg, 3, &flops) == ENC_OK && flops == 616448.0, "enc_clip_flops closed form");
  check(enc_clip_flops(&cfg, 41, &flops) == ENC_ERR_INVALID_ARG, "enc_clip_flops past max_frames");

  check(enc_shard_plan(&cfg, NULL, 10, 3, rank_of, index_of, count, rank_flops) == ENC_OK, "enc_shard_plan");
  for (b = 0; b < 10; ++b)
    if (rank_of[b] != b % 3 || index_of[b] != b / 3) break;
  check(b == 10, "full-length clips go round robin");
  check(count[0] == 4 && count[1] == 3 && count[2] == 3, "clips per rank");
  enc_clip_flops(&cfg, 40, &flops);
  check(rank_flops[0] == 4 * flops && rank_flops[1] == 3 * flops, "FLOPs per rank");
  check(enc_shard_plan(&cfg, NULL, 13, 3, rank_of, NULL, NULL, NULL) == ENC_ERR_INVALID_ARG,
        "more clips than ranks x max_batch");

  printf("%d failures\n", failures);
  return failures ? 1 : 0;
}
