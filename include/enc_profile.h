/*
 * enc_profile.h -- per-kernel timing of enc_forward with CUDA events.
 *
 * When profiling is enabled on a handle, every kernel that enc_forward
 * enqueues is bracketed by a pair of CUDA events on the caller's stream, and
 * its algorithmic work (multiply-add = 2 FLOPs, valid positions only) is
 * recorded with it. enc_profile_collect waits for those events, adds the
 * elapsed times per kernel class and clears the record. Profiling adds two
 * event records per launch and nothing else.
 */
#ifndef AUDIO_ENCODER_TOWER_ENC_PROFILE_H
#define AUDIO_ENCODER_TOWER_ENC_PROFILE_H

#include "enc.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef enum enc_kernel_class {
  ENC_K_MEL = 0,     /* mask + transpose of the mel input */
  ENC_K_CONV1 = 1,   /* conv1 implicit GEMM + GELU */
  ENC_K_CONV2 = 2,   /* conv2 implicit GEMM + GELU + position table */
  ENC_K_LN = 3,      /* pre-attention / pre-FFN LayerNorm */
  ENC_K_QKV = 4,     /* fused q/k/v projection */
  ENC_K_ATTN = 5,    /* attention */
  ENC_K_OUT = 6,     /* output projection + residual */
  ENC_K_FC1 = 7,     /* FFN up-projection + GELU */
  ENC_K_FC2 = 8,     /* FFN down-projection + residual */
  ENC_K_FINAL = 9,   /* final LayerNorm (+ pool, + unpack) */
  ENC_K_PROJ1 = 10,  /* projector fc1 + GELU */
  ENC_K_PROJ2 = 11,  /* projector fc2 (+ scatter) */
  ENC_K_ZERO = 12,   /* zeroing of padded output rows */
  ENC_K_COUNT = 13
} enc_kernel_class;

typedef struct enc_kernel_times {
  double ms[ENC_K_COUNT];        /* summed event time per class */
  double flops[ENC_K_COUNT];     /* summed algorithmic FLOPs per class */
  int64_t launches[ENC_K_COUNT]; /* launches per class */
} enc_kernel_times;

/* Turn event bracketing on or off for the following enc_forward calls. */
ENC_API enc_status enc_profile_enable(enc_handle *h, int32_t enable);

/* Wait for the recorded events, write the sums since the last collect, reset. */
ENC_API enc_status enc_profile_collect(enc_handle *h, enc_kernel_times *out);

/* Kernels enqueued by this handle since it was created (profiling on or off). */
ENC_API int64_t enc_launch_count(const enc_handle *h);

#ifdef __cplusplus
}
#endif

#endif /* AUDIO_ENCODER_TOWER_ENC_PROFILE_H */
