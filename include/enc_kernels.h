/*
 * enc_kernels.h -- single-kernel entry points of the encoder library, for
 * testing and timing one step of the forward pass on its own.
 *
 * Same conventions as enc.h: device pointers, row-major, nothing traps;
 * host-detectable errors return before any launch. These calls allocate
 * nothing; the caller owns every buffer.
 */
#ifndef AUDIO_ENCODER_TOWER_ENC_KERNELS_H
#define AUDIO_ENCODER_TOWER_ENC_KERNELS_H

#include "enc.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Linear layer on the tensor cores (the QKV / out-proj / fc1 / fc2 / projector
 * step of a pre-LN block, Qwen2-Audio-7B-Instruct "(1) AUDIO ENCODER"):
 *   out[M, N] = act(A[M, K] * W[N, K]^T + bias[N])      (act = GELU when gelu != 0)
 * A, W, out: bf16; bias: fp32 [N] or NULL. K a multiple of 64, N a multiple of
 * 128, A/W/out rows 16-byte aligned. With resid != NULL the result is instead
 * accumulated into the fp32 matrix resid[M, N] (resid += A W^T + bias) and out
 * is ignored. status: device int (may be NULL) set to ENC_ERR_TIMEOUT if a
 * bounded wait inside the kernel runs out.
 */
ENC_API enc_status enc_linear_bf16(const void *A, const void *W, const float *bias, void *out, float *resid,
                                   int32_t M, int32_t N, int32_t K, int32_t gelu, int *status,
                                   cudaStream_t stream);

/*
 * Bidirectional multi-head attention, head_dim 64 (Voxtral-Mini-3B-2507
 * "(1) AUDIO ENCODER": 20 heads x 64, MHA), over clips packed row after row,
 * on the tcgen05 tensor cores:
 *   qkv  bf16 [rows, 3d]: q | k | v, head h at columns h*64 of each third;
 *        every row must hold finite values (rows of neighbouring clips are
 *        read by a clip's last key tile and masked out)
 *   cu   device int32 [B+1]: clip b owns rows cu[b] .. cu[b+1]-1 (its keys);
 *        0 <= cu[0] <= cu[1] <= ... <= cu[B] <= rows. These are device values
 *        and are not checked: offsets outside this rule make the kernel write
 *        outside out.
 *   out  bf16 [rows, d] = concat_h softmax(q_h k_h^T / 8) v_h on rows < cu[B]
 * max_n >= max_b (cu[b+1] - cu[b]) (host value). d = 64 * n_heads.
 * status: device int (may be NULL) set to ENC_ERR_TIMEOUT if a bounded wait
 * inside the kernel runs out.
 */
ENC_API enc_status enc_attention_bf16(const void *qkv, void *out, const int32_t *cu, int32_t rows, int32_t B,
                                      int32_t max_n, int32_t n_heads, int *status, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* AUDIO_ENCODER_TOWER_ENC_KERNELS_H */
