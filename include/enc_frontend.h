/*
 * enc_frontend.h -- log-mel front end: 30 s of 16 kHz audio -> the encoder's
 * [n_mels, 3000] input features, on the GPU.
 *
 * The pages fix the geometry: a WhisperFeatureExtractor with 30 s chunks,
 * 480,000 samples at 16 kHz, hop 160, 3000 frames, 128 features
 * (Voxtral-Mini-3B-2507, "Preprocessor"); 80 features for the medium tower
 * (MiniCPM-o-2.6, "(2) AUDIO"). The rest follows the Whisper feature
 * extractor:
 *   - frames of 400 samples centred on samples 0, 160, ..., the clip
 *     reflected at both ends (edge sample not repeated), periodic Hann window
 *   - power of the 201 one-sided DFT bins; 3000 frames (the 3001st dropped)
 *   - Slaney mel filterbank (0 Hz .. 8 kHz, unit-area triangles)
 *   - log10(max(mel, 1e-10)), raised to at least (clip maximum - 8),
 *     then (x + 4) / 4
 * The DFT runs as a GEMM of the overlapping frames against a windowed cos /
 * sin basis on the tensor cores (kind::tf32), with every fp32 operand split
 * into a tf32 part and a tf32 remainder and the three products that matter
 * accumulated in fp32 (about 2^-22 relative to the fp32 product), the power
 * spectrum taken in the same kernel. The filterbank product runs the same way
 * on the tensor cores; log and normalisation run in fp32 on CUDA cores.
 *
 * Same conventions as enc.h: device pointers, row-major, nothing traps;
 * host-detectable errors return before any launch.
 */
#ifndef AUDIO_ENCODER_TOWER_ENC_FRONTEND_H
#define AUDIO_ENCODER_TOWER_ENC_FRONTEND_H

#include "enc.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct enc_frontend enc_frontend;

/*
 * Builds the windowed DFT basis and the filterbank on the current device and
 * allocates the workspace for up to max_batch clips (about 11 MB per clip).
 * n_mels: 80 or 128. Returns ENC_ERR_INVALID_ARG for other values or
 * max_batch < 1, ENC_ERR_UNSUPPORTED off sm_100, ENC_ERR_OOM / ENC_ERR_CUDA on
 * allocation or copy failure (nothing is left allocated then). *out owns the
 * device memory until enc_frontend_destroy.
 */
ENC_API enc_status enc_frontend_create(int32_t n_mels, int32_t max_batch, enc_frontend **out);

/*
 * mel[b] = log-mel features of audio[b], for b < B:
 *   audio  fp32 device [B, 480000]: each clip already padded or cut to 30 s
 *   mel    device [B, n_mels, 3000] in out_dtype (ENC_DTYPE_BF16 or
 *          ENC_DTYPE_FP32): the layout enc_forward takes
 * Enqueued on `stream`; the caller keeps audio and mel alive until the stream
 * reaches this work. One call in flight per handle (shared workspace).
 * Returns ENC_ERR_INVALID_ARG for null pointers, B outside [1, max_batch] or
 * an unknown dtype, before anything is enqueued.
 */
ENC_API enc_status enc_frontend_log_mel(enc_frontend *h, const float *audio, int32_t B, void *mel,
                                        enc_dtype out_dtype, cudaStream_t stream);

/* Frees the handle and its device memory (NULL is ignored). */
ENC_API void enc_frontend_destroy(enc_frontend *h);

#ifdef __cplusplus
}
#endif

#endif /* AUDIO_ENCODER_TOWER_ENC_FRONTEND_H */
