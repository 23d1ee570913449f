/*
 * enc_cache.h -- an embeddings cache in front of enc_forward: encoder outputs
 * kept on the device, looked up by a caller-chosen 64-bit key per clip
 * (the "Multimodal Embeddings Cache" beside the "Multimodal Encoder Side
 * Stream" of the REQUIRED KERNEL CLASS section the pages repeat).
 *
 * A hit copies the cached [P_out, d_out] output block of the clip into `out`;
 * the misses of a call are gathered into one batch, run through enc_forward,
 * written to `out` and inserted (the least recently used entry is replaced
 * when the cache is full). The encoder's result for a clip does not depend on
 * the other clips of its batch (bit for bit), so a hit returns exactly what a
 * fresh forward would.
 *
 * The key must identify the clip's input: its mel features and its length.
 * enc_cache_content_keys derives such a key from the clip's content on the
 * device; a caller may use its own keys instead (for example a hash computed
 * where the audio arrives). enc_forward_cached does not read the mel to check
 * a key: two different clips under one key share one output.
 *
 * Same conventions as enc.h: device pointers, nothing traps, host-detectable
 * errors return before anything is enqueued. All work is enqueued on `stream`;
 * one call in flight per cache (and per encoder handle), on one stream.
 */
#ifndef AUDIO_ENCODER_TOWER_ENC_CACHE_H
#define AUDIO_ENCODER_TOWER_ENC_CACHE_H

#include "enc.h"

#ifdef __cplusplus
extern "C" {
#endif

typedef struct enc_cache enc_cache;

/*
 * A cache of `capacity` clip outputs for encoder handle h (which must outlive
 * it), plus staging for h's max_batch clips. Device memory:
 * (capacity + max_batch) output blocks + max_batch mel blocks, and 12 bytes per
 * clip of max_batch for enc_cache_content_keys.
 * Returns ENC_ERR_INVALID_ARG for a null handle or capacity < 1, ENC_ERR_OOM
 * when an allocation fails (nothing is left allocated then).
 */
ENC_API enc_status enc_cache_create(enc_handle *h, int32_t capacity, enc_cache **out);

/*
 * out[b] = encoder output of clip b, b < B, as enc_forward would write it:
 *   mel, lengths, B, out   as for enc_forward (lengths may be NULL: all T)
 *   keys                   HOST [B]: the clips' keys
 *   hits                   HOST [B] or NULL: set to 1 where the output came
 *                          from the cache, 0 where it was computed
 * A key repeated within one call is computed once.
 */
ENC_API enc_status enc_forward_cached(enc_cache *c, const void *mel, const int32_t *lengths, const uint64_t *keys,
                                      int32_t B, void *out, int32_t *hits, cudaStream_t stream);

/*
 * Content keys: keys[b] (HOST [B]) is a 64-bit hash of clip b's length and of
 * its mel values at frames t < lengths[b], the only frames the encoder reads
 * (frames past the length change neither the output nor the key). With mix()
 * the SplitMix64 output finaliser and g = 0x9E3779B97F4A7C15, element (c, t)
 * of the clip (mel channel c, frame t < lengths[b], T = frames) contributes
 * mix(((c * T + t) << 32 | its 16- or 32-bit pattern) + g); the contributions
 * are summed modulo 2^64 (independent of thread order) into s, and
 * keys[b] = mix(s ^ mix(lengths[b] * g)). Two clips with the same length and
 * the same valid frames get the same key; any other pair collides with a
 * probability of about 2^-64. The hash kernel is enqueued on `stream`, which
 * the call then waits for (the keys are host values). mel, lengths, B as for
 * enc_forward; reads about one byte of HBM per mel byte.
 */
ENC_API enc_status enc_cache_content_keys(enc_cache *c, const void *mel, const int32_t *lengths, int32_t B,
                                          uint64_t *keys, cudaStream_t stream);

/* Number of cached clips (host bookkeeping; no device access). */
ENC_API int32_t enc_cache_size(const enc_cache *c);

/* Frees the cache's device memory (NULL is ignored). The encoder handle stays. */
ENC_API void enc_cache_destroy(enc_cache *c);

#ifdef __cplusplus
}
#endif

#endif /* AUDIO_ENCODER_TOWER_ENC_CACHE_H */
