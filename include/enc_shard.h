/*
 * enc_shard.h -- splitting a batch of clips over data-parallel ranks.
 *
 * The encoder's clips are independent units: attention runs within a clip
 * (Qwen2-Audio-7B-Instruct, "(1) AUDIO ENCODER": one bidirectional pass per
 * 30 s window) and nothing else crosses clips. A batch therefore shards over
 * ranks -- one process per GPU, each with its own encoder handle and a full
 * copy of the weights -- with no collective in the forward pass.
 *
 * With ragged lengths the clips cost different amounts. A clip of `len` valid
 * frames has n = ceil(len / 2) positions and costs, in multiply-add = 2 FLOPs,
 *
 *   conv1  2 * 2n * d * 3 * n_mels
 *   conv2  2 * n * d * 3 * d
 *   L *  ( 6 n d^2            QKV
 *        + 4 d * sum_s n_s^2  attention over the clip's segments: one segment of n
 *                             positions, or chunks of attn_chunk positions
 *        + 2 n d^2            out-proj
 *        + 4 n d F )          fc1 + fc2
 *   proj   2 * n_out * (d * proj_hidden + proj_hidden * proj_out), n_out = floor(n / pool_step)
 *
 * i.e. a term linear in n (the GEMMs, which run over the packed valid rows of
 * the batch) plus a term quadratic in n (attention). The planner balances
 * these costs with the longest-processing-time rule: clips sorted by cost,
 * largest first (equal costs by clip index), each placed on the rank with the
 * smallest total so far among those that still have room (equal totals: the
 * lowest rank). Deterministic: every rank that calls it with the same
 * arguments gets the same plan, so no rank needs to send the plan to another.
 *
 * Host-only calls: no device access, no CUDA context needed.
 */
#ifndef AUDIO_ENCODER_TOWER_ENC_SHARD_H
#define AUDIO_ENCODER_TOWER_ENC_SHARD_H

#include "enc.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * Algorithmic FLOPs of one clip of `length` valid frames under cfg (the
 * formula above). cfg is validated as enc_create validates it (without the
 * device check): ENC_ERR_INVALID_ARG / ENC_ERR_UNSUPPORTED as there;
 * ENC_ERR_INVALID_ARG for length outside [1, cfg->max_frames] or a NULL flops.
 */
ENC_API enc_status enc_clip_flops(const enc_config *cfg, int32_t length, double *flops);

/*
 * Split B clips over `world` ranks that each run batches of up to
 * cfg->max_batch clips.
 *   lengths     HOST [B] valid frames per clip in [1, cfg->max_frames], or NULL (all max_frames)
 *   B, world    1 <= B <= world * cfg->max_batch, world >= 1
 *   rank_of     HOST [B] out: the rank of clip b
 *   index_of    HOST [B] out (may be NULL): clip b's position in its rank's
 *               batch; a rank's clips keep their order in the input
 *   rank_count  HOST [world] out (may be NULL): clips per rank
 *   rank_flops  HOST [world] out (may be NULL): total FLOPs per rank
 * Errors (nothing written then): those of enc_clip_flops, ENC_ERR_INVALID_ARG
 * for a NULL rank_of, world < 1 or B outside the range above.
 */
ENC_API enc_status enc_shard_plan(const enc_config *cfg, const int32_t *lengths, int32_t B, int32_t world,
                                  int32_t *rank_of, int32_t *index_of, int32_t *rank_count, double *rank_flops);

#ifdef __cplusplus
}
#endif

#endif /* AUDIO_ENCODER_TOWER_ENC_SHARD_H */
