/*
 * enc.h -- C ABI of the B200 (sm_100a) Whisper-style audio encoder tower.
 *
 * The library computes one forward pass of the bidirectional audio encoder
 * that audio LLMs put in front of their decoder:
 *
 *   mel [B, n_mels, T]
 *     -> conv1 (n_mels -> d, kernel 3, padding 1) + GELU
 *     -> conv2 (d -> d, kernel 3, stride 2, padding 1) + GELU   (T frames -> ceil(T/2) positions)
 *     -> + sinusoidal position table
 *     -> n_layers pre-LN blocks: x += Wo.MHA(LN1(x)) ; x += W2.GELU(W1.LN2(x))
 *        (non-causal multi-head attention, head_dim 64, key-padding mask per clip)
 *     -> final LayerNorm
 *     -> optional average pool by 2 along time
 *     -> optional 2-layer GELU projector into an LLM's width
 *
 * Defining passages (model pages):
 *   - Qwen2-Audio-7B-Instruct, "(1) AUDIO ENCODER": the tower is the Whisper-large
 *     encoder (d_model 1280, 32 layers, 20 heads, FFN 5120, gelu, 128 mel bins,
 *     1500 positions per 30 s window), a single bidirectional pass with no KV cache.
 *   - Voxtral-Mini-3B-2507, "(1) AUDIO ENCODER" / "Preprocessor" / "PROJECTOR":
 *     head_dim 64 with as many KV heads as heads; 3000 mel frames per 30 s
 *     (16 kHz, hop 160); a 2-layer gelu MLP from 1280 to the 3072-wide LLM.
 *   - MiniCPM-o-2.6, "(2) AUDIO": a 24-layer, d_model 1024, 16-head encoder whose
 *     audio_pool_step 2 halves the token rate (about 750 tokens per 30 s).
 *   - The same pages' "REQUIRED KERNEL CLASS": the encoder runs on its own
 *     schedule, separate from the decoder -- hence the caller's cudaStream_t.
 *
 * Conventions
 *   - All tensors are row-major, PyTorch layouts. Device pointers unless noted.
 *   - Element type of every weight, of mel and of out is cfg.dtype:
 *     ENC_DTYPE_BF16 (tensor-core path: bf16 operands, fp32 accumulation, fp32
 *     residual stream) or ENC_DTYPE_FP32 (check mode: fp32 CUDA-core kernels,
 *     no tensor cores).
 *   - Nothing in this library traps, asserts or aborts. Host-detectable errors
 *     are returned before any work is enqueued; device-side errors (a bounded
 *     wait that ran out) set a status word read by enc_get_status.
 */
#ifndef AUDIO_ENCODER_TOWER_ENC_H
#define AUDIO_ENCODER_TOWER_ENC_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ENC_API __attribute__((visibility("default")))
#else
#define ENC_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same declaration as the CUDA runtime's, so this header needs no CUDA include. */
struct CUstream_st;
typedef struct CUstream_st *cudaStream_t;

typedef enum enc_status {
  ENC_OK = 0,
  ENC_ERR_INVALID_ARG = 1,   /* null pointer, size out of range, bad length */
  ENC_ERR_UNSUPPORTED = 2,   /* geometry or device not supported (needs sm_100) */
  ENC_ERR_OOM = 3,           /* device or pinned allocation failed */
  ENC_ERR_CUDA = 4,          /* a CUDA runtime call or a kernel launch failed */
  ENC_ERR_TIMEOUT = 5,       /* a bounded device-side wait ran out (status word) */
  ENC_ERR_DEVICE_CHECK = 6   /* enc_check_guards: a guard region around a workspace buffer was
                                written (no kernel sets it in the status word: the host
                                validates every input the kernels index by) */
} enc_status;

/*
 * enc_config.flags: ENC_FLAG_GUARD surrounds every workspace buffer of the
 * handle (time-major mel, conv1 output, residual stream, LN output, QKV,
 * attention output, FFN hidden, projector buffers, clip offsets, status word)
 * with 256 KiB guard regions filled with the byte 0xA5, so
 * that enc_check_guards can detect a kernel that wrote outside its buffer.
 * It costs 512 KiB of device memory per buffer and nothing per forward.
 */
#define ENC_FLAG_GUARD 1u

typedef enum enc_dtype {
  ENC_DTYPE_BF16 = 0,
  ENC_DTYPE_FP32 = 1
} enc_dtype;

/* Geometry of the tower; field names follow the Hugging Face audio_config. */
typedef struct enc_config {
  int32_t n_mels;        /* num_mel_bins: 80 or 128 (any multiple of 8, <= 256) */
  int32_t d_model;       /* multiple of 128, <= 2048 */
  int32_t n_layers;      /* encoder_layers, >= 0 */
  int32_t n_heads;       /* encoder_attention_heads; n_heads * head_dim == d_model */
  int32_t head_dim;      /* must be 64 */
  int32_t ffn_dim;       /* encoder_ffn_dim, multiple of 128 */
  int32_t max_frames;    /* T: mel frames of every clip, zero padded (3000 for 30 s) */
  int32_t max_batch;     /* largest B that enc_forward will be given */
  int32_t pool_step;     /* 1 (none), 2 (audio_pool_step: 25 Hz) or 4 (12.5 Hz) */
  int32_t proj_hidden;   /* 0 = no projector, else hidden width (multiple of 128) */
  int32_t proj_out;      /* projector output width (multiple of 128) */
  float ln_eps;          /* LayerNorm epsilon (1e-5) */
  int32_t dtype;         /* enc_dtype */
  uint32_t flags;        /* 0, or ENC_FLAG_GUARD; other bits are reserved and rejected */
  int32_t attn_chunk;    /* 0: full bidirectional attention within each clip; > 0: block-local
                            attention, position i of a clip attending only within its chunk of
                            attn_chunk positions (MiniCPM-o-2.6, "(2) AUDIO": audio_chunk_length
                            1.0 s = 50 positions); max_batch * ceil(P / attn_chunk) <= 65535 */
} enc_config;

/*
 * Weight device pointers in PyTorch layouts, element type cfg.dtype.
 * Per-layer entries are HOST arrays of n_layers device pointers.
 * Any bias / LayerNorm beta may be NULL (read as zeros); a NULL gamma reads as ones.
 * k_b is accepted and ignored (NULL is the usual value): the key projection runs
 * without a bias, because a key bias adds q.k_b to every score of a query row,
 * a per-row constant that softmax cancels exactly, so it cannot change the output.
 */
typedef struct enc_weights {
  const void *conv1_w;   /* [d, n_mels, 3] */
  const void *conv1_b;   /* [d] */
  const void *conv2_w;   /* [d, d, 3] */
  const void *conv2_b;   /* [d] */
  const void *const *ln1_g, *const *ln1_b;   /* [d] each */
  const void *const *q_w, *const *q_b;       /* [d, d], [d] */
  const void *const *k_w, *const *k_b;       /* [d, d], NULL */
  const void *const *v_w, *const *v_b;       /* [d, d], [d] */
  const void *const *o_w, *const *o_b;       /* [d, d], [d] */
  const void *const *ln2_g, *const *ln2_b;   /* [d] each */
  const void *const *fc1_w, *const *fc1_b;   /* [F, d], [F] */
  const void *const *fc2_w, *const *fc2_b;   /* [d, F], [d] */
  const void *lnpost_g, *lnpost_b;           /* [d] */
  const void *proj1_w, *proj1_b;             /* [proj_hidden, d], [proj_hidden] */
  const void *proj2_w, *proj2_b;             /* [proj_out, proj_hidden], [proj_out] */
} enc_weights;

typedef struct enc_handle enc_handle;

/*
 * Create an encoder on the current CUDA device. Synchronous.
 * Passage: Qwen2-Audio-7B-Instruct, "(1) AUDIO ENCODER" (the Whisper-large geometry
 * and weight shapes, e.g. q_proj [1280, 1280]); MiniCPM-o-2.6, "(2) AUDIO" (the
 * medium-sized geometry, audio_pool_step); Voxtral-Mini-3B-2507, "PROJECTOR".
 * Validates cfg (ENC_ERR_UNSUPPORTED for geometry or a device other than sm_100),
 * copies and repacks the weights into library-owned device memory (fused QKV,
 * tap-major conv kernels, fp32 biases, position table) and allocates the
 * workspace for cfg.max_batch clips. The caller may free its weights on return.
 * On failure *out is NULL and nothing stays allocated.
 */
ENC_API enc_status enc_create(const enc_config *cfg, const enc_weights *w, enc_handle **out);

/*
 * Enqueue one forward pass on `stream`. Asynchronous: returns once enqueued.
 * Passage: Qwen2-Audio-7B-Instruct, "(1) AUDIO ENCODER" (one bidirectional pass,
 * 30 s -> 1500 positions); Voxtral-Mini-3B-2507, "Preprocessor" (3000 mel frames
 * per 30 s at 16 kHz, hop 160); "REQUIRED KERNEL CLASS" (the encoder on a schedule
 * of its own, separate from the decoder: the caller's stream).
 *   mel      device [B, n_mels, T], cfg.dtype. Frames t >= lengths[b] are treated
 *            as silence (zero) whatever they hold.
 *   lengths  HOST [B] valid frames per clip, each in [1, T]; NULL means all T.
 *            Read during the call; the caller may reuse it on return.
 *   B        1 <= B <= cfg.max_batch
 *   out      device [B, P_out, d_out], cfg.dtype, where
 *              P = ceil(T/2), P_out = floor(P / pool_step),
 *              d_out = proj_out if a projector is configured, else d_model.
 *            Clip b carries n_b = ceil(lengths[b]/2) positions
 *            (floor(n_b / pool_step) after pooling: only complete windows of
 *            valid positions); its rows past that count are written as exact zeros.
 * mel and out must stay valid until the stream work has completed. One forward
 * may be in flight per handle at a time (the workspace is shared); handles are
 * independent of each other. Host-detectable errors return before enqueueing.
 */
ENC_API enc_status enc_forward(enc_handle *h, const void *mel, const int32_t *lengths, int32_t B,
                       void *out, cudaStream_t stream);

/*
 * Output geometry for a batch, computed on the host (no device work).
 * Passage: Voxtral-Mini-3B-2507, "Preprocessor" and Qwen2-Audio-7B-Instruct,
 * "(1) AUDIO ENCODER" (3000 frames -> 1500 positions); MiniCPM-o-2.6, "(2) AUDIO"
 * (pool step 2: about 750 tokens per 30 s).
 *   n_out  HOST [B] (may be NULL): valid output rows per clip
 *   p_out  (may be NULL): rows per clip in `out` (the row stride is p_out * d_out)
 *   d_out  (may be NULL): width of an output row
 */
ENC_API enc_status enc_output_positions(const enc_handle *h, int32_t B, const int32_t *lengths,
                                int32_t *n_out, int32_t *p_out, int32_t *d_out);

/*
 * Wait for `stream`, then read and clear the device status word of the handle.
 * Returns ENC_ERR_TIMEOUT if a bounded device-side wait ran out since the last
 * call. (No passage: the pages describe the encoder's arithmetic, not how a
 * library reports device-side errors.)
 */
ENC_API enc_status enc_get_status(enc_handle *h, cudaStream_t stream);

/*
 * Self-test of the device-side failure detection (no passage: a property of this
 * library), without a fault: one CTA of
 * two warps on `stream`. Warp 0 waits on an mbarrier phase that nothing
 * completes, with the bounded wait of the GEMM and attention kernels, gives up
 * after limit_ns, records ENC_ERR_TIMEOUT in the handle's status word and
 * raises the CTA's abort flag; warp 1, waiting on a second such phase with a
 * 2 s limit, leaves at its next check of that flag (the path every other warp
 * of a failing CTA takes). Nothing traps and the context stays usable: the
 * next enc_get_status returns ENC_ERR_TIMEOUT and clears the word, and later
 * forwards run normally. Asynchronous.
 *   limit_ns  1,000 .. 100,000,000 (1 us .. 100 ms), else ENC_ERR_INVALID_ARG
 */
ENC_API enc_status enc_selftest_timeout(enc_handle *h, int64_t limit_ns, cudaStream_t stream);

/* Free everything the handle owns. Synchronises the device first. NULL is a no-op.
 * (Library resource management; no passage.) */
ENC_API void enc_destroy(enc_handle *h);

/* Static description of a status code (no passage). */
ENC_API const char *enc_status_string(enc_status s);

/* Library-owned device bytes: repacked weights and workspace (for reporting; no passage). */

/*
 * Guard-band check of a handle created with ENC_FLAG_GUARD (no passage: a
 * race and overrun detector of this library). Synchronises the device, copies
 * every guard region to the host and compares it with the fill byte: a plain
 * device-to-host read, nothing on the device can fault. Returns ENC_OK when
 * every guard is intact, ENC_ERR_DEVICE_CHECK when one is not (what, if not
 * NULL, receives a description such as "qkv: byte +4096 past the end of the
 * buffer changed", truncated to what_len), ENC_ERR_INVALID_ARG for a handle
 * without guards. The static-scratch forward's workspace has no guards.
 */
ENC_API enc_status enc_check_guards(enc_handle *h, char *what, size_t what_len);

/*
 * Self-test of enc_check_guards without a kernel: changes one byte of a guard
 * region of workspace buffer `buffer` (allocation order, 0 = time-major mel)
 * with a host-side cudaMemset (offset < 0: byte -offset before the buffer;
 * offset > 0: byte offset - 1 past its end, |offset| <= 262144), checks that
 * enc_check_guards reports that buffer, restores the byte and checks again.
 * Returns ENC_OK when both checks behaved, ENC_ERR_CUDA when they did not.
 */
ENC_API enc_status enc_guard_selftest(enc_handle *h, int32_t buffer, int64_t offset);
ENC_API size_t enc_device_bytes(const enc_handle *h);

/*
 * enc_forward without any device allocation, for callers that cannot call
 * cudaMalloc once they are running -- for example a serving process whose
 * device memory is handed out up front by its own pool allocator, where a new
 * cudaMalloc would fail or break the pool. (The model pages have no
 * counterpart of this call; it is a property of this library.)
 *
 * Same arguments, output and errors as enc_forward, with the handle's weights.
 * The per-batch workspace (time-major mel, conv1 output, residual stream, LN,
 * QKV, attention and FFN buffers, projector buffers, clip offsets) is carved
 * out of one file-scope static device array of 64 MiB (67,108,864 bytes). The
 * CUDA runtime reserves it on a device when the library's module holding it is
 * loaded there, and keeps it until the process exits.
 *   - Set-up: enc_create looks up the array's device address on its device
 *     (cudaGetSymbolAddress, with that device current); that lookup loads the
 *     module, so the 64 MiB are reserved inside enc_create. This call itself
 *     allocates nothing, its first call included (no cudaMalloc, no cudaFree, no
 *     allocating library routine). If the lookup failed in enc_create (too little
 *     device memory left for the array), enc_create still succeeds and this call
 *     returns ENC_ERR_OOM (ENC_ERR_CUDA for another runtime error).
 *   - Capacity: a batch whose workspace exceeds 64 MiB returns
 *     ENC_ERR_INVALID_ARG before anything is enqueued. One 30 s clip of the
 *     Whisper-large encoder (about 51 MB of workspace) fits; two do not.
 *   - Sharing: every call on a device uses the same array, which keeps the
 *     previous call's contents; the call clears what it reads as zero. Calls
 *     whose GPU work overlaps (other streams, other handles, other threads)
 *     race on the array: order them on one stream or synchronise between them.
 *   - Profiling (enc_profile_enable) does not record this call's kernels.
 */
ENC_API enc_status enc_forward_static_scratch(enc_handle *h, const void *mel, const int32_t *lengths, int32_t B,
                                              void *out, cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* AUDIO_ENCODER_TOWER_ENC_H */
