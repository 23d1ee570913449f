// Launchers shared between the kernel files and the C-ABI layer (not exported).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <atomic>
#include <mutex>

#include "common.cuh"
#include "../../include/enc.h"

namespace enc {

// Geometry checks of enc_create, without the device check (host only).
enc_status validate_config(const enc_config* c);

// Per-device one-time set-up of a launcher (kernel attributes, occupancy
// queries), safe when several host threads launch at once: init() runs at most
// once per device ordinal at a time, under the mutex, and a thread that sees the
// device's bit set (acquire) also sees everything init() wrote before the bit
// was published (release). Device ordinals are taken modulo 64. A failed init()
// leaves the bit clear, so the next call tries again.
struct DeviceOnce {
  std::atomic<unsigned long long> done{0};
  std::mutex m;
  template <typename F>
  bool run(int dev, F&& init) {
    const unsigned long long bit = 1ull << (dev & 63);
    if (done.load(std::memory_order_acquire) & bit) return true;
    std::lock_guard<std::mutex> lock(m);
    if (done.load(std::memory_order_relaxed) & bit) return true;
    if (!init()) return false;
    done.fetch_or(bit, std::memory_order_release);
    return true;
  }
};
// enc_forward_static_scratch set-up (enc_create): the static workspace's device address.
void resolve_static_scratch(enc_handle* h);

// ----------------------------------------------------------- tcgen05 GEMM
// A_DFT (log-mel front end, tf32): A is read as overlapping windows of 416 fp32
// samples over rows of 160; k-block kb of a window part (kb / kb_seg: 0 and 1
// read the rounded-to-tf32 plane, 2 the remainder plane a_lo_rows rows further)
// is columns (w % 5) * 32 of row m + w / 5, w = kb % kb_seg.
// A_SPLIT3 (front end, tf32): k-block kb of part kb / kb_seg is columns
// (kb % kb_seg) * 32 of row m, in the tf32-part plane for parts 0 and 1 and in
// the remainder plane a_lo_rows rows further for part 2.
enum AMode : int { A_PLAIN = 0, A_CONV1 = 1, A_CONV2 = 2, A_DFT = 3, A_SPLIT3 = 4 };

struct GemmTcParams {
  int M, N;        // output rows / columns (N a multiple of 128)
  int num_kb;      // K / 64
  int a_mode;      // AMode
  int kb_seg;      // k-blocks per tap segment (conv modes)
  int tiles_n;     // filled by the launcher
  int num_tiles;   // filled by the launcher
  int tail;        // SM-pair kernel: the last `tail` tiles run as two 256 x 128 halves (launcher)
  int a_lo_rows;   // A_DFT: row offset of the remainder plane
  EpiParams epi;
  int* status;
};

int gemm_tile_n(int n);   // 256 when N % 256 == 0, else 128

// bf16 [rows, cols] output matrix as the target of TMA stores (32 x 64 boxes,
// 128-byte swizzle). Rows past `rows` are never written.
bool make_out_map(CUtensorMap* map, const void* out, uint64_t rows, uint64_t cols);

// 2-D bf16 tensor map with 128-byte swizzle and zero fill outside the tensor.
bool make_tma_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint64_t pitch_bytes,
                 uint32_t box_inner, uint32_t box_rows);

// 2-D fp32 tensor map (tf32 operands): 32-element (128-byte) boxes along the
// inner dimension, 128-byte swizzle, zero fill outside the tensor.
bool make_tma_2d_f32(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint64_t pitch_bytes,
                     uint32_t box_rows);

// Windowed DFT and power spectrum on the tensor cores (kind::tf32, 128 x 128
// tiles on one SM): acc = A W^T over p.num_kb k-blocks of 32 (A_DFT mode),
// W's rows interleaving the cos and sin basis functions of each bin, so that
// pw[r, k] = acc[r, 2k]^2 + acc[r, 2k+1]^2 for k < p.epi.ldo, stored split as
// p.epi.out[r, k] = pw rounded to tf32 and, p.epi.P1 rows further, the
// remainder pw - that (the next tf32 GEMM's operand planes).
cudaError_t launch_dft_power_tf32(const CUtensorMap& map_a, const CUtensorMap& map_b, GemmTcParams p, int sm_count,
                                  cudaStream_t stream);
// fp32 out[r, n] = acc for n < p.epi.ldo (row stride p.epi.ldo), tf32 MMAs, 128 x 128
// tiles on one SM; A in the A_SPLIT3 mode.
cudaError_t launch_gemm_tf32_f32out(const CUtensorMap& map_a, const CUtensorMap& map_b, GemmTcParams p,
                                    int sm_count, cudaStream_t stream);

// fp32 [rows, cols] residual matrix as the target of TMA reduce-adds (32 x 32 boxes,
// 128-byte swizzle). Rows past `rows` are never written.
bool make_resid_map(CUtensorMap* map, const float* resid, uint64_t rows, uint64_t cols);

// map_c: EPI_RESIDUAL: the residual map (required); EPI_STORE / EPI_CONV1: an
// optional bf16 output map from make_out_map (TMA-store epilogue when given).
cudaError_t launch_gemm_tc(const CUtensorMap& map_a, const CUtensorMap& map_b, GemmTcParams p, int sm_count,
                           cudaStream_t stream, const CUtensorMap* map_c = nullptr);

// --------------------------------------------------------- fp32 check path
// C = A[M, K] (row stride lda, rows may overlap) * W[N, K]^T (row stride ldw).
cudaError_t launch_sgemm(const float* A, int lda, const float* W, int ldw, int M, int N, int K, const EpiParams& e,
                         cudaStream_t stream);

// ------------------------------------------------------------- attention
// qkv [R, 3d] packed rows (clip b at rows cu[b] .. cu[b+1]); out [R, d].
// tcgen05 attention: Q (128-row boxes) and K/V (96-row boxes) views of one [rows, 3d] buffer.
struct QkvMaps {
  CUtensorMap q, kv;
};
bool make_qkv_maps(QkvMaps* maps, const void* qkv, int rows, int d);
cudaError_t launch_attention_tc(const QkvMaps& maps, bf16* out, const int* cu, int B, int max_n, int d, int H,
                                int* status, cudaStream_t stream);
cudaError_t launch_attention_f32(const float* qkv, float* out, const int* cu, int B, int max_n, int d, int H,
                                 cudaStream_t stream);

// ------------------------------------------------------------- row kernels
// mel [B, M, T] (clip-major) -> time-major rows [B * Tp, M]: row b*Tp + tp holds
// frame tp - 1 (zero for tp == 0, tp > T and frames >= len[b]).
template <typename T>
cudaError_t launch_mel_stage(const T* mel, const int* len, T* dst, int B, int M, int Tfr, int Tp, cudaStream_t s);

// y = LN(x) * g + b per row; x fp32 [rows, d].
template <typename OutT>
cudaError_t launch_layernorm(const float* x, const float* g, const float* b, OutT* y, int rows, int d, float eps,
                             cudaStream_t s);

// Final LN (+ average pool over `pool` consecutive rows) of packed rows.
// packed == 0: out is [B, p_out, d] with zero rows past each clip's valid count.
// packed == 1: out holds only the valid rows, at cu_out[b] + j.
template <typename OutT>
cudaError_t launch_final_ln(const float* x, const float* g, const float* b, const int* cu, const int* cu_out,
                            OutT* out, int B, int p_out, int d, int pool, int packed, float eps, cudaStream_t s);

// Zero rows j >= cu_out[b+1] - cu_out[b] of out [B, p_out, width].
template <typename OutT>
cudaError_t launch_zero_tail_rows(OutT* out, const int* cu_out, int B, int p_out, int width, cudaStream_t s);

// -------------------------------------------------- encoder handle geometry
// Sizes of one clip's input and output blocks for an encoder handle (for the
// embeddings cache, which sits beside the handle). Returns false for a null handle.
struct HandleGeometry {
  int n_mels, frames, max_batch, device;
  size_t mel_bytes;   // one clip of enc_forward's mel input: n_mels x frames elements
  size_t out_bytes;   // one clip of its output: P_out x d_out elements
};
bool handle_geometry(const enc_handle* h, HandleGeometry* g);

// ------------------------------------------------------------ set-up work
cudaError_t launch_position_table(float* pe, int P, int d, cudaStream_t s);
// src [rows, C, 3] (dtype of src) -> dst [rows, 3, cpad] (dtype of dst), zero padded.
cudaError_t launch_conv_repack(const void* src, bool src_bf16, void* dst, bool dst_bf16, int rows, int C, int cpad,
                               cudaStream_t s);
// n values of src (bf16 or fp32; nullptr -> fill) to fp32.
cudaError_t launch_to_f32(const void* src, bool src_bf16, float* dst, int n, float fill, cudaStream_t s);

}  // namespace enc
