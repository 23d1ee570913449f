// Bandwidth-bound row kernels of the encoder and the set-up kernels:
//   mel stage (mask + transpose to time-major), LayerNorm, final LayerNorm with
//   average pool and unpacking, tail-row zeroing, position table, weight repack.
#include "common.cuh"
#include "internal.h"

namespace enc {

// ------------------------------------------------------------------ mel stage
// One 32 x 32 (frames x channels) tile per block through shared memory so that
// both the clip-major read and the time-major write are coalesced.
template <typename T>
__global__ void mel_stage_kernel(const T* __restrict__ mel, const int* __restrict__ len, T* __restrict__ dst, int M,
                                 int Tfr, int Tp) {
  __shared__ float tile[32][33];
  const int b = blockIdx.z;
  const int tp0 = blockIdx.x * 32, c0 = blockIdx.y * 32;
  const int n = len[b];
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {   // i: channel within tile, tx: padded time
    const int c = c0 + i, tp = tp0 + threadIdx.x, t = tp - 1;
    float v = 0.f;
    if (c < M && t >= 0 && t < Tfr && t < n) v = to_float(mel[((size_t)b * M + c) * Tfr + t]);
    tile[i][threadIdx.x] = v;
  }
  __syncthreads();
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {   // i: padded time within tile, tx: channel
    const int tp = tp0 + i, c = c0 + threadIdx.x;
    if (tp < Tp && c < M) dst[((size_t)b * Tp + tp) * M + c] = from_float<T>(tile[threadIdx.x][i]);
  }
}

template <typename T>
cudaError_t launch_mel_stage(const T* mel, const int* len, T* dst, int B, int M, int Tfr, int Tp, cudaStream_t s) {
  dim3 grid((Tp + 31) / 32, (M + 31) / 32, B), block(32, 8);
  mel_stage_kernel<T><<<grid, block, 0, s>>>(mel, len, dst, M, Tfr, Tp);
  return cudaGetLastError();
}
template cudaError_t launch_mel_stage<bf16>(const bf16*, const int*, bf16*, int, int, int, int, cudaStream_t);
template cudaError_t launch_mel_stage<float>(const float*, const int*, float*, int, int, int, int, cudaStream_t);

// ------------------------------------------------------------------ LayerNorm
// One warp per row; lane l holds float4 columns l, l + 32, ... (NV of them).
template <int NV>
__device__ __forceinline__ void ln_row_stats(const float4 (&v)[NV], int d, float eps, float& mean, float& rstd) {
  float s = 0.f;
#pragma unroll
  for (int i = 0; i < NV; ++i) s += (v[i].x + v[i].y) + (v[i].z + v[i].w);
  mean = warp_sum(s) / d;
  float q = 0.f;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const float a = v[i].x - mean, b = v[i].y - mean, c = v[i].z - mean, e = v[i].w - mean;
    q += (a * a + b * b) + (c * c + e * e);
  }
  rstd = 1.0f / sqrtf(warp_sum(q) / d + eps);
}

template <typename OutT>
__device__ __forceinline__ void store4(OutT* p, float a, float b, float c, float d) {
  if constexpr (sizeof(OutT) == 2) {
    uint2 u;
    u.x = pack_bf16x2(a, b);
    u.y = pack_bf16x2(c, d);
    *reinterpret_cast<uint2*>(p) = u;
  } else {
    *reinterpret_cast<float4*>(p) = make_float4(a, b, c, d);
  }
}

// One warp per row. Blocks take the rows from the last to the first: the GEMM
// that updated x before this kernel (out-proj or fc2, tiles in ascending row
// order) wrote the last rows last, so those are the ones still in L2, and the
// rows this kernel writes last (the first ones) are those the next GEMM reads
// first.
template <typename OutT, int NV>
__global__ void layernorm_kernel(const float* __restrict__ x, const float* __restrict__ g,
                                 const float* __restrict__ bta, OutT* __restrict__ y, int rows, float eps) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = (gridDim.x - 1 - blockIdx.x) * (blockDim.x >> 5) + warp;
  if (row >= rows) return;
  constexpr int d = NV * 128;
  const float4* xr = reinterpret_cast<const float4*>(x + (size_t)row * d);
  float4 v[NV];
#pragma unroll
  for (int i = 0; i < NV; ++i) v[i] = xr[lane + 32 * i];
  float mean, rstd;
  ln_row_stats<NV>(v, d, eps, mean, rstd);
  const float4* g4 = reinterpret_cast<const float4*>(g);
  const float4* b4 = reinterpret_cast<const float4*>(bta);
  OutT* yr = y + (size_t)row * d;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const float4 gg = g4[lane + 32 * i], bb = b4[lane + 32 * i];
    store4<OutT>(yr + 4 * (lane + 32 * i), (v[i].x - mean) * rstd * gg.x + bb.x, (v[i].y - mean) * rstd * gg.y + bb.y,
                 (v[i].z - mean) * rstd * gg.z + bb.z, (v[i].w - mean) * rstd * gg.w + bb.w);
  }
}

#define ENC_NV_SWITCH(d, CALL)                                        \
  switch ((d) / 128) {                                                \
    case 1: CALL(1); break;   case 2: CALL(2); break;                 \
    case 3: CALL(3); break;   case 4: CALL(4); break;                 \
    case 5: CALL(5); break;   case 6: CALL(6); break;                 \
    case 7: CALL(7); break;   case 8: CALL(8); break;                 \
    case 9: CALL(9); break;   case 10: CALL(10); break;               \
    case 11: CALL(11); break; case 12: CALL(12); break;               \
    case 13: CALL(13); break; case 14: CALL(14); break;               \
    case 15: CALL(15); break; case 16: CALL(16); break;               \
    default: return cudaErrorInvalidValue;                            \
  }

template <typename OutT>
cudaError_t launch_layernorm(const float* x, const float* g, const float* b, OutT* y, int rows, int d, float eps,
                             cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  if (d % 128) return cudaErrorInvalidValue;
  const int warps = 8, grid = (rows + warps - 1) / warps;
#define ENC_LN_CALL(NV) layernorm_kernel<OutT, NV><<<grid, warps * 32, 0, s>>>(x, g, b, y, rows, eps)
  ENC_NV_SWITCH(d, ENC_LN_CALL)
#undef ENC_LN_CALL
  return cudaGetLastError();
}
template cudaError_t launch_layernorm<bf16>(const float*, const float*, const float*, bf16*, int, int, float,
                                            cudaStream_t);
template cudaError_t launch_layernorm<float>(const float*, const float*, const float*, float*, int, int, float,
                                             cudaStream_t);

// Final LayerNorm over packed rows, averaged over `pool` consecutive rows.
// One warp per output row (b, j), j < p_out.
template <typename OutT, int NV>
__global__ void final_ln_kernel(const float* __restrict__ x, const float* __restrict__ g,
                                const float* __restrict__ bta, const int* __restrict__ cu,
                                const int* __restrict__ cu_out, OutT* __restrict__ out, int B, int p_out, int pool,
                                int packed, float eps) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int orow = blockIdx.x * (blockDim.x >> 5) + warp;
  if (orow >= B * p_out) return;
  constexpr int d = NV * 128;
  const int b = orow / p_out, j = orow - b * p_out;
  const int n = cu[b + 1] - cu[b];
  const int valid = pool > 1 ? n / pool : n;
  if (j >= valid) {
    if (!packed) {
      OutT* yr = out + (size_t)orow * d;
#pragma unroll
      for (int i = 0; i < NV; ++i) store4<OutT>(yr + 4 * (lane + 32 * i), 0.f, 0.f, 0.f, 0.f);
    }
    return;
  }
  const float4* g4 = reinterpret_cast<const float4*>(g);
  const float4* b4 = reinterpret_cast<const float4*>(bta);
  float4 acc[NV];
#pragma unroll
  for (int i = 0; i < NV; ++i) acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int k = 0; k < pool; ++k) {
    const float4* xr = reinterpret_cast<const float4*>(x + (size_t)(cu[b] + j * pool + k) * d);
    float4 v[NV];
#pragma unroll
    for (int i = 0; i < NV; ++i) v[i] = xr[lane + 32 * i];
    float mean, rstd;
    ln_row_stats<NV>(v, d, eps, mean, rstd);
#pragma unroll
    for (int i = 0; i < NV; ++i) {
      const float4 gg = g4[lane + 32 * i], bb = b4[lane + 32 * i];
      acc[i].x += (v[i].x - mean) * rstd * gg.x + bb.x;
      acc[i].y += (v[i].y - mean) * rstd * gg.y + bb.y;
      acc[i].z += (v[i].z - mean) * rstd * gg.z + bb.z;
      acc[i].w += (v[i].w - mean) * rstd * gg.w + bb.w;
    }
  }
  const float inv = 1.0f / pool;
  const size_t dst = packed ? (size_t)(cu_out[b] + j) : (size_t)orow;
  OutT* yr = out + dst * d;
#pragma unroll
  for (int i = 0; i < NV; ++i)
    store4<OutT>(yr + 4 * (lane + 32 * i), acc[i].x * inv, acc[i].y * inv, acc[i].z * inv, acc[i].w * inv);
}

template <typename OutT>
cudaError_t launch_final_ln(const float* x, const float* g, const float* b, const int* cu, const int* cu_out,
                            OutT* out, int B, int p_out, int d, int pool, int packed, float eps, cudaStream_t s) {
  if (B * p_out <= 0) return cudaSuccess;
  const int warps = 8, grid = (B * p_out + warps - 1) / warps;
#define ENC_FLN_CALL(NV) \
  final_ln_kernel<OutT, NV><<<grid, warps * 32, 0, s>>>(x, g, b, cu, cu_out, out, B, p_out, pool, packed, eps)
  ENC_NV_SWITCH(d, ENC_FLN_CALL)
#undef ENC_FLN_CALL
  return cudaGetLastError();
}
template cudaError_t launch_final_ln<bf16>(const float*, const float*, const float*, const int*, const int*, bf16*,
                                           int, int, int, int, int, float, cudaStream_t);
template cudaError_t launch_final_ln<float>(const float*, const float*, const float*, const int*, const int*, float*,
                                            int, int, int, int, int, float, cudaStream_t);

// ------------------------------------------------------------ tail zeroing
template <typename OutT>
__global__ void zero_tail_rows_kernel(OutT* __restrict__ out, const int* __restrict__ cu_out, int p_out, int width) {
  const int b = blockIdx.y;
  const int valid = cu_out[b + 1] - cu_out[b];
  const size_t begin = ((size_t)b * p_out + valid) * width, end = ((size_t)b + 1) * p_out * width;
  for (size_t i = begin + (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < end; i += (size_t)gridDim.x * blockDim.x)
    out[i] = from_float<OutT>(0.f);
}

template <typename OutT>
cudaError_t launch_zero_tail_rows(OutT* out, const int* cu_out, int B, int p_out, int width, cudaStream_t s) {
  if (B <= 0) return cudaSuccess;
  dim3 grid(64, B);
  zero_tail_rows_kernel<OutT><<<grid, 256, 0, s>>>(out, cu_out, p_out, width);
  return cudaGetLastError();
}
template cudaError_t launch_zero_tail_rows<bf16>(bf16*, const int*, int, int, int, cudaStream_t);
template cudaError_t launch_zero_tail_rows<float>(float*, const int*, int, int, int, cudaStream_t);

// --------------------------------------------------------- position table
// pe[j, i] = sin(j * w_i), pe[j, d/2 + i] = cos(j * w_i), w_i = 10000^(-i / (d/2 - 1)),
// evaluated in double precision and stored as fp32.
__global__ void position_table_kernel(float* pe, int P, int d) {
  const int half = d / 2;
  const size_t total = (size_t)P * half;
  const double log_inc = log(10000.0) / (double)(half - 1);
  for (size_t k = (size_t)blockIdx.x * blockDim.x + threadIdx.x; k < total; k += (size_t)gridDim.x * blockDim.x) {
    const int j = (int)(k / half), i = (int)(k % half);
    const double ang = (double)j * exp(-log_inc * (double)i);
    pe[(size_t)j * d + i] = (float)sin(ang);
    pe[(size_t)j * d + half + i] = (float)cos(ang);
  }
}

cudaError_t launch_position_table(float* pe, int P, int d, cudaStream_t s) {
  position_table_kernel<<<256, 256, 0, s>>>(pe, P, d);
  return cudaGetLastError();
}

// ----------------------------------------------------------- weight repack
__device__ __forceinline__ float load_any(const void* p, bool is_bf16, size_t i) {
  return is_bf16 ? __bfloat162float(reinterpret_cast<const bf16*>(p)[i]) : reinterpret_cast<const float*>(p)[i];
}

__global__ void conv_repack_kernel(const void* src, bool src_bf16, void* dst, bool dst_bf16, int rows, int C,
                                   int cpad) {
  const size_t total = (size_t)rows * 3 * cpad;
  for (size_t k = (size_t)blockIdx.x * blockDim.x + threadIdx.x; k < total; k += (size_t)gridDim.x * blockDim.x) {
    const int o = (int)(k / (3 * (size_t)cpad));
    const int rem = (int)(k - (size_t)o * 3 * cpad);
    const int tap = rem / cpad, c = rem - tap * cpad;
    const float v = c < C ? load_any(src, src_bf16, ((size_t)o * C + c) * 3 + tap) : 0.f;
    if (dst_bf16) reinterpret_cast<bf16*>(dst)[k] = __float2bfloat16_rn(v);
    else reinterpret_cast<float*>(dst)[k] = v;
  }
}

cudaError_t launch_conv_repack(const void* src, bool src_bf16, void* dst, bool dst_bf16, int rows, int C, int cpad,
                               cudaStream_t s) {
  conv_repack_kernel<<<512, 256, 0, s>>>(src, src_bf16, dst, dst_bf16, rows, C, cpad);
  return cudaGetLastError();
}

__global__ void to_f32_kernel(const void* src, bool src_bf16, float* dst, int n, float fill) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x)
    dst[i] = src ? load_any(src, src_bf16, i) : fill;
}

cudaError_t launch_to_f32(const void* src, bool src_bf16, float* dst, int n, float fill, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  to_f32_kernel<<<(n + 255) / 256 < 1024 ? (n + 255) / 256 : 1024, 256, 0, s>>>(src, src_bf16, dst, n, fill);
  return cudaGetLastError();
}

}  // namespace enc
