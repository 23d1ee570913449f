// Log-mel front end on the GPU: 30 s of 16 kHz audio ->
// the encoder's [n_mels, 3000] input features. Geometry from the pages
// (Voxtral-Mini-3B-2507, "Preprocessor": WhisperFeatureExtractor, 480,000
// samples, hop 160, 3000 frames, 128 features; MiniCPM-o-2.6, "(2) AUDIO": 80);
// window, filterbank and compression as the Whisper feature extractor
// (include/enc_frontend.h lists them).
//
// Steps for B clips:
//   1. pad_kernel: each clip reflected by 200 samples at both ends into rows of
//      a buffer whose clip stride is 3003 frames x 160 samples, so frame f of
//      clip b starts at sample (b * 3003 + f) * 160 for every clip. Each
//      sample a is stored twice: a_hi = a rounded to tf32 in one plane, a_lo =
//      a - a_hi (exact in fp32) in a second plane.
//   2. tensor cores (kind::tf32): the windowed DFT of every frame and its power
//      spectrum, P [B * 3003, 204] = |X_k|^2. The product of the frames with the
//      windowed cos / sin basis runs as one GEMM over K = 3 x 416 of
//      [a_hi | a_hi | a_lo] and [w_hi | w_lo | w_hi]: a_hi w_hi + a_hi w_lo +
//      a_lo w_hi is the fp32 product to about 2^-22 relative (the a_lo w_lo term
//      and the tf32 truncation of the remainders are what it leaves out), an
//      error-compensated split of the fp32 operands into tf32 pairs. The basis
//      interleaves cos and sin of each bin, so the epilogue finds both parts of
//      a bin in adjacent accumulator columns.
//      The power spectrum is stored split the same way (tf32 part and
//      remainder planes, 224 bins, zero past 200).
//   3. tensor cores again: power x filterbank^T -> mel [B * 3003, n_mels] fp32,
//      the same three-product split over K = 3 x 224.
//   4. log_max_kernel: log10(max(mel, 1e-10)) in place over the 3000 frames
//      kept, and the clip's maximum
//   5. finish_kernel: max(x, clip max - 8), (x + 4) / 4, transposed to
//      [B, n_mels, 3000]
// Rows 3000..3002 of every clip are computed and dropped (they keep the frame
// stride uniform across clips).
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <new>
#include <vector>

#include "../../include/enc_frontend.h"
#include "common.cuh"
#include "internal.h"

namespace enc {
namespace {

constexpr int kSamples = 480000, kFft = 400, kHop = 160, kFrames = 3000;
constexpr int kBins = kFft / 2 + 1;               // 201
constexpr int kFramesPad = kSamples / kHop + 3;   // 3003 frame rows per clip
constexpr int kClipStride = kFramesPad * kHop;    // 480,480 padded samples per clip
constexpr int kPowCols = 224;                     // 201 bins + 23 zero columns: 7 k-blocks of 32
constexpr int kFbK = 3 * kPowCols;                // [hi | lo | hi] parts of the filterbank
constexpr int kMelRows = 128;                     // filterbank rows, n_mels zero padded
constexpr int kWin = 416;                         // 400-sample window padded to 13 k-blocks of 32
constexpr int kKb = kWin / 32;                    // 13
constexpr int kBasisK = 3 * kWin;                 // [hi | lo | hi] parts
constexpr int kBasisN = 512;                      // 2 x 201 interleaved cos / sin rows, zero padded
constexpr int kSlack = 4 * kHop;                  // read past the last clip by its dropped frame rows
static_assert((kFramesPad - 1 + 2) * kHop + kHop <= kClipStride + kSlack, "slack covers the last windows");
static_assert(kHop % 32 == 0 && kWin <= 3 * kHop, "a window is 13 k-blocks over 3 rows of 160 samples");

// a rounded to the nearest tf32 (10 fraction bits, ties to even); low 13 bits zero
__host__ __device__ inline float round_tf32(float a) {
  uint32_t u;
  memcpy(&u, &a, 4);
  u = (u + 0xFFFu + ((u >> 13) & 1u)) & 0xFFFFE000u;
  float r;
  memcpy(&r, &u, 4);
  return r;
}

// plane 0: the reflect-padded clips rounded to tf32; plane 1 (plane samples on): the remainders
__global__ void pad_kernel(const float* __restrict__ audio, float* __restrict__ padded, int B, size_t plane) {
  const size_t total = static_cast<size_t>(B) * kClipStride;
  for (size_t i = blockIdx.x * static_cast<size_t>(blockDim.x) + threadIdx.x; i < total;
       i += static_cast<size_t>(gridDim.x) * blockDim.x) {
    const int b = static_cast<int>(i / kClipStride);
    int s = static_cast<int>(i - static_cast<size_t>(b) * kClipStride) - kFft / 2;
    if (s < 0) s = -s;                                    // reflect, edge sample not repeated
    if (s >= kSamples) s = 2 * (kSamples - 1) - s;
    const float a = audio[static_cast<size_t>(b) * kSamples + s];
    const float hi = round_tf32(a);
    padded[i] = hi;
    padded[plane + i] = a - hi;
  }
}

// fp32 keys whose unsigned order is the float order (for atomicMax)
__device__ __forceinline__ unsigned order_key(float x) {
  const unsigned u = __float_as_uint(x);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float from_order_key(unsigned k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
}

// grid (ceil(3000 * n_mels / 256 / 8), B): 8 values per thread
__global__ void log_max_kernel(float* __restrict__ M, int n_mels, unsigned* __restrict__ cmax) {
  const int b = blockIdx.y;
  float* m = M + static_cast<size_t>(b) * kFramesPad * n_mels;   // the clip's frame-major rows
  const int count = kFrames * n_mels;
  float best = -INFINITY;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < count; i += gridDim.x * blockDim.x) {
    const float v = log10f(fmaxf(m[i], 1e-10f));
    m[i] = v;
    best = fmaxf(best, v);
  }
  best = fmaxf(best, __shfl_xor_sync(0xffffffffu, best, 16));
  best = fmaxf(best, __shfl_xor_sync(0xffffffffu, best, 8));
  best = fmaxf(best, __shfl_xor_sync(0xffffffffu, best, 4));
  best = fmaxf(best, __shfl_xor_sync(0xffffffffu, best, 2));
  best = fmaxf(best, __shfl_xor_sync(0xffffffffu, best, 1));
  if ((threadIdx.x & 31) == 0 && best > -INFINITY) atomicMax(&cmax[b], order_key(best));
}

// 32 frames x 32 mel channels per block, transposed through shared memory
template <typename OutT>
__global__ void finish_kernel(const float* __restrict__ L, const unsigned* __restrict__ cmax, OutT* __restrict__ mel,
                              int n_mels) {
  __shared__ float tile[32][33];
  const int b = blockIdx.z, f0 = blockIdx.x * 32, m0 = blockIdx.y * 32;
  const float floor_v = from_order_key(cmax[b]) - 8.0f;
  const float* src = L + static_cast<size_t>(b) * kFramesPad * n_mels;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int f = f0 + i, m = m0 + threadIdx.x;
    tile[i][threadIdx.x] = (f < kFrames && m < n_mels) ? src[static_cast<size_t>(f) * n_mels + m] : 0.f;
  }
  __syncthreads();
  OutT* dst = mel + static_cast<size_t>(b) * n_mels * kFrames;
  for (int i = threadIdx.y; i < 32; i += blockDim.y) {
    const int m = m0 + i, f = f0 + threadIdx.x;
    if (m < n_mels && f < kFrames)
      dst[static_cast<size_t>(m) * kFrames + f] = from_float<OutT>((fmaxf(tile[threadIdx.x][i], floor_v) + 4.0f) * 0.25f);
  }
}

// ------------------------------------------------------------ host constants
// Windowed DFT basis [kBasisN, kBasisK]: row 2k = w[n] cos(2 pi k n / 400), row
// 2k + 1 = w[n] sin(2 pi k n / 400), w the periodic Hann window, angles reduced
// exactly ((k n) mod 400) and evaluated in double, then rounded to fp32 and split
// into its tf32 part and remainder: columns [0, 416) hold the tf32 parts,
// [416, 832) the remainders, [832, 1248) the tf32 parts again (n >= 400 and
// rows >= 402 are zero).
std::vector<float> dft_basis() {
  std::vector<float> basis(static_cast<size_t>(kBasisN) * kBasisK, 0.f);
  const double two_pi = 6.283185307179586476925286766559;
  for (int k = 0; k < kBins; ++k)
    for (int n = 0; n < kFft; ++n) {
      const double w = 0.5 - 0.5 * std::cos(two_pi * n / kFft);
      const double a = two_pi * static_cast<double>((k * n) % kFft) / kFft;
      const float v[2] = {static_cast<float>(w * std::cos(a)), static_cast<float>(w * std::sin(a))};
      for (int q = 0; q < 2; ++q) {
        float* row = &basis[static_cast<size_t>(2 * k + q) * kBasisK];
        const float hi = round_tf32(v[q]);
        row[n] = hi;
        row[kWin + n] = v[q] - hi;
        row[2 * kWin + n] = hi;
      }
    }
  return basis;
}

// Slaney mel scale: 3 mels per 200 Hz up to 1 kHz, then 27 mels per factor 6.4.
double slaney_mel(double hz) {
  return hz < 1000.0 ? hz * 3.0 / 200.0 : 15.0 + std::log(hz / 1000.0) * 27.0 / std::log(6.4);
}
double slaney_hz(double mel) {
  return mel < 15.0 ? mel * 200.0 / 3.0 : 1000.0 * std::exp((mel - 15.0) * std::log(6.4) / 27.0);
}

// [kMelRows, kFbK]: row m < n_mels holds the triangle between n_mels + 2
// mel-spaced points from 0 Hz to 8 kHz, on bin frequencies k * 40 Hz, scaled to
// unit area (2 / (upper - lower edge)), rounded to fp32 and split like the DFT
// basis: columns [0, 224) its tf32 parts, [224, 448) the remainders, [448, 672)
// the tf32 parts again; rows >= n_mels and bins > 200 are zero.
std::vector<float> mel_bank(int n_mels) {
  std::vector<double> edge(n_mels + 2);
  const double top = slaney_mel(8000.0);
  for (int i = 0; i < n_mels + 2; ++i) edge[i] = slaney_hz(top * i / (n_mels + 1));
  std::vector<float> fb(static_cast<size_t>(kMelRows) * kFbK, 0.f);
  for (int m = 0; m < n_mels; ++m)
    for (int k = 0; k < kBins; ++k) {
      const double f = 40.0 * k;
      const double rise = (f - edge[m]) / (edge[m + 1] - edge[m]);
      const double fall = (edge[m + 2] - f) / (edge[m + 2] - edge[m + 1]);
      const double t = std::fmax(0.0, std::fmin(rise, fall));
      const float v = static_cast<float>(t * 2.0 / (edge[m + 2] - edge[m]));
      float* row = &fb[static_cast<size_t>(m) * kFbK];
      const float hi = round_tf32(v);
      row[k] = hi;
      row[kPowCols + k] = v - hi;
      row[2 * kPowCols + k] = hi;
    }
  return fb;
}

}  // namespace
}  // namespace enc

struct enc_frontend {
  int n_mels = 0, max_batch = 0, device = 0, sm_count = 0;
  size_t plane = 0;   // samples per plane of the padded buffer (tf32 parts, then remainders)
  int pow_rows = 0;   // rows per plane of the power spectrum (tf32 parts, then remainders)
  float *basis = nullptr, *fb = nullptr, *padded = nullptr, *P = nullptr, *M = nullptr;
  unsigned* cmax = nullptr;
  CUtensorMap map_frames, map_basis, map_pow, map_fb;   // tf32 operands of the two GEMMs
};

extern "C" {

ENC_API void enc_frontend_destroy(enc_frontend* h) {
  if (!h) return;
  int prev = 0;
  const bool have_prev = cudaGetDevice(&prev) == cudaSuccess;
  cudaSetDevice(h->device);
  for (void* p : {static_cast<void*>(h->basis), static_cast<void*>(h->fb), static_cast<void*>(h->padded),
                  static_cast<void*>(h->P), static_cast<void*>(h->M), static_cast<void*>(h->cmax)})
    if (p) cudaFree(p);
  if (have_prev) cudaSetDevice(prev);
  delete h;
}

ENC_API enc_status enc_frontend_create(int32_t n_mels, int32_t max_batch, enc_frontend** out) {
  using namespace enc;
  if (!out) return ENC_ERR_INVALID_ARG;
  *out = nullptr;
  if ((n_mels != 80 && n_mels != 128) || max_batch < 1 || max_batch > 4096) return ENC_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return ENC_ERR_CUDA;
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return ENC_ERR_CUDA;
  if (prop.major != 10 || prop.minor != 0) return ENC_ERR_UNSUPPORTED;
  enc_frontend* h = new (std::nothrow) enc_frontend;
  if (!h) return ENC_ERR_OOM;
  h->n_mels = n_mels;
  h->max_batch = max_batch;
  h->device = dev;
  h->sm_count = prop.multiProcessorCount;
  const size_t rows = static_cast<size_t>(max_batch) * kFramesPad;
  h->plane = static_cast<size_t>(max_batch) * kClipStride + kSlack;
  h->pow_rows = static_cast<int>(rows);
  const size_t padded_n = 2 * h->plane;
  bool ok = cudaMalloc(&h->basis, sizeof(float) * kBasisN * kBasisK) == cudaSuccess &&
            cudaMalloc(&h->fb, sizeof(float) * kMelRows * kFbK) == cudaSuccess &&
            cudaMalloc(&h->padded, sizeof(float) * padded_n) == cudaSuccess &&
            cudaMalloc(&h->P, sizeof(float) * 2 * rows * kPowCols) == cudaSuccess &&
            cudaMalloc(&h->M, sizeof(float) * rows * n_mels) == cudaSuccess &&
            cudaMalloc(&h->cmax, sizeof(unsigned) * max_batch) == cudaSuccess;
  if (!ok) {
    cudaGetLastError();
    enc_frontend_destroy(h);
    return ENC_ERR_OOM;
  }
  const std::vector<float> basis = dft_basis(), fb = mel_bank(n_mels);
  ok = cudaMemcpy(h->basis, basis.data(), sizeof(float) * basis.size(), cudaMemcpyHostToDevice) == cudaSuccess &&
       cudaMemcpy(h->fb, fb.data(), sizeof(float) * fb.size(), cudaMemcpyHostToDevice) == cudaSuccess &&
       cudaMemset(h->padded, 0, sizeof(float) * padded_n) == cudaSuccess;   // the slack stays zero
  // frames: rows of 160 samples over both planes; basis: [512, 1248]
  ok = ok && make_tma_2d_f32(&h->map_frames, h->padded, kHop, padded_n / kHop, kHop * sizeof(float), 128) &&
       make_tma_2d_f32(&h->map_basis, h->basis, kBasisK, kBasisN, kBasisK * sizeof(float), 128) &&
       make_tma_2d_f32(&h->map_pow, h->P, kPowCols, 2 * rows, kPowCols * sizeof(float), 128) &&
       make_tma_2d_f32(&h->map_fb, h->fb, kFbK, kMelRows, kFbK * sizeof(float), 128);
  if (!ok) {
    enc_frontend_destroy(h);
    return ENC_ERR_CUDA;
  }
  *out = h;
  return ENC_OK;
}

ENC_API enc_status enc_frontend_log_mel(enc_frontend* h, const float* audio, int32_t B, void* mel,
                                        enc_dtype out_dtype, cudaStream_t stream) {
  using namespace enc;
  if (!h || !audio || !mel || B < 1 || B > h->max_batch) return ENC_ERR_INVALID_ARG;
  if (out_dtype != ENC_DTYPE_BF16 && out_dtype != ENC_DTYPE_FP32) return ENC_ERR_INVALID_ARG;
  const int rows = B * kFramesPad, nm = h->n_mels;
  cudaError_t e = cudaSuccess;
  auto ok = [&](cudaError_t r) { if (e == cudaSuccess) e = r; return e == cudaSuccess; };
  pad_kernel<<<4 * 148, 256, 0, stream>>>(audio, h->padded, B, h->plane);
  ok(cudaGetLastError());
  GemmTcParams g = {};
  g.M = rows;
  g.N = kBasisN;
  g.num_kb = 3 * kKb;
  g.a_mode = A_DFT;
  g.kb_seg = kKb;
  g.a_lo_rows = static_cast<int>(h->plane / kHop);
  g.epi.out = h->P;
  g.epi.ldo = kPowCols;
  g.epi.P1 = h->pow_rows;   // the remainder plane of the power spectrum
  ok(launch_dft_power_tf32(h->map_frames, h->map_basis, g, h->sm_count, stream));
  GemmTcParams m = {};
  m.M = rows;
  m.N = kMelRows;
  m.num_kb = 3 * (kPowCols / 32);
  m.a_mode = A_SPLIT3;
  m.kb_seg = kPowCols / 32;
  m.a_lo_rows = h->pow_rows;
  m.epi.out = h->M;
  m.epi.ldo = nm;
  ok(launch_gemm_tf32_f32out(h->map_pow, h->map_fb, m, h->sm_count, stream));
  ok(cudaMemsetAsync(h->cmax, 0, sizeof(unsigned) * B, stream));
  log_max_kernel<<<dim3(64, B), 256, 0, stream>>>(h->M, nm, h->cmax);
  ok(cudaGetLastError());
  const dim3 grid((kFrames + 31) / 32, (nm + 31) / 32, B), block(32, 8);
  if (out_dtype == ENC_DTYPE_BF16)
    finish_kernel<bf16><<<grid, block, 0, stream>>>(h->M, h->cmax, static_cast<bf16*>(mel), nm);
  else
    finish_kernel<float><<<grid, block, 0, stream>>>(h->M, h->cmax, static_cast<float*>(mel), nm);
  ok(cudaGetLastError());
  return e == cudaSuccess ? ENC_OK : ENC_ERR_CUDA;
}

}  // extern "C"
