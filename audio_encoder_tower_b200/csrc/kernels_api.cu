// Single-kernel C entry points (include/enc_kernels.h).
#include <string.h>

#include "../../include/enc_kernels.h"
#include "common.cuh"
#include "internal.h"

using namespace enc;

namespace {
int sm_count_current() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
}  // namespace

extern "C" {

enc_status enc_linear_bf16(const void* A, const void* W, const float* bias, void* out, float* resid, int32_t M,
                           int32_t N, int32_t K, int32_t gelu, int* status, cudaStream_t stream) {
  if (!A || !W || (!out && !resid) || M < 0 || N <= 0 || K <= 0) return ENC_ERR_INVALID_ARG;
  if (K % 64 || N % 128) return ENC_ERR_UNSUPPORTED;
  if (!aligned16(A) || !aligned16(W) || (out && !aligned16(out)) || (resid && !aligned16(resid)))
    return ENC_ERR_INVALID_ARG;
  if (M == 0) return ENC_OK;
  const int sms = sm_count_current();
  if (sms <= 0) return ENC_ERR_CUDA;
  CUtensorMap ma, mb;
  if (!make_tma_2d(&ma, A, (uint64_t)K, (uint64_t)M, (uint64_t)K * 2, 64, 128)) return ENC_ERR_CUDA;
  if (!make_tma_2d(&mb, W, (uint64_t)K, (uint64_t)N, (uint64_t)K * 2, 64, 128))
    return ENC_ERR_CUDA;
  GemmTcParams p;
  memset(&p, 0, sizeof(p));
  p.M = M; p.N = N; p.num_kb = K / 64; p.a_mode = A_PLAIN; p.status = status;
  p.epi.mode = resid ? EPI_RESIDUAL : EPI_STORE;
  p.epi.gelu = gelu ? 1 : 0;
  p.epi.bias = bias;
  p.epi.out = out;
  p.epi.resid = resid;
  p.epi.ldo = N;
  CUtensorMap mc;
  if (resid ? !make_resid_map(&mc, resid, (uint64_t)M, (uint64_t)N) : !make_out_map(&mc, out, (uint64_t)M, (uint64_t)N))
    return ENC_ERR_CUDA;
  return launch_gemm_tc(ma, mb, p, sms, stream, &mc) == cudaSuccess ? ENC_OK : ENC_ERR_CUDA;
}

enc_status enc_attention_bf16(const void* qkv, void* out, const int32_t* cu, int32_t rows, int32_t B,
                              int32_t max_n, int32_t n_heads, int* status, cudaStream_t stream) {
  if (!qkv || !out || !cu || rows < 1 || B < 1 || B > 65535 || max_n < 0 || n_heads < 1 || n_heads > 65535)
    return ENC_ERR_INVALID_ARG;
  if (!aligned16(qkv) || !aligned16(out)) return ENC_ERR_INVALID_ARG;
  QkvMaps maps;
  if (!make_qkv_maps(&maps, qkv, rows, 64 * n_heads)) return ENC_ERR_CUDA;
  return launch_attention_tc(maps, reinterpret_cast<bf16*>(out), cu, B, max_n, 64 * n_heads, n_heads, status,
                             stream) == cudaSuccess
             ? ENC_OK
             : ENC_ERR_CUDA;
}

}  // extern "C"
