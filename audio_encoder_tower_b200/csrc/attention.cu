// Non-causal multi-head attention, head_dim 64, bf16 in / bf16 out, fp32
// softmax and accumulation, over ragged clips packed row after row.
//
// For clip b (rows cu[b] .. cu[b+1]) and head h:
//   O = softmax(Q K^T / 8) V, keys j >= n_b masked out (key-padding mask).
// Q, K and V are read in place from the QKV projection output [R, 3d]
// (columns h*64, d + h*64, 2d + h*64).
//
// One CTA = 128 query rows of one (clip, head), 8 warps x 16 rows. K/V tiles of
// 64 keys are double-buffered in shared memory with cp.async. Scores and the
// P.V product use the warp-level bf16 MMA (m16n8k16); the online softmax keeps
// a running row maximum and row sum in registers and rescales the output
// accumulator when the maximum grows.
#include "common.cuh"
#include "internal.h"

namespace enc {

namespace {

constexpr int kQ = 128, kKV = 64, kHD = 64, kWarps = 8;

__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
  const uint32_t d = smem_u32(dst);
  const int n = valid ? 16 : 0;   // 0 bytes read: the 16-byte slot is zero filled
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Shared-memory tile of rows x 64 bf16: 8 chunks of 16 B per row, chunk index
// XOR-swizzled with (row & 7) so that ldmatrix row reads hit distinct banks.
__device__ __forceinline__ uint32_t swz(int row, int chunk) { return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4)); }

}  // namespace

__global__ void __launch_bounds__(kWarps * 32) attention_bf16_kernel(const bf16* __restrict__ qkv,
                                                                     bf16* __restrict__ out,
                                                                     const int* __restrict__ cu, int d,
                                                                     float scale_log2) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* sQ = smem;                       // kQ x 128 B
  uint8_t* sK = sQ + kQ * 128;              // 2 x kKV x 128 B
  uint8_t* sV = sK + 2 * kKV * 128;         // 2 x kKV x 128 B

  const int b = blockIdx.z, h = blockIdx.y;
  const int start = cu[b], n = cu[b + 1] - start;
  const int q0 = blockIdx.x * kQ;
  if (q0 >= n) return;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const size_t ld = 3 * (size_t)d;
  const bf16* Qg = qkv + (size_t)start * ld + h * kHD;
  const bf16* Kg = Qg + d;
  const bf16* Vg = Qg + 2 * d;

  // Q tile (rows past the clip read as zero)
  for (int i = tid; i < kQ * 8; i += kWarps * 32) {
    const int r = i >> 3, ch = i & 7;
    const bool ok = q0 + r < n;
    cp_async16(sQ + swz(r, ch), Qg + (size_t)(ok ? q0 + r : 0) * ld + ch * 8, ok);
  }
  auto load_kv = [&](int t, int buf) {
    const int k0 = t * kKV;
    for (int i = tid; i < kKV * 8; i += kWarps * 32) {
      const int r = i >> 3, ch = i & 7;
      const bool ok = k0 + r < n;
      const size_t off = (size_t)(ok ? k0 + r : 0) * ld + ch * 8;
      cp_async16(sK + buf * kKV * 128 + swz(r, ch), Kg + off, ok);
      cp_async16(sV + buf * kKV * 128 + swz(r, ch), Vg + off, ok);
    }
  };
  load_kv(0, 0);
  cp_async_commit();

  const int n_tiles = (n + kKV - 1) / kKV;
  float m_r[2] = {-INFINITY, -INFINITY};   // running max (log2 domain) of rows lane/4 and lane/4 + 8
  float l_r[2] = {0.f, 0.f};               // running partial row sums (this thread's columns)
  float o_acc[8][4];
#pragma unroll
  for (int j = 0; j < 8; ++j) o_acc[j][0] = o_acc[j][1] = o_acc[j][2] = o_acc[j][3] = 0.f;
  uint32_t qf[4][4];

  const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sVa = smem_u32(sV);
  const int wr = warp * 16;   // first query row of this warp inside the tile

  for (int t = 0; t < n_tiles; ++t) {
    const int buf = t & 1;
    if (t + 1 < n_tiles) {
      load_kv(t + 1, buf ^ 1);
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    if (t == 0) {
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {   // A fragments of the warp's 16 x 64 Q rows
        const int r = wr + (lane & 15), ch = kk * 2 + (lane >> 4);
        ldsm_x4(sQa + swz(r, ch), qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
      }
    }
    // S = Q K^T for 64 keys: 8 n-tiles of 8 keys
    float s[8][4];
#pragma unroll
    for (int j = 0; j < 8; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
    const uint32_t kbase = sKa + buf * kKV * 128;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        const int key = np * 16 + (lane & 7) + ((lane >> 4) << 3);
        const int ch = kk * 2 + ((lane >> 3) & 1);
        uint32_t b0, b1, b2, b3;
        ldsm_x4(kbase + swz(key, ch), b0, b1, b2, b3);
        mma_bf16(s[2 * np], qf[kk], b0, b1);
        mma_bf16(s[2 * np + 1], qf[kk], b2, b3);
      }
    }
    // scale to log2 domain, mask keys past the clip, online softmax
    const int key0 = t * kKV + (lane & 3) * 2;
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int j = 0; j < 8; ++j) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int key = key0 + j * 8 + (e & 1);
        const float v = key < n ? s[j][e] * scale_log2 : -INFINITY;
        s[j][e] = v;
        mx[e >> 1] = fmaxf(mx[e >> 1], v);
      }
    }
    float alpha[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
      const float mnew = fmaxf(m_r[r], mx[r]);   // finite: every tile holds a valid key
      alpha[r] = exp2f(m_r[r] - mnew);           // exp2(-inf) = 0 on the first tile
      m_r[r] = mnew;
      l_r[r] *= alpha[r];
    }
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      s[j][0] = exp2f(s[j][0] - m_r[0]);
      s[j][1] = exp2f(s[j][1] - m_r[0]);
      s[j][2] = exp2f(s[j][2] - m_r[1]);
      s[j][3] = exp2f(s[j][3] - m_r[1]);
      l_r[0] += s[j][0] + s[j][1];
      l_r[1] += s[j][2] + s[j][3];
      o_acc[j][0] *= alpha[0];
      o_acc[j][1] *= alpha[0];
      o_acc[j][2] *= alpha[1];
      o_acc[j][3] *= alpha[1];
    }
    // O += P V: P (16 x 64 keys) as A fragments straight from the score registers
    const uint32_t vbase = sVa + buf * kKV * 128;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t pa[4];
      pa[0] = pack_bf16x2(s[2 * kk][0], s[2 * kk][1]);
      pa[1] = pack_bf16x2(s[2 * kk][2], s[2 * kk][3]);
      pa[2] = pack_bf16x2(s[2 * kk + 1][0], s[2 * kk + 1][1]);
      pa[3] = pack_bf16x2(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
      for (int dp = 0; dp < 4; ++dp) {
        const int key = kk * 16 + (lane & 7) + (((lane >> 3) & 1) << 3);
        const int ch = dp * 2 + (lane >> 4);
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(vbase + swz(key, ch), b0, b1, b2, b3);
        mma_bf16(o_acc[2 * dp], pa, b0, b1);
        mma_bf16(o_acc[2 * dp + 1], pa, b2, b3);
      }
    }
    __syncthreads();   // the buffer read here is refilled by the next prefetch
  }

  // normalise and store
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    l_r[r] += __shfl_xor_sync(0xffffffffu, l_r[r], 1);
    l_r[r] += __shfl_xor_sync(0xffffffffu, l_r[r], 2);
    l_r[r] = 1.f / l_r[r];
  }
  const int row0 = q0 + wr + (lane >> 2);
  bf16* Og = out + (size_t)start * d + h * kHD + (lane & 3) * 2;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (row0 < n)
      *reinterpret_cast<uint32_t*>(Og + (size_t)row0 * d + j * 8) =
          pack_bf16x2(o_acc[j][0] * l_r[0], o_acc[j][1] * l_r[0]);
    if (row0 + 8 < n)
      *reinterpret_cast<uint32_t*>(Og + (size_t)(row0 + 8) * d + j * 8) =
          pack_bf16x2(o_acc[j][2] * l_r[1], o_acc[j][3] * l_r[1]);
  }
}

cudaError_t launch_attention_bf16(const bf16* qkv, bf16* out, const int* cu, int B, int max_n, int d, int H,
                                  cudaStream_t stream) {
  if (B <= 0 || max_n <= 0) return cudaSuccess;
  const size_t smem = (size_t)(kQ + 4 * kKV) * 128;
  dim3 grid((max_n + kQ - 1) / kQ, H, B);
  attention_bf16_kernel<<<grid, kWarps * 32, smem, stream>>>(qkv, out, cu, d, 0.125f * 1.4426950408889634f);
  return cudaGetLastError();
}

}  // namespace enc
