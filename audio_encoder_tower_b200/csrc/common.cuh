// Shared device helpers of the encoder kernels: element types, GELU, warp
// reductions, the epilogue parameter block, and thin inline-PTX wrappers for
// mbarriers, TMA and the tcgen05 (5th-generation tensor core) instructions.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace enc {

using bf16 = __nv_bfloat16;

// ---------------------------------------------------------------- status word
// First error wins; the host reads (and clears) it in enc_get_status.
enum DeviceStatus : int { kDevOk = 0, kDevTimeout = 5, kDevCheck = 6 };

__device__ __forceinline__ void set_status(int* status, int code) {
  if (status) atomicCAS(status, 0, code);
}

// ------------------------------------------------------------------ numerics
// Exact GELU: x * Phi(x) = 0.5 x (1 + erf(x / sqrt 2)).
__device__ __forceinline__ float gelu_erf(float x) {
  return 0.5f * x * (1.0f + erff(x * 0.70710678118654752440f));
}

// 2^x on the MUFU unit (flushes subnormal results to zero).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Packed fp32 pairs (one instruction for two lanes of work on sm_100).
__device__ __forceinline__ void fma2(float& d0, float& d1, float a0, float a1, float b0, float b1, float c0,
                                     float c1) {
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1), "f"(c0), "f"(c1));
}
__device__ __forceinline__ void add2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d0), "=f"(d1)
      : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

// GELU for the tensor-core epilogues (bf16 results). For either sign of x
//   GELU(x) = x Phi(x) = max(x, 0) - |x| q,   q = Phi(-|x|),
// and q = 2^G(|x|) with G(a) = log2(erfc(a / sqrt 2) / 2), a smooth function of
// a that a degree-7 polynomial holds to 1.7e-5 (log2 units) on [0, 6.5]. The
// coefficients below come from Chebyshev interpolation of G on that interval,
// expanded in powers of a. The GELU is then within 1.1e-5 relative (5.1e-7
// absolute) of x Phi(x) for |x| <= 6.5; past 6.5, where Phi(-|x|) < 4.1e-11, q
// keeps its value at 6.5. One exponential per value; the polynomial runs on
// packed fp32 pairs.
namespace gelu_tail {
constexpr float kA = 6.5f;
constexpr float c0 = -9.9999012431e-01f, c1 = -1.1513109512e+00f, c2 = -4.5834896340e-01f,
                c3 = -5.4043046145e-02f, c4 = 8.5355194635e-03f, c5 = -9.3497301463e-04f,
                c6 = 6.1911072665e-05f, c7 = -1.8408538297e-06f;
}  // namespace gelu_tail

__device__ __forceinline__ void gelu_fast2(float& x0, float& x1) {
  using namespace gelu_tail;
  const float a0 = fminf(fabsf(x0), kA), a1 = fminf(fabsf(x1), kA);
  float g0, g1;
  fma2(g0, g1, c7, c7, a0, a1, c6, c6);
  fma2(g0, g1, g0, g1, a0, a1, c5, c5);
  fma2(g0, g1, g0, g1, a0, a1, c4, c4);
  fma2(g0, g1, g0, g1, a0, a1, c3, c3);
  fma2(g0, g1, g0, g1, a0, a1, c2, c2);
  fma2(g0, g1, g0, g1, a0, a1, c1, c1);
  fma2(g0, g1, g0, g1, a0, a1, c0, c0);
  x0 = fmaf(-fabsf(x0), ex2(g0), fmaxf(x0, 0.f));
  x1 = fmaf(-fabsf(x1), ex2(g1), fmaxf(x1, 0.f));
}

__device__ __forceinline__ float gelu_fast(float x) {
  using namespace gelu_tail;
  const float a = fminf(fabsf(x), kA);
  float g = fmaf(c7, a, c6);
  g = fmaf(g, a, c5);
  g = fmaf(g, a, c4);
  g = fmaf(g, a, c3);
  g = fmaf(g, a, c2);
  g = fmaf(g, a, c1);
  g = fmaf(g, a, c0);
  return fmaf(-fabsf(x), ex2(g), fmaxf(x, 0.f));
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

template <typename T> __device__ __forceinline__ T from_float(float v);
template <> __device__ __forceinline__ float from_float<float>(float v) { return v; }
template <> __device__ __forceinline__ bf16 from_float<bf16>(float v) { return __float2bfloat16_rn(v); }

template <typename T> __device__ __forceinline__ float to_float(T v);
template <> __device__ __forceinline__ float to_float<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_float<bf16>(bf16 v) { return __bfloat162float(v); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// ------------------------------------------------------------------ epilogue
// How a GEMM tile's fp32 accumulators become output.
enum EpiMode : int {
  EPI_STORE = 0,      // out[r, c] = acc + bias (optionally GELU)
  EPI_RESIDUAL = 1,   // resid[r, c] += acc + bias          (fp32 residual stream)
  EPI_CONV1 = 2,      // padded-time rows: GELU(acc + bias), exact 0 on pad rows
  EPI_CONV2 = 3,      // resid[cu[b] + j, c] = GELU(acc + bias) + pe[j, c], j < n_b
  EPI_SCATTER = 4,    // packed row -> out[b, j, c] (clip-major output), acc + bias
};

struct EpiParams {
  int mode;
  int gelu;            // apply GELU after the bias (EPI_STORE / EPI_SCATTER)
  const float* bias;   // [N] or nullptr
  void* out;           // output (bf16 or fp32, see kernel) or nullptr
  int ldo;             // row stride of out in elements
  float* resid;        // fp32 residual stream [rows, N]
  const float* pe;     // [P, N] position table (EPI_CONV2)
  const int* cu;       // [B+1] packed row offsets (EPI_CONV2 / EPI_SCATTER)
  int T;               // frames per clip (EPI_CONV1)
  int Tp;              // padded-time rows per clip (EPI_CONV1)
  int P1;              // conv2 rows per clip = P + 1 (EPI_CONV2)
  int B;               // clips (EPI_SCATTER)
  int p_out;           // output rows per clip (EPI_SCATTER)
};

// Destination of accumulator row r: returns false when the row is dropped.
// For EPI_CONV1 `zero` is set on padding rows (written as 0).
__device__ __forceinline__ bool epi_row(const EpiParams& e, int r, int& dst, int& pe_row, bool& zero) {
  zero = false;
  pe_row = 0;
  dst = r;
  if (e.mode == EPI_CONV1) {
    int tp = r % e.Tp;
    zero = (tp == 0) || (tp > e.T);
    return true;
  }
  if (e.mode == EPI_CONV2) {
    int b = r / e.P1, j = r - b * e.P1;
    int n = e.cu[b + 1] - e.cu[b];
    if (j >= n) return false;
    dst = e.cu[b] + j;
    pe_row = j;
    return true;
  }
  if (e.mode == EPI_SCATTER) {
    int lo = 0, hi = e.B;              // largest b with cu[b] <= r
    while (hi - lo > 1) {
      int mid = (lo + hi) >> 1;
      if (e.cu[mid] <= r) lo = mid; else hi = mid;
    }
    dst = lo * e.p_out + (r - e.cu[lo]);
    return true;
  }
  return true;
}

// Apply the epilogue to `n` consecutive columns c0.. of one accumulator row.
// v[] holds the raw accumulators; OutT is the element type of e.out.
template <typename OutT, int n>
__device__ __forceinline__ void epi_apply_run(const EpiParams& e, int dst, int pe_row, bool zero, int c0,
                                              const float* v) {
  // bf16 outputs come from the tensor-core path: the approximate GELU is far below bf16 rounding there
  constexpr bool kFastGelu = sizeof(OutT) == 2;
  if (e.mode == EPI_RESIDUAL) {
    float* x = e.resid + (size_t)dst * e.ldo + c0;
#pragma unroll
    for (int i = 0; i < n; i += 4) {
      float4 r = *reinterpret_cast<float4*>(x + i);
      float b0 = 0.f, b1 = 0.f, b2 = 0.f, b3 = 0.f;
      if (e.bias) { b0 = e.bias[c0 + i]; b1 = e.bias[c0 + i + 1]; b2 = e.bias[c0 + i + 2]; b3 = e.bias[c0 + i + 3]; }
      r.x += v[i] + b0; r.y += v[i + 1] + b1; r.z += v[i + 2] + b2; r.w += v[i + 3] + b3;
      *reinterpret_cast<float4*>(x + i) = r;
    }
    return;
  }
  if (e.mode == EPI_CONV2) {
    float* x = e.resid + (size_t)dst * e.ldo + c0;
    const float* pe = e.pe + (size_t)pe_row * e.ldo + c0;
#pragma unroll
    for (int i = 0; i < n; i += 4) {
      float4 p = *reinterpret_cast<const float4*>(pe + i);
      float b0 = 0.f, b1 = 0.f, b2 = 0.f, b3 = 0.f;
      if (e.bias) { b0 = e.bias[c0 + i]; b1 = e.bias[c0 + i + 1]; b2 = e.bias[c0 + i + 2]; b3 = e.bias[c0 + i + 3]; }
      float4 r;
      if (kFastGelu) {
        float g0 = v[i] + b0, g1 = v[i + 1] + b1, g2 = v[i + 2] + b2, g3 = v[i + 3] + b3;
        gelu_fast2(g0, g1);
        gelu_fast2(g2, g3);
        r.x = g0 + p.x;
        r.y = g1 + p.y;
        r.z = g2 + p.z;
        r.w = g3 + p.w;
      } else {
        r.x = gelu_erf(v[i] + b0) + p.x;
        r.y = gelu_erf(v[i + 1] + b1) + p.y;
        r.z = gelu_erf(v[i + 2] + b2) + p.z;
        r.w = gelu_erf(v[i + 3] + b3) + p.w;
      }
      *reinterpret_cast<float4*>(x + i) = r;
    }
    return;
  }
  // EPI_STORE, EPI_CONV1, EPI_SCATTER: value -> OutT, G columns at a time
  constexpr int G = n < 8 ? n : 8;   // bf16 stores need 8 columns (16 bytes); fp32 stores take 4
  static_assert(n % G == 0 && (sizeof(OutT) == 4 || G == 8), "epilogue run width");
  const bool g = e.gelu || e.mode == EPI_CONV1;
  OutT* o = reinterpret_cast<OutT*>(e.out) + (size_t)dst * e.ldo + c0;
#pragma unroll
  for (int i0 = 0; i0 < n; i0 += G) {
    float t[G];
#pragma unroll
    for (int i = 0; i < G; ++i) t[i] = v[i0 + i] + (e.bias ? e.bias[c0 + i0 + i] : 0.f);
    if (g) {
      if constexpr (kFastGelu) {
#pragma unroll
        for (int i = 0; i < G; i += 2) gelu_fast2(t[i], t[i + 1]);
      } else {
#pragma unroll
        for (int i = 0; i < G; ++i) t[i] = gelu_erf(t[i]);
      }
    }
#pragma unroll
    for (int i = 0; i < G; ++i) t[i] = zero ? 0.f : t[i];
    if constexpr (sizeof(OutT) == 2) {
      uint4 u;
      u.x = pack_bf16x2(t[0], t[1]);
      u.y = pack_bf16x2(t[2], t[3]);
      u.z = pack_bf16x2(t[4], t[5]);
      u.w = pack_bf16x2(t[6], t[7]);
      *reinterpret_cast<uint4*>(o + i0) = u;
    } else {
#pragma unroll
      for (int i = 0; i < G; i += 4)
        *reinterpret_cast<float4*>(o + i0 + i) = make_float4(t[i], t[i + 1], t[i + 2], t[i + 3]);
    }
  }
}

// ------------------------------------------------------- PTX: smem, mbarrier
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_test(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// mbar_test with a suspend-time hint: while the phase is incomplete the thread
// sleeps in the instruction until the phase completes or about `hint_ns` have
// passed, instead of returning at once to spin (a spinning warp takes issue
// slots from the warps that share its scheduler).
__device__ __forceinline__ bool mbar_test_sleep(uint32_t bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// Wait for the phase of `bar` with the given parity to complete, for at most
// `limit_ns` nanoseconds or until *abort (when given) becomes non-zero. Returns false when
// the wait gave up (the caller records the error and unwinds). Each retry sleeps for at
// most 20 us, so the limit and the abort flag are looked at every 320 us or sooner.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, const volatile int* abort,
                                          uint64_t limit_ns) {
  const uint32_t a = smem_u32(bar);
  if (mbar_test(a, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_test_sleep(a, parity, 20000u)) return true;
    if ((it & 15u) == 0u) {
      if (abort && *abort) return false;
      if (globaltimer_ns() - t0 > limit_ns) return false;
    }
  }
}

// mbar_wait by every lane of a converged warp; true only if all lanes saw the phase.
__device__ __forceinline__ bool mbar_wait_warp(uint64_t* bar, uint32_t parity, const volatile int* abort,
                                               uint64_t limit_ns) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort, limit_ns));
}

// One lane of a converged warp (the lowest active one) for single-thread issue.
// tcgen05.mma issued from converged warp code with warp-uniform operands costs a
// fraction of the issue cycles it takes from divergent single-lane code.
__device__ __forceinline__ bool elect_one() {
  uint32_t p;
  asm volatile(
      "{\n\t.reg .pred P;\n\t.reg .b32 R;\n\telect.sync R|P, 0xffffffff;\n\tselp.u32 %0, 1, 0, P;\n\t}"
      : "=r"(p));
  return p != 0;
}

// ---------------------------------------------------------------- PTX: TMA
__device__ __forceinline__ void tma_prefetch_desc(const void* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 2-D tiled bulk tensor load global -> shared, completion on an mbarrier.
__device__ __forceinline__ void tma_load_2d(void* dst, const void* map, uint64_t* bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::
          "r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

// ------------------------------------------------------------ PTX: tcgen05
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, kind::f16 (bf16 inputs, fp32 accumulate).
__device__ __forceinline__ void umma_f16_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive (once) on `bar` when all previously issued tcgen05.mma of this thread are done.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp receives lane
// (base lane + i), columns col .. col+31 of the accumulator.
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),
        "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
        "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

// Shared-memory matrix descriptor of a K-major bf16 tile written by TMA with
// 128-byte swizzle: rows of 64 elements (128 B), 8-row atoms of 1024 B.
//   bits  0-13 start address >> 4     bits 16-29 leading byte offset >> 4 (unused here: 1)
//   bits 32-45 stride byte offset >> 4 (1024 B between 8-row groups)
//   bits 46-47 descriptor version 1   bits 61-63 layout: 2 = 128-byte swizzle
__device__ __forceinline__ uint64_t smem_desc_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>(1) << 16;
  d |= static_cast<uint64_t>(1024 >> 4) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}

// Instruction descriptor, kind::f16: fp32 accumulator, bf16 A and B, both K-major.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int m, int n) {
  return (1u << 4)                                // D format: f32
         | (1u << 7)                              // A format: bf16
         | (1u << 10)                             // B format: bf16
         | (static_cast<uint32_t>(n >> 3) << 17)  // N / 8
         | (static_cast<uint32_t>(m >> 4) << 24); // M / 16
}

}  // namespace enc
