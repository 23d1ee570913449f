// Non-causal multi-head attention on the 5th-generation tensor cores
// (tcgen05), head_dim 64, over ragged clips packed row after row.
//
// For clip b (packed rows cu[b] .. cu[b+1]) and head h:
//   O = softmax(Q K^T / 8) V, keys j >= n_b masked out (key-padding mask),
// with Q, K, V read in place from the QKV projection output [R, 3d]
// (columns h*64, d + h*64, 2d + h*64) -- the single bidirectional pass of the
// Whisper encoder (Qwen2-Audio-7B-Instruct, "(1) AUDIO ENCODER"; head_dim 64,
// MHA: Voxtral-Mini-3B-2507, "(1) AUDIO ENCODER").
//
// One CTA = 128 query rows of one (clip, head). Warp roles:
//   warp 0      TMA: the Q tile once, then K and V tiles of 128 keys into a
//               3-stage ring (128-byte swizzle).
//   warp 1      MMA issuer: S_j = Q K_j^T (M=128, N=128, K=64) into one of two
//               TMEM score buffers, then O += P_j V_j with P_j read from TMEM
//               (A operand in tensor memory) and V_j from shared memory.
//   warps 2..9  softmax: two threads per query row (the row's TMEM lane), each
//               owning 64 of the tile's 128 keys, holding its scores in
//               registers; the two half-row maxima meet in shared memory.
//               exp2, row sum, P_j = bf16 into TMEM; the output accumulator O
//               is rescaled only when a row's running maximum grows by more
//               than 2^8 (otherwise the stale maximum is kept: P <= 256).
//               At the end O / l is written out as bf16.
// S_{j+1} is computed while the softmax works on S_j.
//
// TMEM (512 columns): S0 [0,128) S1 [128,256) O [256,320) P0 [320,384) P1 [384,448).
#include "common.cuh"
#include "internal.h"

namespace enc {

namespace {

constexpr int kQT = 128, kKT = 128, kHD = 64, kStages = 3;
constexpr int kSoftWarps = 8;
constexpr int kThreads = 64 + 32 * kSoftWarps;
constexpr uint32_t kTileBytes = 128 * 64 * 2;   // one 128 x 64 bf16 tile
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColS = 0, kColO = 256, kColP = 320;
constexpr uint64_t kWaitNs = 2000000000ull;
constexpr float kRescaleThreshold = 8.0f;       // log2 units

constexpr size_t kSmemBytes = 1024 + kTileBytes * (1 + 2 * kStages) + 256 + 2 * 2 * 128 * 4 + 2 * 128 * 4;

__device__ __forceinline__ void umma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tmem_st_32x32b_x16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Shared-memory descriptor of a 128-byte-swizzled tile whose rows of 128 B run
// along the N (MN-major) dimension: 8-row atoms of 1024 B follow each other
// along K (stride byte offset 1024); one atom spans the whole N = 64.
__device__ __forceinline__ uint64_t smem_desc_sw128_mn(uint32_t saddr) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr & 0x3FFFFu) >> 4);
  d |= static_cast<uint64_t>(1) << 16;
  d |= static_cast<uint64_t>(1024 >> 4) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(2) << 61;
  return d;
}

}  // namespace

__global__ void __launch_bounds__(kThreads, 1)
attention_tc_kernel(const __grid_constant__ CUtensorMap map_qkv, bf16* __restrict__ out, const int* __restrict__ cu,
                    int d, float scale_log2, int* status) {
  const int b = blockIdx.z, h = blockIdx.y;
  const int start = cu[b], n = cu[b + 1] - start;
  const int q0 = blockIdx.x * kQT;
  if (q0 >= n) return;
  const int nkv = (n + kKT - 1) / kKT;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + kTileBytes;                  // kStages tiles
  uint8_t* sV = sK + kStages * kTileBytes;        // kStages tiles
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + kStages * kTileBytes);
  uint64_t* q_full = bars;
  uint64_t* kv_full = bars + 1;
  uint64_t* kv_empty = kv_full + kStages;
  uint64_t* s_full = kv_empty + kStages;          // [2]
  uint64_t* s_empty = s_full + 2;                 // [2]
  uint64_t* p_full = s_empty + 2;                 // [2]
  uint64_t* pv_done = p_full + 2;                 // [2]
  uint64_t* drain = pv_done + 2;
  uint64_t* red_bar = drain + 1;                  // [2] half-row maxima written
  uint64_t* sum_bar = red_bar + 2;                // half-row sums written
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sum_bar + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  float* red_max = reinterpret_cast<float*>(bars + 32);   // [2 tiles][2 halves][128 rows]
  float* red_sum = red_max + 2 * 2 * 128;                  // [2 halves][128 rows]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < kStages; ++s) { mbar_init(&kv_full[s], 1); mbar_init(&kv_empty[s], 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], 32 * kSoftWarps);
      mbar_init(&p_full[i], 32 * kSoftWarps);
      mbar_init(&pv_done[i], 1);
    }
    mbar_init(drain, 1);
    mbar_init(&red_bar[0], 32 * kSoftWarps);
    mbar_init(&red_bar[1], 32 * kSoftWarps);
    mbar_init(sum_bar, 32 * kSoftWarps);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) tma_prefetch_desc(&map_qkv);
  if (warp == 1) { tmem_alloc(tmem_slot, kTmemCols); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  volatile int* abort_v = abort_flag;

  if (warp == 0) {
    // -------------------------------------------------------------- TMA
    if (lane == 0) {
      bool ok = true;
      uint32_t armed = 0, armed_ph = 0;
      mbar_arrive_expect_tx(q_full, kTileBytes);
      tma_load_2d(sQ, &map_qkv, q_full, h * kHD, start + q0);
      int st = 0;
      uint32_t ph = 0;
      for (int j = 0; j < nkv; ++j) {
        if (!mbar_wait(&kv_empty[st], ph ^ 1u, abort_v, kWaitNs)) { ok = false; break; }
        mbar_arrive_expect_tx(&kv_full[st], 2 * kTileBytes);
        tma_load_2d(sK + st * kTileBytes, &map_qkv, &kv_full[st], d + h * kHD, start + j * kKT);
        tma_load_2d(sV + st * kTileBytes, &map_qkv, &kv_full[st], 2 * d + h * kHD, start + j * kKT);
        armed |= 1u << st;
        armed_ph = (armed_ph & ~(1u << st)) | (ph << st);
        if (++st == kStages) { st = 0; ph ^= 1u; }
      }
      if (!ok) {
        set_status(status, kDevTimeout);
        *abort_v = 1;
        mbar_wait(q_full, 0, nullptr, kWaitNs / 4);
        for (int s = 0; s < kStages; ++s)
          if (armed & (1u << s)) mbar_wait(&kv_full[s], (armed_ph >> s) & 1u, nullptr, kWaitNs / 4);
      }
    }
  } else if (warp == 1) {
    // -------------------------------------------------------------- MMA
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, kKT);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, kHD) | (1u << 16);   // B (V) MN-major
      bool ok = mbar_wait(q_full, 0, abort_v, kWaitNs);
      bool issued = false;
      const uint64_t qdesc = smem_desc_sw128(smem_u32(sQ));
      auto issue_s = [&](int j, int stage) {
        const uint64_t kdesc = smem_desc_sw128(smem_u32(sK + stage * kTileBytes));
        const uint32_t dS = tmem + kColS + static_cast<uint32_t>((j & 1) * kKT);
#pragma unroll
        for (int k = 0; k < kHD / 16; ++k)
          umma_f16_ss(dS, qdesc + static_cast<uint64_t>(2 * k), kdesc + static_cast<uint64_t>(2 * k), idesc_s,
                      k > 0 ? 1u : 0u);
        umma_commit(&s_full[j & 1]);
        issued = true;
      };
      int st = 0;
      uint32_t ph = 0;
      if (ok) ok = mbar_wait(&kv_full[0], 0, abort_v, kWaitNs);
      if (ok) { tc_fence_after(); issue_s(0, 0); }
      for (int j = 0; ok && j < nkv; ++j) {
        const int st1 = (st + 1 == kStages) ? 0 : st + 1;
        const uint32_t ph1 = (st + 1 == kStages) ? (ph ^ 1u) : ph;
        if (j + 1 < nkv) {
          if (!mbar_wait(&kv_full[st1], ph1, abort_v, kWaitNs)) { ok = false; break; }
          // the score buffer of tile j+1 was last read by the softmax of tile j-1
          if (!mbar_wait(&s_empty[(j + 1) & 1], (((j + 1) >> 1) & 1u) ^ 1u, abort_v, kWaitNs)) { ok = false; break; }
          tc_fence_after();
          issue_s(j + 1, st1);
        }
        if (!mbar_wait(&p_full[j & 1], (j >> 1) & 1u, abort_v, kWaitNs)) { ok = false; break; }
        tc_fence_after();
        const uint64_t vdesc = smem_desc_sw128_mn(smem_u32(sV + st * kTileBytes));
        const uint32_t aP = tmem + kColP + static_cast<uint32_t>((j & 1) * (kKT / 2));
#pragma unroll
        for (int k = 0; k < kKT / 16; ++k)   // 16 keys per step: 8 TMEM columns of P, 2048 B of V
          umma_f16_ts(tmem + kColO, aP + static_cast<uint32_t>(8 * k), vdesc + static_cast<uint64_t>(128 * k),
                      idesc_pv, (j > 0 || k > 0) ? 1u : 0u);
        umma_commit(&pv_done[j & 1]);
        umma_commit(&kv_empty[st]);
        st = st1;
        ph = ph1;
      }
      if (!ok) { set_status(status, kDevTimeout); *abort_v = 1; }
      if (issued) {
        umma_commit(drain);
        mbar_wait(drain, 0, nullptr, kWaitNs);
      }
    }
  } else {
    // ----------------------------------------------------------- softmax
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;      // keys [64*half, 64*half + 64) of each tile
    const int row = quarter * 32 + lane;   // query row inside the tile = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    float m_run = -INFINITY, l_run = 0.f;
    bool ok = true;
    for (int j = 0; j < nkv; ++j) {
      const int sb = j & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[sb], (j >> 1) & 1u, abort_v, kWaitNs))) { ok = false; break; }
      tc_fence_after();
      const uint32_t tS = tmem + lane_off + kColS + static_cast<uint32_t>(sb * kKT + 64 * half);
      uint32_t v[64];
      tmem_ld_32x32b_x32(tS, *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
      tmem_ld_32x32b_x32(tS + 32u, *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
      tmem_wait_ld();
      const int kvalid = n - j * kKT - 64 * half;   // keys of this half-tile inside the clip
      const bool full = kvalid >= 64;
      float mx = -INFINITY;
      if (full) {
#pragma unroll
        for (int e = 0; e < 64; ++e) mx = fmaxf(mx, __uint_as_float(v[e]));
      } else {
#pragma unroll
        for (int e = 0; e < 64; ++e)
          if (e < kvalid) mx = fmaxf(mx, __uint_as_float(v[e]));
      }
      // the other half of the row (slot sb is rewritten two tiles later, after
      // both threads of the row have passed the next tile's exchange)
      red_max[(sb * 2 + half) * 128 + row] = mx;
      mbar_arrive(&red_bar[sb]);
      if (!__all_sync(0xffffffffu, mbar_wait(&red_bar[sb], (j >> 1) & 1u, abort_v, kWaitNs))) { ok = false; break; }
      mx = fmaxf(mx, red_max[(sb * 2 + (half ^ 1)) * 128 + row]) * scale_log2;
      if (j == 0) {
        m_run = mx;
      } else {
        const bool need = mx > m_run + kRescaleThreshold;
        if (__any_sync(0xffffffffu, need)) {
          // O must hold P_{j-1} V_{j-1} before it is rescaled
          if (!__all_sync(0xffffffffu, mbar_wait(&pv_done[(j - 1) & 1], ((j - 1) >> 1) & 1u, abort_v, kWaitNs))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const float alpha = need ? ex2(m_run - mx) : 1.f;
          if (need) { m_run = mx; l_run *= alpha; }
          uint32_t o[32];
          const uint32_t tO = tmem + lane_off + kColO + static_cast<uint32_t>(32 * half);
          tmem_ld_32x32b_x32(tO, o);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st_32x32b_x32(tO, o);
          tmem_wait_st();
        }
      }
      // P = exp2(s * scale_log2 - m) (0 on masked keys) as bf16 pairs into TMEM
      const uint32_t tP = tmem + lane_off + kColP + static_cast<uint32_t>(sb * (kKT / 2) + 32 * half);
      const float neg_m = -m_run;
      uint32_t pk[32];
      if (full) {
#pragma unroll
        for (int e = 0; e < 64; e += 2) {
          const float p0 = ex2(fmaf(__uint_as_float(v[e]), scale_log2, neg_m));
          const float p1 = ex2(fmaf(__uint_as_float(v[e + 1]), scale_log2, neg_m));
          l_run += p0 + p1;
          pk[e >> 1] = pack_bf16x2(p0, p1);
        }
      } else {
#pragma unroll
        for (int e = 0; e < 64; e += 2) {
          float p0 = ex2(fmaf(__uint_as_float(v[e]), scale_log2, neg_m));
          float p1 = ex2(fmaf(__uint_as_float(v[e + 1]), scale_log2, neg_m));
          if (e >= kvalid) p0 = 0.f;
          if (e + 1 >= kvalid) p1 = 0.f;
          l_run += p0 + p1;
          pk[e >> 1] = pack_bf16x2(p0, p1);
        }
      }
      tmem_st_32x32b_x32(tP, pk);
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&s_empty[sb]);
      mbar_arrive(&p_full[sb]);
    }
    if (ok && !__all_sync(0xffffffffu, mbar_wait(&pv_done[(nkv - 1) & 1], ((nkv - 1) >> 1) & 1u, abort_v, kWaitNs)))
      ok = false;
    // the row sum is split between the two halves
    red_sum[half * 128 + row] = l_run;
    mbar_arrive(sum_bar);
    if (ok && !__all_sync(0xffffffffu, mbar_wait(sum_bar, 0, abort_v, kWaitNs))) ok = false;
    if (!__all_sync(0xffffffffu, ok)) {
      set_status(status, kDevTimeout);
      *abort_v = 1;
    } else {
      tc_fence_after();
      const float inv = 1.f / (l_run + red_sum[(half ^ 1) * 128 + row]);
      const bool valid = q0 + row < n;
      bf16* orow = out + (size_t)(start + q0 + row) * d + h * kHD + 32 * half;
      uint32_t o[32];
      tmem_ld_32x32b_x32(tmem + lane_off + kColO + static_cast<uint32_t>(32 * half), o);
      tmem_wait_ld();
      if (valid) {
#pragma unroll
        for (int e = 0; e < 32; e += 8) {
          uint4 u;
          u.x = pack_bf16x2(__uint_as_float(o[e]) * inv, __uint_as_float(o[e + 1]) * inv);
          u.y = pack_bf16x2(__uint_as_float(o[e + 2]) * inv, __uint_as_float(o[e + 3]) * inv);
          u.z = pack_bf16x2(__uint_as_float(o[e + 4]) * inv, __uint_as_float(o[e + 5]) * inv);
          u.w = pack_bf16x2(__uint_as_float(o[e + 6]) * inv, __uint_as_float(o[e + 7]) * inv);
          *reinterpret_cast<uint4*>(orow + e) = u;
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

bool make_qkv_map(CUtensorMap* map, const void* qkv, int rows, int d) {
  return make_tma_2d(map, qkv, 3 * (uint64_t)d, (uint64_t)rows, 6 * (uint64_t)d, 64, 128);
}

cudaError_t launch_attention_tc(const CUtensorMap& map_qkv, bf16* out, const int* cu, int B, int max_n, int d, int H,
                                int* status, cudaStream_t stream) {
  if (B <= 0 || max_n <= 0) return cudaSuccess;
  static unsigned long long done = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidValue;
  if (!(done & (1ull << (dev & 63)))) {
    cudaError_t e = cudaFuncSetAttribute(attention_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    done |= 1ull << (dev & 63);
  }
  dim3 grid((max_n + kQT - 1) / kQT, H, B);
  attention_tc_kernel<<<grid, kThreads, kSmemBytes, stream>>>(map_qkv, out, cu, d, 0.125f * 1.4426950408889634f,
                                                              status);
  return cudaGetLastError();
}

}  // namespace enc
