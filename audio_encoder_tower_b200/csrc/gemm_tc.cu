// tcgen05 (UMMA) GEMM with fused epilogues for the encoder's dense contractions:
//   conv1 / conv2 (implicit GEMM over TMA-staged taps), QKV, out-proj, fc1, fc2,
//   projector fc1 / fc2.
//
//   C[M, N] = A[M, K] * W[N, K]^T, bf16 operands, fp32 accumulation in TMEM.
//
// Design (one CTA per SM, persistent over 128 x BN output tiles):
//   warp 0      TMA producer: 64-wide K slices of A (128 rows) and W (BN rows)
//               into a kStages-deep shared-memory ring, 128-byte swizzle.
//   warp 1      MMA issuer: one thread issues tcgen05.mma (M=128, N=BN, K=16)
//               into a double-buffered TMEM accumulator (2 x BN columns) and
//               frees ring slots / publishes finished tiles with tcgen05.commit.
//   warps 2..9  epilogue: tcgen05.ld the accumulator (one row per thread;
//               warps w and w+4 share TMEM lanes and split the columns),
//               apply bias / GELU / residual / position-table / scatter, store.
// The epilogue of tile i overlaps the MMAs of tile i+1.
//
// The A operand of the convolutions is never materialised as an im2col matrix:
//   conv1: tap k of output row r is row r + k - 1 of the time-major mel buffer
//          (a shifted TMA box; row -1 and rows past the end read as zeros);
//   conv2: the conv1 output [rows, d] is viewed as [rows/2, 2d] ("pairs");
//          output j needs pair j (taps 0, 1) and the first half of pair j + 1.
#include <cudaTypedefs.h>

#include "common.cuh"
#include "internal.h"

namespace enc {

namespace {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int kEpiWarps = 8;   // two per TMEM lane quarter, each with half of the tile's columns
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr uint64_t kWaitLimitNs = 2000000000ull;   // 2 s: far above any legitimate wait

template <int BN>
struct TcCfg {
  static constexpr int kStages = BN == 256 ? 4 : 6;
  static constexpr uint32_t kABytes = BM * BK * 2;
  static constexpr uint32_t kBBytes = BN * BK * 2;
  static constexpr uint32_t kStageBytes = kABytes + kBBytes;
  static constexpr uint32_t kTmemCols = 2 * BN;
  static constexpr size_t kStagingBytes = kEpiWarps * 32 * 32 * 4;   // one 32x32 fp32 tile per epilogue warp
  static constexpr size_t kSmemBytes =
      1024 /*align slack*/ + kStages * (size_t)kStageBytes + 1024 /*barriers*/ + kStagingBytes;
};

__device__ __forceinline__ void a_coords(const GemmTcParams& p, int m0, int kb, int& x, int& y) {
  if (p.a_mode == A_CONV1) {
    const int tap = kb / p.kb_seg;
    x = (kb - tap * p.kb_seg) * BK;
    y = m0 + tap - 1;
  } else if (p.a_mode == A_CONV2) {
    if (kb < 2 * p.kb_seg) { x = kb * BK; y = m0; }
    else { x = (kb - 2 * p.kb_seg) * BK; y = m0 + 1; }
  } else if (p.a_mode == A_DFT) {
    const int part = kb / p.kb_seg, w = kb - part * p.kb_seg;
    x = (w % 5) * 32;
    y = m0 + w / 5 + (part == 2 ? p.a_lo_rows : 0);
  } else if (p.a_mode == A_SPLIT3) {
    const int part = kb / p.kb_seg;
    x = (kb - part * p.kb_seg) * 32;
    y = m0 + (part == 2 ? p.a_lo_rows : 0);
  } else {
    x = kb * BK;
    y = m0;
  }
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// resid[y .. y+32, x .. x+32) += the 32x32 fp32 tile at smem (tensor-map layout,
// 128-byte swizzle), reduced in L2 by the TMA unit; rows past the map's end are
// skipped. Completion is tracked with bulk groups.
__device__ __forceinline__ void tma_reduce_add_2d(const void* map, const void* smem, int x, int y) {
  asm volatile("cp.reduce.async.bulk.tensor.2d.global.shared::cta.add.tile.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(smem)), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// x[r0 .. r0+32, n0 .. n0+32*NC) += acc + bias for the warp's 32 accumulator rows.
// Each 32-column chunk goes through the warp's 4 KB staging tile: thread = row
// writes its 32 values (16-byte pieces XOR-swizzled by row, as the tensor map's
// 128-byte swizzle expects: conflict-free), then one lane hands the tile to the
// TMA unit as a reduce-add into the fp32 residual, which happens in L2. The SM
// never loads the residual and nothing here waits on global memory, except for
// the previous chunk's bulk read of the staging tile.
template <int NC>
__device__ __forceinline__ void epi_residual_tile(const EpiParams& e, const CUtensorMap* map_c, int r0, int n0,
                                                  uint32_t taddr, float* tile, int lane) {
#pragma unroll 1
  for (int c = 0; c < NC; ++c) {
    uint32_t v[32];
    tmem_ld_32x32b_x32(taddr + static_cast<uint32_t>(c * 32), v);
    if (lane == 0) bulk_wait_read0();   // the previous reduce has read the staging tile
    tmem_wait_ld();
    __syncwarp();
    const float* bias = e.bias ? e.bias + n0 + c * 32 : nullptr;
    float4* row = reinterpret_cast<float4*>(tile + lane * 32);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float4 b = bias ? *reinterpret_cast<const float4*>(bias + 4 * j) : make_float4(0.f, 0.f, 0.f, 0.f);
      row[j ^ (lane & 7)] = make_float4(__uint_as_float(v[4 * j]) + b.x, __uint_as_float(v[4 * j + 1]) + b.y,
                                        __uint_as_float(v[4 * j + 2]) + b.z, __uint_as_float(v[4 * j + 3]) + b.w);
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_reduce_add_2d(map_c, tile, n0 + c * 32, r0);
      bulk_commit();
    }
  }
}

// out[y .. y+32, x .. x+64) = the 32x64 bf16 tile at smem (tensor-map layout,
// 128-byte swizzle); rows past the map's end are skipped.
__device__ __forceinline__ void tma_store_2d(const void* map, const void* smem, int x, int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(smem_u32(smem)), "r"(x), "r"(y)
               : "memory");
}

// out[r0 .. r0+32, n0 .. n0+64*NC) = act(acc + bias) as bf16 for the warp's 32
// accumulator rows (EPI_STORE, EPI_CONV1). Each 64-column chunk is converted
// into the warp's 4 KB staging tile (thread = row, 16-byte pieces XOR-swizzled
// by row as the tensor map's 128-byte swizzle expects) and written by one TMA
// bulk store, so global writes are whole lines and asynchronous.
template <int NC>
__device__ __forceinline__ void epi_store_tile(const EpiParams& e, const CUtensorMap* map_c, int r0, int n0,
                                               uint32_t taddr, uint32_t* tile, int lane) {
  const int r = r0 + lane;
  bool zero = false;   // conv1: padding rows of the padded time axis are exact zeros
  if (e.mode == EPI_CONV1) {
    const int tp = r % e.Tp;
    zero = (tp == 0) || (tp > e.T);
  }
  const bool g = e.gelu || e.mode == EPI_CONV1;
#pragma unroll 1
  for (int c = 0; c < NC; ++c) {
    uint32_t v[64];
    tmem_ld_32x32b_x32(taddr + static_cast<uint32_t>(c * 64), *reinterpret_cast<uint32_t(*)[32]>(&v[0]));
    tmem_ld_32x32b_x32(taddr + static_cast<uint32_t>(c * 64 + 32), *reinterpret_cast<uint32_t(*)[32]>(&v[32]));
    if (lane == 0) bulk_wait_read0();   // the previous store has read the staging tile
    tmem_wait_ld();
    __syncwarp();
    const float4* bias = e.bias ? reinterpret_cast<const float4*>(e.bias + n0 + c * 64) : nullptr;
    uint4* row = reinterpret_cast<uint4*>(tile + lane * 32);
#pragma unroll
    for (int j = 0; j < 8; ++j) {   // 8 columns -> one 16-byte piece
      float t[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) t[i] = __uint_as_float(v[8 * j + i]);
      if (bias) {   // the same 32 bytes for every lane: one broadcast load
        const float4 b0 = __ldg(bias + 2 * j), b1 = __ldg(bias + 2 * j + 1);
        add2(t[0], t[1], t[0], t[1], b0.x, b0.y);
        add2(t[2], t[3], t[2], t[3], b0.z, b0.w);
        add2(t[4], t[5], t[4], t[5], b1.x, b1.y);
        add2(t[6], t[7], t[6], t[7], b1.z, b1.w);
      }
      if (g) {
#pragma unroll
        for (int i = 0; i < 8; i += 2) gelu_fast2(t[i], t[i + 1]);
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) t[i] = zero ? 0.f : t[i];
      row[j ^ (lane & 7)] = make_uint4(pack_bf16x2(t[0], t[1]), pack_bf16x2(t[2], t[3]), pack_bf16x2(t[4], t[5]),
                                       pack_bf16x2(t[6], t[7]));
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_2d(map_c, tile, n0 + c * 64, r0);
      bulk_commit();
    }
  }
}

// ------------------------------------------------------ pairs of CTAs (2-SM MMA)
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// shared::cluster address of the same shared variable in CTA `rank` of the cluster
__device__ __forceinline__ uint32_t peer_addr(const void* p, uint32_t rank) {
  uint32_t a;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(smem_u32(p)), "r"(rank));
  return a;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// TMA load into this CTA's shared memory whose transaction bytes count on the
// barrier of the pair's first CTA (the one that issues the MMAs). Not a
// multicast: every CTA loads only its own operand halves.
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const void* map, uint32_t bar_cluster, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
      "%4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(x), "r"(y)
      : "memory");
}
// D[tmem of both CTAs] (+)= A[smem of both] * B[smem of both]^T, M = 256 over the pair.
__device__ __forceinline__ void umma_f16_ss_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                                 uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on `bar` in every CTA of `mask` once the pair's previously issued MMAs are done.
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          smem_u32(bar)),
      "h"(mask)
      : "memory");
}

// Epilogue instantiations: each keeps the whole register budget to itself.
enum EpiKind : int {
  EK_GENERIC = 0,   // per-thread stores (conv2 scatter + position table, projector scatter)
  EK_RESID = 1,     // fp32 residual via TMA reduce-add
  EK_STORE = 2,     // bf16 output via TMA store (plain rows, conv1)
  EK_POWER = 3,     // tf32 operands; out[r, k] = acc[r, 2k]^2 + acc[r, 2k+1]^2, split into tf32 planes
  EK_F32 = 4,       // tf32 operands; fp32 out[r, n] = acc (log-mel front end: the filterbank)
};
// a rounded to the nearest tf32 (10 fraction bits, ties to even); low 13 bits zero
__device__ __forceinline__ float round_tf32_dev(float a) {
  return __uint_as_float((__float_as_uint(a) + 0xFFFu + ((__float_as_uint(a) >> 13) & 1u)) & 0xFFFFE000u);
}

// D[tmem] (+)= A[smem] * B[smem]^T, kind::tf32 (fp32 operands read as tf32, fp32 accumulate).
__device__ __forceinline__ void umma_tf32_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor, kind::tf32: fp32 accumulator, tf32 A and B, both K-major.
__host__ __device__ constexpr uint32_t idesc_tf32_f32(int m, int n) {
  return (1u << 4)                                // D format: f32
         | (2u << 7)                              // A format: tf32
         | (2u << 10)                             // B format: tf32
         | (static_cast<uint32_t>(n >> 3) << 17)  // N / 8
         | (static_cast<uint32_t>(m >> 4) << 24); // M / 16
}
template <int BN, int kEpi>
__global__ void __launch_bounds__(kThreads, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
               const __grid_constant__ CUtensorMap map_c, const GemmTcParams p) {
  using C = TcCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::kStages * C::kABytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + C::kStages * C::kBBytes);
  uint64_t* empty = full + C::kStages;
  uint64_t* tfull = empty + C::kStages;    // [2] accumulator ready
  uint64_t* tempty = tfull + 2;            // [2] accumulator drained
  uint64_t* drain = tempty + 2;            // all MMAs of this CTA complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  float* stage_c = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(full) + 1024);   // [kEpiWarps][32 x 32]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(&tfull[a], 1); mbar_init(&tempty[a], kEpiWarps * 32); }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) { tma_prefetch_desc(&map_a); tma_prefetch_desc(&map_b); }
  if (warp == 1) { tmem_alloc(tmem_slot, C::kTmemCols); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  volatile int* abort_v = abort_flag;

  // producer lane: bit s of `armed` = ring slot s received a load, whose phase parity is bit s of armed_phase
  uint32_t armed = 0, armed_phase = 0;
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x) {
        const int m0 = (tile / p.tiles_n) * BM, n0 = (tile % p.tiles_n) * BN;
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_v, kWaitLimitNs)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[stage], C::kStageBytes);
          int ax, ay;
          a_coords(p, m0, kb, ax, ay);
          tma_load_2d(sA + stage * C::kABytes, &map_a, &full[stage], ax, ay);
          // a k-block is 128 bytes of K: 64 bf16 or 32 tf32 elements
          constexpr int kx = (kEpi == EK_POWER || kEpi == EK_F32) ? 32 : BK;
#pragma unroll
          for (int half_b = 0; half_b < BN / 128; ++half_b)   // weight maps use 128-row boxes
            tma_load_2d(sB + stage * C::kBBytes + half_b * (128 * BK * 2), &map_b, &full[stage], kb * kx,
                        n0 + half_b * 128);
          armed |= 1u << stage;
          armed_phase = (armed_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        set_status(p.status, kDevTimeout);
        *abort_v = 1;
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    // The whole warp walks the schedule and one elected lane issues and commits.
    constexpr bool kTf32 = kEpi == EK_POWER || kEpi == EK_F32;
    constexpr uint32_t idesc = kTf32 ? idesc_tf32_f32(BM, BN) : idesc_bf16_f32(BM, BN);
    const uint64_t adesc0 = smem_desc_sw128(smem_u32(sA)), bdesc0 = smem_desc_sw128(smem_u32(sB));
    int stage = 0, acc = 0;
    uint32_t phase = 0, acc_phase = 0;
    bool ok = true, issued = false;
    for (int tile = blockIdx.x; ok && tile < p.num_tiles; tile += gridDim.x) {
      if (!mbar_wait_warp(&tempty[acc], acc_phase ^ 1u, abort_v, kWaitLimitNs)) { ok = false; break; }
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
      for (int kb = 0; kb < p.num_kb; ++kb) {
        if (!mbar_wait_warp(&full[stage], phase, abort_v, kWaitLimitNs)) { ok = false; break; }
        tc_fence_after();
        // descriptor start addresses advance in 16-byte units
        const uint64_t adesc = adesc0 + static_cast<uint64_t>(stage) * (C::kABytes >> 4);
        const uint64_t bdesc = bdesc0 + static_cast<uint64_t>(stage) * (C::kBBytes >> 4);
        if (elect_one()) {
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {   // +32 bytes along K inside the swizzled row
            if constexpr (kTf32)
              umma_tf32_ss(d_tmem, adesc + static_cast<uint64_t>(2 * k), bdesc + static_cast<uint64_t>(2 * k),
                           idesc, (kb | k) != 0 ? 1u : 0u);
            else
              umma_f16_ss(d_tmem, adesc + static_cast<uint64_t>(2 * k), bdesc + static_cast<uint64_t>(2 * k),
                          idesc, (kb | k) != 0 ? 1u : 0u);
          }
          umma_commit(&empty[stage]);
        }
        __syncwarp();
        issued = true;
        if (++stage == C::kStages) { stage = 0; phase ^= 1u; }
      }
      if (!ok) break;
      if (elect_one()) umma_commit(&tfull[acc]);
      __syncwarp();
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    if (!ok && lane == 0) { set_status(p.status, kDevTimeout); *abort_v = 1; }
    if (issued) {   // every MMA done before TMEM is released
      if (elect_one()) umma_commit(drain);
      __syncwarp();
      mbar_wait_warp(drain, 0, nullptr, kWaitLimitNs);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    constexpr int NC = BN / 64;            // 32-column chunks per epilogue warp
    const int quarter = warp & 3;          // TMEM lanes this warp may read: 32*quarter ..
    const int half = (warp - 2) >> 2;      // which half of the tile's columns
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int tile = blockIdx.x; tile < p.num_tiles; tile += gridDim.x) {
      const int m0 = (tile / p.tiles_n) * BM, n0 = (tile % p.tiles_n) * BN + half * (BN / 2);
      if (!mbar_wait(&tfull[acc], acc_phase, abort_v, kWaitLimitNs)) {
        set_status(p.status, kDevTimeout);
        *abort_v = 1;
        break;
      }
      tc_fence_after();
      const int r = m0 + quarter * 32 + lane;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                             static_cast<uint32_t>(acc * BN + half * (BN / 2));
      if constexpr (kEpi == EK_RESID) {
        epi_residual_tile<NC>(p.epi, &map_c, m0 + quarter * 32, n0, taddr, stage_c + (warp - 2) * 32 * 32, lane);
      } else if constexpr (kEpi == EK_STORE) {
        epi_store_tile<NC / 2>(p.epi, &map_c, m0 + quarter * 32, n0, taddr,
                               reinterpret_cast<uint32_t*>(stage_c + (warp - 2) * 32 * 32), lane);
      } else if constexpr (kEpi == EK_POWER) {
        // columns 2k and 2k+1 hold the cos and sin parts of bin k: 16 bins per 32 columns
        float* prow = reinterpret_cast<float*>(p.epi.out) + (size_t)r * p.epi.ldo;
#pragma unroll 1
        for (int c = 0; c < NC; ++c) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(taddr + static_cast<uint32_t>(c * 32), v);
          tmem_wait_ld();
          const int k0 = (n0 + c * 32) >> 1;
          if (r < p.M && k0 < p.epi.ldo) {
#pragma unroll
            for (int i = 0; i < 16; i += 4) {
              float q[4];
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const float re = __uint_as_float(v[2 * (i + j)]), im = __uint_as_float(v[2 * (i + j) + 1]);
                q[j] = fmaf(re, re, im * im);
              }
              if (k0 + i < p.epi.ldo) {
                float hi[4], lo[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                  hi[j] = round_tf32_dev(q[j]);
                  lo[j] = q[j] - hi[j];
                }
                *reinterpret_cast<float4*>(prow + k0 + i) = make_float4(hi[0], hi[1], hi[2], hi[3]);
                *reinterpret_cast<float4*>(prow + (size_t)p.epi.P1 * p.epi.ldo + k0 + i) =
                    make_float4(lo[0], lo[1], lo[2], lo[3]);
              }
            }
          }
        }
      } else if constexpr (kEpi == EK_F32) {
        float* orow = reinterpret_cast<float*>(p.epi.out) + (size_t)r * p.epi.ldo;
#pragma unroll 1
        for (int c = 0; c < NC; ++c) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(taddr + static_cast<uint32_t>(c * 32), v);
          tmem_wait_ld();
          const int c0 = n0 + c * 32;
          if (r < p.M && c0 < p.epi.ldo) {
#pragma unroll
            for (int i = 0; i < 32; i += 4)
              if (c0 + i < p.epi.ldo)
                *reinterpret_cast<float4*>(orow + c0 + i) =
                    make_float4(__uint_as_float(v[i]), __uint_as_float(v[i + 1]), __uint_as_float(v[i + 2]),
                                __uint_as_float(v[i + 3]));
          }
        }
      } else {
        int dst = 0, pe_row = 0;
        bool zero = false;
        const bool row_ok = (r < p.M) && epi_row(p.epi, r, dst, pe_row, zero);
#pragma unroll 1
        for (int c = 0; c < NC; ++c) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(taddr + static_cast<uint32_t>(c * 32), v);
          tmem_wait_ld();
          if (row_ok)
            epi_apply_run<bf16, 32>(p.epi, dst, pe_row, zero, n0 + c * 32, reinterpret_cast<const float*>(v));
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    if constexpr (kEpi != EK_GENERIC && kEpi != EK_POWER && kEpi != EK_F32) {
      if (lane == 0) bulk_wait0();   // the bulk stores / reduces have landed
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0 && lane == 0 && *abort_v) {
    // a CTA that gave up may still have copies in flight (issued, never consumed):
    // let them land before its shared memory goes away
    for (int s = 0; s < C::kStages; ++s)
      if (armed & (1u << s)) mbar_wait(&full[s], (armed_phase >> s) & 1u, nullptr, kWaitLimitNs / 4);
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// Pair kernel: a cluster of two CTAs on two SMs computes 256 x 256 output tiles
// with tcgen05.mma.cta_group::2 (M = 256). CTA r of the pair holds rows
// 128r .. 128r+127 of the A tile and rows 128r .. 128r+127 of the B tile (half
// of the tile's columns) in a 6-stage ring of 32 KB per stage; the MMA reads
// both CTAs' halves. Against the single-CTA kernel each SM loads a third less
// operand data per MMA and keeps more stages in flight.
//   warp 0 (both CTAs)  TMA producer for the CTA's own halves; the bytes count
//                       on the first CTA's stage barrier.
//   warp 1 (first CTA)  MMA issuer; multicast commits free the stage in both
//                       CTAs and publish the accumulator to both epilogues.
//   warps 2..9 (both)   epilogue of the CTA's 128 rows, as in the single-CTA
//                       kernel; they release the accumulator on the first
//                       CTA's barrier.
// ---------------------------------------------------------------------------
constexpr int kPairStages = 6;

// Work units of the pair kernel: the p.num_tiles tiles of 256 x 256 in row-major
// tile order, except that the last p.tail tiles are each split into two units
// of 256 x 128 (their column halves). The launcher sets p.tail so that the last
// wave of a schedule that would run under half full instead runs twice as many
// units of half the work. Every output element still comes from one unit, with
// the same K order, so results do not depend on the split.
struct PairUnit {
  int m0, n0, width;   // rows m0 .. m0+255, columns n0 .. n0+width-1 (width 256 or 128)
};
__device__ __forceinline__ int pair_units(const GemmTcParams& p) { return p.num_tiles + p.tail; }
__device__ __forceinline__ PairUnit pair_unit(const GemmTcParams& p, int u) {
  const int nfull = p.num_tiles - p.tail;
  if (u < nfull) return {(u / p.tiles_n) * 256, (u % p.tiles_n) * 256, 256};
  const int h = u - nfull, tile = nfull + (h >> 1);
  return {(tile / p.tiles_n) * 256, (tile % p.tiles_n) * 256 + (h & 1) * 128, 128};
}

// Epilogue of one CTA's 128 rows of a unit: each epilogue warp drains its TMEM
// lane quarter over its half of the unit's columns (NC 32-column chunks).
template <int kEpi, int NC>
__device__ __forceinline__ void pair_epilogue(const GemmTcParams& p, const CUtensorMap* map_c, int m0, int n0,
                                              uint32_t taddr, float* stage, int lane, int quarter) {
  if constexpr (kEpi == EK_RESID) {
    epi_residual_tile<NC>(p.epi, map_c, m0 + quarter * 32, n0, taddr, stage, lane);
  } else if constexpr (kEpi == EK_STORE) {
    epi_store_tile<NC / 2>(p.epi, map_c, m0 + quarter * 32, n0, taddr, reinterpret_cast<uint32_t*>(stage), lane);
  } else {
    const int r = m0 + quarter * 32 + lane;
    int dst = 0, pe_row = 0;
    bool zero = false;
    const bool row_ok = (r < p.M) && epi_row(p.epi, r, dst, pe_row, zero);
#pragma unroll 1
    for (int c = 0; c < NC; ++c) {
      uint32_t v[32];
      tmem_ld_32x32b_x32(taddr + static_cast<uint32_t>(c * 32), v);
      tmem_wait_ld();
      if (row_ok) epi_apply_run<bf16, 32>(p.epi, dst, pe_row, zero, n0 + c * 32, reinterpret_cast<const float*>(v));
    }
  }
}
constexpr uint32_t kPairABytes = 128 * BK * 2;   // this CTA's 128 rows of A
constexpr uint32_t kPairBBytes = 128 * BK * 2;   // this CTA's 128 rows of B
constexpr size_t kPairSmemBytes = 1024 + kPairStages * (size_t)(kPairABytes + kPairBBytes) + 1024 +
                                  (size_t)kEpiWarps * 32 * 32 * 4;

template <int kEpi>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
gemm_tc2_kernel(const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
                const __grid_constant__ CUtensorMap map_c, const GemmTcParams p) {
  constexpr int BN = 256;
  constexpr uint32_t kTmemCols = 2 * BN;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + kPairStages * kPairABytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + kPairStages * kPairBBytes);   // used in the first CTA
  uint64_t* empty = full + kPairStages;
  uint64_t* tfull = empty + kPairStages;   // [2]
  uint64_t* tempty = tfull + 2;            // [2] used in the first CTA
  uint64_t* drain = tempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);
  float* stage_c = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(full) + 1024);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int cluster = blockIdx.x >> 1, nclusters = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPairStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    for (int a = 0; a < 2; ++a) { mbar_init(&tfull[a], 1); mbar_init(&tempty[a], 2 * kEpiWarps * 32); }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) { tma_prefetch_desc(&map_a); tma_prefetch_desc(&map_b); }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();   // both CTAs' barriers exist before any remote arrive or transaction
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  volatile int* abort_v = abort_flag;

  // producer lane: bit s of `armed` = ring slot s received a load, whose phase parity is bit s of armed_phase
  uint32_t armed = 0, armed_phase = 0;
  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int u = cluster; ok && u < pair_units(p); u += nclusters) {
        const PairUnit t = pair_unit(p, u);
        const int m0 = t.m0 + 128 * static_cast<int>(rank);
        // this CTA's half of the unit's weight rows; a 128-wide unit uses the
        // first 64 rows of each CTA's 128-row box (the rest is loaded and unused)
        const int n0 = t.n0 + (t.width / 2) * static_cast<int>(rank);
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_v, kWaitLimitNs)) { ok = false; break; }
          if (leader) mbar_arrive_expect_tx(&full[stage], 2 * (kPairABytes + kPairBBytes));
          const uint32_t bar = peer_addr(&full[stage], 0);
          int ax, ay;
          a_coords(p, m0, kb, ax, ay);
          tma_load_2d_pair(sA + stage * kPairABytes, &map_a, bar, ax, ay);
          tma_load_2d_pair(sB + stage * kPairBBytes, &map_b, bar, kb * BK, n0);
          armed |= 1u << stage;
          armed_phase = (armed_phase & ~(1u << stage)) | (phase << stage);
          if (++stage == kPairStages) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        set_status(p.status, kDevTimeout);
        *abort_v = 1;
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------- MMA issuer
    // first CTA only: the whole warp walks the schedule, one elected lane issues
    if (leader) {
      constexpr uint32_t idesc_full = idesc_bf16_f32(256, BN), idesc_half = idesc_bf16_f32(256, BN / 2);
      const uint64_t adesc0 = smem_desc_sw128(smem_u32(sA)), bdesc0 = smem_desc_sw128(smem_u32(sB));
      int stage = 0, acc = 0;
      uint32_t phase = 0, acc_phase = 0;
      bool ok = true, issued = false;
      for (int u = cluster; ok && u < pair_units(p); u += nclusters) {
        const uint32_t idesc = pair_unit(p, u).width == BN ? idesc_full : idesc_half;
        if (!mbar_wait_warp(&tempty[acc], acc_phase ^ 1u, abort_v, kWaitLimitNs)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = 0; kb < p.num_kb; ++kb) {
          if (!mbar_wait_warp(&full[stage], phase, abort_v, kWaitLimitNs)) { ok = false; break; }
          tc_fence_after();
          const uint64_t adesc = adesc0 + static_cast<uint64_t>(stage) * (kPairABytes >> 4);
          const uint64_t bdesc = bdesc0 + static_cast<uint64_t>(stage) * (kPairBBytes >> 4);
          if (elect_one()) {
#pragma unroll
            for (int k = 0; k < BK / 16; ++k)
              umma_f16_ss_pair(d_tmem, adesc + static_cast<uint64_t>(2 * k), bdesc + static_cast<uint64_t>(2 * k),
                               idesc, (kb | k) != 0 ? 1u : 0u);
            umma_commit_pair(&empty[stage], 0x3);
          }
          __syncwarp();
          issued = true;
          if (++stage == kPairStages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        if (elect_one()) umma_commit_pair(&tfull[acc], 0x3);
        __syncwarp();
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      if (!ok && lane == 0) { set_status(p.status, kDevTimeout); *abort_v = 1; }
      if (issued) {   // every MMA done before the pair's TMEM and shared memory go away
        if (elect_one()) umma_commit_pair(drain, 0x1);
        __syncwarp();
        mbar_wait_warp(drain, 0, nullptr, kWaitLimitNs);
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    constexpr int NC = BN / 64;            // 32-column chunks per epilogue warp
    const int quarter = warp & 3;
    const int half = (warp - 2) >> 2;
    const uint32_t tempty_leader[2] = {peer_addr(&tempty[0], 0), peer_addr(&tempty[1], 0)};
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int u = cluster; u < pair_units(p); u += nclusters) {
      const PairUnit t = pair_unit(p, u);
      const int m0 = t.m0 + 128 * static_cast<int>(rank);
      const int n0 = t.n0 + half * (t.width / 2);
      if (!mbar_wait(&tfull[acc], acc_phase, abort_v, kWaitLimitNs)) {
        set_status(p.status, kDevTimeout);
        *abort_v = 1;
        break;
      }
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                             static_cast<uint32_t>(acc * BN + half * (t.width / 2));
      float* stage = stage_c + (warp - 2) * 32 * 32;
      if (t.width == BN) pair_epilogue<kEpi, NC>(p, &map_c, m0, n0, taddr, stage, lane, quarter);
      else pair_epilogue<kEpi, NC / 2>(p, &map_c, m0, n0, taddr, stage, lane, quarter);
      tc_fence_before();
      mbar_arrive_cluster(tempty_leader[acc]);
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    if constexpr (kEpi != EK_GENERIC) {
      if (lane == 0) bulk_wait0();
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0 && lane == 0 && leader && *abort_v) {
    // the first CTA's stage barriers count both CTAs' copies: after a failure, let
    // every copy issued into the pair's rings land before either CTA leaves
    for (int s = 0; s < kPairStages; ++s)
      if (armed & (1u << s)) mbar_wait(&full[s], (armed_phase >> s) & 1u, nullptr, kWaitLimitNs / 4);
  }
  cluster_sync();   // no CTA leaves while its pair may still read its memory
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(kTmemCols)
                 : "memory");
  }
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  // looked up once, by whichever thread comes first (a function-local static
  // is initialised exactly once even when threads race for it)
  static const PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    return nullptr;
  }();
  return fn;
}

template <int BN, int kEpi>
bool configure_once() {
  static DeviceOnce once;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  return once.run(dev, [] {
    return cudaFuncSetAttribute(gemm_tc_kernel<BN, kEpi>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)TcCfg<BN>::kSmemBytes) == cudaSuccess;
  });
}

template <int BN, int kEpi>
cudaError_t launch_one(const CUtensorMap& map_a, const CUtensorMap& map_b, const CUtensorMap& map_c,
                       const GemmTcParams& p, int grid, cudaStream_t stream) {
  if (!configure_once<BN, kEpi>()) return cudaErrorInvalidValue;
  gemm_tc_kernel<BN, kEpi><<<grid, kThreads, TcCfg<BN>::kSmemBytes, stream>>>(map_a, map_b, map_c, p);
  return cudaGetLastError();
}

}  // namespace

int gemm_tile_n(int n) { return (n % 256 == 0) ? 256 : 128; }

bool make_tma_2d(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint64_t pitch_bytes,
                 uint32_t box_inner, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn || !base) return false;
  if ((reinterpret_cast<uintptr_t>(base) & 15u) || (pitch_bytes & 15u)) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {pitch_bytes};
  cuuint32_t box[2] = {box_inner, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_out_map(CUtensorMap* map, const void* out, uint64_t rows, uint64_t cols) {
  return make_tma_2d(map, out, cols, rows, cols * 2, 64, 32);
}

bool make_resid_map(CUtensorMap* map, const float* resid, uint64_t rows, uint64_t cols) {
  auto fn = encode_fn();
  if (!fn || !resid || (reinterpret_cast<uintptr_t>(resid) & 15u) || ((cols * 4) & 15u)) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 4};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(resid), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_tma_2d_f32(CUtensorMap* map, const void* base, uint64_t inner, uint64_t rows, uint64_t pitch_bytes,
                     uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn || !base) return false;
  if ((reinterpret_cast<uintptr_t>(base) & 15u) || (pitch_bytes & 15u)) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {pitch_bytes};
  cuuint32_t box[2] = {32, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_dft_power_tf32(const CUtensorMap& map_a, const CUtensorMap& map_b, GemmTcParams p, int sm_count,
                                  cudaStream_t stream) {
  if (p.M <= 0) return cudaSuccess;
  if (p.N % 128 || p.a_mode != A_DFT || !p.epi.out) return cudaErrorInvalidValue;
  p.tiles_n = p.N / 128;
  p.num_tiles = ((p.M + BM - 1) / BM) * p.tiles_n;
  const int grid = p.num_tiles < sm_count ? p.num_tiles : sm_count;
  return launch_one<128, EK_POWER>(map_a, map_b, map_a, p, grid, stream);
}

cudaError_t launch_gemm_tf32_f32out(const CUtensorMap& map_a, const CUtensorMap& map_b, GemmTcParams p,
                                    int sm_count, cudaStream_t stream) {
  if (p.M <= 0) return cudaSuccess;
  if (p.N % 128 || p.a_mode != A_SPLIT3 || !p.epi.out || p.epi.ldo % 4) return cudaErrorInvalidValue;
  p.tiles_n = p.N / 128;
  p.num_tiles = ((p.M + BM - 1) / BM) * p.tiles_n;
  const int grid = p.num_tiles < sm_count ? p.num_tiles : sm_count;
  return launch_one<128, EK_F32>(map_a, map_b, map_a, p, grid, stream);
}

template <int kEpi>
cudaError_t launch_pair(const CUtensorMap& map_a, const CUtensorMap& map_b, const CUtensorMap& map_c,
                        const GemmTcParams& p, int sm_count, cudaStream_t stream) {
  static DeviceOnce once;
  static int max_clusters[64] = {};   // written under once's mutex, read after its acquire
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidValue;
  cudaError_t setup_error = cudaSuccess;
  const bool ready = once.run(dev, [&] {
    cudaError_t e = cudaFuncSetAttribute(gemm_tc2_kernel<kEpi>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kPairSmemBytes);
    if (e != cudaSuccess) {
      setup_error = e;
      return false;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * (sm_count / 2), 1, 1);
    cfg.blockDim = dim3(kThreads, 1, 1);
    cfg.dynamicSmemBytes = kPairSmemBytes;
    cudaLaunchAttribute attr;
    attr.id = cudaLaunchAttributeClusterDimension;
    attr.val.clusterDim.x = 2;
    attr.val.clusterDim.y = 1;
    attr.val.clusterDim.z = 1;
    cfg.attrs = &attr;
    cfg.numAttrs = 1;
    int n = 0;
    e = cudaOccupancyMaxActiveClusters(&n, gemm_tc2_kernel<kEpi>, &cfg);
    if (e != cudaSuccess || n < 1) n = sm_count / 2;   // every SM pairs up
    cudaGetLastError();
    if (n < 1) {
      setup_error = cudaErrorInvalidValue;
      return false;
    }
    max_clusters[dev & 63] = n;
    return true;
  });
  if (!ready) return setup_error != cudaSuccess ? setup_error : cudaErrorInvalidValue;
  // a last wave that would run at most half full runs as two 128-wide halves per tile
  const int ncl = max_clusters[dev & 63];
  const int tail = p.num_tiles % ncl;
  GemmTcParams q = p;
  q.tail = (2 * tail <= ncl) ? tail : 0;
  const int units = q.num_tiles + q.tail;
  const int clusters = units < ncl ? units : ncl;
  gemm_tc2_kernel<kEpi><<<2 * clusters, kThreads, kPairSmemBytes, stream>>>(map_a, map_b, map_c, q);
  return cudaGetLastError();
}

cudaError_t launch_gemm_tc(const CUtensorMap& map_a, const CUtensorMap& map_b, GemmTcParams p, int sm_count,
                           cudaStream_t stream, const CUtensorMap* map_c) {
  if (p.M <= 0) return cudaSuccess;
  const int bn = gemm_tile_n(p.N);
  const bool resid = p.epi.mode == EPI_RESIDUAL;
  if (resid && !map_c) return cudaErrorInvalidValue;
  // bf16 row outputs go through TMA stores when the caller supplied the output map
  const bool store = !resid && map_c && (p.epi.mode == EPI_STORE || p.epi.mode == EPI_CONV1);
  const CUtensorMap& mc = map_c ? *map_c : map_a;
  p.tiles_n = p.N / bn;
  if (bn == 256) {   // 256 x 256 tiles on pairs of SMs
    p.num_tiles = ((p.M + 255) / 256) * p.tiles_n;
    if (resid) return launch_pair<EK_RESID>(map_a, map_b, mc, p, sm_count, stream);
    if (store) return launch_pair<EK_STORE>(map_a, map_b, mc, p, sm_count, stream);
    return launch_pair<EK_GENERIC>(map_a, map_b, mc, p, sm_count, stream);
  }
  p.num_tiles = ((p.M + BM - 1) / BM) * p.tiles_n;
  const int grid = p.num_tiles < sm_count ? p.num_tiles : sm_count;
  if (resid) return launch_one<128, EK_RESID>(map_a, map_b, mc, p, grid, stream);
  if (store) return launch_one<128, EK_STORE>(map_a, map_b, mc, p, grid, stream);
  return launch_one<128, EK_GENERIC>(map_a, map_b, mc, p, grid, stream);
}

}  // namespace enc
