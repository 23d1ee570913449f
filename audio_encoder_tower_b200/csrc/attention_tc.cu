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
// Work items of 128 query rows of one (clip, head); two CTAs share an SM, each
// taking a run of items, so one CTA's exponentials overlap the other's waits
// and a CTA's next item's loads overlap its current item. K/V stream in tiles
// of 96 keys; t below counts a CTA's key tiles across its items.
//   warp 0      TMA: an item's Q, then K_t and V_t into a 3-stage ring (128-byte swizzle).
//   warp 1      TMEM allocation; otherwise idle (it completes warpgroup 0 for
//               the register split).
//   warp 2      score issuer (whole warp, one elected lane): S_t = Q K_t^T
//               (M=128, N=96, K=64) goes to score buffer t%2, so S_{t+1} is
//               ready while the softmax works on S_t. S_{t+2} reuses that buffer
//               only after P_t V_t has completed.
//   warp 3      P V issuer (whole warp, one elected lane): O += P_t V_t reads P_t
//               from TMEM (A operand in tensor memory): the softmax writes P_t
//               (bf16) over the first 48 columns of S_t's own buffer.
//               The two issuers sit on two warp schedulers (warp w runs on
//               scheduler w % 4, beside softmax warp 4 + w % 4): issuing a
//               tile's ten MMAs from one warp held back the softmax warp that
//               shares its scheduler, and P V waits for the slowest softmax warp.
//   warps 4..7  softmax: one query row per thread (its TMEM lane), the whole
//               96-key score row in registers: exp2, row sum, P. The row's
//               maximum is taken once, over an item's first key tile, and kept: later
//               tiles need no max pass. A tile whose row sum exceeds 2^16 (a
//               score grew far past that maximum) is redone against its own
//               maximum, with O and l scaled down, after the previous P V has
//               completed. At the end O / l is stored as bf16.
// Registers: launched at 128 per thread (256 threads, two CTAs per SM); the
// control warpgroup drops to 56 and the softmax warpgroup rises to 200
// (setmaxnreg): 128*56 + 128*200 = 256*128.
//
// TMEM (256 columns per CTA): S0/P0 [0,96), S1/P1 [96,192), O [192,256).
#include <type_traits>

#include "common.cuh"
#include "internal.h"

namespace enc {

namespace {

constexpr int kQT = 128, kKT = 96, kHD = 64, kStages = 3;
constexpr int kThreads = 256;
// registers per thread: launch / control warpgroup / softmax warpgroup (setmaxnreg)
constexpr int kRegsLaunch = 128, kRegsLow = 56, kRegsHigh = 200;
static_assert(128 * kRegsLow + 128 * kRegsHigh == kThreads * kRegsLaunch, "register split must match the launch");
constexpr uint32_t kQBytes = kQT * kHD * 2;      // 16 KB
constexpr uint32_t kKVBytes = kKT * kHD * 2;     // 12 KB
constexpr uint32_t kTmemCols = 256;              // two CTAs share an SM's 512 columns
constexpr uint32_t kColS = 0, kColO = 2 * kKT;   // S buffers [0,96) [96,192), O [192,256)
constexpr uint64_t kWaitNs = 2000000000ull;
// A tile's exponentials are taken against the row maximum of the CTA's first key
// tile (held fixed); only a tile whose row sum exceeds this bound (or is not
// finite) moves the row to a new maximum, rescales O and redoes its exponentials.
// Every P is then <= 2^16: far from fp32 / bf16 overflow, and bf16 rounds
// relative to a value's own size, so the fixed maximum costs no precision.
constexpr float kSumLimit = 65536.0f;
#ifndef ENC_ATTN_POLY_OF8
#define ENC_ATTN_POLY_OF8 2
#endif
constexpr int kPolyOf8 = ENC_ATTN_POLY_OF8;      // of every 8 score pairs, this many take exp2_poly2
constexpr size_t kSmemBytes = 1024 + kQBytes + 2 * kStages * kKVBytes + 256;

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

__device__ __forceinline__ void tmem_ld_32x32b_x8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
}

__device__ __forceinline__ void tmem_st_32x32b_x8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
               "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }


// 2^x for two values on the FMA pipe (the MUFU unit is the softmax's bottleneck):
// Cody-Waite split x = n + f, n = round(x) (adding 1.5 * 2^23 rounds to an
// integer held in the low mantissa bits), f in [-1/2, 1/2]; 2^f by a cubic
// fitted here for least maximum relative error on [-1/2, 1/2] (7.5e-5, far
// below the bf16 rounding of P); 2^n enters through the exponent bits. x is
// clamped to [-126, 126] so the exponent never wraps (2^-126 is zero for P; a
// clamped 2^126 fails the tile's row-sum bound and the tile is redone).
__device__ __forceinline__ void exp2_poly2(float x0, float x1, float& y0, float& y1) {
  constexpr float kMagic = 12582912.0f;   // 1.5 * 2^23
  constexpr float c0 = 0.99992810936f, c1 = 0.69326098561f, c2 = 0.24261054228f, c3 = 0.05517132143f;
  x0 = fminf(fmaxf(x0, -126.0f), 126.0f);
  x1 = fminf(fmaxf(x1, -126.0f), 126.0f);
  float t0, t1, n0, n1, f0, f1, p0, p1;
  add2(t0, t1, x0, x1, kMagic, kMagic);
  add2(n0, n1, t0, t1, -kMagic, -kMagic);
  fma2(f0, f1, n0, n1, -1.0f, -1.0f, x0, x1);   // f = x - n
  fma2(p0, p1, f0, f1, c3, c3, c2, c2);
  fma2(p0, p1, p0, p1, f0, f1, c1, c1);
  fma2(p0, p1, p0, p1, f0, f1, c0, c0);
  // (bits of t) << 23 == n << 23 modulo 2^32: the 1.5 * 2^23 offset shifts out
  y0 = __uint_as_float(__float_as_uint(p0) + (__float_as_uint(t0) << 23));
  y1 = __uint_as_float(__float_as_uint(p1) + (__float_as_uint(t1) << 23));
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

// P = exp2(s * scale_log2 - m) for one 96-key score row (this thread's TMEM
// lane), written as bf16 pairs over the row's first 48 columns, 32 keys at a
// time; row sums into ps. kMasked zeroes keys >= kvalid (the clip's last key
// tile only, so full tiles carry no compare-and-select per key).
template <bool kMasked, int c>
__device__ __forceinline__ void softmax_exps_group(const uint32_t (&v)[kKT], uint32_t tS, float scale_log2,
                                                   float neg_m, int kvalid, float (&ps)[8]) {
  {
    uint32_t pk[16];
    if (kMasked && 32 * c >= kvalid) {   // 32 keys past the clip: P = 0 without exponentials
#pragma unroll
      for (int e = 0; e < 16; ++e) pk[e] = 0u;
      tmem_st_32x32b_x16(tS + static_cast<uint32_t>(16 * c), pk);
      return;
    }
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
      const int k = 32 * c + e;
      const int q = (e >> 1) & 3;
      float x0, x1, p0, p1;
      fma2(x0, x1, __uint_as_float(v[k]), __uint_as_float(v[k + 1]), scale_log2, scale_log2, neg_m, neg_m);
      if (((e >> 1) & 7) < kPolyOf8) {
        exp2_poly2(x0, x1, p0, p1);
      } else {
        p0 = ex2(x0);
        p1 = ex2(x1);
      }
      if constexpr (kMasked) {
        if (k >= kvalid) p0 = 0.f;
        if (k + 1 >= kvalid) p1 = 0.f;
      }
      add2(ps[2 * q], ps[2 * q + 1], ps[2 * q], ps[2 * q + 1], p0, p1);
      pk[e >> 1] = pack_bf16x2(p0, p1);
    }
    tmem_st_32x32b_x16(tS + static_cast<uint32_t>(16 * c), pk);
  }
}

template <bool kMasked>
__device__ __forceinline__ void softmax_exps(const uint32_t (&v)[kKT], uint32_t tS, float scale_log2, float neg_m,
                                             int kvalid, float (&ps)[8]) {
  softmax_exps_group<kMasked, 0>(v, tS, scale_log2, neg_m, kvalid, ps);
  softmax_exps_group<kMasked, 1>(v, tS, scale_log2, neg_m, kvalid, ps);
  softmax_exps_group<kMasked, 2>(v, tS, scale_log2, neg_m, kvalid, ps);
}

}  // namespace

// Work items: (segment b, head h, query tile qt), qt fastest, then h, then b
// (items of one clip and head run side by side, so their K/V stay in L2). A
// CTA takes items blockIdx.x, blockIdx.x + gridDim.x, ... (two CTAs per SM),
// so that its next item's Q and K/V loads and first scores overlap the
// current item's last tiles and output. Items whose query tile starts past the
// segment are skipped by every role alike.
struct AttnItem {
  int start, n, h, q0;
};
__device__ __forceinline__ AttnItem attn_item(const int* __restrict__ cu, int it, int H, int qtiles) {
  const int qt = it % qtiles, h = (it / qtiles) % H, b = it / (qtiles * H);
  const int start = cu[b];
  return {start, cu[b + 1] - start, h, qt * kQT};
}

__global__ void __launch_bounds__(kThreads, 2)
attention_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_kv,
                    bf16* __restrict__ out, const int* __restrict__ cu, int n_items, int H, int qtiles, int d,
                    float scale_log2, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = sQ + kQBytes;                     // kStages tiles of 96 keys
  uint8_t* sV = sK + kStages * kKVBytes;          // kStages tiles of 96 keys
  uint64_t* bars = reinterpret_cast<uint64_t*>(sV + kStages * kKVBytes);
  uint64_t* q_full = bars;                        // Q of the CTA's i-th item landed (phase i)
  uint64_t* q_empty = q_full + 1;                 // every S MMA of the i-th item complete: Q free
  uint64_t* kv_full = q_empty + 1;
  uint64_t* kv_empty = kv_full + kStages;
  uint64_t* s_full = kv_empty + kStages;          // [2] score buffer t%2 holds S_t (t: the CTA's tile count)
  uint64_t* p_full = s_full + 2;                  // [2] softmax read S_t and wrote P_t
  uint64_t* pv_done = p_full + 2;                 // [2] P_t V_t complete
  uint64_t* o_done = pv_done + 2;                 // every MMA of the i-th item complete: O final
  uint64_t* o_empty = o_done + 1;                 // the softmax has read O of the i-th item
  uint64_t* drain = o_empty + 1;                  // [2] every S MMA / every P V MMA of the CTA complete
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 2);
  int* abort_flag = reinterpret_cast<int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < kStages; ++s) { mbar_init(&kv_full[s], 1); mbar_init(&kv_empty[s], 1); }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&p_full[i], 128);
      mbar_init(&pv_done[i], 1);
    }
    mbar_init(o_done, 1);
    mbar_init(o_empty, 128);
    mbar_init(&drain[0], 1);
    mbar_init(&drain[1], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) { tma_prefetch_desc(&map_q); tma_prefetch_desc(&map_kv); }
  if (warp == 1) { tmem_alloc(tmem_slot, kTmemCols); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  volatile int* abort_v = abort_flag;
  // K/V tile t (counted over the CTA's items) sits in ring slot t % kStages,
  // filled for the (t / kStages)-th time; its scores use buffer t % 2
  auto slot = [](int t) { return t % kStages; };
  auto fill_parity = [](int t) { return static_cast<uint32_t>((t / kStages) & 1); };
  int armed_upto = 0, q_loads = 0;   // TMA lane: K/V tiles and Q tiles whose loads were issued

  if (warp < 4) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsLow));
    if (warp == 0 && lane == 0) {
      // ------------------------------------------------------------ TMA
      bool ok = true;
      for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x) {
        const AttnItem w = attn_item(cu, it, H, qtiles);
        if (w.q0 >= w.n) continue;
        // Q of the previous item is free once its S MMAs are complete
        if (q_loads > 0 && !mbar_wait(q_empty, (q_loads - 1) & 1, abort_v, kWaitNs)) { ok = false; break; }
        mbar_arrive_expect_tx(q_full, kQBytes);
        tma_load_2d(sQ, &map_q, q_full, w.h * kHD, w.start + w.q0);
        ++q_loads;
        const int nkv = (w.n + kKT - 1) / kKT;
        for (int j = 0; j < nkv; ++j) {
          const int t = armed_upto, st = slot(t);
          if (!mbar_wait(&kv_empty[st], fill_parity(t) ^ 1u, abort_v, kWaitNs)) { ok = false; break; }
          mbar_arrive_expect_tx(&kv_full[st], 2 * kKVBytes);
          tma_load_2d(sK + st * kKVBytes, &map_kv, &kv_full[st], d + w.h * kHD, w.start + j * kKT);
          tma_load_2d(sV + st * kKVBytes, &map_kv, &kv_full[st], 2 * d + w.h * kHD, w.start + j * kKT);
          armed_upto = t + 1;
        }
      }
      if (!ok) {
        set_status(status, kDevTimeout);
        *abort_v = 1;
      }
    } else if (warp == 2 || warp == 3) {
      // ------------------------------------------------------------ MMA
      // Two issuers on two schedulers: warp 2 issues the scores S_t, warp 3 the
      // products P_t V_t. The whole warp walks the schedule and one elected lane
      // issues, so the operands stay warp-uniform.
      constexpr uint32_t idesc_s = idesc_bf16_f32(128, kKT);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, kHD) | (1u << 16);   // B (V) MN-major
      constexpr uint64_t kSlotDesc = kKVBytes >> 4;   // one ring slot in descriptor address units
      auto wait_all = [&](uint64_t* bar, uint32_t parity) { return mbar_wait_warp(bar, parity, abort_v, kWaitNs); };
      const uint64_t qdesc = smem_desc_sw128(smem_u32(sQ));
      const uint64_t kdesc0 = smem_desc_sw128(smem_u32(sK));
      const uint64_t vdesc0 = smem_desc_sw128_mn(smem_u32(sV));
      const bool s_role = warp == 2;
      bool issued = false, ok = true;
      int t0 = 0, ic = 0;   // tiles and items of this CTA so far
      for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x) {
        const AttnItem w = attn_item(cu, it, H, qtiles);
        if (w.q0 >= w.n) continue;
        const int nkv = (w.n + kKT - 1) / kKT;
        if (s_role) {
          ok = wait_all(q_full, static_cast<uint32_t>(ic & 1));
          // S_t = Q K_t^T into buffer t % 2, after that buffer's previous P (tile t - 2)
          // has been read by its P V, and K_t has landed; the last S of an item frees Q
          for (int j = 0; ok && j < nkv; ++j) {
            const int t = t0 + j;
            const uint32_t bf = static_cast<uint32_t>(t & 1);
            if (t >= 2) ok = wait_all(&pv_done[bf], static_cast<uint32_t>(((t - 2) >> 1) & 1));
            if (ok) ok = wait_all(&kv_full[slot(t)], fill_parity(t));
            if (!ok) break;
            tc_fence_after();
            const uint64_t kdesc = kdesc0 + static_cast<uint64_t>(slot(t)) * kSlotDesc;
            if (elect_one()) {
#pragma unroll
              for (int k = 0; k < kHD / 16; ++k)
                umma_f16_ss(tmem + kColS + bf * kKT, qdesc + static_cast<uint64_t>(2 * k),
                            kdesc + static_cast<uint64_t>(2 * k), idesc_s, k > 0 ? 1u : 0u);
              umma_commit(&s_full[bf]);
              if (j == nkv - 1) umma_commit(q_empty);
            }
            __syncwarp();
            issued = true;
          }
        } else {
          for (int j = 0; ok && j < nkv; ++j) {
            const int t = t0 + j;
            const uint32_t bf = static_cast<uint32_t>(t & 1), use = static_cast<uint32_t>((t >> 1) & 1);
            // the softmax has read S_t (so S_t is complete) and written P_t
            ok = wait_all(&p_full[bf], use);
            // the item's first P V overwrites O: the softmax must have read the previous item's O
            if (ok && j == 0 && ic > 0) ok = wait_all(o_empty, static_cast<uint32_t>((ic - 1) & 1));
            if (!ok) break;
            tc_fence_after();
            // O += P_t V_t: P_t in the first 48 columns of buffer t % 2, 16 keys (8 columns) per step
            const uint64_t vdesc = vdesc0 + static_cast<uint64_t>(slot(t)) * kSlotDesc;
            if (elect_one()) {
#pragma unroll
              for (int k = 0; k < kKT / 16; ++k)
                umma_f16_ts(tmem + kColO, tmem + kColS + bf * kKT + static_cast<uint32_t>(8 * k),
                            vdesc + static_cast<uint64_t>(128 * k), idesc_pv, (j > 0 || k > 0) ? 1u : 0u);
              // K_t was read by S_t, complete before the softmax saw it; V_t by these MMAs
              umma_commit(&pv_done[bf]);
              umma_commit(&kv_empty[slot(t)]);
              if (j == nkv - 1) umma_commit(o_done);
            }
            __syncwarp();
            issued = true;
          }
        }
        t0 += nkv;
        ++ic;
      }
      if (!ok && lane == 0) { set_status(status, kDevTimeout); *abort_v = 1; }
      if (issued) {   // this warp's MMAs done before TMEM is released: this wait ignores the abort flag
        uint64_t* dr = &drain[s_role ? 0 : 1];
        if (elect_one()) umma_commit(dr);
        __syncwarp();
        mbar_wait_warp(dr, 0, nullptr, kWaitNs);
      }
    }
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsHigh));
    // ------------------------------------------------------------ softmax
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;    // query row inside the tile = TMEM lane
    const uint32_t lane_off = static_cast<uint32_t>(quarter * 32) << 16;
    const uint32_t tO = tmem + lane_off + kColO;
    bool ok = true;
    int t0 = 0, ic = 0;
    for (int it = blockIdx.x; ok && it < n_items; it += gridDim.x) {
      const AttnItem w = attn_item(cu, it, H, qtiles);
      if (w.q0 >= w.n) continue;
      const int n = w.n, nkv = (n + kKT - 1) / kKT;
      const int qrow = w.q0 + row;            // query row inside the segment
      float m_run = -INFINITY, l_run = 0.f;
      // a warp whose 32 query rows all lie past the segment (its last query tile)
      // computes nothing: its P rows only feed O rows that are never stored. It
      // still follows the score buffers' phases so that its arrivals count for
      // the right tile.
      const bool warp_idle = !__any_sync(0xffffffffu, qrow < n);
      for (int j = 0; j < nkv; ++j) {
        const int t = t0 + j;
        const int bf = t & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(&s_full[bf], (t >> 1) & 1u, abort_v, kWaitNs))) {
          ok = false;
          break;
        }
        if (warp_idle) {
          tc_fence_before();
          mbar_arrive(&p_full[bf]);
          continue;
        }
        tc_fence_after();
        const uint32_t tS = tmem + lane_off + kColS + static_cast<uint32_t>(bf * kKT);
        uint32_t v[kKT];
        auto load_group = [&](int c) {
          tmem_ld_32x32b_x32(tS + static_cast<uint32_t>(32 * c), *reinterpret_cast<uint32_t(*)[32]>(&v[32 * c]));
        };
        const int kvalid = n - j * kKT;       // keys of this tile inside the segment
        const bool full = kvalid >= kKT;
#pragma unroll
        for (int c = 0; c < kKT / 32; ++c) load_group(c);
        tmem_wait_ld();
        // row maximum of this tile's valid scores, in log2 units
        auto tile_max = [&]() {
          float pm[8];   // eight independent partial maxima, then a tree
#pragma unroll
          for (int q = 0; q < 8; ++q) pm[q] = -INFINITY;
          if (full) {
#pragma unroll
            for (int e = 0; e < kKT; ++e) pm[e & 7] = fmaxf(pm[e & 7], __uint_as_float(v[e]));
          } else {
#pragma unroll
            for (int e = 0; e < kKT; ++e)
              if (e < kvalid) pm[e & 7] = fmaxf(pm[e & 7], __uint_as_float(v[e]));
          }
          return scale_log2 * fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])),
                                    fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
        };
        // P = exp2(s * scale_log2 - m) as bf16 pairs over the first 48 columns of
        // this score buffer; only the segment's last key tile takes the masked copy
        auto exps = [&]() {
          float ps[8];   // eight independent partial row sums (four packed pairs)
#pragma unroll
          for (int q = 0; q < 8; ++q) ps[q] = 0.f;
          if (full) {
            softmax_exps<false>(v, tS, scale_log2, -m_run, kvalid, ps);
          } else {
            softmax_exps<true>(v, tS, scale_log2, -m_run, kvalid, ps);
          }
          return ((ps[0] + ps[1]) + (ps[2] + ps[3])) + ((ps[4] + ps[5]) + (ps[6] + ps[7]));
        };
        if (j == 0) m_run = tile_max();       // the first tile fixes the row's maximum
        float lt = exps();
        const bool over = !(lt <= kSumLimit);  // also true for an infinite sum
        if (__any_sync(0xffffffffu, over)) {
          // rare: a row whose scores grew far past its maximum moves to the tile's
          // maximum, O and l are scaled down to it, and the tile is redone (the
          // other rows of the warp recompute the same P: TMEM stores are collective)
          float alpha = 1.f;
          if (over) {
            const float m_new = fmaxf(m_run, tile_max());
            alpha = ex2(m_run - m_new);
            m_run = m_new;
            l_run *= alpha;
          }
          lt = exps();
          // O must hold P_{t-1} V_{t-1} before it is scaled (the item's first tile has no O yet)
          if (j > 0 && !__all_sync(0xffffffffu, mbar_wait(&pv_done[(t - 1) & 1], ((t - 1) >> 1) & 1u, abort_v,
                                                            kWaitNs))) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; j > 0 && c < kHD / 8; ++c) {   // 8 columns at a time: the score row is still in registers
            uint32_t o[8];
            tmem_ld_32x32b_x8(tO + static_cast<uint32_t>(8 * c), o);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 8; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
            tmem_st_32x32b_x8(tO + static_cast<uint32_t>(8 * c), o);
          }
        }
        l_run += lt;
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&p_full[bf]);
      }
      if (ok && !__all_sync(0xffffffffu, mbar_wait(o_done, static_cast<uint32_t>(ic & 1), abort_v, kWaitNs)))
        ok = false;
      if (!__all_sync(0xffffffffu, ok)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const float inv = 1.f / l_run;
      const bool valid = qrow < n;
      bf16* orow = out + (size_t)(w.start + qrow) * d + w.h * kHD;
#pragma unroll
      for (int c = 0; !warp_idle && c < kHD / 32; ++c) {
        uint32_t o[32];
        tmem_ld_32x32b_x32(tO + static_cast<uint32_t>(32 * c), o);
        tmem_wait_ld();
        if (valid) {
#pragma unroll
          for (int e = 0; e < 32; e += 8) {
            uint4 u;
            u.x = pack_bf16x2(__uint_as_float(o[e]) * inv, __uint_as_float(o[e + 1]) * inv);
            u.y = pack_bf16x2(__uint_as_float(o[e + 2]) * inv, __uint_as_float(o[e + 3]) * inv);
            u.z = pack_bf16x2(__uint_as_float(o[e + 4]) * inv, __uint_as_float(o[e + 5]) * inv);
            u.w = pack_bf16x2(__uint_as_float(o[e + 6]) * inv, __uint_as_float(o[e + 7]) * inv);
            *reinterpret_cast<uint4*>(orow + 32 * c + e) = u;
          }
        }
      }
      tc_fence_before();
      mbar_arrive(o_empty);   // O of this item read: the next item's first P V may overwrite it
      t0 += nkv;
      ++ic;
    }
    if (!ok) {
      set_status(status, kDevTimeout);
      *abort_v = 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0 && lane == 0 && *abort_v) {
    // a CTA that gave up may still have copies in flight (issued before the
    // failure, never consumed): let them land before its shared memory goes away
    if (q_loads > 0) mbar_wait(q_full, (q_loads - 1) & 1, nullptr, kWaitNs / 4);
    for (int t = armed_upto - kStages; t < armed_upto; ++t)
      if (t >= 0) mbar_wait(&kv_full[slot(t)], fill_parity(t), nullptr, kWaitNs / 4);
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

bool make_qkv_maps(QkvMaps* maps, const void* qkv, int rows, int d) {
  return make_tma_2d(&maps->q, qkv, 3 * (uint64_t)d, (uint64_t)rows, 6 * (uint64_t)d, 64, kQT) &&
         make_tma_2d(&maps->kv, qkv, 3 * (uint64_t)d, (uint64_t)rows, 6 * (uint64_t)d, 64, kKT);
}

cudaError_t launch_attention_tc(const QkvMaps& maps, bf16* out, const int* cu, int B, int max_n, int d, int H,
                                int* status, cudaStream_t stream) {
  if (B <= 0 || max_n <= 0) return cudaSuccess;
  static DeviceOnce once;
  static int sm_count[64] = {};   // written under once's mutex, read after its acquire
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidValue;
  cudaError_t setup_error = cudaSuccess;
  const bool ready = once.run(dev, [&] {
    // setmaxnreg redistributes the registers the CTA was launched with: refuse to
    // launch unless the compiled kernel holds exactly the planned count per thread
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, attention_tc_kernel);
    if (e == cudaSuccess && fa.numRegs != kRegsLaunch) e = cudaErrorInvalidConfiguration;
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(attention_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemBytes);
    int n = 0;
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess && n < 1) e = cudaErrorInvalidValue;
    if (e != cudaSuccess) {
      setup_error = e;
      return false;
    }
    sm_count[dev & 63] = n;
    return true;
  });
  if (!ready) return setup_error != cudaSuccess ? setup_error : cudaErrorInvalidValue;
  const int qtiles = (max_n + kQT - 1) / kQT;
  const long long items = (long long)B * H * qtiles;
  if (items > 0x7fffffffLL) return cudaErrorInvalidValue;
  // two CTAs per SM, each taking a run of items: a CTA's next Q and K/V loads and
  // first scores overlap its current item's last tiles and output
  const long long resident = 2LL * sm_count[dev & 63];
  const int grid = items > resident ? (int)resident : (int)items;
  attention_tc_kernel<<<grid, kThreads, kSmemBytes, stream>>>(maps.q, maps.kv, out, cu, (int)items, H, qtiles, d,
                                                              0.125f * 1.4426950408889634f, status);
  return cudaGetLastError();
}

}  // namespace enc
