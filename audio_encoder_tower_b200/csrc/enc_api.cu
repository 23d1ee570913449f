// C ABI of the encoder tower: argument checks, weight repacking, workspace,
// tensor maps, and the stream-ordered launch sequence of one forward pass.
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <vector>

#include <nvtx3/nvToolsExt.h>

#include "../../include/enc.h"
#include "../../include/enc_profile.h"
#include "common.cuh"
#include "internal.h"

using namespace enc;

namespace {

inline int ceil_div(int a, int b) { return (a + b - 1) / b; }
inline int round_up(int a, int b) { return ceil_div(a, b) * b; }

struct LayerMaps {
  CUtensorMap qkv, o, fc1, fc2;
};

}  // namespace

struct enc_handle {
  enc_config cfg;
  int device = 0, sm_count = 0;
  bool bf16 = true;
  size_t esz = 2;            // bytes per element of cfg.dtype
  // geometry
  int T = 0, Tp = 0, P = 0, P1 = 0, p_out = 0, d_out = 0, mpad = 0;
  // allocations (all library-owned)
  std::vector<void*> allocs;
  size_t bytes = 0;
  int alloc_calls = 0;       // device allocations attempted (ENC_FAIL_ALLOC test hook)
  // ENC_FLAG_GUARD: guard regions around every workspace buffer
  struct Guard { const char* name; unsigned char* buf; size_t bytes; };
  std::vector<Guard> guards;
  // enc_forward_static_scratch: device address of the library's static workspace
  // on this handle's device, resolved in enc_create (nullptr when that failed)
  unsigned char* static_scratch = nullptr;
  enc_status static_scratch_status = ENC_ERR_CUDA;
  // repacked weights
  void* conv1_w = nullptr;   // [d, 3, mpad] (bf16) or [d, 3, n_mels] (fp32)
  void* conv2_w = nullptr;   // [d, 3, d]
  float *conv1_b = nullptr, *conv2_b = nullptr, *pe = nullptr;
  std::vector<void*> qkv_w, o_w, fc1_w, fc2_w;                 // per layer
  std::vector<float*> qkv_b, o_b, fc1_b, fc2_b, ln1_g, ln1_b, ln2_g, ln2_b;
  float *lnpost_g = nullptr, *lnpost_b = nullptr;
  void *proj1_w = nullptr, *proj2_w = nullptr;
  float *proj1_b = nullptr, *proj2_b = nullptr;
  // workspace
  void* melT = nullptr;      // [2 + max_batch * Tp, n_mels]; data starts one row in
  void* y1 = nullptr;        // [max_batch * Tp + 2, d]
  float* x = nullptr;        // [max_batch * P, d] residual stream
  void *a = nullptr, *qkv = nullptr, *o = nullptr, *f = nullptr, *e = nullptr, *p1 = nullptr;
  int* meta = nullptr;       // device [cu (B+1) | cu_out (B+1) | len (B) | cu_attn (segments+1)]
  int meta_ints = 0;         // capacity of meta / h_meta
  int* h_meta = nullptr;     // pinned host staging of meta
  int* status = nullptr;     // device status word
  cudaEvent_t meta_free = nullptr;
  bool meta_pending = false;
  // tensor maps (bf16 path)
  CUtensorMap m_conv1_a, m_conv2_a, m_a, m_o, m_f, m_e, m_p1, m_x;
  CUtensorMap m_out_y1, m_out_qkv, m_out_f, m_out_p1;   // bf16 outputs written by TMA stores
  QkvMaps m_qkv;
  CUtensorMap m_conv1_w, m_conv2_w, m_proj1_w, m_proj2_w;
  std::vector<LayerMaps> lmaps;
  // profiling
  bool profile = false;
  int64_t launches = 0;
  struct Rec { int cls; cudaEvent_t a, b; double flops; };
  std::vector<Rec> recs;
  std::vector<cudaEvent_t> event_pool;
};

namespace {

enc_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return ENC_OK;
  if (e == cudaErrorMemoryAllocation) return ENC_ERR_OOM;
  return ENC_ERR_CUDA;
}

#define ENC_TRY(expr)                                       \
  do {                                                      \
    cudaError_t _e = (expr);                                \
    if (_e != cudaSuccess) return cuda_status(_e);          \
  } while (0)

template <typename P>
enc_status dev_alloc(enc_handle* h, P** out, size_t bytes) {
  void* p = nullptr;
  if (bytes == 0) bytes = 16;
  // Test hook: ENC_FAIL_ALLOC=N makes the handle's N-th device allocation (1-based,
  // counted per handle, so every enc_create starts again at 1) report failure.
  ++h->alloc_calls;
  const char* env = getenv("ENC_FAIL_ALLOC");
  if (env && atoi(env) > 0 && h->alloc_calls == atoi(env)) return ENC_ERR_OOM;
  cudaError_t e = cudaMalloc(&p, bytes);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return ENC_ERR_OOM;
  }
  h->allocs.push_back(p);
  h->bytes += bytes;
  *out = reinterpret_cast<P*>(p);
  return ENC_OK;
}

#define ENC_CHECK(expr)                        \
  do {                                         \
    enc_status _s = (expr);                    \
    if (_s != ENC_OK) return _s;               \
  } while (0)

constexpr size_t kGuardBytes = 256u << 10;   // each side of a guarded workspace buffer
constexpr unsigned char kGuardByte = 0xA5;

// A workspace buffer of the handle. With ENC_FLAG_GUARD it sits between two
// guard regions of kGuardBytes filled with kGuardByte (the buffer keeps 256-byte
// alignment); enc_check_guards reads them back.
template <typename P>
enc_status ws_alloc(enc_handle* h, P** out, size_t bytes, const char* name) {
  if (!(h->cfg.flags & ENC_FLAG_GUARD)) return dev_alloc(h, out, bytes);
  const size_t inner = (bytes + 255) & ~size_t(255);
  unsigned char* base = nullptr;
  ENC_CHECK(dev_alloc(h, &base, inner + 2 * kGuardBytes));
  if (cudaMemset(base, kGuardByte, kGuardBytes) != cudaSuccess ||
      cudaMemset(base + kGuardBytes + inner, kGuardByte, kGuardBytes) != cudaSuccess)
    return ENC_ERR_CUDA;
  h->guards.push_back({name, base + kGuardBytes, inner});
  *out = reinterpret_cast<P*>(base + kGuardBytes);
  return ENC_OK;
}

void free_all(enc_handle* h) {
  for (void* p : h->allocs) cudaFree(p);
  h->allocs.clear();
  if (h->h_meta) cudaFreeHost(h->h_meta);
  h->h_meta = nullptr;
  if (h->meta_free) cudaEventDestroy(h->meta_free);
  h->meta_free = nullptr;
  for (auto& r : h->recs) { cudaEventDestroy(r.a); cudaEventDestroy(r.b); }
  h->recs.clear();
  for (cudaEvent_t e : h->event_pool) cudaEventDestroy(e);
  h->event_pool.clear();
}

}  // namespace

enc_status enc::validate_config(const enc_config* c) {
  if (!c) return ENC_ERR_INVALID_ARG;
  if (c->flags & ~ENC_FLAG_GUARD) return ENC_ERR_INVALID_ARG;
  if (c->dtype != ENC_DTYPE_BF16 && c->dtype != ENC_DTYPE_FP32) return ENC_ERR_INVALID_ARG;
  if (c->n_mels <= 0 || c->d_model <= 0 || c->n_layers < 0 || c->n_heads <= 0 || c->ffn_dim <= 0 ||
      c->max_frames <= 0 || c->max_batch <= 0)
    return ENC_ERR_INVALID_ARG;
  if (c->pool_step != 1 && c->pool_step != 2 && c->pool_step != 4) return ENC_ERR_UNSUPPORTED;
  if (c->head_dim != 64 || c->n_heads * c->head_dim != c->d_model) return ENC_ERR_UNSUPPORTED;
  if (c->d_model % 128 || c->d_model > 2048) return ENC_ERR_UNSUPPORTED;
  if (c->ffn_dim % 128) return ENC_ERR_UNSUPPORTED;
  if (c->n_mels % 8 || c->n_mels > 256) return ENC_ERR_UNSUPPORTED;
  if (c->proj_hidden < 0 || c->proj_out < 0) return ENC_ERR_INVALID_ARG;
  if (c->proj_hidden && (c->proj_hidden % 128 || c->proj_out <= 0 || c->proj_out % 128)) return ENC_ERR_UNSUPPORTED;
  if (!(c->ln_eps > 0.f)) return ENC_ERR_INVALID_ARG;
  // block-local attention: every chunk is one attention segment (grid z <= 65535)
  if (c->attn_chunk < 0) return ENC_ERR_INVALID_ARG;
  if (c->attn_chunk > 0) {
    const long long p = (c->max_frames + 1) / 2;
    if ((long long)c->max_batch * ((p + c->attn_chunk - 1) / c->attn_chunk) > 65535) return ENC_ERR_UNSUPPORTED;
  }
  // index arithmetic stays in 32 bits
  const long long rows = (long long)c->max_batch * (c->max_frames + 4);
  if (rows * (long long)(3 * c->d_model > c->ffn_dim ? 3 * c->d_model : c->ffn_dim) > (1ll << 31) - 1)
    return ENC_ERR_UNSUPPORTED;
  return ENC_OK;
}

namespace {

// Copy `n` elements (cfg dtype) device to device into fresh library memory.
enc_status copy_weight(enc_handle* h, const void* src, size_t n, void** dst) {
  if (!src) return ENC_ERR_INVALID_ARG;
  ENC_CHECK(dev_alloc(h, dst, n * h->esz));
  ENC_TRY(cudaMemcpy(*dst, src, n * h->esz, cudaMemcpyDeviceToDevice));
  return ENC_OK;
}

enc_status to_f32(enc_handle* h, const void* src, int n, float fill, float** dst) {
  ENC_CHECK(dev_alloc(h, dst, (size_t)n * 4));
  ENC_TRY(launch_to_f32(src, h->bf16, *dst, n, fill, 0));
  return ENC_OK;
}

bool map_rows(CUtensorMap* m, const void* base, int inner, long long rows, int box_rows) {
  return make_tma_2d(m, base, (uint64_t)inner, (uint64_t)rows, (uint64_t)inner * 2, 64, (uint32_t)box_rows);
}

enc_status build(enc_handle* h, const enc_weights* w) {
  const enc_config& c = h->cfg;
  const int d = c.d_model, F = c.ffn_dim, L = c.n_layers, M = c.n_mels, Bm = c.max_batch;
  // ---- weights
  if (!w->conv1_w || !w->conv2_w) return ENC_ERR_INVALID_ARG;
  h->mpad = h->bf16 ? round_up(M, 64) : M;
  ENC_CHECK(dev_alloc(h, &h->conv1_w, (size_t)d * 3 * h->mpad * h->esz));
  ENC_TRY(launch_conv_repack(w->conv1_w, h->bf16, h->conv1_w, h->bf16, d, M, h->mpad, 0));
  ENC_CHECK(dev_alloc(h, &h->conv2_w, (size_t)d * 3 * d * h->esz));
  ENC_TRY(launch_conv_repack(w->conv2_w, h->bf16, h->conv2_w, h->bf16, d, d, d, 0));
  ENC_CHECK(to_f32(h, w->conv1_b, d, 0.f, &h->conv1_b));
  ENC_CHECK(to_f32(h, w->conv2_b, d, 0.f, &h->conv2_b));
  if (L > 0 && (!w->ln1_g || !w->ln1_b || !w->q_w || !w->q_b || !w->k_w || !w->v_w || !w->v_b || !w->o_w ||
                !w->o_b || !w->ln2_g || !w->ln2_b || !w->fc1_w || !w->fc1_b || !w->fc2_w || !w->fc2_b))
    return ENC_ERR_INVALID_ARG;
  h->qkv_w.resize(L); h->o_w.resize(L); h->fc1_w.resize(L); h->fc2_w.resize(L);
  h->qkv_b.resize(L); h->o_b.resize(L); h->fc1_b.resize(L); h->fc2_b.resize(L);
  h->ln1_g.resize(L); h->ln1_b.resize(L); h->ln2_g.resize(L); h->ln2_b.resize(L);
  const size_t dd = (size_t)d * d;
  for (int l = 0; l < L; ++l) {
    if (!w->q_w[l] || !w->k_w[l] || !w->v_w[l] || !w->o_w[l] || !w->fc1_w[l] || !w->fc2_w[l])
      return ENC_ERR_INVALID_ARG;
    ENC_CHECK(dev_alloc(h, &h->qkv_w[l], 3 * dd * h->esz));
    uint8_t* q = reinterpret_cast<uint8_t*>(h->qkv_w[l]);
    ENC_TRY(cudaMemcpy(q, w->q_w[l], dd * h->esz, cudaMemcpyDeviceToDevice));
    ENC_TRY(cudaMemcpy(q + dd * h->esz, w->k_w[l], dd * h->esz, cudaMemcpyDeviceToDevice));
    ENC_TRY(cudaMemcpy(q + 2 * dd * h->esz, w->v_w[l], dd * h->esz, cudaMemcpyDeviceToDevice));
    ENC_CHECK(dev_alloc(h, &h->qkv_b[l], 3 * (size_t)d * 4));
    ENC_TRY(launch_to_f32(w->q_b[l], h->bf16, h->qkv_b[l], d, 0.f, 0));
    // a key bias shifts every score of a query row equally and cancels in softmax: k runs unbiased
    ENC_TRY(launch_to_f32(nullptr, h->bf16, h->qkv_b[l] + d, d, 0.f, 0));
    ENC_TRY(launch_to_f32(w->v_b[l], h->bf16, h->qkv_b[l] + 2 * d, d, 0.f, 0));
    ENC_CHECK(copy_weight(h, w->o_w[l], dd, &h->o_w[l]));
    ENC_CHECK(copy_weight(h, w->fc1_w[l], (size_t)F * d, &h->fc1_w[l]));
    ENC_CHECK(copy_weight(h, w->fc2_w[l], (size_t)d * F, &h->fc2_w[l]));
    ENC_CHECK(to_f32(h, w->o_b[l], d, 0.f, &h->o_b[l]));
    ENC_CHECK(to_f32(h, w->fc1_b[l], F, 0.f, &h->fc1_b[l]));
    ENC_CHECK(to_f32(h, w->fc2_b[l], d, 0.f, &h->fc2_b[l]));
    ENC_CHECK(to_f32(h, w->ln1_g[l], d, 1.f, &h->ln1_g[l]));
    ENC_CHECK(to_f32(h, w->ln1_b[l], d, 0.f, &h->ln1_b[l]));
    ENC_CHECK(to_f32(h, w->ln2_g[l], d, 1.f, &h->ln2_g[l]));
    ENC_CHECK(to_f32(h, w->ln2_b[l], d, 0.f, &h->ln2_b[l]));
  }
  ENC_CHECK(to_f32(h, w->lnpost_g, d, 1.f, &h->lnpost_g));
  ENC_CHECK(to_f32(h, w->lnpost_b, d, 0.f, &h->lnpost_b));
  const int ph = c.proj_hidden, po = c.proj_out;
  if (ph) {
    ENC_CHECK(copy_weight(h, w->proj1_w, (size_t)ph * d, &h->proj1_w));
    ENC_CHECK(copy_weight(h, w->proj2_w, (size_t)po * ph, &h->proj2_w));
    ENC_CHECK(to_f32(h, w->proj1_b, ph, 0.f, &h->proj1_b));
    ENC_CHECK(to_f32(h, w->proj2_b, po, 0.f, &h->proj2_b));
  }
  // ---- position table
  ENC_CHECK(dev_alloc(h, &h->pe, (size_t)h->P * d * 4));
  ENC_TRY(launch_position_table(h->pe, h->P, d, 0));
  // ---- workspace
  const long long rows_t = (long long)Bm * h->Tp, rows_p = (long long)Bm * h->P, rows_o = (long long)Bm * h->p_out;
  ENC_CHECK(ws_alloc(h, &h->melT, (size_t)(rows_t + 2) * M * h->esz, "melT"));
  ENC_CHECK(ws_alloc(h, &h->y1, (size_t)(rows_t + 2) * d * h->esz, "y1"));
  ENC_TRY(cudaMemset(h->melT, 0, (size_t)(rows_t + 2) * M * h->esz));
  ENC_TRY(cudaMemset(h->y1, 0, (size_t)(rows_t + 2) * d * h->esz));
  ENC_CHECK(ws_alloc(h, &h->x, (size_t)rows_p * d * 4, "x"));
  ENC_CHECK(ws_alloc(h, &h->a, (size_t)rows_p * d * h->esz, "a"));
  ENC_CHECK(ws_alloc(h, &h->qkv, (size_t)rows_p * 3 * d * h->esz, "qkv"));
  ENC_CHECK(ws_alloc(h, &h->o, (size_t)rows_p * d * h->esz, "o"));
  ENC_CHECK(ws_alloc(h, &h->f, (size_t)rows_p * F * h->esz, "f"));
  if (ph) {
    ENC_CHECK(ws_alloc(h, &h->e, (size_t)rows_o * d * h->esz, "e"));
    ENC_CHECK(ws_alloc(h, &h->p1, (size_t)rows_o * ph * h->esz, "p1"));
  }
  ENC_TRY(cudaMemset(h->x, 0, (size_t)rows_p * d * 4));
  ENC_TRY(cudaMemset(h->a, 0, (size_t)rows_p * d * h->esz));
  ENC_TRY(cudaMemset(h->qkv, 0, (size_t)rows_p * 3 * d * h->esz));
  ENC_TRY(cudaMemset(h->o, 0, (size_t)rows_p * d * h->esz));
  ENC_TRY(cudaMemset(h->f, 0, (size_t)rows_p * F * h->esz));
  // block-local attention adds the chunk boundaries: at most ceil(P / chunk) per clip
  h->meta_ints = 3 * Bm + 2 + (c.attn_chunk > 0 ? Bm * ((h->P + c.attn_chunk - 1) / c.attn_chunk) + 1 : 0);
  ENC_CHECK(ws_alloc(h, &h->meta, (size_t)h->meta_ints * 4, "meta"));
  ENC_CHECK(ws_alloc(h, &h->status, 4, "status"));
  ENC_TRY(cudaMemset(h->status, 0, 4));
  if (cudaMallocHost(&h->h_meta, (size_t)h->meta_ints * 4) != cudaSuccess) {
    cudaGetLastError();
    h->h_meta = nullptr;
    return ENC_ERR_OOM;
  }
  ENC_TRY(cudaEventCreateWithFlags(&h->meta_free, cudaEventDisableTiming));
  // ---- tensor maps (tensor-core path)
  if (h->bf16) {
    const uint8_t* melT_data = reinterpret_cast<const uint8_t*>(h->melT) + (size_t)M * 2;
    bool ok = map_rows(&h->m_conv1_a, melT_data, M, rows_t, 128);
    ok = ok && make_tma_2d(&h->m_conv2_a, h->y1, 2 * (uint64_t)d, (uint64_t)rows_t / 2, 4 * (uint64_t)d, 64, 128);
    ok = ok && map_rows(&h->m_a, h->a, d, rows_p, 128);
    ok = ok && map_rows(&h->m_o, h->o, d, rows_p, 128);
    ok = ok && map_rows(&h->m_f, h->f, F, rows_p, 128);
    ok = ok && make_qkv_maps(&h->m_qkv, h->qkv, (int)rows_p, d);
    ok = ok && make_resid_map(&h->m_x, h->x, (uint64_t)rows_p, (uint64_t)d);
    ok = ok && make_out_map(&h->m_out_y1, h->y1, (uint64_t)rows_t, (uint64_t)d);
    ok = ok && make_out_map(&h->m_out_qkv, h->qkv, (uint64_t)rows_p, 3 * (uint64_t)d);
    ok = ok && make_out_map(&h->m_out_f, h->f, (uint64_t)rows_p, (uint64_t)F);
    ok = ok && map_rows(&h->m_conv1_w, h->conv1_w, 3 * h->mpad, d, 128);
    ok = ok && map_rows(&h->m_conv2_w, h->conv2_w, 3 * d, d, 128);
    if (ph) {
      ok = ok && map_rows(&h->m_e, h->e, d, rows_o, 128);
      ok = ok && map_rows(&h->m_p1, h->p1, ph, rows_o, 128);
      ok = ok && make_out_map(&h->m_out_p1, h->p1, (uint64_t)rows_o, (uint64_t)ph);
      ok = ok && map_rows(&h->m_proj1_w, h->proj1_w, d, ph, 128);
      ok = ok && map_rows(&h->m_proj2_w, h->proj2_w, ph, po, 128);
    }
    h->lmaps.resize(L);
    for (int l = 0; ok && l < L; ++l) {
      ok = ok && map_rows(&h->lmaps[l].qkv, h->qkv_w[l], d, 3 * d, 128);
      ok = ok && map_rows(&h->lmaps[l].o, h->o_w[l], d, d, 128);
      ok = ok && map_rows(&h->lmaps[l].fc1, h->fc1_w[l], d, F, 128);
      ok = ok && map_rows(&h->lmaps[l].fc2, h->fc2_w[l], F, d, 128);
    }
    if (!ok) return ENC_ERR_CUDA;
  }
  ENC_TRY(cudaDeviceSynchronize());
  return ENC_OK;
}

EpiParams epi_base(int mode) {
  EpiParams e;
  memset(&e, 0, sizeof(e));
  e.mode = mode;
  return e;
}

cudaEvent_t pooled_event(enc_handle* h) {
  if (!h->event_pool.empty()) {
    cudaEvent_t e = h->event_pool.back();
    h->event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

// NVTX range names of the kernel classes (include/enc_profile.h order). The
// ranges mark host-side enqueueing for a tool such as Nsight Systems; with no
// tool attached each push / pop is a check of one pointer.
const char* const kRangeNames[ENC_K_COUNT] = {"mel stage", "conv1", "conv2", "layernorm", "qkv", "attention",
                                              "out-proj", "fc1", "fc2", "final layernorm", "projector fc1",
                                              "projector fc2", "zero rows"};

// RAII NVTX range
struct Range {
  explicit Range(const char* name) { nvtxRangePushA(name); }
  ~Range() { nvtxRangePop(); }
};

// Enqueue one kernel: bracket it with events when profiling, count it.
template <typename F>
cudaError_t run(enc_handle* h, cudaStream_t s, int cls, double flops, F&& launch) {
  Range range(cls >= 0 && cls < ENC_K_COUNT ? kRangeNames[cls] : "kernel");
  cudaEvent_t a = nullptr, b = nullptr;
  if (h->profile) {
    a = pooled_event(h);
    b = pooled_event(h);
    if (a) cudaEventRecord(a, s);
  }
  cudaError_t e = launch();
  ++h->launches;
  if (h->profile && a && b) {
    cudaEventRecord(b, s);
    h->recs.push_back({cls, a, b, flops});
  }
  return e;
}

#define ENC_RUN(cls, flops, expr) ENC_TRY(run(h, s, (cls), (flops), [&]() { return (expr); }))

// ------------------------------------------------------------- forward (bf16)
// Sizes of one batch: packed rows, pooled/packed output rows, longest clip,
// and sum of n_b^2 (attention work).
struct Work {
  int B, R, R_out, max_n;
  double sum_n2;
  int nseg, max_seg;   // attention segments: the clips, or their chunks with block-local attention
  double sum_seg2;
};

int valid_out(const enc_handle* h, int n);   // output rows of a clip with n positions

// Per-clip counts of one batch, staged into hm for upload:
//   [cu (B+1) | cu_out (B+1) | len (B) | cu_attn (nseg+1), block-local attention only]
// n_b = ceil(len_b / 2) positions; cu_attn cuts every clip into chunks of
// cfg.attn_chunk positions (the last one shorter). Returns the ints to upload,
// or 0 when a length is outside [1, T].
int stage_meta(const enc_handle* h, const int32_t* lengths, int B, int* hm, Work* wk) {
  int* cu = hm;
  int* cu_out = hm + (B + 1);
  int* len = hm + 2 * (B + 1);
  int max_n = 0;
  double sum_n2 = 0.0;
  cu[0] = cu_out[0] = 0;
  for (int b = 0; b < B; ++b) {
    len[b] = lengths ? lengths[b] : h->T;
    if (len[b] < 1 || len[b] > h->T) return 0;
    const int n = (len[b] + 1) / 2;
    cu[b + 1] = cu[b] + n;
    cu_out[b + 1] = cu_out[b] + valid_out(h, n);
    if (n > max_n) max_n = n;
    sum_n2 += (double)n * n;
  }
  int total = 3 * B + 2;
  int nseg = B, max_seg = max_n;
  double sum_seg2 = sum_n2;
  const int chunk = h->cfg.attn_chunk;
  if (chunk > 0) {
    int* ca = hm + total;
    nseg = 0;
    max_seg = 0;
    sum_seg2 = 0.0;
    ca[0] = 0;
    for (int b = 0; b < B; ++b)
      for (int c0 = cu[b]; c0 < cu[b + 1]; c0 += chunk) {
        const int c1 = c0 + chunk < cu[b + 1] ? c0 + chunk : cu[b + 1];
        ca[++nseg] = c1;
        if (c1 - c0 > max_seg) max_seg = c1 - c0;
        sum_seg2 += (double)(c1 - c0) * (c1 - c0);
      }
    total += nseg + 1;
  }
  *wk = Work{B, cu[B], cu_out[B], max_n, sum_n2, nseg, max_seg, sum_seg2};
  return total;
}

enc_status forward_bf16(enc_handle* h, const void* mel, void* out, const Work& wk, cudaStream_t s) {
  const enc_config& c = h->cfg;
  const int d = c.d_model, F = c.ffn_dim, M = c.n_mels, B = wk.B, R = wk.R;
  const double Rd = (double)R * d;
  const int* cu = h->meta;
  const int* cu_out = h->meta + (B + 1);
  const int* len = h->meta + 2 * (B + 1);
  const int* cu_att = c.attn_chunk > 0 ? h->meta + 3 * B + 2 : cu;   // attention segments
  bf16* melT_data = reinterpret_cast<bf16*>(h->melT) + M;
  ENC_RUN(ENC_K_MEL, 0.0,
          launch_mel_stage<bf16>(reinterpret_cast<const bf16*>(mel), len, melT_data, B, M, h->T, h->Tp, s));

  GemmTcParams g;
  memset(&g, 0, sizeof(g));
  g.status = h->status;
  // conv1: rows = padded time of every clip
  g.M = B * h->Tp; g.N = d; g.a_mode = A_CONV1; g.kb_seg = h->mpad / 64; g.num_kb = 3 * g.kb_seg;
  g.epi = epi_base(EPI_CONV1);
  g.epi.bias = h->conv1_b; g.epi.out = h->y1; g.epi.ldo = d; g.epi.T = h->T; g.epi.Tp = h->Tp;
  ENC_RUN(ENC_K_CONV1, 2.0 * 2 * Rd * 3 * M,
          launch_gemm_tc(h->m_conv1_a, h->m_conv1_w, g, h->sm_count, s, &h->m_out_y1));
  // conv2 (+ GELU + position table) -> packed residual stream
  g.M = B * h->P1; g.N = d; g.a_mode = A_CONV2; g.kb_seg = d / 64; g.num_kb = 3 * g.kb_seg;
  g.epi = epi_base(EPI_CONV2);
  g.epi.bias = h->conv2_b; g.epi.resid = h->x; g.epi.ldo = d; g.epi.pe = h->pe; g.epi.cu = cu; g.epi.P1 = h->P1;
  ENC_RUN(ENC_K_CONV2, 2.0 * Rd * 3 * d, launch_gemm_tc(h->m_conv2_a, h->m_conv2_w, g, h->sm_count, s));

  bf16* a = reinterpret_cast<bf16*>(h->a);
  for (int l = 0; l < c.n_layers; ++l) {
    Range block("encoder block");
    const LayerMaps& lm = h->lmaps[l];
    ENC_RUN(ENC_K_LN, 0.0, launch_layernorm<bf16>(h->x, h->ln1_g[l], h->ln1_b[l], a, R, d, c.ln_eps, s));
    g.M = R; g.a_mode = A_PLAIN; g.kb_seg = 0;
    g.N = 3 * d; g.num_kb = d / 64;
    g.epi = epi_base(EPI_STORE);
    g.epi.bias = h->qkv_b[l]; g.epi.out = h->qkv; g.epi.ldo = 3 * d;
    ENC_RUN(ENC_K_QKV, 6.0 * Rd * d, launch_gemm_tc(h->m_a, lm.qkv, g, h->sm_count, s, &h->m_out_qkv));
    ENC_RUN(ENC_K_ATTN, 4.0 * wk.sum_seg2 * d,
            launch_attention_tc(h->m_qkv, reinterpret_cast<bf16*>(h->o), cu_att, wk.nseg, wk.max_seg, d, c.n_heads,
                                h->status, s));
    g.N = d; g.num_kb = d / 64;
    g.epi = epi_base(EPI_RESIDUAL);
    g.epi.bias = h->o_b[l]; g.epi.resid = h->x; g.epi.ldo = d;
    ENC_RUN(ENC_K_OUT, 2.0 * Rd * d, launch_gemm_tc(h->m_o, lm.o, g, h->sm_count, s, &h->m_x));
    ENC_RUN(ENC_K_LN, 0.0, launch_layernorm<bf16>(h->x, h->ln2_g[l], h->ln2_b[l], a, R, d, c.ln_eps, s));
    g.N = F; g.num_kb = d / 64;
    g.epi = epi_base(EPI_STORE);
    g.epi.gelu = 1; g.epi.bias = h->fc1_b[l]; g.epi.out = h->f; g.epi.ldo = F;
    ENC_RUN(ENC_K_FC1, 2.0 * Rd * F, launch_gemm_tc(h->m_a, lm.fc1, g, h->sm_count, s, &h->m_out_f));
    g.N = d; g.num_kb = F / 64;
    g.epi = epi_base(EPI_RESIDUAL);
    g.epi.bias = h->fc2_b[l]; g.epi.resid = h->x; g.epi.ldo = d;
    ENC_RUN(ENC_K_FC2, 2.0 * Rd * F, launch_gemm_tc(h->m_f, lm.fc2, g, h->sm_count, s, &h->m_x));
  }

  if (!c.proj_hidden) {
    ENC_RUN(ENC_K_FINAL, 0.0,
            launch_final_ln<bf16>(h->x, h->lnpost_g, h->lnpost_b, cu, cu_out, reinterpret_cast<bf16*>(out), B,
                                  h->p_out, d, c.pool_step, 0, c.ln_eps, s));
    return ENC_OK;
  }
  const int ph = c.proj_hidden, po = c.proj_out;
  const double Ro = wk.R_out;
  ENC_RUN(ENC_K_FINAL, 0.0,
          launch_final_ln<bf16>(h->x, h->lnpost_g, h->lnpost_b, cu, cu_out, reinterpret_cast<bf16*>(h->e), B,
                                h->p_out, d, c.pool_step, 1, c.ln_eps, s));
  g.M = wk.R_out; g.a_mode = A_PLAIN; g.kb_seg = 0;
  g.N = ph; g.num_kb = d / 64;
  g.epi = epi_base(EPI_STORE);
  g.epi.gelu = 1; g.epi.bias = h->proj1_b; g.epi.out = h->p1; g.epi.ldo = ph;
  ENC_RUN(ENC_K_PROJ1, 2.0 * Ro * d * ph, launch_gemm_tc(h->m_e, h->m_proj1_w, g, h->sm_count, s, &h->m_out_p1));
  g.N = po; g.num_kb = ph / 64;
  g.epi = epi_base(EPI_SCATTER);
  g.epi.bias = h->proj2_b; g.epi.out = out; g.epi.ldo = po; g.epi.cu = cu_out; g.epi.B = B; g.epi.p_out = h->p_out;
  ENC_RUN(ENC_K_PROJ2, 2.0 * Ro * ph * po, launch_gemm_tc(h->m_p1, h->m_proj2_w, g, h->sm_count, s));
  ENC_RUN(ENC_K_ZERO, 0.0, launch_zero_tail_rows<bf16>(reinterpret_cast<bf16*>(out), cu_out, B, h->p_out, po, s));
  return ENC_OK;
}

// -------------------------------------------------------- forward (fp32 check)
enc_status forward_f32(enc_handle* h, const void* mel, void* out, const Work& wk, cudaStream_t s) {
  const enc_config& c = h->cfg;
  const int d = c.d_model, F = c.ffn_dim, M = c.n_mels, B = wk.B, R = wk.R;
  const double Rd = (double)R * d;
  const int* cu = h->meta;
  const int* cu_out = h->meta + (B + 1);
  const int* len = h->meta + 2 * (B + 1);
  const int* cu_att = c.attn_chunk > 0 ? h->meta + 3 * B + 2 : cu;   // attention segments
  float* melT = reinterpret_cast<float*>(h->melT);
  float* y1 = reinterpret_cast<float*>(h->y1);
  ENC_RUN(ENC_K_MEL, 0.0,
          launch_mel_stage<float>(reinterpret_cast<const float*>(mel), len, melT + M, B, M, h->T, h->Tp, s));

  EpiParams e = epi_base(EPI_CONV1);
  e.bias = h->conv1_b; e.out = y1; e.ldo = d; e.T = h->T; e.Tp = h->Tp;
  // conv1 row r reads mel rows r-1, r, r+1: A starts at the guard row, rows overlap (lda = M)
  ENC_RUN(ENC_K_CONV1, 2.0 * 2 * Rd * 3 * M,
          launch_sgemm(melT, M, reinterpret_cast<const float*>(h->conv1_w), 3 * M, B * h->Tp, d, 3 * M, e, s));
  e = epi_base(EPI_CONV2);
  e.bias = h->conv2_b; e.resid = h->x; e.ldo = d; e.pe = h->pe; e.cu = cu; e.P1 = h->P1;
  // conv2 row j reads conv1 rows 2j, 2j+1, 2j+2 (padded time): lda = 2d, K = 3d
  ENC_RUN(ENC_K_CONV2, 2.0 * Rd * 3 * d,
          launch_sgemm(y1, 2 * d, reinterpret_cast<const float*>(h->conv2_w), 3 * d, B * h->P1, d, 3 * d, e, s));

  float* a = reinterpret_cast<float*>(h->a);
  float* qkv = reinterpret_cast<float*>(h->qkv);
  float* o = reinterpret_cast<float*>(h->o);
  float* f = reinterpret_cast<float*>(h->f);
  for (int l = 0; l < c.n_layers; ++l) {
    Range block("encoder block");
    ENC_RUN(ENC_K_LN, 0.0, launch_layernorm<float>(h->x, h->ln1_g[l], h->ln1_b[l], a, R, d, c.ln_eps, s));
    e = epi_base(EPI_STORE);
    e.bias = h->qkv_b[l]; e.out = qkv; e.ldo = 3 * d;
    ENC_RUN(ENC_K_QKV, 6.0 * Rd * d,
            launch_sgemm(a, d, reinterpret_cast<const float*>(h->qkv_w[l]), d, R, 3 * d, d, e, s));
    ENC_RUN(ENC_K_ATTN, 4.0 * wk.sum_seg2 * d,
            launch_attention_f32(qkv, o, cu_att, wk.nseg, wk.max_seg, d, c.n_heads, s));
    e = epi_base(EPI_RESIDUAL);
    e.bias = h->o_b[l]; e.resid = h->x; e.ldo = d;
    ENC_RUN(ENC_K_OUT, 2.0 * Rd * d, launch_sgemm(o, d, reinterpret_cast<const float*>(h->o_w[l]), d, R, d, d, e, s));
    ENC_RUN(ENC_K_LN, 0.0, launch_layernorm<float>(h->x, h->ln2_g[l], h->ln2_b[l], a, R, d, c.ln_eps, s));
    e = epi_base(EPI_STORE);
    e.gelu = 1; e.bias = h->fc1_b[l]; e.out = f; e.ldo = F;
    ENC_RUN(ENC_K_FC1, 2.0 * Rd * F, launch_sgemm(a, d, reinterpret_cast<const float*>(h->fc1_w[l]), d, R, F, d, e, s));
    e = epi_base(EPI_RESIDUAL);
    e.bias = h->fc2_b[l]; e.resid = h->x; e.ldo = d;
    ENC_RUN(ENC_K_FC2, 2.0 * Rd * F, launch_sgemm(f, F, reinterpret_cast<const float*>(h->fc2_w[l]), F, R, d, F, e, s));
  }
  if (!c.proj_hidden) {
    ENC_RUN(ENC_K_FINAL, 0.0,
            launch_final_ln<float>(h->x, h->lnpost_g, h->lnpost_b, cu, cu_out, reinterpret_cast<float*>(out), B,
                                   h->p_out, d, c.pool_step, 0, c.ln_eps, s));
    return ENC_OK;
  }
  const int ph = c.proj_hidden, po = c.proj_out;
  const double Ro = wk.R_out;
  float* ev = reinterpret_cast<float*>(h->e);
  float* p1 = reinterpret_cast<float*>(h->p1);
  ENC_RUN(ENC_K_FINAL, 0.0,
          launch_final_ln<float>(h->x, h->lnpost_g, h->lnpost_b, cu, cu_out, ev, B, h->p_out, d, c.pool_step, 1,
                                 c.ln_eps, s));
  e = epi_base(EPI_STORE);
  e.gelu = 1; e.bias = h->proj1_b; e.out = p1; e.ldo = ph;
  ENC_RUN(ENC_K_PROJ1, 2.0 * Ro * d * ph,
          launch_sgemm(ev, d, reinterpret_cast<const float*>(h->proj1_w), d, wk.R_out, ph, d, e, s));
  e = epi_base(EPI_SCATTER);
  e.bias = h->proj2_b; e.out = out; e.ldo = po; e.cu = cu_out; e.B = B; e.p_out = h->p_out;
  ENC_RUN(ENC_K_PROJ2, 2.0 * Ro * ph * po,
          launch_sgemm(p1, ph, reinterpret_cast<const float*>(h->proj2_w), ph, wk.R_out, po, ph, e, s));
  ENC_RUN(ENC_K_ZERO, 0.0, launch_zero_tail_rows<float>(reinterpret_cast<float*>(out), cu_out, B, h->p_out, po, s));
  return ENC_OK;
}

int valid_out(const enc_handle* h, int n) { return h->cfg.pool_step > 1 ? n / h->cfg.pool_step : n; }

constexpr uint64_t kSelftestOtherNs = 2000000000ull;   // warp 1's own limit: 2 s

// Failure detection without a fault (enc_selftest_timeout): two mbarrier
// phases that nothing completes. Warp 0 gives up after limit_ns and raises
// the abort flag; warp 1 leaves at its next check of the flag.
__global__ void __launch_bounds__(64) selftest_timeout_kernel(int* status, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bars[2];
  __shared__ int abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  volatile int* abort_v = &abort_flag;
  if (warp == 0) {
    if (!mbar_wait_warp(&bars[0], 0, abort_v, limit_ns) && lane == 0) {
      set_status(status, kDevTimeout);
      *abort_v = 1;
    }
  } else {
    mbar_wait_warp(&bars[1], 0, abort_v, kSelftestOtherNs);
  }
}

}  // namespace

extern "C" {

const char* enc_status_string(enc_status s) {
  switch (s) {
    case ENC_OK: return "ok";
    case ENC_ERR_INVALID_ARG: return "invalid argument";
    case ENC_ERR_UNSUPPORTED: return "unsupported geometry or device (needs sm_100)";
    case ENC_ERR_OOM: return "out of memory";
    case ENC_ERR_CUDA: return "CUDA runtime error";
    case ENC_ERR_TIMEOUT: return "device-side wait timed out";
    case ENC_ERR_DEVICE_CHECK: return "device-side range check failed";
  }
  return "unknown status";
}

enc_status enc_create(const enc_config* cfg, const enc_weights* w, enc_handle** out) {
  if (!out) return ENC_ERR_INVALID_ARG;
  *out = nullptr;
  if (!w) return ENC_ERR_INVALID_ARG;
  enc_status st = validate_config(cfg);
  if (st != ENC_OK) return st;
  int dev = 0;
  cudaDeviceProp prop;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaGetDeviceProperties(&prop, dev) != cudaSuccess) {
    cudaGetLastError();
    return ENC_ERR_CUDA;
  }
  if (prop.major != 10 || prop.minor != 0) return ENC_ERR_UNSUPPORTED;
  enc_handle* h = new enc_handle();
  h->cfg = *cfg;
  h->device = dev;
  h->sm_count = prop.multiProcessorCount;
  h->bf16 = cfg->dtype == ENC_DTYPE_BF16;
  h->esz = h->bf16 ? 2 : 4;
  h->T = cfg->max_frames;
  h->Tp = round_up(h->T + 2, 2);
  h->P = (h->T + 1) / 2;
  h->P1 = h->P + 1;
  h->p_out = cfg->pool_step > 1 ? h->P / cfg->pool_step : h->P;
  h->d_out = cfg->proj_hidden ? cfg->proj_out : cfg->d_model;
  st = build(h, w);
  if (st == ENC_OK) resolve_static_scratch(h);
  if (st != ENC_OK) {
    cudaDeviceSynchronize();
    cudaGetLastError();
    free_all(h);
    delete h;
    return st;
  }
  *out = h;
  return ENC_OK;
}

enc_status enc_output_positions(const enc_handle* h, int32_t B, const int32_t* lengths, int32_t* n_out,
                                int32_t* p_out, int32_t* d_out) {
  if (!h || B < 1) return ENC_ERR_INVALID_ARG;
  if (n_out) {
    for (int b = 0; b < B; ++b) {
      const int len = lengths ? lengths[b] : h->T;
      if (len < 1 || len > h->T) return ENC_ERR_INVALID_ARG;
      n_out[b] = valid_out(h, (len + 1) / 2);
    }
  }
  if (p_out) *p_out = h->p_out;
  if (d_out) *d_out = h->d_out;
  return ENC_OK;
}

enc_status enc_forward(enc_handle* h, const void* mel, const int32_t* lengths, int32_t B, void* out,
                       cudaStream_t stream) {
  if (!h || !mel || !out || B < 1 || B > h->cfg.max_batch) return ENC_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(mel) | reinterpret_cast<uintptr_t>(out)) & 15u) return ENC_ERR_INVALID_ARG;
  if (cudaSetDevice(h->device) != cudaSuccess) return ENC_ERR_CUDA;
  // the pinned staging buffer may still feed the previous forward's upload
  if (h->meta_pending) ENC_TRY(cudaEventSynchronize(h->meta_free));
  Work wk;
  const int nints = stage_meta(h, lengths, B, h->h_meta, &wk);
  if (nints == 0) return ENC_ERR_INVALID_ARG;
  ENC_TRY(cudaMemcpyAsync(h->meta, h->h_meta, (size_t)nints * 4, cudaMemcpyHostToDevice, stream));
  ENC_TRY(cudaEventRecord(h->meta_free, stream));
  h->meta_pending = true;
  Range range("enc_forward");
  return h->bf16 ? forward_bf16(h, mel, out, wk, stream) : forward_f32(h, mel, out, wk, stream);
}

enc_status enc_get_status(enc_handle* h, cudaStream_t stream) {
  if (!h) return ENC_ERR_INVALID_ARG;
  if (cudaSetDevice(h->device) != cudaSuccess) return ENC_ERR_CUDA;
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_status(e);
  int v = 0;
  ENC_TRY(cudaMemcpy(&v, h->status, 4, cudaMemcpyDeviceToHost));
  if (v != 0) ENC_TRY(cudaMemset(h->status, 0, 4));
  if (v == kDevTimeout) return ENC_ERR_TIMEOUT;
  if (v == kDevCheck) return ENC_ERR_DEVICE_CHECK;
  return v == 0 ? ENC_OK : ENC_ERR_CUDA;
}

enc_status enc_selftest_timeout(enc_handle* h, int64_t limit_ns, cudaStream_t stream) {
  if (!h || limit_ns < 1000 || limit_ns > 100000000) return ENC_ERR_INVALID_ARG;
  if (cudaSetDevice(h->device) != cudaSuccess) return ENC_ERR_CUDA;
  selftest_timeout_kernel<<<1, 64, 0, stream>>>(h->status, static_cast<uint64_t>(limit_ns));
  return cuda_status(cudaGetLastError());
}

void enc_destroy(enc_handle* h) {
  if (!h) return;
  cudaSetDevice(h->device);
  cudaDeviceSynchronize();
  free_all(h);
  delete h;
}

size_t enc_device_bytes(const enc_handle* h) { return h ? h->bytes : 0; }

enc_status enc_guard_selftest(enc_handle* h, int32_t buffer, int64_t offset) {
  if (!h || !(h->cfg.flags & ENC_FLAG_GUARD) || buffer < 0 || buffer >= (int32_t)h->guards.size())
    return ENC_ERR_INVALID_ARG;
  const auto& g = h->guards[buffer];
  if (offset == 0 || offset < -(int64_t)kGuardBytes || offset > (int64_t)kGuardBytes) return ENC_ERR_INVALID_ARG;
  // offset < 0: byte -offset before the buffer; offset > 0: byte offset - 1 past its end
  unsigned char* p = offset < 0 ? g.buf + offset : g.buf + g.bytes + (offset - 1);
  if (cudaSetDevice(h->device) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) return ENC_ERR_CUDA;
  if (cudaMemset(p, kGuardByte ^ 0xFF, 1) != cudaSuccess) return ENC_ERR_CUDA;
  char msg[128];
  const enc_status seen = enc_check_guards(h, msg, sizeof msg);
  if (cudaMemset(p, kGuardByte, 1) != cudaSuccess) return ENC_ERR_CUDA;
  if (seen != ENC_ERR_DEVICE_CHECK || strncmp(msg, g.name, strlen(g.name)) != 0) return ENC_ERR_CUDA;
  return enc_check_guards(h, nullptr, 0);
}

enc_status enc_check_guards(enc_handle* h, char* what, size_t what_len) {
  if (!h) return ENC_ERR_INVALID_ARG;
  if (what && what_len) what[0] = 0;
  if (!(h->cfg.flags & ENC_FLAG_GUARD)) return ENC_ERR_INVALID_ARG;
  if (cudaSetDevice(h->device) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) return ENC_ERR_CUDA;
  std::vector<unsigned char> buf(kGuardBytes);
  for (const auto& g : h->guards) {
    for (int side = 0; side < 2; ++side) {
      const unsigned char* src = side ? g.buf + g.bytes : g.buf - kGuardBytes;
      if (cudaMemcpy(buf.data(), src, kGuardBytes, cudaMemcpyDeviceToHost) != cudaSuccess) return ENC_ERR_CUDA;
      for (size_t i = 0; i < kGuardBytes; ++i) {
        if (buf[i] == kGuardByte) continue;
        if (what && what_len)
          snprintf(what, what_len, "%s: byte %s%zu %s the buffer changed", g.name, side ? "+" : "-",
                   side ? i : kGuardBytes - i, side ? "past the end of" : "before the start of");
        return ENC_ERR_DEVICE_CHECK;
      }
    }
  }
  return ENC_OK;
}

enc_status enc_profile_enable(enc_handle* h, int32_t enable) {
  if (!h) return ENC_ERR_INVALID_ARG;
  h->profile = enable != 0;
  return ENC_OK;
}

enc_status enc_profile_collect(enc_handle* h, enc_kernel_times* out) {
  if (!h || !out) return ENC_ERR_INVALID_ARG;
  memset(out, 0, sizeof(*out));
  if (cudaSetDevice(h->device) != cudaSuccess) return ENC_ERR_CUDA;
  enc_status st = ENC_OK;
  for (const auto& r : h->recs) {
    float ms = 0.f;
    if (st == ENC_OK) {
      cudaError_t e = cudaEventSynchronize(r.b);
      if (e == cudaSuccess) e = cudaEventElapsedTime(&ms, r.a, r.b);
      if (e != cudaSuccess) st = cuda_status(e);
    }
    if (r.cls >= 0 && r.cls < ENC_K_COUNT) {
      out->ms[r.cls] += ms;
      out->flops[r.cls] += r.flops;
      out->launches[r.cls] += 1;
    }
    h->event_pool.push_back(r.a);
    h->event_pool.push_back(r.b);
  }
  h->recs.clear();
  return st;
}

int64_t enc_launch_count(const enc_handle* h) { return h ? h->launches : 0; }

}  // extern "C"

// ---------------------------------------------------------------------------
// enc_forward_static_scratch: the forward pass with its workspace in a fixed
// static device array instead of handle-owned memory, so that the call itself
// needs no device allocation. Reuses the launch sequence above unchanged.
// ---------------------------------------------------------------------------
#define ENC_STATIC_SCRATCH_BYTES (64ull << 20)

// Reserved by the CUDA runtime on every device that loads this library, until exit.
static __device__ __align__(256) unsigned char enc_static_scratch[ENC_STATIC_SCRATCH_BYTES];

namespace {

size_t align256(size_t n) { return (n + 255) & ~size_t(255); }

}  // namespace

// Set-up of enc_forward_static_scratch, run by enc_create with the handle's
// device current. In host code the array's name only stands in for it, so the
// runtime is asked for its device address. The first lookup on a device loads
// this file's module there, which is when the 64 MiB are reserved: in
// enc_create, not inside enc_forward_static_scratch.
void enc::resolve_static_scratch(enc_handle* h) {
  void* p = nullptr;
  const cudaError_t e = cudaGetSymbolAddress(&p, enc_static_scratch);
  if (e == cudaSuccess && p) {
    h->static_scratch = reinterpret_cast<unsigned char*>(p);
    h->static_scratch_status = ENC_OK;
  } else {
    cudaGetLastError();
    h->static_scratch = nullptr;
    h->static_scratch_status = e == cudaErrorMemoryAllocation ? ENC_ERR_OOM : ENC_ERR_CUDA;
  }
}

extern "C" enc_status enc_forward_static_scratch(enc_handle* h, const void* mel, const int32_t* lengths, int32_t B,
                                                 void* out, cudaStream_t stream) {
  if (!h || !mel || !out || B < 1 || B > h->cfg.max_batch) return ENC_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(mel) | reinterpret_cast<uintptr_t>(out)) & 15u) return ENC_ERR_INVALID_ARG;
  for (int b = 0; b < B; ++b) {
    const int len = lengths ? lengths[b] : h->T;
    if (len < 1 || len > h->T) return ENC_ERR_INVALID_ARG;
  }
  const enc_config& c = h->cfg;
  const int d = c.d_model, F = c.ffn_dim, M = c.n_mels;
  if (cudaSetDevice(h->device) != cudaSuccess) return ENC_ERR_CUDA;
  unsigned char* base = h->static_scratch;   // resolved by enc_create
  if (!base) return h->static_scratch_status;
  enc_status st = ENC_OK;

  // per-clip counts, written straight into the handle's pinned staging buffer
  if (h->meta_pending) ENC_TRY(cudaEventSynchronize(h->meta_free));
  Work wk;
  const int nints = stage_meta(h, lengths, B, h->h_meta, &wk);
  if (nints == 0) return ENC_ERR_INVALID_ARG;
  const int R = wk.R, R_out = wk.R_out;

  // carve the workspace of this batch out of the static array
  const size_t rows_t = (size_t)B * h->Tp;
  size_t off = 0;
  auto take = [&](size_t bytes) { unsigned char* p = base + off; off += align256(bytes); return p; };
  unsigned char* melT = take((rows_t + 2) * M * h->esz);
  unsigned char* y1 = take((rows_t + 2) * d * h->esz);
  unsigned char* x = take((size_t)R * d * 4);
  unsigned char* a = take((size_t)R * d * h->esz);
  unsigned char* qkv = take((size_t)R * 3 * d * h->esz);
  unsigned char* o = take((size_t)R * d * h->esz);
  unsigned char* f = take((size_t)R * F * h->esz);
  unsigned char* e = c.proj_hidden ? take((size_t)R_out * d * h->esz) : nullptr;
  unsigned char* p1 = c.proj_hidden ? take((size_t)R_out * c.proj_hidden * h->esz) : nullptr;
  unsigned char* meta = take((size_t)nints * 4);
  if (off > ENC_STATIC_SCRATCH_BYTES) return ENC_ERR_INVALID_ARG;   // batch too large for the array

  // the array keeps the previous call's contents: clear what is read as zero
  // (the guard rows around the time-major mel)
  ENC_TRY(cudaMemsetAsync(melT, 0, (size_t)M * h->esz, stream));
  ENC_TRY(cudaMemsetAsync(melT + (rows_t + 1) * M * h->esz, 0, (size_t)M * h->esz, stream));

  // point the handle at the static workspace for this call, then restore it
  void *s_melT = h->melT, *s_y1 = h->y1, *s_a = h->a, *s_qkv = h->qkv, *s_o = h->o, *s_f = h->f, *s_e = h->e,
       *s_p1 = h->p1;
  float* s_x = h->x;
  int* s_meta = h->meta;
  const CUtensorMap s_conv1_a = h->m_conv1_a, s_conv2_a = h->m_conv2_a, s_ma = h->m_a, s_mo = h->m_o,
                    s_mf = h->m_f, s_me = h->m_e, s_mp1 = h->m_p1, s_mx = h->m_x;
  const QkvMaps s_mqkv = h->m_qkv;
  const CUtensorMap s_oy1 = h->m_out_y1, s_oqkv = h->m_out_qkv, s_of = h->m_out_f, s_op1 = h->m_out_p1;
  const bool s_profile = h->profile;
  h->melT = melT; h->y1 = y1; h->x = reinterpret_cast<float*>(x); h->a = a; h->qkv = qkv; h->o = o; h->f = f;
  h->e = e; h->p1 = p1; h->meta = reinterpret_cast<int*>(meta);
  h->profile = false;   // event records would grow host-side lists
  st = ENC_OK;
  if (h->bf16) {
    bool ok = map_rows(&h->m_conv1_a, melT + (size_t)M * 2, M, (long long)rows_t, 128);
    ok = ok && make_tma_2d(&h->m_conv2_a, y1, 2 * (uint64_t)d, (uint64_t)rows_t / 2, 4 * (uint64_t)d, 64, 128);
    ok = ok && map_rows(&h->m_a, a, d, R, 128);
    ok = ok && map_rows(&h->m_o, o, d, R, 128);
    ok = ok && map_rows(&h->m_f, f, F, R, 128);
    ok = ok && make_qkv_maps(&h->m_qkv, qkv, R, d);
    ok = ok && make_resid_map(&h->m_x, reinterpret_cast<float*>(x), (uint64_t)R, (uint64_t)d);
    ok = ok && make_out_map(&h->m_out_y1, y1, (uint64_t)rows_t, (uint64_t)d);
    ok = ok && make_out_map(&h->m_out_qkv, qkv, (uint64_t)R, 3 * (uint64_t)d);
    ok = ok && make_out_map(&h->m_out_f, f, (uint64_t)R, (uint64_t)F);
    if (c.proj_hidden) {
      ok = ok && map_rows(&h->m_e, e, d, R_out > 0 ? R_out : 1, 128);
      ok = ok && map_rows(&h->m_p1, p1, c.proj_hidden, R_out > 0 ? R_out : 1, 128);
      ok = ok && make_out_map(&h->m_out_p1, p1, (uint64_t)(R_out > 0 ? R_out : 1), (uint64_t)c.proj_hidden);
    }
    if (!ok) st = ENC_ERR_CUDA;
  }
  if (st == ENC_OK) {
    cudaError_t ce = cudaMemcpyAsync(h->meta, h->h_meta, (size_t)nints * 4, cudaMemcpyHostToDevice, stream);
    if (ce == cudaSuccess) ce = cudaEventRecord(h->meta_free, stream);
    if (ce != cudaSuccess) st = cuda_status(ce);
    else h->meta_pending = true;
  }
  if (st == ENC_OK) {
    st = h->bf16 ? forward_bf16(h, mel, out, wk, stream) : forward_f32(h, mel, out, wk, stream);
  }
  h->melT = s_melT; h->y1 = s_y1; h->x = s_x; h->a = s_a; h->qkv = s_qkv; h->o = s_o; h->f = s_f; h->e = s_e;
  h->p1 = s_p1; h->meta = s_meta;
  h->m_conv1_a = s_conv1_a; h->m_conv2_a = s_conv2_a; h->m_a = s_ma; h->m_o = s_mo; h->m_f = s_mf; h->m_e = s_me;
  h->m_p1 = s_mp1;
  h->m_qkv = s_mqkv;
  h->m_x = s_mx;
  h->m_out_y1 = s_oy1; h->m_out_qkv = s_oqkv; h->m_out_f = s_of; h->m_out_p1 = s_op1;
  h->profile = s_profile;
  return st;
}

namespace enc {
bool handle_geometry(const enc_handle* h, HandleGeometry* g) {
  if (!h || !g) return false;
  g->n_mels = h->cfg.n_mels;
  g->frames = h->T;
  g->max_batch = h->cfg.max_batch;
  g->device = h->device;
  g->mel_bytes = (size_t)h->cfg.n_mels * h->T * h->esz;
  g->out_bytes = (size_t)h->p_out * h->d_out * h->esz;
  return true;
}
}  // namespace enc
