// Embeddings cache in front of enc_forward (include/enc_cache.h): encoder
// outputs kept on the device and looked up by a caller-chosen 64-bit key per
// clip, the "Multimodal Embeddings Cache" of the REQUIRED KERNEL CLASS section
// the model pages repeat. Host bookkeeping only: every device transfer is one
// cudaMemcpyAsync on the caller's stream, so hits, the forward of the misses
// and the insertions stay in stream order.
#include <stdint.h>

#include <new>
#include <unordered_map>
#include <vector>

#include "../../include/enc_cache.h"
#include "internal.h"

struct enc_cache {
  enc_handle* h = nullptr;
  enc::HandleGeometry g{};
  int capacity = 0;
  unsigned char* slots = nullptr;       // [capacity] output blocks
  unsigned char* out_stage = nullptr;   // [max_batch] output blocks of the misses
  unsigned char* mel_stage = nullptr;   // [max_batch] mel blocks of the misses
  std::unordered_map<uint64_t, int> where;   // key -> slot
  std::vector<uint64_t> slot_key;
  std::vector<uint64_t> slot_tick;            // last use; 0 = free
  uint64_t tick = 0;
};

namespace {

// a free slot, else the least recently used one (its key leaves the map)
int take_slot(enc_cache* c) {
  int best = 0;
  for (int s = 0; s < c->capacity; ++s) {
    if (c->slot_tick[s] == 0) return s;
    if (c->slot_tick[s] < c->slot_tick[best]) best = s;
  }
  c->where.erase(c->slot_key[best]);
  c->slot_tick[best] = 0;
  return best;
}

}  // namespace

extern "C" {

ENC_API void enc_cache_destroy(enc_cache* c) {
  if (!c) return;
  int prev = 0;
  const bool have_prev = cudaGetDevice(&prev) == cudaSuccess;
  cudaSetDevice(c->g.device);
  if (c->slots) cudaFree(c->slots);
  if (c->out_stage) cudaFree(c->out_stage);
  if (c->mel_stage) cudaFree(c->mel_stage);
  if (have_prev) cudaSetDevice(prev);
  delete c;
}

ENC_API enc_status enc_cache_create(enc_handle* h, int32_t capacity, enc_cache** out) {
  if (!out) return ENC_ERR_INVALID_ARG;
  *out = nullptr;
  enc::HandleGeometry g;
  if (!enc::handle_geometry(h, &g) || capacity < 1) return ENC_ERR_INVALID_ARG;
  enc_cache* c = new (std::nothrow) enc_cache;
  if (!c) return ENC_ERR_OOM;
  c->h = h;
  c->g = g;
  c->capacity = capacity;
  c->slot_key.assign(capacity, 0);
  c->slot_tick.assign(capacity, 0);
  if (cudaSetDevice(g.device) != cudaSuccess) {
    delete c;
    return ENC_ERR_CUDA;
  }
  const bool ok = cudaMalloc(&c->slots, g.out_bytes * capacity) == cudaSuccess &&
                  cudaMalloc(&c->out_stage, g.out_bytes * g.max_batch) == cudaSuccess &&
                  cudaMalloc(&c->mel_stage, g.mel_bytes * g.max_batch) == cudaSuccess;
  if (!ok) {
    cudaGetLastError();
    enc_cache_destroy(c);
    return ENC_ERR_OOM;
  }
  *out = c;
  return ENC_OK;
}

ENC_API int32_t enc_cache_size(const enc_cache* c) { return c ? static_cast<int32_t>(c->where.size()) : 0; }

ENC_API enc_status enc_forward_cached(enc_cache* c, const void* mel, const int32_t* lengths, const uint64_t* keys,
                                      int32_t B, void* out, int32_t* hits, cudaStream_t stream) {
  if (!c || !mel || !out || !keys || B < 1 || B > c->g.max_batch) return ENC_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(mel) | reinterpret_cast<uintptr_t>(out)) & 15u) return ENC_ERR_INVALID_ARG;
  for (int b = 0; b < B; ++b)
    if (lengths && (lengths[b] < 1 || lengths[b] > c->g.frames)) return ENC_ERR_INVALID_ARG;
  if (cudaSetDevice(c->g.device) != cudaSuccess) return ENC_ERR_CUDA;
  const size_t ob = c->g.out_bytes, mb = c->g.mel_bytes;
  auto* dst = static_cast<unsigned char*>(out);
  const auto* src = static_cast<const unsigned char*>(mel);
  auto copy = [&](void* to, const void* from, size_t bytes) {
    return cudaMemcpyAsync(to, from, bytes, cudaMemcpyDeviceToDevice, stream) == cudaSuccess;
  };

  // hits first (in stream order before any insertion of this call)
  std::vector<int> miss;                         // clips computed here
  std::vector<int> miss_of(B, -1);               // clip -> index in miss of the clip computing its key
  std::unordered_map<uint64_t, int> first;       // key -> index in miss
  for (int b = 0; b < B; ++b) {
    auto it = c->where.find(keys[b]);
    if (it != c->where.end()) {
      if (!copy(dst + ob * b, c->slots + ob * it->second, ob)) return ENC_ERR_CUDA;
      c->slot_tick[it->second] = ++c->tick;
      if (hits) hits[b] = 1;
      continue;
    }
    if (hits) hits[b] = 0;
    auto f = first.find(keys[b]);
    if (f != first.end()) {
      miss_of[b] = f->second;
      continue;
    }
    first.emplace(keys[b], static_cast<int>(miss.size()));
    miss_of[b] = static_cast<int>(miss.size());
    miss.push_back(b);
  }
  if (miss.empty()) return ENC_OK;

  // the misses as one batch
  const int k = static_cast<int>(miss.size());
  std::vector<int32_t> len(k);
  for (int i = 0; i < k; ++i) {
    if (!copy(c->mel_stage + mb * i, src + mb * miss[i], mb)) return ENC_ERR_CUDA;
    len[i] = lengths ? lengths[miss[i]] : c->g.frames;
  }
  const enc_status st = enc_forward(c->h, c->mel_stage, len.data(), k, c->out_stage, stream);
  if (st != ENC_OK) return st;
  for (int b = 0; b < B; ++b)
    if (miss_of[b] >= 0 && !copy(dst + ob * b, c->out_stage + ob * miss_of[b], ob)) return ENC_ERR_CUDA;
  for (int i = 0; i < k; ++i) {
    const int s = take_slot(c);
    if (!copy(c->slots + ob * s, c->out_stage + ob * i, ob)) return ENC_ERR_CUDA;
    c->slot_key[s] = keys[miss[i]];
    c->slot_tick[s] = ++c->tick;
    c->where[keys[miss[i]]] = s;
  }
  return ENC_OK;
}

}  // extern "C"
