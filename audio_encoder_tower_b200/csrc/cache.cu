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
  unsigned long long* d_sums = nullptr; // [max_batch] content-hash sums (enc_cache_content_keys)
  int* d_len = nullptr;                 // [max_batch] clip lengths for the hash kernel
  std::unordered_map<uint64_t, int> where;   // key -> slot
  std::vector<uint64_t> slot_key;
  std::vector<uint64_t> slot_tick;            // last use; 0 = free
  uint64_t tick = 0;
};

namespace {

// SplitMix64 output finaliser (Steele, Lea and Flood, "Fast splittable
// pseudorandom number generators", OOPSLA 2014): a bijective 64-bit mixer.
__host__ __device__ __forceinline__ uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}
constexpr uint64_t kGolden = 0x9E3779B97F4A7C15ull;

// sums[b] += sum over the valid frames t < len[b] of clip b of
// mix64(((c * T + t) << 32 | value bits) + golden): each element contributes the
// mix of its position and its bits, and the contributions are added modulo
// 2^64, so the result does not depend on the order the threads add them in.
template <typename E>
__global__ void __launch_bounds__(256) content_hash_kernel(const E* __restrict__ mel, const int* __restrict__ len,
                                                           int n_mels, int T, unsigned long long* sums) {
  const int b = blockIdx.y;
  const int L = len[b];
  const E* clip = mel + (size_t)b * n_mels * T;
  const long long n = (long long)n_mels * T;
  uint64_t acc = 0;
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x) {
    const int t = (int)(i % T);
    if (t >= L) continue;
    uint64_t bits;
    if constexpr (sizeof(E) == 2) bits = *reinterpret_cast<const uint16_t*>(clip + i);
    else bits = *reinterpret_cast<const uint32_t*>(clip + i);
    acc += mix64(((static_cast<uint64_t>(i) << 32) | bits) + kGolden);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  __shared__ uint64_t part[8];
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = acc;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint64_t s = 0;
    for (int w = 0; w < (int)(blockDim.x >> 5); ++w) s += part[w];
    atomicAdd(&sums[b], static_cast<unsigned long long>(s));
  }
}

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
  if (c->d_sums) cudaFree(c->d_sums);
  if (c->d_len) cudaFree(c->d_len);
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
                  cudaMalloc(&c->mel_stage, g.mel_bytes * g.max_batch) == cudaSuccess &&
                  cudaMalloc(&c->d_sums, sizeof(unsigned long long) * g.max_batch) == cudaSuccess &&
                  cudaMalloc(&c->d_len, sizeof(int) * g.max_batch) == cudaSuccess;
  if (!ok) {
    cudaGetLastError();
    enc_cache_destroy(c);
    return ENC_ERR_OOM;
  }
  *out = c;
  return ENC_OK;
}

ENC_API int32_t enc_cache_size(const enc_cache* c) { return c ? static_cast<int32_t>(c->where.size()) : 0; }

ENC_API enc_status enc_cache_content_keys(enc_cache* c, const void* mel, const int32_t* lengths, int32_t B,
                                          uint64_t* keys, cudaStream_t stream) {
  if (!c || !mel || !keys || B < 1 || B > c->g.max_batch) return ENC_ERR_INVALID_ARG;
  std::vector<int> len(B);
  for (int b = 0; b < B; ++b) {
    len[b] = lengths ? lengths[b] : c->g.frames;
    if (len[b] < 1 || len[b] > c->g.frames) return ENC_ERR_INVALID_ARG;
  }
  if (cudaSetDevice(c->g.device) != cudaSuccess) return ENC_ERR_CUDA;
  const int n_mels = c->g.n_mels, T = c->g.frames;
  const long long per_clip = (long long)n_mels * T;
  const int blocks = (int)((per_clip + 256 * 8 - 1) / (256 * 8));   // about 8 elements per thread
  std::vector<unsigned long long> sums(B);
  cudaError_t e = cudaMemsetAsync(c->d_sums, 0, sizeof(unsigned long long) * B, stream);
  if (e == cudaSuccess) e = cudaMemcpyAsync(c->d_len, len.data(), sizeof(int) * B, cudaMemcpyHostToDevice, stream);
  if (e == cudaSuccess) {
    const dim3 grid(blocks < 1 ? 1 : blocks, B);
    if (c->g.mel_bytes == (size_t)per_clip * 2)
      content_hash_kernel<uint16_t><<<grid, 256, 0, stream>>>(static_cast<const uint16_t*>(mel), c->d_len, n_mels,
                                                               T, c->d_sums);
    else
      content_hash_kernel<uint32_t><<<grid, 256, 0, stream>>>(static_cast<const uint32_t*>(mel), c->d_len, n_mels,
                                                               T, c->d_sums);
    e = cudaGetLastError();
  }
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(sums.data(), c->d_sums, sizeof(unsigned long long) * B, cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return ENC_ERR_CUDA;
  }
  for (int b = 0; b < B; ++b)   // the length enters through its own mix, then the sum is mixed once more
    keys[b] = mix64(sums[b] ^ mix64(static_cast<uint64_t>(len[b]) * kGolden));
  return ENC_OK;
}

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
