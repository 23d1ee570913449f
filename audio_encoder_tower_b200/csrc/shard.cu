// Splitting a batch of clips over data-parallel ranks (include/enc_shard.h).
// Host code only: the cost of a clip is its algorithmic FLOP count, linear in
// its positions (the GEMMs over packed rows) plus quadratic (attention within
// the clip or its chunks), and the plan is the longest-processing-time rule
// with a per-rank capacity of max_batch clips.
#include <stdint.h>

#include <algorithm>
#include <numeric>
#include <vector>

#include "../../include/enc_shard.h"
#include "internal.h"

namespace {

double clip_flops(const enc_config& c, int len) {
  const int np = (len + 1) / 2;   // positions after the stride-2 conv
  const double n = np, d = c.d_model, m = c.n_mels, f = c.ffn_dim;
  double attn = 0.0;   // sum over attention segments of (segment length)^2
  const int seg = c.attn_chunk > 0 ? c.attn_chunk : np;
  for (int s0 = 0; s0 < np; s0 += seg) {
    const double s = std::min(seg, np - s0);
    attn += s * s;
  }
  double t = 2.0 * (2.0 * n) * d * 3.0 * m + 2.0 * n * d * 3.0 * d;
  t += c.n_layers * (6.0 * n * d * d + 4.0 * attn * d + 2.0 * n * d * d + 4.0 * n * d * f);
  if (c.proj_hidden > 0) {
    const double no = c.pool_step > 1 ? np / c.pool_step : np;
    t += 2.0 * no * (d * c.proj_hidden + double(c.proj_hidden) * c.proj_out);
  }
  return t;
}

}  // namespace

extern "C" {

ENC_API enc_status enc_clip_flops(const enc_config* cfg, int32_t length, double* flops) {
  const enc_status st = enc::validate_config(cfg);
  if (st != ENC_OK) return st;
  if (!flops || length < 1 || length > cfg->max_frames) return ENC_ERR_INVALID_ARG;
  *flops = clip_flops(*cfg, length);
  return ENC_OK;
}

ENC_API enc_status enc_shard_plan(const enc_config* cfg, const int32_t* lengths, int32_t B, int32_t world,
                                  int32_t* rank_of, int32_t* index_of, int32_t* rank_count, double* rank_flops) {
  const enc_status st = enc::validate_config(cfg);
  if (st != ENC_OK) return st;
  if (!rank_of || world < 1 || B < 1 || (long long)B > (long long)world * cfg->max_batch) return ENC_ERR_INVALID_ARG;
  std::vector<double> cost(B);
  for (int b = 0; b < B; ++b) {
    const int len = lengths ? lengths[b] : cfg->max_frames;
    if (len < 1 || len > cfg->max_frames) return ENC_ERR_INVALID_ARG;
    cost[b] = clip_flops(*cfg, len);
  }
  // largest cost first; equal costs in clip order
  std::vector<int> order(B);
  std::iota(order.begin(), order.end(), 0);
  std::stable_sort(order.begin(), order.end(), [&](int a, int b) { return cost[a] > cost[b]; });
  std::vector<double> load(world, 0.0);
  std::vector<int> count(world, 0), rank(B);
  for (int b : order) {
    int best = -1;
    for (int r = 0; r < world; ++r)
      if (count[r] < cfg->max_batch && (best < 0 || load[r] < load[best])) best = r;
    rank[b] = best;   // B <= world * max_batch: some rank always has room
    load[best] += cost[b];
    ++count[best];
  }
  std::vector<int> next(world, 0);
  for (int b = 0; b < B; ++b) {
    rank_of[b] = rank[b];
    const int i = next[rank[b]]++;
    if (index_of) index_of[b] = i;
  }
  for (int r = 0; r < world; ++r) {
    if (rank_count) rank_count[r] = count[r];
    if (rank_flops) rank_flops[r] = load[r];
  }
  return ENC_OK;
}

}  // extern "C"
