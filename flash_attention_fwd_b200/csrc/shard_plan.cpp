/*
 * shard_plan.cpp — host-side partition of one packed batch over several GPUs
 * (one process per GPU), declared in include/varlen_attn.h.
 *
 * The forward has no exchange step: a (sequence, key/value head) pair and
 * the query heads that map onto that key/value head (kv_h = h / (H / Hkv),
 * the GQA head map of the boostr 0.2.0 source page
 * src/ops/cpu/attention/varlen_attention.rs, varlen_attention_fwd) form a
 * unit that needs nothing from any other unit.  So a batch can be split with
 * no collective on the data path, in one of two ways:
 *
 *   key/value-head groups  every rank computes every sequence for a
 *                          contiguous range of key/value heads and their
 *                          query heads (the tensor-parallel layout: each rank
 *                          holds [T, heads / P, D] slices of q, k, v, out);
 *   sequences              every rank computes all heads of a subset of the
 *                          sequences, chosen to even out the unmasked
 *                          (query, key) pairs, the forward's unit of work.
 *
 * This is host code only; it reads host arrays and allocates nothing on a
 * device.
 */
#include <stdint.h>

#include <algorithm>
#include <numeric>
#include <vector>

#include "varlen_attn.h"

namespace {

// Unmasked (query, key) pairs of one sequence for one query head: query qi
// sees key ki iff ki < lk, qi - left <= ki (left >= 0), ki <= qi + right
// (right >= 0), and not (causal and qi < ki).
int64_t sequence_pairs(int64_t lq, int64_t lk, int causal, int left, int right) {
  if (lq <= 0 || lk <= 0) return 0;
  if (causal) right = 0;  // the causal rule is the right bound 0
  if (left < 0 && right < 0) return lq * lk;
  if (left < 0 && right == 0) {  // plain causal: min(qi + 1, lk) keys
    const int64_t n = std::min(lq, lk);
    return n * (n + 1) / 2 + std::max<int64_t>(0, lq - lk) * lk;
  }
  int64_t total = 0;
  for (int64_t qi = 0; qi < lq; ++qi) {
    const int64_t lo = left >= 0 ? std::max<int64_t>(0, qi - left) : 0;
    const int64_t hi = right >= 0 ? std::min<int64_t>(lk, qi + right + 1) : lk;
    total += std::max<int64_t>(0, hi - lo);
  }
  return total;
}

}  // namespace

extern "C" int varlen_attn_plan_shards(const int32_t *cu_seqlens_q, const int32_t *cu_seqlens_k,
                                       const int32_t *seqused_k, int batch, int num_heads,
                                       int num_kv_heads, int causal, int window_left,
                                       int window_right, int world, int mode, int32_t *seq_rank,
                                       int32_t *kv_head_lo, int32_t *kv_head_hi,
                                       int64_t *rank_pairs) {
  if (batch < 0 || num_heads <= 0 || num_kv_heads <= 0 || num_heads % num_kv_heads != 0 ||
      world < 1 || mode < VARLEN_SHARD_AUTO || mode > VARLEN_SHARD_SEQUENCES)
    return VARLEN_ERR_SHAPE;
  if (!kv_head_lo || !kv_head_hi || !rank_pairs) return VARLEN_ERR_NULL;
  if (batch > 0 && (!cu_seqlens_q || !cu_seqlens_k || !seq_rank)) return VARLEN_ERR_NULL;
  if (mode == VARLEN_SHARD_KV_HEADS && world > num_kv_heads) return VARLEN_ERR_SHAPE;
  const int group = num_heads / num_kv_heads;

  // pairs of each sequence, summed over one key/value head's query heads
  std::vector<int64_t> unit(batch);
  for (int b = 0; b < batch; ++b) {
    const int64_t lq = (int64_t)cu_seqlens_q[b + 1] - cu_seqlens_q[b];
    int64_t lk = (int64_t)cu_seqlens_k[b + 1] - cu_seqlens_k[b];
    if (lq < 0 || lk < 0) return VARLEN_ERR_SHAPE;
    if (seqused_k) lk = std::min<int64_t>(lk, std::max<int32_t>(seqused_k[b], 0));
    unit[b] = group * sequence_pairs(lq, lk, causal, window_left, window_right);
  }
  const int64_t per_kv_head = std::accumulate(unit.begin(), unit.end(), (int64_t)0);

  // key/value-head groups: the first Hkv mod P ranks take one head more
  std::vector<int64_t> heads_load(world, 0);
  if (world <= num_kv_heads) {
    for (int r = 0; r < world; ++r) {
      const int base = num_kv_heads / world, extra = num_kv_heads % world;
      heads_load[r] = (base + (r < extra ? 1 : 0)) * per_kv_head;
    }
  }
  // sequences: longest first, each to the least-loaded rank (lowest on ties)
  std::vector<int32_t> owner(batch, 0);
  std::vector<int64_t> seq_load(world, 0);
  {
    std::vector<int> order(batch);
    std::iota(order.begin(), order.end(), 0);
    std::stable_sort(order.begin(), order.end(),
                     [&](int a, int b) { return unit[a] > unit[b]; });
    for (int b : order) {
      const int r = (int)(std::min_element(seq_load.begin(), seq_load.end()) - seq_load.begin());
      owner[b] = r;
      seq_load[r] += unit[b] * num_kv_heads;
    }
  }
  if (mode == VARLEN_SHARD_AUTO) {
    const int64_t max_heads =
        world <= num_kv_heads ? *std::max_element(heads_load.begin(), heads_load.end()) : -1;
    const int64_t max_seqs = *std::max_element(seq_load.begin(), seq_load.end());
    mode = (max_heads >= 0 && max_heads <= max_seqs) ? VARLEN_SHARD_KV_HEADS
                                                     : VARLEN_SHARD_SEQUENCES;
  }
  if (mode == VARLEN_SHARD_KV_HEADS) {
    int lo = 0;
    for (int r = 0; r < world; ++r) {
      const int n = num_kv_heads / world + (r < num_kv_heads % world ? 1 : 0);
      kv_head_lo[r] = lo;
      kv_head_hi[r] = lo + n;
      rank_pairs[r] = heads_load[r];
      lo += n;
    }
    for (int b = 0; b < batch; ++b) seq_rank[b] = -1;
  } else {
    for (int r = 0; r < world; ++r) {
      kv_head_lo[r] = 0;
      kv_head_hi[r] = num_kv_heads;
      rank_pairs[r] = seq_load[r];
    }
    for (int b = 0; b < batch; ++b) seq_rank[b] = owner[b];
  }
  return mode;
}
