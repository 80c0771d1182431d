// partition.cu -- dsa_partition_queries: one chunk's queries split over
// several GPUs (host code only; no device is touched).
//
// Query rows are independent given the cache, so a chunk can be split into
// contiguous query ranges, one per rank, each rank running dsa_prefill_layer
// on its range against the same cache. The work of a row grows with its
// position t: the indexer scores t + 1 causal keys and the top-k reads them,
// while the attention takes min(top_k, t + 1) keys. Equal row counts would
// leave the last rank with the most work, so the ranges are cut where the
// cumulative useful work crosses equal shares:
//   work(t) = (t + 1) * 2 * H_I * D_I  +  min(top_k, t + 1) * 2 * H * (2 Dc + Dr)
// (the indexer's and the attention's multiply-adds per row, the same count
// the throughput figures use). Boundaries are multiples of the smallest row
// count g that keeps every per-row tensor offset 16-byte aligned (g = 1 for
// the 32-head shapes at a top_k that is a multiple of 4; at most 8).
//
// The pages split a model over two machines by experts and attention heads
// (the TensorFold guide on localai.co.kr); a split by queries is what keeps
// the indexer, the top-k and the attention of a row on one GPU, so the only
// exchanges are the chunk's new cache rows before the layer and, when the
// consumer is not itself split by queries, the outputs after it.
#include <stdint.h>

#include <vector>

#include "dsa.h"

extern "C" dsa_status dsa_partition_queries(const dsa_dims* d, int32_t n_parts, int32_t* starts) {
  if (!d || !starts) return DSA_ERR_NULL;
  if (n_parts < 1 || d->n_q < 0 || d->q_pos0 < 0 || d->top_k < 1 || d->n_heads < 1 ||
      d->n_idx_heads < 1 || d->d_idx < 1 || d->d_latent < 1 || d->d_rope < 0)
    return DSA_ERR_DIMS;
  if (static_cast<int64_t>(d->q_pos0) + d->n_q > d->ctx_len) return DSA_ERR_CAUSAL;
  const double w_idx = 2.0 * d->n_idx_heads * d->d_idx;
  const double w_att = 2.0 * d->n_heads * (2.0 * d->d_latent + d->d_rope);
  // prefix[i] = work of rows 0 .. i-1
  std::vector<double> prefix(static_cast<size_t>(d->n_q) + 1, 0.0);
  for (int32_t i = 0; i < d->n_q; ++i) {
    const double keys = static_cast<double>(d->q_pos0) + i + 1;
    const double sel = keys < d->top_k ? keys : static_cast<double>(d->top_k);
    prefix[i + 1] = prefix[i] + keys * w_idx + sel * w_att;
  }
  // rows per step that keep q, q_idx, w_idx, out, lse and idx row offsets
  // 16-byte aligned
  const int64_t row_bytes[6] = {2LL * d->n_heads * (d->d_latent + d->d_rope),
                                2LL * d->n_idx_heads * d->d_idx, 4LL * d->n_idx_heads,
                                2LL * d->n_heads * d->d_latent, 4LL * d->n_heads, 4LL * d->top_k};
  int32_t g = 1;
  for (int64_t rb : row_bytes)
    while ((rb * g) % 16 != 0) g *= 2;  // every row size is even, so g stays <= 8
  const double total = prefix[d->n_q];
  starts[0] = 0;
  int32_t i = 0;
  for (int32_t p = 1; p < n_parts; ++p) {
    const double target = total * p / n_parts;
    while (i < d->n_q && prefix[i] < target) ++i;
    // the nearer of the two row boundaries around the target, rounded to a
    // multiple of g rows
    int32_t b = i;
    if (b > 0 && target - prefix[b - 1] < prefix[b] - target) --b;
    b = (b + g / 2) / g * g;
    if (b > d->n_q) b = d->n_q;
    if (b < starts[p - 1]) b = starts[p - 1];
    starts[p] = b;
  }
  starts[n_parts] = d->n_q;
  return DSA_OK;
}
