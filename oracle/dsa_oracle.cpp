// dsa_oracle.cpp -- TEST INFRASTRUCTURE ONLY.
//
// A plain, slow, float64 CPU reference ("the oracle") for one DSA sparse-attention
// prefill layer: lightning-indexer scores, per-query top-k selection, and sparse
// MLA-style attention over the selected keys. Only tests/, the smoke check in
// __graft_entry__.py and the CPU-baseline leg of bench.py may load this library.
// The CUDA library never includes, links or calls it, and it includes nothing from
// the CUDA library: the two share no code, header, table or constant.
//
// What the pages say. The one page that describes this layer is the post on
// feedman.me/posts/wy2HU (an M3 Ultra + M5 Ultra prefill/decode split for
// GLM-5.3-Flash):
//   * its per-component prefill table has the rows "DSA indexer" and
//     "DSA sparse-attention core";
//   * the paragraph after the table calls the attention step "the per-query
//     top-2048 gather kernel for sparse attention";
//   * the paragraph "Two levers fell out of this" says that kernel takes one
//     query, gathers that query's 2,048 keys and forms dot products with them;
//   * the paragraph "Why the hand-off is cheap" says the sparse-attention layers
//     keep a 512-wide latent KV per token.
// The pages print no formula for any of the three steps. The definitions used
// here are the plainest reading of DeepSeek-style sparse attention (DSA) that
// agrees with those facts; each is stated at the function that implements it.
//
// Arithmetic rules (so that "bit-exact selection" has one meaning):
//   * every product and sum is an IEEE float64 operation in the order written,
//     with no fused multiply-add (built with -ffp-contract=off, no fast-math);
//   * bf16 inputs are widened exactly (bf16 -> float32 -> float64);
//   * float32 inputs (indexer head weights) are widened exactly.
//
// Pins (see tests/test_oracle.py): hand-computed 4-token cases, brute-force full
// causal attention through torch's float64 scaled-dot-product attention when
// k >= context, exact rational arithmetic on tiny inputs, a numpy lexsort
// selection, and invariants (set sizes, causality, softmax normalisation,
// convex hull, permutation and duplicate-row invariance).

#include <cmath>
#include <cstdint>
#include <cstring>
#include <algorithm>
#include <limits>
#include <thread>
#include <vector>

extern "C" {

// Shapes of one prefill chunk. Query i sits at absolute position t = q_pos0 + i
// and may attend to cache rows s = 0..t (the chunk's own rows are already in
// the cache, so every query sees itself).
typedef struct oracle_dims {
  int32_t n_q;          // queries in the chunk
  int32_t q_pos0;       // absolute position of query 0
  int32_t ctx_len;      // cache rows T (>= q_pos0 + n_q)
  int32_t n_heads;      // attention heads H
  int32_t d_latent;     // latent width Dc (the value is the latent)
  int32_t d_rope;       // rotary part width Dr
  int32_t n_idx_heads;  // indexer heads H_I
  int32_t d_idx;        // indexer head width D_I
  int32_t top_k;        // keys kept per query
  double softmax_scale; // multiplies the attention logits
} oracle_dims;

}  // extern "C"

namespace {

double bf16_to_double(uint16_t h) {
  uint32_t bits = static_cast<uint32_t>(h) << 16;
  float f;
  std::memcpy(&f, &bits, sizeof f);
  return static_cast<double>(f);
}

// Runs body(r) for r in [0, n) on up to n_threads threads (static interleave).
template <class F>
void parallel_rows(int64_t n, int n_threads, F body) {
  if (n_threads < 1) n_threads = 1;
  if (n_threads > n) n_threads = static_cast<int>(n > 0 ? n : 1);
  if (n_threads == 1) {
    for (int64_t r = 0; r < n; ++r) body(r);
    return;
  }
  std::vector<std::thread> pool;
  for (int w = 0; w < n_threads; ++w)
    pool.emplace_back([=, &body] {
      for (int64_t r = w; r < n; r += n_threads) body(r);
    });
  for (auto& th : pool) th.join();
}

bool dims_ok(const oracle_dims* d) {
  return d && d->n_q >= 0 && d->q_pos0 >= 0 && d->ctx_len >= d->q_pos0 + d->n_q &&
         d->n_heads > 0 && d->d_latent > 0 && d->d_rope >= 0 && d->n_idx_heads > 0 &&
         d->d_idx > 0 && d->top_k > 0;
}

// Indexer score of query row i against key s (s <= t), float64, in the order
// the contract fixes:
//   d_j = sum_{c=0}^{D_I-1} qI[i,j,c] * kI[s,c]      (sequential in c)
//   r_j = d_j if d_j > 0 else +0                     (ReLU)
//   I   = sum_{j=0}^{H_I-1} w[i,j] * r_j             (sequential in j)
// One key vector per cache row is shared by all indexer heads; the heads are
// query-side only, and each query weighs its heads with its own w[i,:].
double index_score(const oracle_dims* d, const uint16_t* q_idx, const uint16_t* k_idx,
                   const float* w_idx, int64_t i, int64_t s) {
  const int HI = d->n_idx_heads, DI = d->d_idx;
  double score = 0.0;
  for (int j = 0; j < HI; ++j) {
    const uint16_t* qrow = q_idx + (i * HI + j) * static_cast<int64_t>(DI);
    const uint16_t* krow = k_idx + s * static_cast<int64_t>(DI);
    double dot = 0.0;
    for (int c = 0; c < DI; ++c) dot = dot + bf16_to_double(qrow[c]) * bf16_to_double(krow[c]);
    double relu = dot > 0.0 ? dot : 0.0;
    score = score + static_cast<double>(w_idx[i * HI + j]) * relu;
  }
  return score;
}

// Selection for one query: among candidates s = 0..t, order by (score
// descending, s ascending) and keep the first min(k, t+1); report them in
// ascending s, with -1 in the unused tail of the k slots.
void select_row(const double* row, int64_t t, int k, int32_t* out) {
  std::vector<int32_t> cand(static_cast<size_t>(t + 1));
  for (int64_t s = 0; s <= t; ++s) cand[static_cast<size_t>(s)] = static_cast<int32_t>(s);
  std::sort(cand.begin(), cand.end(), [row](int32_t a, int32_t b) {
    if (row[a] != row[b]) return row[a] > row[b];
    return a < b;
  });
  const int64_t keep = std::min<int64_t>(k, t + 1);
  cand.resize(static_cast<size_t>(keep));
  std::sort(cand.begin(), cand.end());
  for (int64_t c = 0; c < k; ++c) out[c] = c < keep ? cand[static_cast<size_t>(c)] : -1;
}

// Sparse attention for query row i, head h, over the listed keys (-1 ends the
// list's valid part; entries are used in the order given):
//   z_s = scale * ( sum_{c<Dc} q[i,h,c]*latent[s,c] + sum_{c<Dr} q[i,h,Dc+c]*rope[s,c] )
//   p_s = exp(z_s - m) / sum_s' exp(z_s' - m),  m = max_s z_s
//   o   = sum_s p_s * latent[s, :]               (the value is the latent)
//   lse = m + log(sum_s exp(z_s - m))
// q's rotary part and the rope rows are taken as already rotated.
void attend_head(const oracle_dims* d, const uint16_t* q, const uint16_t* latent,
                 const uint16_t* rope, const int32_t* sel, int64_t i, int h, double* o,
                 double* lse) {
  const int Dc = d->d_latent, Dr = d->d_rope, H = d->n_heads, k = d->top_k;
  const uint16_t* qh = q + (i * H + h) * static_cast<int64_t>(Dc + Dr);
  std::vector<double> z;
  std::vector<int32_t> keys;
  for (int c = 0; c < k; ++c) {
    const int32_t s = sel[c];
    if (s < 0) continue;
    const uint16_t* lrow = latent + static_cast<int64_t>(s) * Dc;
    const uint16_t* rrow = rope + static_cast<int64_t>(s) * Dr;
    double dot = 0.0;
    for (int c2 = 0; c2 < Dc; ++c2) dot = dot + bf16_to_double(qh[c2]) * bf16_to_double(lrow[c2]);
    for (int c2 = 0; c2 < Dr; ++c2)
      dot = dot + bf16_to_double(qh[Dc + c2]) * bf16_to_double(rrow[c2]);
    z.push_back(d->softmax_scale * dot);
    keys.push_back(s);
  }
  for (int c2 = 0; c2 < Dc; ++c2) o[c2] = 0.0;
  if (keys.empty()) {  // no key: defined as a zero output and lse = -inf
    if (lse) *lse = -std::numeric_limits<double>::infinity();
    return;
  }
  double m = z[0];
  for (double v : z) m = std::max(m, v);
  double denom = 0.0;
  for (double v : z) denom = denom + std::exp(v - m);
  for (size_t e = 0; e < keys.size(); ++e) {
    const double p = std::exp(z[e] - m) / denom;
    const uint16_t* lrow = latent + static_cast<int64_t>(keys[e]) * Dc;
    for (int c2 = 0; c2 < Dc; ++c2) o[c2] = o[c2] + p * bf16_to_double(lrow[c2]);
  }
  if (lse) *lse = m + std::log(denom);
}

// rows == nullptr means "all n_q rows"; otherwise rows[0..n_rows) are query row
// indices and outputs are packed in that order.
int64_t row_at(const int32_t* rows, int64_t r) { return rows ? rows[r] : r; }

}  // namespace

extern "C" {

// Indexer scores, float64. scores is [n_rows, ctx_len] (row-major). Entries
// s > t are set to -inf (a causal mask; they are never candidates).
int oracle_index_scores(const oracle_dims* d, const uint16_t* q_idx, const uint16_t* k_idx,
                        const float* w_idx, const int32_t* rows, int32_t n_rows,
                        double* scores, int n_threads) {
  if (!dims_ok(d) || !q_idx || !k_idx || !w_idx || !scores) return -1;
  const int64_t nr = rows ? n_rows : d->n_q;
  const int64_t T = d->ctx_len;
  parallel_rows(nr, n_threads, [&](int64_t r) {
    const int64_t i = row_at(rows, r);
    const int64_t t = d->q_pos0 + i;
    double* out = scores + r * T;
    for (int64_t s = 0; s < T; ++s)
      out[s] = s <= t ? index_score(d, q_idx, k_idx, w_idx, i, s)
                      : -std::numeric_limits<double>::infinity();
  });
  return 0;
}

// Top-k selection on given float64 scores. scores row r (leading dimension ld)
// belongs to query row row_at(r); only entries 0..t are read. idx is [n_rows, k].
int oracle_topk_select(const oracle_dims* d, const double* scores, int64_t ld,
                       const int32_t* rows, int32_t n_rows, int32_t* idx, int n_threads) {
  if (!dims_ok(d) || !scores || !idx || ld < d->ctx_len) return -1;
  const int64_t nr = rows ? n_rows : d->n_q;
  parallel_rows(nr, n_threads, [&](int64_t r) {
    const int64_t t = d->q_pos0 + row_at(rows, r);
    select_row(scores + r * ld, t, d->top_k, idx + r * d->top_k);
  });
  return 0;
}

// Same selection on float32 scores (each widened exactly to float64 first).
int oracle_topk_select_f32(const oracle_dims* d, const float* scores, int64_t ld,
                           const int32_t* rows, int32_t n_rows, int32_t* idx,
                           int n_threads) {
  if (!dims_ok(d) || !scores || !idx || ld < d->ctx_len) return -1;
  const int64_t nr = rows ? n_rows : d->n_q;
  parallel_rows(nr, n_threads, [&](int64_t r) {
    const int64_t t = d->q_pos0 + row_at(rows, r);
    std::vector<double> row(static_cast<size_t>(t + 1));
    for (int64_t s = 0; s <= t; ++s) row[static_cast<size_t>(s)] = scores[r * ld + s];
    select_row(row.data(), t, d->top_k, idx + r * d->top_k);
  });
  return 0;
}

// Sparse attention over given selections. idx row r is [k] keys of query row
// row_at(r). out is [n_rows, H, Dc] float64; lse is [n_rows, H] or null.
int oracle_sparse_attn(const oracle_dims* d, const uint16_t* q, const uint16_t* latent,
                       const uint16_t* rope, const int32_t* idx, const int32_t* rows,
                       int32_t n_rows, double* out, double* lse, int n_threads) {
  if (!dims_ok(d) || !q || !latent || (d->d_rope > 0 && !rope) || !idx || !out) return -1;
  const int64_t nr = rows ? n_rows : d->n_q;
  const int H = d->n_heads, Dc = d->d_latent;
  parallel_rows(nr, n_threads, [&](int64_t r) {
    const int64_t i = row_at(rows, r);
    for (int h = 0; h < H; ++h)
      attend_head(d, q, latent, rope, idx + r * d->top_k, i, h, out + (r * H + h) * Dc,
                  lse ? lse + r * H + h : nullptr);
  });
  return 0;
}

// FP8 (e4m3) form of indexer inputs, for the FP8 indexer variant. The pages do
// not describe one; this follows the layer's published design in spirit (an
// 8-bit indexer) with the plainest exact rules:
//   scale  the smallest power of two s = 2^k with max_c |x[r,c]| <= 448 s
//          (448 is the largest finite e4m3 value; s = 1 for an all-zero row);
//   x8     x / s rounded to the nearest e4m3 value, ties to even: 4
//          significant bits for |x/s| >= 2^-6, multiples of 2^-9 below
//          (subnormals); the sign is kept, also on a zero;
//   xhat   x8 * s, the dequantized value (exact, and a bf16 value).
// The FP8 indexer's score contract is the bf16 contract (index_score) applied
// to the dequantized rows xhat.
// x: bf16 [rows, cols]; x8: e4m3 bit patterns [rows, cols]; scale: float
// [rows]; xhat: bf16 [rows, cols].
int oracle_quantize_fp8(const uint16_t* x, int64_t rows, int32_t cols, uint8_t* x8, float* scale,
                        uint16_t* xhat) {
  if (!x || !x8 || !scale || !xhat || rows < 0 || cols < 1) return -1;
  for (int64_t r = 0; r < rows; ++r) {
    const uint16_t* xr = x + r * cols;
    double amax = 0.0;
    for (int c = 0; c < cols; ++c) amax = std::max(amax, std::fabs(bf16_to_double(xr[c])));
    int k = 0;
    if (amax > 0.0) {
      k = std::ilogb(amax) - 9;  // 448 * 2^k < amax here; step up to the first k that covers it
      while (amax > std::ldexp(448.0, k)) ++k;
    }
    scale[r] = static_cast<float>(std::ldexp(1.0, k));
    for (int c = 0; c < cols; ++c) {
      const double xv = bf16_to_double(xr[c]);
      const double v = std::ldexp(xv, -k);  // exact
      const double av = std::fabs(v);
      double qv = 0.0;  // |x8| as a value
      if (av > 0.0) {
        const int e = std::ilogb(av);
        const double quantum = e < -6 ? std::ldexp(1.0, -9) : std::ldexp(1.0, e - 3);
        qv = std::nearbyint(av / quantum) * quantum;  // round half to even
      }
      uint8_t bits = std::signbit(v) ? 0x80 : 0x00;
      if (qv > 0.0) {
        const int e2 = std::ilogb(qv);
        if (e2 < -6) {
          bits |= static_cast<uint8_t>(qv / std::ldexp(1.0, -9));           // subnormal: m * 2^-9
        } else {
          const int mant = static_cast<int>(qv / std::ldexp(1.0, e2 - 3)) - 8;  // 1.mmm * 2^e2
          bits |= static_cast<uint8_t>(((e2 + 7) << 3) | mant);
        }
      }
      x8[r * cols + c] = bits;
      const double hat = std::signbit(v) ? -std::ldexp(qv, k) : std::ldexp(qv, k);
      const float hf = static_cast<float>(hat);  // exact: 4 significant bits
      uint32_t hb;
      std::memcpy(&hb, &hf, sizeof hb);
      xhat[r * cols + c] = static_cast<uint16_t>(hb >> 16);
    }
  }
  return 0;
}

// The whole layer for the listed query rows: scores -> selection -> attention.
// idx_out ([n_rows, k]) and lse ([n_rows, H]) may be null.
int oracle_prefill_layer(const oracle_dims* d, const uint16_t* q, const uint16_t* latent,
                         const uint16_t* rope, const uint16_t* q_idx, const uint16_t* k_idx,
                         const float* w_idx, const int32_t* rows, int32_t n_rows,
                         double* out, double* lse, int32_t* idx_out, int n_threads) {
  if (!dims_ok(d) || !q || !latent || !q_idx || !k_idx || !w_idx || !out) return -1;
  const int64_t nr = rows ? n_rows : d->n_q;
  const int64_t T = d->ctx_len;
  const int H = d->n_heads, Dc = d->d_latent, k = d->top_k;
  parallel_rows(nr, n_threads, [&](int64_t r) {
    const int64_t i = row_at(rows, r);
    const int64_t t = d->q_pos0 + i;
    std::vector<double> row(static_cast<size_t>(T), -std::numeric_limits<double>::infinity());
    for (int64_t s = 0; s <= t; ++s)
      row[static_cast<size_t>(s)] = index_score(d, q_idx, k_idx, w_idx, i, s);
    std::vector<int32_t> sel(static_cast<size_t>(k));
    select_row(row.data(), t, k, sel.data());
    if (idx_out)
      for (int c = 0; c < k; ++c) idx_out[r * k + c] = sel[static_cast<size_t>(c)];
    for (int h = 0; h < H; ++h)
      attend_head(d, q, latent, rope, sel.data(), i, h, out + (r * H + h) * Dc,
                  lse ? lse + r * H + h : nullptr);
  });
  return 0;
}

}  // extern "C"
