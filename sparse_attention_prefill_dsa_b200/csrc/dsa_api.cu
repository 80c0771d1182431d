// dsa_api.cu -- the C ABI: argument checks, workspace layout and launch order.
//
// Every entry point validates its arguments completely before it launches
// anything (a lesson the TensorFold issue #743 thread draws from a sparse
// attention kernel that launched past a hardware limit on some GPUs: here a
// shape the kernels were not built for is an error, never a launch).
#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include "dsa.h"
#include "dsa_internal.cuh"

using dsa::WsHeader;

namespace dsa {
namespace {
constexpr int kMaxDevices = 64;
int g_device_ok[kMaxDevices];  // 0 unknown, 1 sm_100, -1 other
}  // namespace

dsa_status check_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DSA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return DSA_ERR_DEVICE;
  if (g_device_ok[dev] == 0) {
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
      return DSA_ERR_CUDA;
    g_device_ok[dev] = (major == 10 && minor == 0) ? 1 : -1;
  }
  return g_device_ok[dev] == 1 ? DSA_OK : DSA_ERR_DEVICE;
}

}  // namespace dsa

namespace {

dsa_status check_device() { return dsa::check_current_device(); }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool attn_shape_ok(const dsa_dims& d) {
  return (d.n_heads == 4 && d.d_latent == 64 && d.d_rope == 16) ||
         (d.n_heads == 32 && d.d_latent == 512 && d.d_rope == 64);
}

bool indexer_shape_ok(const dsa_dims& d) {
  return (d.n_idx_heads == 2 && d.d_idx == 32) || (d.n_idx_heads == 32 && d.d_idx == 128);
}

// Common shape checks. `need_attn` / `need_indexer` select which head shapes
// the call uses.
dsa_status check_dims(const dsa_dims* d, bool need_attn, bool need_indexer,
                      uint32_t allowed_flags = 0u) {
  if (!d) return DSA_ERR_NULL;
  if ((d->flags & ~allowed_flags) != 0u) return DSA_ERR_DIMS;
  if (d->n_q < 0 || d->q_pos0 < 0 || d->ctx_len < 1 || d->ctx_len > DSA_MAX_CTX)
    return DSA_ERR_DIMS;
  if (d->top_k < 1 || d->top_k > DSA_MAX_TOPK) return DSA_ERR_DIMS;
  if (need_attn && !attn_shape_ok(*d)) return DSA_ERR_DIMS;
  if (need_indexer && !indexer_shape_ok(*d)) return DSA_ERR_DIMS;
  if (need_attn && !(d->softmax_scale > 0.0f && d->softmax_scale < 1e30f)) return DSA_ERR_DIMS;
  if (static_cast<int64_t>(d->q_pos0) + d->n_q > d->ctx_len) return DSA_ERR_CAUSAL;
  return DSA_OK;
}

int64_t layer_ld(const dsa_dims& d) { return (static_cast<int64_t>(d.ctx_len) + 127) / 128 * 128; }

bool l2_scores(const dsa_dims& d) { return (d.flags & DSA_FLAG_L2_SCORES) != 0u; }

// DSA_FLAG_L2_SCORES: query rows per sub-block, so that a sub-block's float32
// scores (rows x ld) take at most 64 MiB of the 126 MB L2 and stay there
// between the indexer that writes them and the top-k that reads them; a
// multiple of 64 rows, at least 64
int l2_subblock_rows(const dsa_dims& d) {
  const int64_t rows = (static_cast<int64_t>(64) << 20) / (layer_ld(d) * 4);
  const int64_t r = rows < 64 ? 64 : rows / 64 * 64;
  return static_cast<int>(r < d.n_q ? r : d.n_q);
}

size_t layer_scores_bytes(const dsa_dims& d) {
  const int64_t rows = l2_scores(d) ? l2_subblock_rows(d) : d.n_q;
  return static_cast<size_t>(rows) * layer_ld(d) * sizeof(float);
}


size_t r256(size_t b) { return (b + 255) / 256 * 256; }

bool fp8_indexer(const dsa_dims& d) { return (d.flags & DSA_FLAG_FP8_INDEXER) != 0u; }

// e4m3 codes, scales and dequantized bf16 copies of `rows` rows of `cols`
size_t fp8_rows_bytes(size_t rows, int cols) {
  return r256(rows * cols) + r256(rows * 4) + r256(rows * cols * 2);
}

// decode: the split attention's partials follow the header (attention alone)
// or the layer's other regions (whole layer)
size_t decode_part_bytes(const dsa_dims& d) {
  const int n_split = dsa::attn_decode_split(d);
  return n_split > 1 ? dsa::attn_split_bytes(d.n_q, n_split, d.n_heads, d.d_latent) : 0;
}

// Byte offsets of the layer's workspace regions: the header; with the FP8
// indexer the keys' e4m3 form (it depends on the cache only, so sub-chunks of
// one chunk find it at the same place); the float32 scores; the selection;
// with the FP8 indexer the queries' e4m3 form; for decode the split
// attention's partials; for rows of more than 49,152 keys the top-k's
// candidate buffer. Without these this is header | scores | idx.
struct LayerWs {
  size_t kfp8, scores, idx, qfp8, part, cand, total;
};

LayerWs layer_ws(const dsa_dims& d, bool decode) {
  const bool f8 = fp8_indexer(d);
  const size_t idx_bytes = static_cast<size_t>(d.n_q) * d.top_k * sizeof(int32_t);
  LayerWs w;
  w.kfp8 = dsa::kWsHeaderBytes;
  w.scores = w.kfp8 + (f8 ? fp8_rows_bytes(static_cast<size_t>(d.ctx_len), d.d_idx) : 0);
  w.idx = w.scores + layer_scores_bytes(d);
  w.qfp8 = w.idx + (f8 || decode ? r256(idx_bytes) : idx_bytes);
  w.part = w.qfp8 + (f8 ? fp8_rows_bytes(static_cast<size_t>(d.n_q) * d.n_idx_heads, d.d_idx) : 0);
  w.cand = w.part + (decode ? decode_part_bytes(d) : 0);
  w.total = w.cand + dsa::topk_cand_bytes(d);
  return w;
}

// Pointers of one FP8 region (codes, scales, dequantized rows) at byte `off`.
struct Fp8Rows {
  uint8_t* x8;
  float* scale;
  uint16_t* xhat;
};

Fp8Rows fp8_rows(void* ws, size_t off, size_t rows, int cols) {
  char* b = static_cast<char*>(ws) + off;
  Fp8Rows r;
  r.x8 = reinterpret_cast<uint8_t*>(b);
  r.scale = reinterpret_cast<float*>(b + r256(rows * cols));
  r.xhat = reinterpret_cast<uint16_t*>(b + r256(rows * cols) + r256(rows * 4));
  return r;
}

dsa_status check_ws(const dsa_dims& d, int which, void* ws, size_t bytes) {
  if (!ws) return DSA_ERR_WORKSPACE;
  if (!aligned16(ws)) return DSA_ERR_ALIGN;
  if (bytes < dsa_workspace_size(&d, which)) return DSA_ERR_WORKSPACE;
  return DSA_OK;
}

dsa_status from_cuda(cudaError_t e) { return e == cudaSuccess ? DSA_OK : DSA_ERR_CUDA; }

dsa_status clear_header(void* ws, cudaStream_t st) {
  return from_cuda(cudaMemsetAsync(ws, 0, dsa::kWsHeaderBytes, st));
}

// The prefill attention: on SM pairs when the caller asks for it
// (DSA_FLAG_ATTN_PAIR) and the shape has that kernel, else one SM per query.
cudaError_t attention(const dsa_dims& d, const uint16_t* q, const uint16_t* latent,
                      const uint16_t* rope, const int32_t* idx, uint16_t* out, float* lse,
                      bool prefix_valid, WsHeader* h, cudaStream_t st) {
  if ((d.flags & DSA_FLAG_ATTN_PAIR) != 0u && dsa::attn_pair_supported(d))
    return dsa::launch_sparse_attn_pair(d, q, latent, rope, idx, out, lse, prefix_valid, h, st);
  return dsa::launch_sparse_attn(d, q, latent, rope, idx, out, lse, prefix_valid, h, st);
}

// The layer's kernels on validated arguments (the workspace header cleared
// by the caller): scores -> exact top-k -> attention. The two key-norm passes
// (max ||k_idx[s]|| for the top-k band, max ||[latent_s, rope_s]|| for the
// attention's score bound) depend only on the cache, so a caller that runs
// several sub-chunks against one cache and one header computes them once
// (norms_ready = false on the first sub-chunk only).
dsa_status enqueue_layer(const dsa_dims& d, const uint16_t* q, const uint16_t* latent,
                         const uint16_t* rope, const uint16_t* q_idx, const uint16_t* k_idx,
                         const float* w_idx, uint16_t* out, float* lse, int32_t* idx_out, void* ws,
                         cudaStream_t st, bool norms_ready = false, bool decode = false) {
  if (d.n_q == 0) return DSA_OK;
  WsHeader* h = static_cast<WsHeader*>(ws);
  const LayerWs w = layer_ws(d, decode);
  float* scores = reinterpret_cast<float*>(static_cast<char*>(ws) + w.scores);
  const int64_t ld = layer_ld(d);
  // The selection goes to the caller's idx_out when given, else to the
  // workspace region after the score matrix.
  int32_t* idx = idx_out ? idx_out : reinterpret_cast<int32_t*>(static_cast<char*>(ws) + w.idx);
  void* cand = static_cast<char*>(ws) + w.cand;
  cudaError_t e = cudaSuccess;
  if (fp8_indexer(d)) {
    // FP8 indexer: the e4m3 forms of k_idx (once per cache) and q_idx; the
    // exact top-k orders by the float64 contract on their dequantized rows
    const Fp8Rows k8 = fp8_rows(ws, w.kfp8, static_cast<size_t>(d.ctx_len), d.d_idx);
    const size_t q_rows = static_cast<size_t>(d.n_q) * d.n_idx_heads;
    const Fp8Rows q8 = fp8_rows(ws, w.qfp8, q_rows, d.d_idx);
    if (!norms_ready) {
      e = dsa::launch_quantize_fp8(k_idx, d.ctx_len, d.d_idx, k8.x8, k8.scale, k8.xhat, st);
      if (e == cudaSuccess) e = dsa::launch_key_norm_max(d, k8.xhat, h, st);
      if (e == cudaSuccess) e = dsa::launch_attn_key_norm_max(d, latent, rope, h, st);
    }
    if (e == cudaSuccess)
      e = dsa::launch_quantize_fp8(q_idx, static_cast<int64_t>(q_rows), d.d_idx, q8.x8, q8.scale,
                                   q8.xhat, st);
    if (e == cudaSuccess)
      e = dsa::launch_index_scores_fp8(d, q8.x8, q8.scale, k8.x8, k8.scale, w_idx, scores, ld, h, st);
    if (e != cudaSuccess) return DSA_ERR_CUDA;
    e = dsa::launch_topk(d, scores, ld, q8.xhat, k8.xhat, w_idx, idx, h, cand, st);
  } else {
    if (!norms_ready) {
      e = dsa::launch_key_norm_max(d, k_idx, h, st);
      if (e == cudaSuccess) e = dsa::launch_attn_key_norm_max(d, latent, rope, h, st);
    }
    // scores then selection, over the whole chunk or (DSA_FLAG_L2_SCORES)
    // over query sub-blocks whose scores stay in L2; a row's scores and
    // selection do not depend on the rows launched with it
    const int step = l2_scores(d) ? l2_subblock_rows(d) : d.n_q;
    for (int r0 = 0; r0 < d.n_q && e == cudaSuccess; r0 += step) {
      dsa_dims ds = d;
      ds.n_q = d.n_q - r0 < step ? d.n_q - r0 : step;
      ds.q_pos0 = d.q_pos0 + r0;
      const uint16_t* qi = q_idx + static_cast<int64_t>(r0) * d.n_idx_heads * d.d_idx;
      const float* wi = w_idx + static_cast<int64_t>(r0) * d.n_idx_heads;
      e = dsa::launch_index_scores(ds, qi, k_idx, wi, scores, ld, h, st);
      if (e == cudaSuccess)
        e = dsa::launch_topk(ds, scores, ld, qi, k_idx, wi, idx + static_cast<int64_t>(r0) * d.top_k, h,
                             cand, st);
    }
  }
  if (e != cudaSuccess) return DSA_ERR_CUDA;
  if (decode) {
    const int n_split = dsa::attn_decode_split(d);
    void* part = n_split > 1 ? static_cast<char*>(ws) + w.part : nullptr;
    return from_cuda(
        dsa::launch_sparse_attn(d, q, latent, rope, idx, out, lse, true, h, st, n_split, part));
  }
  return from_cuda(attention(d, q, latent, rope, idx, out, lse, true, h, st));
}

cudaError_t h2d(void* dst, const void* src, size_t bytes, cudaStream_t st) {
  return bytes ? cudaMemcpyAsync(dst, src, bytes, cudaMemcpyHostToDevice, st) : cudaSuccess;
}

cudaError_t d2h(void* dst, const void* src, size_t bytes, cudaStream_t st) {
  return bytes ? cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToHost, st) : cudaSuccess;
}

}  // namespace

extern "C" {

size_t dsa_workspace_size(const dsa_dims* d, int32_t which) {
  if (!d || d->n_q < 0 || d->ctx_len < 1) return 0;
  switch (which) {
    case DSA_WS_INDEX_SCORES:
    case DSA_WS_ATTN:
      return dsa::kWsHeaderBytes;
    case DSA_WS_TOPK:
      return dsa::kWsHeaderBytes + dsa::topk_cand_bytes(*d);
    case DSA_WS_LAYER:
      return layer_ws(*d, false).total;
    case DSA_WS_DECODE_ATTN:
      return dsa::kWsHeaderBytes + decode_part_bytes(*d);
    case DSA_WS_DECODE_LAYER:
      return layer_ws(*d, true).total;
    case DSA_WS_BLOCK_ATTN:
      return dsa::kWsHeaderBytes + dsa::block_attn_scratch_bytes(*d, DSA_MAX_BLOCK_QUERIES);
    default:
      return 0;
  }
}

dsa_status dsa_index_scores(const dsa_dims* d, const uint16_t* q_idx, const uint16_t* k_idx,
                            const float* w_idx, float* scores, int64_t ld, void* ws,
                            size_t ws_bytes, void* stream) {
  dsa_status s = check_dims(d, false, true);
  if (s != DSA_OK) return s;
  if (!q_idx || !k_idx || !w_idx || !scores) return DSA_ERR_NULL;
  if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(w_idx) || !aligned16(scores) ||
      ld % 4 != 0)
    return DSA_ERR_ALIGN;
  if (ld < d->ctx_len) return DSA_ERR_DIMS;
  if ((s = check_ws(*d, DSA_WS_INDEX_SCORES, ws, ws_bytes)) != DSA_OK) return s;
  if ((s = check_device()) != DSA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((s = clear_header(ws, st)) != DSA_OK) return s;
  if (d->n_q == 0) return DSA_OK;
  return from_cuda(dsa::launch_index_scores(*d, q_idx, k_idx, w_idx, scores, ld,
                                            static_cast<WsHeader*>(ws), st));
}

dsa_status dsa_topk_select(const dsa_dims* d, const float* scores, int64_t ld,
                           const uint16_t* q_idx, const uint16_t* k_idx, const float* w_idx,
                           int32_t* idx, void* ws, size_t ws_bytes, void* stream) {
  const int given = (q_idx != nullptr) + (k_idx != nullptr) + (w_idx != nullptr);
  dsa_status s = check_dims(d, false, given == 3);
  if (s != DSA_OK) return s;
  if (!scores || !idx || (given != 0 && given != 3)) return DSA_ERR_NULL;
  if (!aligned16(scores) || !aligned16(idx) || ld % 4 != 0) return DSA_ERR_ALIGN;
  if (given == 3 && (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(w_idx)))
    return DSA_ERR_ALIGN;
  if (ld < d->ctx_len) return DSA_ERR_DIMS;
  if ((s = check_ws(*d, DSA_WS_TOPK, ws, ws_bytes)) != DSA_OK) return s;
  if ((s = check_device()) != DSA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((s = clear_header(ws, st)) != DSA_OK) return s;
  if (d->n_q == 0) return DSA_OK;
  WsHeader* h = static_cast<WsHeader*>(ws);
  if (given == 3) {
    cudaError_t e = dsa::launch_key_norm_max(*d, k_idx, h, st);
    if (e != cudaSuccess) return DSA_ERR_CUDA;
  }
  return from_cuda(dsa::launch_topk(*d, scores, ld, q_idx, k_idx, w_idx, idx, h,
                                    static_cast<char*>(ws) + dsa::kWsHeaderBytes, st));
}

dsa_status dsa_sparse_attn_prefill(const dsa_dims* d, const uint16_t* q, const uint16_t* latent,
                                   const uint16_t* rope, const int32_t* idx, uint16_t* out,
                                   float* lse, void* ws, size_t ws_bytes, void* stream) {
  dsa_status s = check_dims(d, true, false, DSA_FLAG_ATTN_PAIR);
  if (s != DSA_OK) return s;
  if (!q || !latent || !rope || !idx || !out) return DSA_ERR_NULL;
  if (!aligned16(q) || !aligned16(latent) || !aligned16(rope) || !aligned16(idx) ||
      !aligned16(out) || (lse && !aligned16(lse)))
    return DSA_ERR_ALIGN;
  if ((s = check_ws(*d, DSA_WS_ATTN, ws, ws_bytes)) != DSA_OK) return s;
  if ((s = check_device()) != DSA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((s = clear_header(ws, st)) != DSA_OK) return s;
  if (d->n_q == 0) return DSA_OK;
  WsHeader* h = static_cast<WsHeader*>(ws);
  cudaError_t e = dsa::launch_attn_key_norm_max(*d, latent, rope, h, st);
  if (e != cudaSuccess) return DSA_ERR_CUDA;
  return from_cuda(attention(*d, q, latent, rope, idx, out, lse, false, h, st));
}

dsa_status dsa_sparse_attn_decode(const dsa_dims* d, const uint16_t* q, const uint16_t* latent,
                                  const uint16_t* rope, const int32_t* idx, uint16_t* out,
                                  float* lse, void* ws, size_t ws_bytes, void* stream) {
  dsa_status s = check_dims(d, true, false);
  if (s != DSA_OK) return s;
  if (!q || !latent || !rope || !idx || !out) return DSA_ERR_NULL;
  if (!aligned16(q) || !aligned16(latent) || !aligned16(rope) || !aligned16(idx) ||
      !aligned16(out) || (lse && !aligned16(lse)))
    return DSA_ERR_ALIGN;
  if ((s = check_ws(*d, DSA_WS_DECODE_ATTN, ws, ws_bytes)) != DSA_OK) return s;
  if ((s = check_device()) != DSA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((s = clear_header(ws, st)) != DSA_OK) return s;
  if (d->n_q == 0) return DSA_OK;
  WsHeader* h = static_cast<WsHeader*>(ws);
  cudaError_t e = dsa::launch_attn_key_norm_max(*d, latent, rope, h, st);
  if (e != cudaSuccess) return DSA_ERR_CUDA;
  const int n_split = dsa::attn_decode_split(*d);
  void* part = n_split > 1 ? static_cast<char*>(ws) + dsa::kWsHeaderBytes : nullptr;
  return from_cuda(dsa::launch_sparse_attn(*d, q, latent, rope, idx, out, lse, false, h, st,
                                           n_split, part));
}

dsa_status dsa_quantize_fp8(const uint16_t* x, int64_t rows, int32_t cols, uint8_t* x8,
                            float* scale, uint16_t* xhat, void* stream) {
  if (rows < 0 || cols < 1 || cols > 128) return DSA_ERR_DIMS;
  if (!x || !x8 || !scale || !xhat) return DSA_ERR_NULL;
  if (!aligned16(x) || !aligned16(x8) || !aligned16(scale) || !aligned16(xhat)) return DSA_ERR_ALIGN;
  dsa_status s = check_device();
  if (s != DSA_OK) return s;
  return from_cuda(dsa::launch_quantize_fp8(x, rows, cols, x8, scale, xhat,
                                            static_cast<cudaStream_t>(stream)));
}

dsa_status dsa_index_scores_fp8(const dsa_dims* d, const uint8_t* q8, const float* q_scale,
                                const uint8_t* k8, const float* k_scale, const float* w_idx,
                                float* scores, int64_t ld, void* ws, size_t ws_bytes, void* stream) {
  dsa_status s = check_dims(d, false, true);
  if (s != DSA_OK) return s;
  if (!q8 || !q_scale || !k8 || !k_scale || !w_idx || !scores) return DSA_ERR_NULL;
  if (!aligned16(q8) || !aligned16(q_scale) || !aligned16(k8) || !aligned16(k_scale) ||
      !aligned16(w_idx) || !aligned16(scores) || ld % 4 != 0)
    return DSA_ERR_ALIGN;
  if (ld < d->ctx_len) return DSA_ERR_DIMS;
  if ((s = check_ws(*d, DSA_WS_INDEX_SCORES, ws, ws_bytes)) != DSA_OK) return s;
  if ((s = check_device()) != DSA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((s = clear_header(ws, st)) != DSA_OK) return s;
  if (d->n_q == 0) return DSA_OK;
  return from_cuda(dsa::launch_index_scores_fp8(*d, q8, q_scale, k8, k_scale, w_idx, scores, ld,
                                                static_cast<WsHeader*>(ws), st));
}

dsa_status dsa_sparse_attn_block(const dsa_dims* d, const uint16_t* q, const uint16_t* latent,
                                 const uint16_t* rope, const int32_t* idx, uint16_t* out,
                                 float* lse, int32_t block_queries, void* ws, size_t ws_bytes,
                                 void* stream) {
  dsa_status s = check_dims(d, true, false);
  if (s != DSA_OK) return s;
  if (block_queries < 1 || block_queries > DSA_MAX_BLOCK_QUERIES) return DSA_ERR_DIMS;
  if (!q || !latent || !rope || !idx || !out) return DSA_ERR_NULL;
  if (!aligned16(q) || !aligned16(latent) || !aligned16(rope) || !aligned16(idx) ||
      !aligned16(out) || (lse && !aligned16(lse)))
    return DSA_ERR_ALIGN;
  if ((s = check_ws(*d, DSA_WS_BLOCK_ATTN, ws, ws_bytes)) != DSA_OK) return s;
  if ((s = check_device()) != DSA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((s = clear_header(ws, st)) != DSA_OK) return s;
  if (d->n_q == 0) return DSA_OK;
  return from_cuda(dsa::launch_block_attn(*d, q, latent, rope, idx, out, lse, block_queries,
                                          static_cast<WsHeader*>(ws),
                                          static_cast<char*>(ws) + dsa::kWsHeaderBytes, st));
}

dsa_status dsa_decode_layer(const dsa_dims* d, const uint16_t* q, const uint16_t* latent,
                            const uint16_t* rope, const uint16_t* q_idx, const uint16_t* k_idx,
                            const float* w_idx, uint16_t* out, float* lse, int32_t* idx_out,
                            void* ws, size_t ws_bytes, void* stream) {
  dsa_status s = check_dims(d, true, true, DSA_FLAG_FP8_INDEXER | DSA_FLAG_ATTN_PAIR);
  if (s != DSA_OK) return s;
  if (!q || !latent || !rope || !q_idx || !k_idx || !w_idx || !out) return DSA_ERR_NULL;
  if (!aligned16(q) || !aligned16(latent) || !aligned16(rope) || !aligned16(q_idx) ||
      !aligned16(k_idx) || !aligned16(w_idx) || !aligned16(out) || (lse && !aligned16(lse)) ||
      (idx_out && !aligned16(idx_out)))
    return DSA_ERR_ALIGN;
  if ((s = check_ws(*d, DSA_WS_DECODE_LAYER, ws, ws_bytes)) != DSA_OK) return s;
  if ((s = check_device()) != DSA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((s = clear_header(ws, st)) != DSA_OK) return s;
  return enqueue_layer(*d, q, latent, rope, q_idx, k_idx, w_idx, out, lse, idx_out, ws, st,
                       /*norms_ready=*/false, /*decode=*/true);
}

dsa_status dsa_prefill_layer(const dsa_dims* d, const uint16_t* q, const uint16_t* latent,
                             const uint16_t* rope, const uint16_t* q_idx, const uint16_t* k_idx,
                             const float* w_idx, uint16_t* out, float* lse, int32_t* idx_out,
                             void* ws, size_t ws_bytes, void* stream) {
  dsa_status s =
      check_dims(d, true, true, DSA_FLAG_FP8_INDEXER | DSA_FLAG_ATTN_PAIR | DSA_FLAG_L2_SCORES);
  if (s != DSA_OK) return s;
  if (fp8_indexer(*d) && l2_scores(*d)) return DSA_ERR_DIMS;  // sub-blocks: bf16 indexer only
  if (!q || !latent || !rope || !q_idx || !k_idx || !w_idx || !out) return DSA_ERR_NULL;
  if (!aligned16(q) || !aligned16(latent) || !aligned16(rope) || !aligned16(q_idx) ||
      !aligned16(k_idx) || !aligned16(w_idx) || !aligned16(out) || (lse && !aligned16(lse)) ||
      (idx_out && !aligned16(idx_out)))
    return DSA_ERR_ALIGN;
  if ((s = check_ws(*d, DSA_WS_LAYER, ws, ws_bytes)) != DSA_OK) return s;
  if ((s = check_device()) != DSA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((s = clear_header(ws, st)) != DSA_OK) return s;
  return enqueue_layer(*d, q, latent, rope, q_idx, k_idx, w_idx, out, lse, idx_out, ws, st);
}

dsa_status dsa_prefill_layer_host(const dsa_dims* d, const uint16_t* q, const uint16_t* latent,
                                  const uint16_t* rope, const uint16_t* q_idx, const uint16_t* k_idx,
                                  const float* w_idx, uint16_t* out, float* lse, int32_t* idx_out,
                                  const dsa_device_tensors* dev, void* ws, size_t ws_bytes,
                                  void* const streams[3], void* const events[2], int32_t n_sub) {
  dsa_status s =
      check_dims(d, true, true, DSA_FLAG_FP8_INDEXER | DSA_FLAG_ATTN_PAIR | DSA_FLAG_HOST_UNORDERED);
  if (s != DSA_OK) return s;
  if (!q || !latent || !rope || !q_idx || !k_idx || !w_idx || !out || !dev || !streams || !events)
    return DSA_ERR_NULL;
  if (!events[0] || !events[1]) return DSA_ERR_NULL;
  if (!dev->q || !dev->latent || !dev->rope || !dev->q_idx || !dev->k_idx || !dev->w_idx ||
      !dev->out || (lse && !dev->lse) || (idx_out && !dev->idx))
    return DSA_ERR_NULL;
  if (!aligned16(dev->q) || !aligned16(dev->latent) || !aligned16(dev->rope) ||
      !aligned16(dev->q_idx) || !aligned16(dev->k_idx) || !aligned16(dev->w_idx) ||
      !aligned16(dev->out) || (dev->lse && !aligned16(dev->lse)) ||
      (dev->idx && !aligned16(dev->idx)))
    return DSA_ERR_ALIGN;
  if (n_sub < 1) return DSA_ERR_DIMS;
  if ((s = check_ws(*d, DSA_WS_LAYER, ws, ws_bytes)) != DSA_OK) return s;
  if ((s = check_device()) != DSA_OK) return s;
  cudaStream_t s_in = static_cast<cudaStream_t>(streams[0]);
  cudaStream_t s_run = static_cast<cudaStream_t>(streams[1]);
  cudaStream_t s_out = static_cast<cudaStream_t>(streams[2]);
  cudaEvent_t ev_a = static_cast<cudaEvent_t>(events[0]);
  cudaEvent_t ev_b = static_cast<cudaEvent_t>(events[1]);
  // work already on the streams (an earlier call) ends before this call's
  // copies overwrite the inputs its layers read and its layers overwrite the
  // outputs its copies read (unless the caller orders the calls itself)
  cudaError_t e = cudaSuccess;
  if ((d->flags & DSA_FLAG_HOST_UNORDERED) == 0u) {
    e = cudaEventRecord(ev_a, s_run);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s_in, ev_a, 0);
    if (e == cudaSuccess) e = cudaEventRecord(ev_b, s_out);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s_run, ev_b, 0);
    if (e != cudaSuccess) return DSA_ERR_CUDA;
  }
  if ((s = clear_header(ws, s_run)) != DSA_OK) return s;  // once: sub-chunks keep each other's status
  if (d->n_q == 0) return DSA_OK;
  const size_t T = static_cast<size_t>(d->ctx_len);
  const size_t q_row = static_cast<size_t>(d->n_heads) * (d->d_latent + d->d_rope);
  const size_t qi_row = static_cast<size_t>(d->n_idx_heads) * d->d_idx;
  const size_t w_row = static_cast<size_t>(d->n_idx_heads);
  const size_t o_row = static_cast<size_t>(d->n_heads) * d->d_latent;
  const size_t l_row = static_cast<size_t>(d->n_heads);
  const size_t i_row = static_cast<size_t>(d->top_k);
  e = h2d(dev->latent, latent, T * d->d_latent * 2, s_in);
  if (e == cudaSuccess) e = h2d(dev->rope, rope, T * d->d_rope * 2, s_in);
  if (e == cudaSuccess) e = h2d(dev->k_idx, k_idx, T * d->d_idx * 2, s_in);
  if (e != cudaSuccess) return DSA_ERR_CUDA;
  // sub-chunks of a multiple of 4 rows keep every row offset 16-byte aligned
  int rows = (d->n_q + n_sub - 1) / n_sub;
  rows = (rows + 3) & ~3;
  for (int r0 = 0; r0 < d->n_q; r0 += rows) {
    const int nr = d->n_q - r0 < rows ? d->n_q - r0 : rows;
    const size_t o = static_cast<size_t>(r0), n = static_cast<size_t>(nr);
    e = h2d(dev->q + o * q_row, q + o * q_row, n * q_row * 2, s_in);
    if (e == cudaSuccess) e = h2d(dev->q_idx + o * qi_row, q_idx + o * qi_row, n * qi_row * 2, s_in);
    if (e == cudaSuccess) e = h2d(dev->w_idx + o * w_row, w_idx + o * w_row, n * w_row * 4, s_in);
    if (e == cudaSuccess) e = cudaEventRecord(ev_a, s_in);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s_run, ev_a, 0);
    if (e != cudaSuccess) return DSA_ERR_CUDA;
    dsa_dims sub = *d;
    sub.n_q = nr;
    sub.q_pos0 = d->q_pos0 + r0;
    s = enqueue_layer(sub, dev->q + o * q_row, dev->latent, dev->rope, dev->q_idx + o * qi_row,
                      dev->k_idx, dev->w_idx + o * w_row, dev->out + o * o_row,
                      lse ? dev->lse + o * l_row : nullptr, idx_out ? dev->idx + o * i_row : nullptr,
                      ws, s_run, /*norms_ready=*/r0 > 0);
    if (s != DSA_OK) return s;
    e = cudaEventRecord(ev_b, s_run);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s_out, ev_b, 0);
    if (e == cudaSuccess) e = d2h(out + o * o_row, dev->out + o * o_row, n * o_row * 2, s_out);
    if (e == cudaSuccess && lse) e = d2h(lse + o * l_row, dev->lse + o * l_row, n * l_row * 4, s_out);
    if (e == cudaSuccess && idx_out)
      e = d2h(idx_out + o * i_row, dev->idx + o * i_row, n * i_row * 4, s_out);
    if (e != cudaSuccess) return DSA_ERR_CUDA;
  }
  return DSA_OK;
}

dsa_status dsa_selftest_bounded_wait(void* ws, size_t ws_bytes, int64_t* cycles, void* stream) {
  if (!ws || ws_bytes < dsa::kWsHeaderBytes) return DSA_ERR_WORKSPACE;
  if (!aligned16(ws) || (cycles && (reinterpret_cast<uintptr_t>(cycles) & 7u))) return DSA_ERR_ALIGN;
  dsa_status s = check_device();
  if (s != DSA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((s = clear_header(ws, st)) != DSA_OK) return s;
  return from_cuda(dsa::launch_bounded_wait_selftest(static_cast<dsa::WsHeader*>(ws),
                                                     reinterpret_cast<long long*>(cycles), st));
}

dsa_status dsa_selftest_mma_layout(void* ws, size_t ws_bytes, int32_t* mismatches,
                                   float* cycles_per_mma, void* stream) {
  if (!ws || ws_bytes < dsa::kWsHeaderBytes + 32) return DSA_ERR_WORKSPACE;
  if (!aligned16(ws)) return DSA_ERR_ALIGN;
  dsa_status s = check_device();
  if (s != DSA_OK) return s;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((s = clear_header(ws, st)) != DSA_OK) return s;
  unsigned char* out = static_cast<unsigned char*>(ws) + dsa::kWsHeaderBytes;
  int* dev_counts = reinterpret_cast<int*>(out);
  float* dev_cycles = reinterpret_cast<float*>(out + 16);
  if ((s = from_cuda(dsa::launch_mma_layout_selftest(static_cast<dsa::WsHeader*>(ws), dev_counts,
                                                     dev_cycles, st))) != DSA_OK)
    return s;
  if (mismatches &&
      cudaMemcpyAsync(mismatches, dev_counts, 4 * sizeof(int32_t), cudaMemcpyDeviceToHost, st) !=
          cudaSuccess)
    return DSA_ERR_CUDA;
  if (cycles_per_mma &&
      cudaMemcpyAsync(cycles_per_mma, dev_cycles, 4 * sizeof(float), cudaMemcpyDeviceToHost, st) !=
          cudaSuccess)
    return DSA_ERR_CUDA;
  if ((mismatches || cycles_per_mma) && cudaStreamSynchronize(st) != cudaSuccess) return DSA_ERR_CUDA;
  return DSA_OK;
}

dsa_status dsa_device_status(void* ws, void* stream) {
  if (!ws) return DSA_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return DSA_ERR_CUDA;
  unsigned int code = 0;
  if (cudaMemcpy(&code, ws, sizeof code, cudaMemcpyDeviceToHost) != cudaSuccess)
    return DSA_ERR_CUDA;
  if (code != 0 && cudaMemset(ws, 0, 2 * sizeof(unsigned int)) != cudaSuccess)
    return DSA_ERR_CUDA;
  if (code == dsa::kDevTimeout) return DSA_ERR_TIMEOUT;
  if (code == dsa::kDevRange) return DSA_ERR_RANGE;
  if (code == dsa::kDevLayout) return DSA_ERR_LAYOUT;
  return code == 0 ? DSA_OK : DSA_ERR_CUDA;
}

const char* dsa_status_string(dsa_status s) {
  switch (s) {
    case DSA_OK: return "ok";
    case DSA_ERR_NULL: return "a required pointer is NULL";
    case DSA_ERR_ALIGN: return "a pointer is not 16-byte aligned, or ld is not a multiple of 4";
    case DSA_ERR_DIMS: return "unsupported or inconsistent shape, or nonzero flags";
    case DSA_ERR_CAUSAL: return "q_pos0 + n_q exceeds ctx_len";
    case DSA_ERR_WORKSPACE: return "workspace missing or smaller than dsa_workspace_size()";
    case DSA_ERR_TIMEOUT: return "a device-side bounded wait gave up";
    case DSA_ERR_CUDA: return "CUDA runtime or launch error";
    case DSA_ERR_DEVICE: return "current device is not an sm_100 (B200) GPU";
    case DSA_ERR_RANGE: return "a selected index was outside the causal range 0..t of its query";
    case DSA_ERR_LAYOUT:
      return "the tensor-core layout self-test found an accumulator element that differs";
    case DSA_ERR_SCRATCH_LIMIT:
      return "the chunk needs more scratch than the no-alloc entry point's static array holds";
    default: return "unknown status";
  }
}

}  // extern "C"
