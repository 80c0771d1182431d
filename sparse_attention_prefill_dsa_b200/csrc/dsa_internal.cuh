// dsa_internal.cuh -- shared definitions of the CUDA library (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "dsa.h"

namespace dsa {

// First 256 bytes of every workspace.
struct WsHeader {
  unsigned int status;        // 0 or a positive code: kDevTimeout / kDevRange / ...
  unsigned int status_info;   // first failing site (kernel-specific)
  unsigned long long kmax_bits;  // float64 bit pattern of max_s ||k_idx[s]||_2 (>= 0)
  unsigned int akmax_bits;       // float32 bit pattern of max_s ||[latent_s, rope_s]||_2 (>= 0)
  unsigned int unit_next;        // the indexer's work queue: next unit to hand out
  unsigned int topk_redo;        // rows the top-k's window select handed to the bucket select
  unsigned char pad[228];
};
static_assert(sizeof(WsHeader) == 256, "workspace header is 256 bytes");

constexpr unsigned int kDevTimeout = 1;
constexpr unsigned int kDevRange = 2;
constexpr unsigned int kDevInternal = 3;  // an internal consistency check failed
constexpr unsigned int kDevLayout = 4;    // the tensor-core layout self-test found a wrong element
// wait sites of the bounded-wait self-test (the kernels use sites below 100)
constexpr unsigned int kSelftestSiteShort = 101;
constexpr unsigned int kSelftestSiteLong = 102;
constexpr size_t kWsHeaderBytes = 256;

// Records the first device-side failure in the workspace header.
__device__ __forceinline__ void report(WsHeader* ws, unsigned int code, unsigned int info) {
  if (atomicCAS(&ws->status, 0u, code) == 0u) ws->status_info = info;
}

// Bounds checks of the checking build (compiled with -DDSA_CHECK=1, shipped
// as libdsa_check.so): an index outside its buffer records kDevInternal with
// kCheckSiteBase + site as the failing site, and the caller skips the access.
// This stands in for a memory checker: nothing traps, and the status is read
// like any other device-side failure. In the normal build every check is the
// constant true and compiles away.
constexpr unsigned int kCheckSiteBase = 1000;
__device__ __forceinline__ bool check_bound(WsHeader* ws, long long i, long long cap,
                                            unsigned int site) {
  if (i >= 0 && i < cap) return true;
  report(ws, kDevInternal, kCheckSiteBase + site);
  return false;
}
#if defined(DSA_CHECK) && DSA_CHECK
#define DSA_IN_BOUNDS(ws, i, cap, site) \
  ::dsa::check_bound((ws), static_cast<long long>(i), static_cast<long long>(cap), (site))
#else
#define DSA_IN_BOUNDS(ws, i, cap, site) true
#endif


__device__ __forceinline__ float bf16_to_f32(uint16_t h) {
  return __uint_as_float(static_cast<unsigned int>(h) << 16);
}

__device__ __forceinline__ double bf16_to_f64(uint16_t h) {
  return static_cast<double>(__uint_as_float(static_cast<unsigned int>(h) << 16));
}

// float32 -> bf16 bits, round to nearest even (finite inputs).
__device__ __forceinline__ uint16_t f32_to_bf16_rne(float f) {
  unsigned int b = __float_as_uint(f);
  b += 0x7FFFu + ((b >> 16) & 1u);
  return static_cast<uint16_t>(b >> 16);
}

// Launchers (one per kernel family), defined in the .cu files. Each returns
// cudaGetLastError() after its launches.
cudaError_t launch_index_scores(const dsa_dims& d, const uint16_t* q_idx, const uint16_t* k_idx,
                                const float* w_idx, float* scores, int64_t ld, WsHeader* ws,
                                cudaStream_t st);
// FP8 indexer: e4m3 codes with per-row power-of-two scales (quantize first).
cudaError_t launch_index_scores_fp8(const dsa_dims& d, const uint8_t* q8, const float* q_scale,
                                    const uint8_t* k8, const float* k_scale, const float* w_idx,
                                    float* scores, int64_t ld, WsHeader* ws, cudaStream_t st);
cudaError_t launch_quantize_fp8(const uint16_t* x, int64_t rows, int cols, uint8_t* x8,
                                float* scale, uint16_t* xhat, cudaStream_t st);
cudaError_t launch_key_norm_max(const dsa_dims& d, const uint16_t* k_idx, WsHeader* ws,
                                cudaStream_t st);
// Rows longer than one CTA stages (more than 49,152 keys) are selected in two
// passes through a candidate buffer of topk_cand_bytes(d) bytes (0 for shorter
// rows, where `cand` may be null).
size_t topk_cand_bytes(const dsa_dims& d);
cudaError_t launch_topk(const dsa_dims& d, const float* scores, int64_t ld,
                        const uint16_t* q_idx, const uint16_t* k_idx, const float* w_idx,
                        int32_t* idx, WsHeader* ws, void* cand, cudaStream_t st);
// max_s ||[latent_s, rope_s]|| into the header, read by launch_sparse_attn's
// kernel (launch it first, on the same stream, with the header's field zero).
cudaError_t launch_attn_key_norm_max(const dsa_dims& d, const uint16_t* latent, const uint16_t* rope,
                                     WsHeader* ws, cudaStream_t st);
// prefix_valid: every idx row holds its min(top_k, t+1) valid keys first (as the
// selections of dsa_topk_select do), so tiles past them are skipped.
// n_split > 1 cuts every query's key tiles into n_split ranges on different
// SMs (decode); `part` is then the partials' scratch of
// attn_split_bytes(n_q, n_split, n_heads, d_latent) bytes, 16-byte aligned,
// and a combine pass writes out / lse.
cudaError_t launch_sparse_attn(const dsa_dims& d, const uint16_t* q, const uint16_t* latent,
                               const uint16_t* rope, const int32_t* idx, uint16_t* out,
                               float* lse, bool prefix_valid, WsHeader* ws, cudaStream_t st,
                               int n_split = 1, void* part = nullptr);
// The same attention on SM pairs (a cluster of two CTAs per query, each with
// half of every key's dims), for the 32-head 512 + 64 shape only.
bool attn_pair_supported(const dsa_dims& d);
cudaError_t launch_sparse_attn_pair(const dsa_dims& d, const uint16_t* q, const uint16_t* latent,
                                    const uint16_t* rope, const int32_t* idx, uint16_t* out,
                                    float* lse, bool prefix_valid, WsHeader* ws, cudaStream_t st);
// The split the decode entry points use: as many ranges per query as leave no
// SM idle, at most one per 128-key tile of top_k.
int attn_decode_split(const dsa_dims& d);
inline size_t attn_split_ml_bytes(int n_q, int n_split, int H) {
  return (static_cast<size_t>(n_q) * n_split * H * 8 + 255) / 256 * 256;
}
inline size_t attn_split_bytes(int n_q, int n_split, int H, int DC) {
  return attn_split_ml_bytes(n_q, n_split, H) + static_cast<size_t>(n_q) * n_split * H * DC * 4;
}

// DSA_OK when the current device is an sm_100 GPU, else DSA_ERR_DEVICE (or
// DSA_ERR_CUDA when the runtime cannot say). Cached per device.
dsa_status check_current_device();

// Block-sparse attention over groups of qb (1 or 2) neighbouring queries:
// the union of each group's selections (built into `scratch`, of
// block_attn_scratch_bytes(d, qb) bytes, 16-byte aligned), then QK^T / PV on
// the union with per-query masks.
size_t block_attn_scratch_bytes(const dsa_dims& d, int qb);
cudaError_t launch_block_attn(const dsa_dims& d, const uint16_t* q, const uint16_t* latent,
                              const uint16_t* rope, const int32_t* idx, uint16_t* out, float* lse,
                              int qb, WsHeader* ws, void* scratch, cudaStream_t st);

// The bounded-wait self-test (one CTA, two warps on mbarriers nothing signals).
cudaError_t launch_bounded_wait_selftest(WsHeader* ws, long long* cycles, cudaStream_t st);
cudaError_t launch_mma_layout_selftest(WsHeader* ws, int* mismatches, float* cycles_per_mma,
                                      cudaStream_t st);

}  // namespace dsa
