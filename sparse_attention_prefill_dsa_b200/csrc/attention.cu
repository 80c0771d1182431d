// attention.cu -- sparse MLA-style attention over the selected keys
// (component-table row "DSA sparse-attention core" of the feedman.me post
// feedman.me/posts/wy2HU).
//
//   z_s = scale * (q[:Dc] . latent[s] + q[Dc:] . rope[s]),  out = softmax(z) @ latent
//
// Straightforward CUDA-core version: one CTA per query, one warp per head;
// lanes split the 576-wide dot, a warp reduction forms each logit, and an
// online softmax (running max and sum in float32) accumulates the latent rows.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "dsa_internal.cuh"

namespace dsa {
namespace {

template <int H, int DC, int DR>
__global__ void __launch_bounds__(H * 32) sparse_attn_simple(
    const uint16_t* __restrict__ q, const uint16_t* __restrict__ latent,
    const uint16_t* __restrict__ rope, const int32_t* __restrict__ idx,
    uint16_t* __restrict__ out, float* __restrict__ lse, int k, int ctx_len, float scale,
    WsHeader* ws) {
  constexpr int QPL = (DC + DR + 31) / 32;  // q elements per lane
  constexpr int OPL = DC / 32;              // output elements per lane
  const int i = blockIdx.x;
  const int h = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint16_t* qh = q + (static_cast<int64_t>(i) * H + h) * (DC + DR);
  float qv[QPL];
#pragma unroll
  for (int e = 0; e < QPL; ++e) {
    const int c = lane + 32 * e;
    qv[e] = c < DC + DR ? bf16_to_f32(qh[c]) : 0.f;
  }
  float o[OPL];
#pragma unroll
  for (int e = 0; e < OPL; ++e) o[e] = 0.f;
  float m = -INFINITY, l = 0.f;
  const int32_t* sel = idx + static_cast<int64_t>(i) * k;
  for (int e = 0; e < k; ++e) {
    const int s = sel[e];
    if (s < 0) continue;
    if (s >= ctx_len) {
      if (lane == 0 && h == 0) report(ws, kDevRange, static_cast<unsigned>(i));
      continue;
    }
    const uint16_t* lr = latent + static_cast<int64_t>(s) * DC;
    const uint16_t* rr = rope + static_cast<int64_t>(s) * DR;
    float dot = 0.f;
#pragma unroll
    for (int e2 = 0; e2 < QPL; ++e2) {
      const int c = lane + 32 * e2;
      float kv = 0.f;
      if (c < DC) kv = bf16_to_f32(lr[c]);
      else if (c < DC + DR) kv = bf16_to_f32(rr[c - DC]);
      dot = fmaf(qv[e2], kv, dot);
    }
#pragma unroll
    for (int off = 16; off; off >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, off);
    const float z = dot * scale;
    const float m_new = fmaxf(m, z);
    const float corr = __expf(m - m_new);
    const float p = __expf(z - m_new);
    l = l * corr + p;
#pragma unroll
    for (int e2 = 0; e2 < OPL; ++e2) o[e2] = o[e2] * corr + p * bf16_to_f32(lr[lane + 32 * e2]);
    m = m_new;
  }
  const float inv = l > 0.f ? 1.f / l : 0.f;
  uint16_t* oh = out + (static_cast<int64_t>(i) * H + h) * DC;
#pragma unroll
  for (int e2 = 0; e2 < OPL; ++e2) oh[lane + 32 * e2] = f32_to_bf16_rne(o[e2] * inv);
  if (lse && lane == 0) lse[static_cast<int64_t>(i) * H + h] = l > 0.f ? m + logf(l) : -INFINITY;
}

template <int H, int DC, int DR>
cudaError_t launch(const dsa_dims& d, const uint16_t* q, const uint16_t* latent,
                   const uint16_t* rope, const int32_t* idx, uint16_t* out, float* lse,
                   WsHeader* ws, cudaStream_t st) {
  sparse_attn_simple<H, DC, DR><<<d.n_q, H * 32, 0, st>>>(q, latent, rope, idx, out, lse,
                                                          d.top_k, d.ctx_len, d.softmax_scale,
                                                          ws);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_sparse_attn(const dsa_dims& d, const uint16_t* q, const uint16_t* latent,
                               const uint16_t* rope, const int32_t* idx, uint16_t* out,
                               float* lse, WsHeader* ws, cudaStream_t st) {
  if (d.n_heads == 32 && d.d_latent == 512 && d.d_rope == 64)
    return launch<32, 512, 64>(d, q, latent, rope, idx, out, lse, ws, st);
  if (d.n_heads == 4 && d.d_latent == 64 && d.d_rope == 16)
    return launch<4, 64, 16>(d, q, latent, rope, idx, out, lse, ws, st);
  return cudaErrorInvalidValue;
}

}  // namespace dsa
