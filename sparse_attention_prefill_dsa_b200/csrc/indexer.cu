// indexer.cu -- lightning-indexer scores (component-table row "DSA indexer" of
// the feedman.me post feedman.me/posts/wy2HU).
//
//   I[i,s] = sum_j w[i,j] * ReLU( sum_c qI[i,j,c] * kI[s,c] ),  s <= t = q_pos0 + i
//
// Straightforward CUDA-core version: a CTA takes 4 queries x 128 keys, stages
// the queries' indexer rows and the key tile (transposed) in shared memory as
// float32 and accumulates each head's dot product with sequential float32 FMAs
// (error <= 128 * 2^-24 * sum|q*k|, inside the selection's 2^-14 bound).
// Key tiles entirely above the causal boundary are skipped.
#include <cuda_runtime.h>
#include <stdint.h>

#include "dsa_internal.cuh"

namespace dsa {
namespace {

constexpr int kKeys = 128;  // keys per CTA (one per thread)
constexpr int kQB = 4;      // queries per CTA

template <int HI, int DI>
__global__ void __launch_bounds__(kKeys) index_scores_simple(
    const uint16_t* __restrict__ q_idx, const uint16_t* __restrict__ k_idx,
    const float* __restrict__ w_idx, float* __restrict__ scores, int64_t ld, int n_q,
    int q_pos0) {
  extern __shared__ __align__(16) float sm[];
  float* qf = sm;                            // [kQB][HI][DI]
  float* kT = qf + kQB * HI * DI;            // [DI][kKeys]
  float* ws = kT + DI * kKeys;               // [kQB][HI]
  const int i0 = blockIdx.y * kQB;
  const int s0 = blockIdx.x * kKeys;
  const int t_max = q_pos0 + min(i0 + kQB, n_q) - 1;
  if (s0 > t_max) return;  // whole tile is masked for every query of the block

  for (int e = threadIdx.x; e < kQB * HI * DI; e += kKeys) {
    const int qi = e / (HI * DI);
    qf[e] = (i0 + qi < n_q) ? bf16_to_f32(q_idx[static_cast<int64_t>(i0) * HI * DI + e]) : 0.f;
  }
  for (int e = threadIdx.x; e < kQB * HI; e += kKeys) {
    const int qi = e / HI;
    ws[e] = (i0 + qi < n_q) ? w_idx[static_cast<int64_t>(i0) * HI + e] : 0.f;
  }
  for (int e = threadIdx.x; e < kKeys * DI; e += kKeys) {
    const int key = e / DI, c = e - key * DI;
    const int s = s0 + key;
    kT[c * kKeys + key] = (s <= t_max) ? bf16_to_f32(k_idx[static_cast<int64_t>(s) * DI + c]) : 0.f;
  }
  __syncthreads();

  const int s = s0 + threadIdx.x;
  for (int qi = 0; qi < kQB; ++qi) {
    const int i = i0 + qi;
    if (i >= n_q) break;
    const int t = q_pos0 + i;
    if (s > t) continue;
    float acc = 0.f;
    for (int j = 0; j < HI; ++j) {
      const float* q = qf + (qi * HI + j) * DI;
      float dot = 0.f;
#pragma unroll 8
      for (int c = 0; c < DI; ++c) dot = fmaf(q[c], kT[c * kKeys + threadIdx.x], dot);
      acc = fmaf(ws[qi * HI + j], fmaxf(dot, 0.f), acc);
    }
    scores[static_cast<int64_t>(i) * ld + s] = acc;
  }
}

template <int HI, int DI>
cudaError_t launch(const dsa_dims& d, const uint16_t* q_idx, const uint16_t* k_idx,
                   const float* w_idx, float* scores, int64_t ld, cudaStream_t st) {
  const size_t smem = sizeof(float) * (kQB * HI * DI + DI * kKeys + kQB * HI);
  cudaFuncSetAttribute(index_scores_simple<HI, DI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       static_cast<int>(smem));
  const int T_used = d.q_pos0 + d.n_q;
  dim3 grid((T_used + kKeys - 1) / kKeys, (d.n_q + kQB - 1) / kQB);
  index_scores_simple<HI, DI><<<grid, kKeys, smem, st>>>(q_idx, k_idx, w_idx, scores, ld, d.n_q,
                                                         d.q_pos0);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_index_scores(const dsa_dims& d, const uint16_t* q_idx, const uint16_t* k_idx,
                                const float* w_idx, float* scores, int64_t ld, WsHeader* ws,
                                cudaStream_t st) {
  (void)ws;
  if (d.n_idx_heads == 32 && d.d_idx == 128)
    return launch<32, 128>(d, q_idx, k_idx, w_idx, scores, ld, st);
  if (d.n_idx_heads == 2 && d.d_idx == 32)
    return launch<2, 32>(d, q_idx, k_idx, w_idx, scores, ld, st);
  return cudaErrorInvalidValue;
}

}  // namespace dsa
