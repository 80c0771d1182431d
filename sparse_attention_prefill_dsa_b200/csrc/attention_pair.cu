// attention_pair.cu -- the sparse attention on pairs of SMs (a thread-block
// cluster of two CTAs per query), for the 32-head, 512 + 64 layer shape
// (component-table row "DSA sparse-attention core" of the feedman.me post
// feedman.me/posts/wy2HU).
//
// The per-query kernel (attention.cu) holds a whole 128-key tile, 576 dims
// of every key (144 KB), in one SM's shared memory, which leaves room for one
// tile and one extra 128-dim pair: the next tile's last pairs can only be
// gathered once the current tile's PV releases them, and the tile period is a
// chain of softmax, PV, gather latency and QK^T. Here the two CTAs of a
// cluster work on the same query and split every key's dims:
//   CTA r gathers latent dims [256 r, 256 r + 256) and rope dims
//   [32 r, 32 r + 32) of each selected key (72 KB per tile), so its ring holds
//   two whole tiles and the gather of tile t + 1 runs while tile t is in
//   softmax and PV;
//   QK^T   each CTA forms its partial S^T over its 288 dims (M = 128 keys,
//          N = 32 heads) in TMEM;
//   S      each CTA owns the softmax of 16 heads: it sends the other CTA's
//          16 heads of its partial to that CTA's shared memory (distributed
//          shared memory, st.shared::cluster) and adds the 16 received
//          columns to its own;
//   P      each CTA writes the bf16 P of its 16 heads into both CTAs' P
//          buffers, together with each head's rescale factor of the running
//          maximum, so each CTA has P for all 32 heads;
//   PV     each CTA accumulates O^T for its 256 dims and all 32 heads
//          (two 128-dim blocks), rescaling columns of either CTA's heads when
//          their maximum grows;
//   out    row sums are exchanged once per query; each CTA writes its 256
//          dims of every head, the owner of a head writes its lse.
// Buffers that the other CTA writes (received partials, P, rescale factors)
// are double-buffered by tile parity. Their reuse two tiles later needs no
// extra signal: S of tile t + 2 exists in a CTA only after its PV of tile t
// has released the tile's pairs, and the other CTA sends its part of tile
// t + 2 only after receiving that S.
// Roles per CTA (416 threads, one CTA per SM): warps 0-3 cp.async gathers,
// warp 4 TMEM owner and MMA issuer, warps 5-12 softmax and epilogue (two per
// TMEM lane quarter, eight heads each). Every wait is bounded; a CTA that
// gives up records DSA_ERR_TIMEOUT, and the other CTA's waits on it then run
// out as well. Before exiting, each CTA waits (bounded) until the other has
// finished writing into its shared memory.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "dsa_internal.cuh"
#include "sm100_primitives.cuh"

namespace dsa {
namespace {

using namespace sm100;

struct PairCfg {
  static constexpr int H = 32, DC = 512, DR = 64;
  static constexpr int kKeys = 128;
  static constexpr int kOwnHeads = 16;                      // softmax heads of each CTA
  static constexpr int HH = 8;                              // heads per softmax warp
  static constexpr int kDims = DC / 2;                      // latent dims of a CTA
  static constexpr int kRopeDims = DR / 2;                  // rope dims of a CTA
  static constexpr int NL = kDims / 64;                     // latent chunks of a CTA's tile
  static constexpr int MB = kDims / 128;                    // PV blocks (latent pairs) of a CTA's tile
  static constexpr int kChunkBytes = kKeys * 128;           // 64 dims of 128 keys
  static constexpr int kPairBytes = 2 * kChunkBytes;
  static constexpr int kRopeBytes = kKeys * kRopeDims * 2;  // 64-byte rows
  static constexpr int kSlots = 2;                          // tiles in flight
  static constexpr int kPairs = kSlots * MB;
  static constexpr int kQChunkBytes = H * 128;
  static constexpr int kQRopeBytes = H * kRopeDims * 2;
  static constexpr uint32_t kQBytes = NL * kQChunkBytes + kQRopeBytes;
  static constexpr int kPRowBytes = H * 2;                  // 64
  static constexpr int kPBytes = kKeys * kPRowBytes;
  static constexpr int kRecvBytes = kKeys * kOwnHeads * 4;  // [key][16] floats
  static constexpr int kSoftmaxWarps = 8;
  static constexpr int kSoftmaxThreads = 32 * kSoftmaxWarps;
  static constexpr int kProducerThreads = 128;
  static constexpr int kThreads = 32 * (5 + kSoftmaxWarps);
  static constexpr int kRowsPerThread = kKeys / 16;
  static constexpr uint32_t kIdescQK = idesc_bf16_f32(128, H, false, false);
  static constexpr uint32_t kIdescPV = idesc_bf16_f32(128, H, true, true);
  static constexpr int kTmemS = 0;                          // S^T[2]
  static constexpr int kTmemO = 2 * H;                      // O^T[2 queries][MB]
  static constexpr int kTmemCols = 256;
  // shared memory (offsets from a 1024-byte aligned base)
  static constexpr int kOffPairs = 0;
  static constexpr int kOffRope = kOffPairs + kPairs * kPairBytes;
  static constexpr int kOffQ = kOffRope + kSlots * kRopeBytes;
  static constexpr int kOffQRope = kOffQ + NL * kQChunkBytes;
  static constexpr int kOffP = kOffQRope + kQRopeBytes;           // [2] x kPBytes
  static constexpr int kOffRecv = kOffP + 2 * kPBytes;            // [2] x kRecvBytes
  static constexpr int kOffAlpha = kOffRecv + 2 * kRecvBytes;     // [2][32] floats
  static constexpr int kOffL = kOffAlpha + 2 * H * 4;             // [2][32] floats
  static constexpr int kOffRed = kOffL + 2 * H * 4;               // [2][8 warps][8] floats
  static constexpr int kOffNorm = kOffRed + 2 * kSoftmaxWarps * HH * 4;  // [16] floats
  static constexpr int kOffBar = kOffNorm + kOwnHeads * 4;
  static constexpr int kNumBars = 3 * kPairs + 2 * kSlots + 1 + 2 * 9 + 3;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;
  static_assert(kOffQ % 1024 == 0 && kOffQRope % 512 == 0 && kOffP % 1024 == 0, "alignment");
  static_assert(kOffRope % 1024 == 0 && kOffRecv % 16 == 0 && kOffBar % 8 == 0, "alignment");
  static_assert(kSmemBytes <= 232448, "shared memory");
};

struct PairBars {
  using C = PairCfg;
  static constexpr int kPairFull = 0;                     // [kPairs][2]
  static constexpr int kPairEmpty = 2 * C::kPairs;        // [kPairs]
  static constexpr int kRopeFull = 3 * C::kPairs;         // [kSlots]
  static constexpr int kRopeEmpty = kRopeFull + C::kSlots;  // [kSlots]
  static constexpr int kQFull = kRopeEmpty + C::kSlots;
  static constexpr int kSFull = kQFull + 1;               // [2]
  static constexpr int kSEmpty = kSFull + 2;              // [2]
  static constexpr int kRecvFull = kSEmpty + 2;           // [2] the other CTA's partials arrived
  static constexpr int kPFull = kRecvFull + 2;            // [2] both halves of P arrived
  static constexpr int kOReady = kPFull + 2;              // [2] O rescaled, PV may run
  static constexpr int kOFull = kOReady + 2;              // [2]
  static constexpr int kOEmpty = kOFull + 2;              // [2]
  static constexpr int kExch = kOEmpty + 2;               // [2]
  static constexpr int kLFull = kExch + 2;                // [2] both CTAs' row sums arrived
  static constexpr int kOStep = kLFull + 2;
  static constexpr int kMmaDone = kOStep + 1;
  static constexpr int kExit = kMmaDone + 1;
  static constexpr int kCount = kExit + 1;
  static_assert(kCount == C::kNumBars, "barrier count");
};

struct PairParams {
  const uint16_t* latent;
  const uint16_t* rope;
  const int32_t* idx;
  uint16_t* out;
  float* lse;
  const uint16_t* q;
  int n_q, q_pos0, ctx_len, k, n_clusters;
  int prefix_valid;
  float scale_log2;
  WsHeader* ws;
};

__device__ __forceinline__ int pair_n_valid(const PairParams& p, int i) {
  return p.prefix_valid ? min(p.k, p.q_pos0 + i + 1) : p.k;
}

__device__ __forceinline__ int pair_selected_row(const PairParams& p, int i, int sel) {
  return sel < pair_n_valid(p, i) ? __ldg(p.idx + static_cast<int64_t>(i) * p.k + sel) : -1;
}

__device__ __forceinline__ uint64_t pdesc_add(uint64_t d, uint32_t bytes) {
  return d + static_cast<uint64_t>(bytes >> 4);
}

__device__ __forceinline__ void pair_drain_wait(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity))
    if (clock64() - t0 > kWaitLimitCycles) break;
}

// NV (power of two <= 32) values reduced over the warp; lane l gets the
// result for value l % NV.
template <int NV, bool kMax>
__device__ __forceinline__ float pair_transpose_reduce(float (&v)[NV]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int s = 16; s >= NV; s >>= 1) {
#pragma unroll
    for (int e = 0; e < NV; ++e) {
      const float o = __shfl_xor_sync(0xffffffffu, v[e], s);
      v[e] = kMax ? fmaxf(v[e], o) : v[e] + o;
    }
  }
#pragma unroll
  for (int s = NV / 2; s >= 1; s >>= 1) {
    const bool upper = (lane & s) != 0;
#pragma unroll
    for (int e = 0; e < s; ++e) {
      const float send = upper ? v[e] : v[e + s];
      const float keep = upper ? v[e + s] : v[e];
      const float o = __shfl_xor_sync(0xffffffffu, send, s);
      v[e] = kMax ? fmaxf(keep, o) : keep + o;
    }
  }
  return v[0];
}

__device__ __forceinline__ bool pwarp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                           WsHeader* ws, unsigned site) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, ws, site));
}

__device__ __forceinline__ bool pwarp_wait_cluster(uint64_t* bar, uint32_t parity,
                                                   volatile int* abort_flag, WsHeader* ws,
                                                   unsigned site) {
  return __all_sync(0xffffffffu, mbar_wait_cluster(bar, parity, abort_flag, ws, site));
}

template <int NC>
__device__ __forceinline__ void ptmem_ld(uint32_t taddr, float (&x)[NC]) {
  uint32_t r[NC];
  if constexpr (NC == 16) tmem_ld_32x32b_x16(taddr, r);
  else tmem_ld_32x32b_x8(taddr, r);
  tmem_ld_wait();
#pragma unroll
  for (int e = 0; e < NC; ++e) x[e] = __uint_as_float(r[e]);
}

template <int NC>
__device__ __forceinline__ void ptmem_st(uint32_t taddr, const float (&x)[NC]) {
  uint32_t r[NC];
#pragma unroll
  for (int e = 0; e < NC; ++e) r[e] = __float_as_uint(x[e]);
  if constexpr (NC == 16) tmem_st_32x32b_x16(taddr, r);
  else tmem_st_32x32b_x8(taddr, r);
}

// QK^T on latent pair mb of tile tc (both 64-dim chunks, each once it lands).
__device__ __forceinline__ bool pair_qk(const PairParams& p, volatile int* abort_flag, uint64_t* bars,
                                        uint64_t dpair_k, uint64_t dq, uint32_t tc, int mb, uint32_t d_s) {
  using C = PairCfg;
  using B = PairBars;
  const uint32_t pi = (tc % C::kSlots) * C::MB + mb;
  const uint32_t par = (tc / C::kSlots) & 1;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    if (!pwarp_wait(&bars[B::kPairFull + 2 * pi + half], par, abort_flag, p.ws, 63)) return false;
    fence_proxy_async_smem();
    tc_fence_after();
    const uint64_t a = pdesc_add(dpair_k, pi * C::kPairBytes + half * C::kChunkBytes);
    const uint64_t b = pdesc_add(dq, (2 * mb + half) * C::kQChunkBytes);
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
      mma_bf16_ss_warp(d_s, pdesc_add(a, ks * 32), pdesc_add(b, ks * 32), C::kIdescQK, 1u);
  }
  return true;
}

// O^T += latent_r^T P^T for tile tc (query slot qi), releasing each pair.
__device__ __forceinline__ bool pair_pv(const PairParams& p, volatile int* abort_flag, uint64_t* bars,
                                        uint32_t tmem_base, uint64_t dpair_mn, uint64_t dp, uint32_t tc,
                                        uint32_t qi, bool first, bool last) {
  using C = PairCfg;
  using B = PairBars;
  const uint32_t pb = tc & 1;
  if (!pwarp_wait(&bars[B::kOReady + pb], (tc >> 1) & 1, abort_flag, p.ws, 64)) return false;
  if (first && !pwarp_wait(&bars[B::kOEmpty + (qi & 1)], ((qi >> 1) & 1) ^ 1, abort_flag, p.ws, 65))
    return false;
  fence_proxy_async_smem();
  tc_fence_after();
  const uint32_t d_o = tmem_base + C::kTmemO + (qi & 1) * C::MB * C::H;
  const uint64_t dpb = pdesc_add(dp, pb * C::kPBytes);
#pragma unroll
  for (int mb = 0; mb < C::MB; ++mb) {
    const uint32_t pi = (tc % C::kSlots) * C::MB + mb;
    const uint64_t a = pdesc_add(dpair_mn, pi * C::kPairBytes);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
      mma_bf16_ss_warp(d_o + mb * C::H, pdesc_add(a, kk * 2048), pdesc_add(dpb, kk * 16 * C::kPRowBytes),
                       C::kIdescPV, (first && kk == 0) ? 0u : 1u);
    mma_commit_warp(&bars[B::kPairEmpty + pi]);
  }
  mma_commit_warp(&bars[B::kOStep]);
  if (last) mma_commit_warp(&bars[B::kOFull + (qi & 1)]);
  return true;
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PairCfg::kThreads, 1)
    sparse_attn_pair(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_qr,
                     const PairParams p) {
  using C = PairCfg;
  using B = PairBars;
  constexpr int H = C::H;
  constexpr int HH = C::HH;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* sPairs = smem + C::kOffPairs;
  unsigned char* sRope = smem + C::kOffRope;
  unsigned char* sQ = smem + C::kOffQ;
  unsigned char* sQR = smem + C::kOffQRope;
  unsigned char* sP = smem + C::kOffP;
  float* sRecv = reinterpret_cast<float*>(smem + C::kOffRecv);
  float* sAlpha = reinterpret_cast<float*>(smem + C::kOffAlpha);
  float* sL = reinterpret_cast<float*>(smem + C::kOffL);
  float* sRed = reinterpret_cast<float*>(smem + C::kOffRed);
  float* sNorm = reinterpret_cast<float*>(smem + C::kOffNorm);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int cluster = blockIdx.x >> 1;

  for (int e = threadIdx.x * 16; e < C::kOffBar; e += C::kThreads * 16)
    *reinterpret_cast<uint4*>(smem + e) = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    for (int s = 0; s < 2 * C::kPairs; ++s) mbar_init(&bars[B::kPairFull + s], C::kProducerThreads);
    for (int s = 0; s < C::kPairs; ++s) mbar_init(&bars[B::kPairEmpty + s], 1);
    for (int s = 0; s < C::kSlots; ++s) {
      mbar_init(&bars[B::kRopeFull + s], C::kProducerThreads);
      mbar_init(&bars[B::kRopeEmpty + s], 1);
    }
    mbar_init(&bars[B::kQFull], 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bars[B::kSFull + b], 1);
      mbar_init(&bars[B::kSEmpty + b], C::kSoftmaxThreads);
      // one arrival per softmax warp: the other CTA's warps, or both CTAs' warps
      mbar_init(&bars[B::kRecvFull + b], C::kSoftmaxWarps);
      mbar_init(&bars[B::kPFull + b], 2 * C::kSoftmaxWarps);
      mbar_init(&bars[B::kOReady + b], C::kSoftmaxWarps);
      mbar_init(&bars[B::kOFull + b], 1);
      mbar_init(&bars[B::kOEmpty + b], C::kSoftmaxThreads);
      mbar_init(&bars[B::kExch + b], C::kSoftmaxThreads);
      mbar_init(&bars[B::kLFull + b], 2 * C::kSoftmaxWarps);
    }
    mbar_init(&bars[B::kOStep], 1);
    mbar_init(&bars[B::kMmaDone], 1);
    mbar_init(&bars[B::kExit], 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 4) tmem_alloc(tmem_slot, C::kTmemCols);
  __syncthreads();
  // both CTAs' barriers are initialised before either arrives on the other's
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp < 4) {
    // -------------------------------------------------------------- producers
    constexpr int R = C::kRowsPerThread;
    const int kbase = 32 * warp + (lane >> 3);
    const int part = lane & 7;
    uint32_t doff[R], roff[R];
#pragma unroll
    for (int e = 0; e < R; ++e) {
      const int key = kbase + 4 * e;
      doff[e] = key * 128 + ((part ^ (key & 7)) << 4);
      roff[e] = key * 64 + (((part & 3) ^ ((key >> 1) & 3)) << 4);  // 64-byte rows, 64B swizzle
    }
    int cur[R], nxt[R];
    if (cluster < p.n_q) {
#pragma unroll
      for (int e = 0; e < R; ++e) cur[e] = pair_selected_row(p, cluster, kbase + 4 * e);
    }
    uint32_t tc = 0;
    bool ok = true;
    for (int i = cluster; i < p.n_q && ok; i += p.n_clusters) {
      const int nt = (pair_n_valid(p, i) + 127) / 128;
      for (int j = 0; j < nt && ok; ++j, ++tc) {
        const int ni = j + 1 < nt ? i : i + p.n_clusters;
        const int nj = j + 1 < nt ? j + 1 : 0;
        if (ni < p.n_q) {
#pragma unroll
          for (int e = 0; e < R; ++e) nxt[e] = pair_selected_row(p, ni, nj * 128 + kbase + 4 * e);
        }
        const uint16_t* lsrc[R];
        const uint16_t* rsrc[R];
#pragma unroll
        for (int e = 0; e < R; ++e) {
          int row = cur[e];
          if (row > p.q_pos0 + i) {  // past the query's own position (t < ctx_len)
            report(p.ws, kDevRange, static_cast<unsigned>(i));
            row = -1;
          }
          if (row < 0) row = 0;  // masked key: any valid row, weight zero
          if (!DSA_IN_BOUNDS(p.ws, row, p.ctx_len, 40)) row = 0;
          lsrc[e] = p.latent + static_cast<int64_t>(row) * C::DC + rank * C::kDims + part * 8;
          rsrc[e] = p.rope + static_cast<int64_t>(row) * C::DR + rank * C::kRopeDims + (part & 3) * 8;
        }
        const uint32_t sl = tc % C::kSlots, par = ((tc / C::kSlots) & 1) ^ 1;
        ok = __all_sync(0xffffffffu, mbar_wait(&bars[B::kRopeEmpty + sl], par, abort_flag, p.ws, 60));
        if (!ok) break;
        if (part < 4) {
#pragma unroll
          for (int e = 0; e < R; ++e) cp_async_16(sRope + sl * C::kRopeBytes + roff[e], rsrc[e]);
        }
        cp_async_arrive_noinc(&bars[B::kRopeFull + sl]);
#pragma unroll
        for (int mb = 0; mb < C::MB; ++mb) {
          const uint32_t pi = sl * C::MB + mb;
          ok = __all_sync(0xffffffffu, mbar_wait(&bars[B::kPairEmpty + pi], par, abort_flag, p.ws, 61));
          if (!ok) break;
          unsigned char* dst = sPairs + pi * C::kPairBytes;
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            const int c = 2 * mb + half;
#pragma unroll
            for (int e = 0; e < R; ++e) cp_async_16(dst + half * C::kChunkBytes + doff[e], lsrc[e] + c * 64);
            cp_async_arrive_noinc(&bars[B::kPairFull + 2 * pi + half]);
          }
        }
#pragma unroll
        for (int e = 0; e < R; ++e) cur[e] = nxt[e];
      }
    }
    cp_async_wait_all();
  } else if (warp == 4) {
    // ------------------------------------------------------------ MMA issuer
    const uint64_t dq = smem_desc(smem_u32(sQ), 16, 1024, 2);
    const uint64_t dqr = smem_desc(smem_u32(sQR), 16, 512, 4);
    const uint64_t drope = smem_desc(smem_u32(sRope), 16, 512, 4);
    const uint64_t dpair_k = smem_desc(smem_u32(sPairs), 16, 1024, 2);
    const uint64_t dpair_mn = smem_desc(smem_u32(sPairs), C::kChunkBytes, 1024, 2);
    const uint64_t dp = smem_desc(smem_u32(sP), 8 * C::kPRowBytes, 8 * C::kPRowBytes, 4);
    bool pend = false, pend_first = false, pend_last = false;
    uint32_t pend_tc = 0, pend_qi = 0;
    uint32_t tc = 0, qi = 0;
    bool ok = true;
    for (int i = cluster; i < p.n_q && ok; i += p.n_clusters, ++qi) {
      const int nt = (pair_n_valid(p, i) + 127) / 128;
      for (int j = 0; j < nt; ++j, ++tc) {
        const int sb = tc & 1;
        const uint32_t sl = tc % C::kSlots;
        const uint32_t d_s = tmem_base + C::kTmemS + sb * H;
        if (j == 0) {
          if (pend && !(ok = pair_pv(p, abort_flag, bars, tmem_base, dpair_mn, dp, pend_tc, pend_qi,
                                     pend_first, pend_last)))
            break;
          pend = false;
          if (!(ok = pwarp_wait(&bars[B::kQFull], qi & 1, abort_flag, p.ws, 66))) break;
          tc_fence_after();
        }
        if (!(ok = pwarp_wait(&bars[B::kSEmpty + sb], ((tc >> 1) & 1) ^ 1, abort_flag, p.ws, 67))) break;
        if (!(ok = pwarp_wait(&bars[B::kRopeFull + sl], (tc / C::kSlots) & 1, abort_flag, p.ws, 68))) break;
        fence_proxy_async_smem();
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < C::kRopeDims / 16; ++ks)
          mma_bf16_ss_warp(d_s, pdesc_add(drope, sl * C::kRopeBytes + ks * 32), pdesc_add(dqr, ks * 32),
                           C::kIdescQK, ks > 0 ? 1u : 0u);
        mma_commit_warp(&bars[B::kRopeEmpty + sl]);
        // all of QK^T(t) first, so that the softmax of tile t runs while the
        // tensor pipe does PV(t-1); two tiles in flight keep the gather ahead
        for (int mb = 0; mb < C::MB && ok; ++mb) ok = pair_qk(p, abort_flag, bars, dpair_k, dq, tc, mb, d_s);
        if (!ok) break;
        mma_commit_warp(&bars[B::kSFull + sb]);
        if (pend && !(ok = pair_pv(p, abort_flag, bars, tmem_base, dpair_mn, dp, pend_tc, pend_qi, pend_first,
                                   pend_last)))
          break;
        pend = false;
        pend = true;
        pend_tc = tc;
        pend_qi = qi;
        pend_first = j == 0;
        pend_last = j == nt - 1;
      }
    }
    if (ok && pend)
      ok = pair_pv(p, abort_flag, bars, tmem_base, dpair_mn, dp, pend_tc, pend_qi, pend_first, pend_last);
    mma_commit_warp(&bars[B::kMmaDone]);
    pair_drain_wait(&bars[B::kMmaDone], 0);
  } else {
    // ------------------------------------------------- softmax and epilogue
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;        // key lane (dim lane in the epilogue)
    const int sw = warp - 5;                  // 0..7
    const int hh = sw >> 2;                   // which eight of this CTA's heads
    const int own0 = 16 * rank + HH * hh;     // this warp's heads in the CTA's S columns
    const int oth0 = 16 * peer + HH * hh;     // the other CTA's heads it forwards
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const bool q_loader = warp == 5 && lane == 0;
    // the other CTA's buffers
    const uint32_t rRecv = mapa_shared(smem_u32(sRecv), peer);
    const uint32_t rP = mapa_shared(smem_u32(sP), peer);
    const uint32_t rAlpha = mapa_shared(smem_u32(sAlpha), peer);
    const uint32_t rL = mapa_shared(smem_u32(sL), peer);
    const uint32_t rRecvFull = mapa_shared(smem_u32(&bars[B::kRecvFull]), peer);
    const uint32_t rPFull = mapa_shared(smem_u32(&bars[B::kPFull]), peer);
    const uint32_t rLFull = mapa_shared(smem_u32(&bars[B::kLFull]), peer);
    int q_loads = 0;
    if (q_loader && cluster < p.n_q) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_qr);
      mbar_arrive_expect_tx(&bars[B::kQFull], C::kQBytes);
      for (int c = 0; c < C::NL; ++c)
        tma_load_2d(sQ + c * C::kQChunkBytes, &tm_q, rank * C::kDims + c * 64, cluster * H, &bars[B::kQFull]);
      tma_load_2d(sQR, &tm_qr, C::DC + rank * C::kRopeDims, cluster * H, &bars[B::kQFull]);
      q_loads = 1;
    }
    uint32_t tc = 0, qi = 0, xc = 0;
    bool ok = true;
    int row_next = cluster < p.n_q ? pair_selected_row(p, cluster, r) : -1;
    const float kmax = __uint_as_float(*reinterpret_cast<volatile unsigned int*>(&p.ws->akmax_bits));
    const float bound_scale = fabsf(p.scale_log2) * kmax;
    for (int i = cluster; i < p.n_q && ok; i += p.n_clusters, ++qi) {
      const int nt = (pair_n_valid(p, i) + 127) / 128;
      const int ob = qi & 1;
      const bool next_q = i + p.n_clusters < p.n_q;
      // ||q_h||^2 of this CTA's 16 heads over all 576 dims (plain loads of
      // the q rows): thread t takes 36 dims of head t / 16
      {
        const int t = threadIdx.x - 160;
        const int hl = t >> 4, part16 = t & 15;
        const uint16_t* qrow = p.q + (static_cast<int64_t>(i) * H + 16 * rank + hl) * (C::DC + C::DR) + part16 * 36;
        float ss = 0.f;
        for (int e = 0; e < 36; e += 2) {
          const uint32_t w2 = __ldg(reinterpret_cast<const uint32_t*>(qrow + e));
          const float a = __uint_as_float(w2 << 16), b = __uint_as_float(w2 & 0xFFFF0000u);
          ss = fmaf(a, a, fmaf(b, b, ss));
        }
#pragma unroll
        for (int o = 8; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
        if (part16 == 0) sNorm[hl] = ss;  // read after the first tile's exchange
      }
      float m_lane = -INFINITY;     // running max (log2 units) of head 16 rank + lane (lane < 16)
      float bound_lane = INFINITY;  // B of that head
      bool fixed_m = false;
      float lpart[HH];
#pragma unroll
      for (int h = 0; h < HH; ++h) lpart[h] = 0.f;
      for (int j = 0; j < nt; ++j, ++tc) {
        const int sb = tc & 1;
        const int row = row_next;
        {
          const int ni = j + 1 < nt ? i : i + p.n_clusters;
          const int nj = j + 1 < nt ? j + 1 : 0;
          row_next = ni < p.n_q ? pair_selected_row(p, ni, nj * 128 + r) : -1;
        }
        ok = pwarp_wait(&bars[B::kSFull + sb], (tc >> 1) & 1, abort_flag, p.ws, 70);
        if (!ok) break;
        tc_fence_after();
        float xo[HH], xp[HH];
        ptmem_ld<HH>(tmem_base + lane_addr + C::kTmemS + sb * H + own0, xo);
        ptmem_ld<HH>(tmem_base + lane_addr + C::kTmemS + sb * H + oth0, xp);
        tc_fence_before();
        mbar_arrive(&bars[B::kSEmpty + sb]);
        // this CTA's partial of the other CTA's heads -> its receive buffer
        {
          const uint32_t dst = rRecv + sb * C::kRecvBytes + r * 64 + hh * 32;
          st_cluster_v4(dst, __float_as_uint(xp[0]), __float_as_uint(xp[1]), __float_as_uint(xp[2]),
                        __float_as_uint(xp[3]));
          st_cluster_v4(dst + 16, __float_as_uint(xp[4]), __float_as_uint(xp[5]), __float_as_uint(xp[6]),
                        __float_as_uint(xp[7]));
          __syncwarp();
          if (lane == 0) mbar_arrive_remote(rRecvFull + sb * 8);  // releases the warp's stores
        }
        ok = pwarp_wait_cluster(&bars[B::kRecvFull + sb], (tc >> 1) & 1, abort_flag, p.ws, 71);
        if (!ok) break;
        float x[HH];
        {
          const float4 a = *reinterpret_cast<const float4*>(sRecv + sb * (C::kRecvBytes / 4) + r * 16 + hh * 8);
          const float4 b = *reinterpret_cast<const float4*>(sRecv + sb * (C::kRecvBytes / 4) + r * 16 + hh * 8 + 4);
          const float in[HH] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
          for (int h = 0; h < HH; ++h) x[h] = xo[h] + in[h];
        }
        const bool issue_q = j == nt - 1 && q_loader && next_q;
        const bool valid = row >= 0 && row <= p.q_pos0 + i;
        float alpha_lane = 1.f;
        if (!fixed_m) {
          float red[HH];
#pragma unroll
          for (int h = 0; h < HH; ++h) red[h] = valid ? x[h] * p.scale_log2 : -INFINITY;
          const float wmax = pair_transpose_reduce<HH, true>(red);
          float* xbuf = sRed + (xc & 1) * (C::kSoftmaxWarps * HH);
          if (lane < HH) xbuf[sw * HH + lane] = wmax;
          mbar_arrive(&bars[B::kExch + (xc & 1)]);
          ok = pwarp_wait(&bars[B::kExch + (xc & 1)], (xc >> 1) & 1, abort_flag, p.ws, 72);
          ++xc;
          if (!ok) break;
          float tmax = -INFINITY;
          if (lane < 16) {
            const int g = lane >> 3, jj = lane & 7;  // head 16 rank + lane: warps 4g .. 4g + 3, entry jj
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) tmax = fmaxf(tmax, xbuf[(4 * g + qq) * HH + jj]);
          }
          if (j == 0 && lane < 16)
            bound_lane = bound_scale * sqrtf(sNorm[lane]) * (1.f + 0.00390625f);
          const bool need = lane < 16 && tmax > -INFINITY && (m_lane == -INFINITY || tmax > m_lane + 8.f);
          if (__any_sync(0xffffffffu, need)) {
            const float m_new = fmaxf(m_lane, tmax);
            alpha_lane = m_lane == -INFINITY ? 0.f : ex2_approx(m_lane - m_new);
            m_lane = m_new;
#pragma unroll
            for (int h = 0; h < HH; ++h) lpart[h] *= __shfl_sync(0xffffffffu, alpha_lane, HH * hh + h);
          }
          fixed_m = __all_sync(0xffffffffu, lane >= 16 || bound_lane <= m_lane + 64.f);
        }
        if (issue_q) {
          // every QK^T of query i has completed: the next query's q rows
          mbar_arrive_expect_tx(&bars[B::kQFull], C::kQBytes);
          const int inext = i + p.n_clusters;
          for (int c = 0; c < C::NL; ++c)
            tma_load_2d(sQ + c * C::kQChunkBytes, &tm_q, rank * C::kDims + c * 64, inext * H, &bars[B::kQFull]);
          tma_load_2d(sQR, &tm_qr, C::DC + rank * C::kRopeDims, inext * H, &bars[B::kQFull]);
          ++q_loads;
        }
        // P of this warp's eight heads (16 bytes per key) into both CTAs' P
        // buffers, and the heads' rescale factors
        const int pb = tc & 1;
        uint32_t w4[4];
#pragma unroll
        for (int e2 = 0; e2 < 4; ++e2) {
          float pv[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int h = 2 * e2 + e;
            const float mh = __shfl_sync(0xffffffffu, m_lane, HH * hh + h);
            pv[e] = (valid && mh > -INFINITY) ? ex2_approx(fmaf(x[h], p.scale_log2, -mh)) : 0.f;
            lpart[h] += pv[e];
          }
          const __nv_bfloat162 b2 = __floats2bfloat162_rn(pv[0], pv[1]);
          w4[e2] = *reinterpret_cast<const uint32_t*>(&b2);
        }
        const int chunk = (2 * static_cast<int>(rank) + hh) ^ ((r >> 1) & 3);
        const uint32_t poff = pb * C::kPBytes + r * C::kPRowBytes + (chunk << 4);
        *reinterpret_cast<uint4*>(sP + poff) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        st_cluster_v4(rP + poff, w4[0], w4[1], w4[2], w4[3]);
        if (sw == 0 && lane < 16) {
          sAlpha[pb * H + 16 * rank + lane] = alpha_lane;
          st_cluster_f32(rAlpha + (pb * H + 16 * rank + lane) * 4, alpha_lane);
        }
        fence_proxy_async_all();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&bars[B::kPFull + pb]);
          mbar_arrive_remote(rPFull + pb * 8);
        }
        ok = pwarp_wait_cluster(&bars[B::kPFull + pb], (tc >> 1) & 1, abort_flag, p.ws, 73);
        if (!ok) break;
        // rescale O^T columns of every head whose maximum grew (this CTA's or
        // the other's) once the previous tile's PV is complete
        if (j > 0) {
          const float4* al = reinterpret_cast<const float4*>(sAlpha + pb * H);
          bool any = false;
#pragma unroll
          for (int e = 0; e < H / 4; ++e) {
            const float4 v = al[e];
            any |= v.x != 1.f || v.y != 1.f || v.z != 1.f || v.w != 1.f;
          }
          if (any) {
            ok = pwarp_wait(&bars[B::kOStep], (tc - 1) & 1, abort_flag, p.ws, 74);
            if (!ok) break;
            tc_fence_after();
#pragma unroll 1
            for (int mb = 0; mb < C::MB; ++mb) {
              const uint32_t ta = tmem_base + lane_addr + C::kTmemO + (ob * C::MB + mb) * H + 16 * hh;
              float o[16];
              ptmem_ld<16>(ta, o);
#pragma unroll
              for (int h = 0; h < 16; ++h) o[h] *= sAlpha[pb * H + 16 * hh + h];
              ptmem_st<16>(ta, o);
            }
            tmem_st_wait();
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bars[B::kOReady + pb]);
      }
      if (!ok) break;
      // ---- epilogue of query i
      ok = pwarp_wait(&bars[B::kOFull + ob], (qi >> 1) & 1, abort_flag, p.ws, 75);
      if (!ok) break;
      tc_fence_after();
      const float lsum = pair_transpose_reduce<HH, false>(lpart);
      float* xbuf = sRed + (xc & 1) * (C::kSoftmaxWarps * HH);
      if (lane < HH) xbuf[sw * HH + lane] = lsum;
      mbar_arrive(&bars[B::kExch + (xc & 1)]);
      ok = pwarp_wait(&bars[B::kExch + (xc & 1)], (xc >> 1) & 1, abort_flag, p.ws, 76);
      ++xc;
      if (!ok) break;
      if (sw == 0 && lane < 16) {
        const int g = lane >> 3, jj = lane & 7;
        float l = 0.f;
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) l += xbuf[(4 * g + qq) * HH + jj];
        sL[ob * H + 16 * rank + lane] = l;
        st_cluster_f32(rL + (ob * H + 16 * rank + lane) * 4, l);
        if (p.lse)
          p.lse[static_cast<int64_t>(i) * H + 16 * rank + lane] =
              l > 0.f ? (m_lane + log2f(l)) * 0.6931471805599453f : -INFINITY;
      }
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&bars[B::kLFull + ob]);
        mbar_arrive_remote(rLFull + ob * 8);
      }
      ok = pwarp_wait_cluster(&bars[B::kLFull + ob], (qi >> 1) & 1, abort_flag, p.ws, 77);
      if (!ok) break;
#pragma unroll 1
      for (int mb = 0; mb < C::MB; ++mb) {
        float o[16];
        ptmem_ld<16>(tmem_base + lane_addr + C::kTmemO + (ob * C::MB + mb) * H + 16 * hh, o);
        const int d = rank * C::kDims + mb * 128 + r;
        uint16_t* orow = p.out + (static_cast<int64_t>(i) * H + 16 * hh) * C::DC + d;
#pragma unroll
        for (int h = 0; h < 16; ++h) {
          const float l = sL[ob * H + 16 * hh + h];
          orow[h * C::DC] = f32_to_bf16_rne(l > 0.f ? o[h] / l : 0.f);
        }
      }
      tc_fence_before();
      mbar_arrive(&bars[B::kOEmpty + ob]);
    }
    if (!ok && q_loader && q_loads > 0) pair_drain_wait(&bars[B::kQFull], (q_loads - 1) & 1);
  }

  __syncthreads();
  // no exit while the other CTA may still write into this CTA's shared
  // memory: each CTA signals the other once all its threads are done, then
  // waits (bounded) for the other's signal
  if (threadIdx.x == 0) {
    mbar_arrive_remote(mapa_shared(smem_u32(&bars[B::kExit]), peer));
    const long long t0 = clock64();
    while (!mbar_try_wait_cluster(&bars[B::kExit], 0))
      if (clock64() - t0 > 2 * kWaitLimitCycles) {
        report(p.ws, kDevTimeout, 79);
        break;
      }
  }
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

int pair_num_sms() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

}  // namespace

bool attn_pair_supported(const dsa_dims& d) {
  return d.n_heads == 32 && d.d_latent == 512 && d.d_rope == 64;
}

cudaError_t launch_sparse_attn_pair(const dsa_dims& d, const uint16_t* q, const uint16_t* latent,
                                    const uint16_t* rope, const int32_t* idx, uint16_t* out,
                                    float* lse, bool prefix_valid, WsHeader* ws, cudaStream_t st) {
  using C = PairCfg;
  if (!attn_pair_supported(d)) return cudaErrorInvalidValue;
  PairParams p;
  p.latent = latent;
  p.rope = rope;
  p.idx = idx;
  p.out = out;
  p.lse = lse;
  p.q = q;
  p.n_q = d.n_q;
  p.q_pos0 = d.q_pos0;
  p.ctx_len = d.ctx_len;
  p.k = d.top_k;
  p.prefix_valid = prefix_valid ? 1 : 0;
  p.scale_log2 = d.softmax_scale * 1.4426950408889634f;
  p.ws = ws;
  CUtensorMap tm_q, tm_qr;
  if (!make_tmap_bf16_2d(&tm_q, q, C::DC + C::DR, static_cast<uint64_t>(d.n_q) * C::H, 64, C::H,
                         CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_bf16_2d(&tm_qr, q, C::DC + C::DR, static_cast<uint64_t>(d.n_q) * C::H, C::kRopeDims,
                         C::H, CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(sparse_attn_pair, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       C::kSmemBytes);
  if (e != cudaSuccess) return e;
  int max_clusters = pair_num_sms() / 2;
  {
    cudaLaunchConfig_t cfg = {};
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.gridDim = dim3(2 * max_clusters, 1, 1);
    cfg.blockDim = dim3(C::kThreads, 1, 1);
    cfg.dynamicSmemBytes = C::kSmemBytes;
    cfg.stream = st;
    cfg.attrs = attr;
    cfg.numAttrs = 0;  // the kernel's own __cluster_dims__ gives the cluster shape
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, sparse_attn_pair, &cfg) == cudaSuccess && n > 0 &&
        n < max_clusters)
      max_clusters = n;
    cudaGetLastError();
  }
  const int n_clusters = d.n_q < max_clusters ? d.n_q : max_clusters;
  p.n_clusters = n_clusters;
  sparse_attn_pair<<<2 * n_clusters, C::kThreads, C::kSmemBytes, st>>>(tm_q, tm_qr, p);
  return cudaGetLastError();
}

}  // namespace dsa
