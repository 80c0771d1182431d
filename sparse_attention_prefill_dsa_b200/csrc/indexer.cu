// indexer.cu -- lightning-indexer scores on tcgen05 tensor cores (component-
// table row "DSA indexer" of the feedman.me post feedman.me/posts/wy2HU).
//
//   I[i,s] = sum_j w[i,j] * ReLU( sum_c qI[i,j,c] * kI[s,c] ),  s <= t = q_pos0 + i
//
// The head dot products form one dense GEMM per (query block, key tile):
//   D[s, (i,j)] = sum_c kI[s,c] * qI[i,j,c]
// with the 128 keys of a tile as the MMA's M dimension and 256 / H_I queries x
// H_I heads (= 256 columns, query-major, the natural layout of q_idx) as N,
// K = D_I. Putting keys on M leaves each key's whole row of head dots in one
// TMEM lane, so the epilogue thread that owns that lane forms ReLU, the
// w-weighted head sum and the store with no cross-thread traffic, and a warp
// writes 32 consecutive keys of a query row (128 coalesced bytes).
//
// Persistent, warp-specialised CTA (one per SM, 576 threads):
//   warp 0      TMA producer: takes work units from a queue (an atomic
//               counter in the workspace header, reset before each launch),
//               hands each unit to the other warps through a four-slot ring
//               in shared memory (a -1 ends the stream), and loads the
//               block's q_idx rows (once per unit), a 4-stage ring of key
//               tiles, 128-byte (or 64-byte) swizzled, and the block's head
//               weights into a double-buffered slot;
//   warp 1      TMEM owner and MMA issuer (tcgen05.mma kind::f16, bf16 x bf16
//               -> f32), issued warp-collectively by one elected lane with
//               base descriptors plus compile-time offsets, accumulating each
//               tile into one of two 256-column TMEM buffers;
//   warps 2-17  epilogue: four warpgroups split the 256 columns (64 each);
//               each thread reads its key's columns with tcgen05.ld, hands
//               the accumulator buffer back as soon as they are in registers
//               (the next tile but one accumulates there while this one is
//               summed), and writes the scores.
// A work unit is (query block, up to 32 consecutive causal key tiles). The
// queue hands units out in slot-major order with the later (longer) query
// blocks first, so every block's first 32 tiles go out before any block's
// second and the units come roughly longest first. Key tiles past the last
// query of a block are never loaded (causal skip); rows of a partial tile
// past the context read as zero and no score past t is written.
// Every wait is bounded: on a timeout the CTA records DSA_ERR_TIMEOUT in the
// workspace, all roles stop, outstanding TMA loads and MMAs are drained, and
// TMEM is freed before the CTA exits.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "dsa_internal.cuh"
#include "sm100_primitives.cuh"

namespace dsa {
namespace {

using namespace sm100;

// FP8: the operands are e4m3 codes (1 byte, K = 32 per MMA, kind::f8f6f4)
// with a power-of-two scale per key row and per (query, head) row; else bf16.
template <int HI, int DI, bool FP8 = false>
struct IdxCfg {
  static constexpr int kM = 128;                       // keys per tile (MMA M)
  static constexpr int kN = 256;                       // (query, head) columns (MMA N)
  static constexpr int kQB = kN / HI;                  // queries per block
  static constexpr int kEB = FP8 ? 1 : 2;              // bytes per element
  static constexpr int kChunk = DI * kEB < 128 ? DI : 128 / kEB;  // elements per swizzled row
  static constexpr int kNChunk = DI / kChunk;
  static constexpr int kRowBytes = kChunk * kEB;       // 128, 64 or 32
  static constexpr uint32_t kSwzCode = kRowBytes == 128 ? 2u : (kRowBytes == 64 ? 4u : 6u);
  static constexpr CUtensorMapSwizzle kSwzMap =
      kRowBytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                       : (kRowBytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B);
  static constexpr int kSbo = 8 * kRowBytes;           // bytes between 8-row groups
  static constexpr int kKChunkBytes = kM * kRowBytes;
  static constexpr int kQChunkBytes = kN * kRowBytes;
  static constexpr int kKTileBytes = kKChunkBytes * kNChunk;
  static constexpr int kQBytes = kQChunkBytes * kNChunk;
  static constexpr int kStages = 4;
  static constexpr int kKPerMma = FP8 ? 32 : 16;       // elements of K per MMA (32 bytes)
  static constexpr int kKSteps = DI / kKPerMma;
  static constexpr int kStepsPerChunk = kChunk / kKPerMma;
  static constexpr int kTilesPerUnit = 32;             // key tiles per work unit (fewer for small chunks)
  static constexpr int kEpiWarps = 16;                 // warps 2-17: four per TMEM lane quarter
  static constexpr int kEpiGroups = kEpiWarps / 4;     // column ranges, one per warpgroup
  static constexpr int kColsPerWg = kN / kEpiGroups;   // accumulator columns per epilogue warp
  static constexpr int kGroups = kColsPerWg / 32;      // 32-column TMEM loads per tile and warp
  static constexpr int kThreads = 32 * (2 + kEpiWarps);
  static constexpr uint32_t kIdesc = FP8 ? idesc_e4m3_f32(kM, kN) : idesc_bf16_f32(kM, kN, false, false);
  // shared memory carve (offsets from a 1024-byte aligned base)
  static constexpr int kOffQ = 0;
  static constexpr int kOffK = kOffQ + kQBytes;
  static constexpr int kOffW = kOffK + kStages * kKTileBytes;        // 2 x 256 floats
  static constexpr int kOffBar = kOffW + 2 * kN * 4;
  static constexpr int kUnitRing = 4;                  // units handed from the producer to the others
  static constexpr int kNumBars = 2 * kStages + 2 + 2 + 2 + 2 + 2 + 1 + 2 * kUnitRing;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kOffUnit = kOffMisc + 16;                     // int [kUnitRing]
  static constexpr int kSmemBytes = kOffUnit + 4 * kUnitRing + 1024;  // + alignment slack
  static_assert(DI % kKPerMma == 0 && kN % HI == 0 && HI <= 32 && 32 % HI == 0, "shape");
};

struct IdxParams {
  const float* w_idx;
  const float* q_scale;  // FP8: [n_q * H_I] power-of-two scale of each (query, head) row
  const float* k_scale;  // FP8: [ctx_len] scale of each key row
  int ctx_len;
  float* scores;
  int64_t ld;
  int n_q, q_pos0;
  int n_units, n_qb;  // units: n_qb query blocks x (up to) tpu-tile slots
  int tpu;            // key tiles per unit: kTilesPerUnit, or fewer when that leaves SMs idle
  WsHeader* ws;
};

template <class C>
__device__ __forceinline__ bool unit_range(const IdxParams& p, int u, int& qb, int& kt0,
                                           int& kt1) {
  // slot-major, later (longer) query blocks first: the queue hands out every
  // block's first 32 key tiles before any block's second, so units arrive in
  // roughly decreasing size and the CTAs finish close together
  const int c = u / p.n_qb;
  qb = p.n_qb - 1 - (u - c * p.n_qb);
  const int last_q = min((qb + 1) * C::kQB, p.n_q) - 1;
  const int ntiles = (p.q_pos0 + last_q) / C::kM + 1;
  kt0 = c * p.tpu;
  kt1 = min(kt0 + p.tpu, ntiles);
  return kt0 < kt1;
}

// The un-th unit of this CTA from the producer's ring (-1: the queue is
// exhausted, or a wait gave up and *ok is false). Warp-collective; the warp
// frees the slot once every lane has read it.
template <class C>
__device__ __forceinline__ int take_unit(uint64_t* unit_full, uint64_t* unit_empty, volatile int* sUnit,
                                         uint32_t un, volatile int* abort_flag, WsHeader* ws, unsigned site,
                                         bool& ok) {
  const int slot = static_cast<int>(un % C::kUnitRing);
  ok = __all_sync(0xffffffffu, mbar_wait(&unit_full[slot], (un / C::kUnitRing) & 1, abort_flag, ws, site));
  if (!ok) return -1;
  const int u = sUnit[slot];
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(&unit_empty[slot]);
  return u;
}

// Wait without the abort shortcut, used only to drain in-flight work.
__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity))
    if (clock64() - t0 > kWaitLimitCycles) break;
}

template <int HI, int DI, bool FP8>
__global__ void __launch_bounds__(IdxCfg<HI, DI, FP8>::kThreads, 1)
    index_scores_tc(const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_q, const IdxParams p) {
  using C = IdxCfg<HI, DI, FP8>;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* sQ = smem + C::kOffQ;
  unsigned char* sK = smem + C::kOffK;
  float* sW = reinterpret_cast<float*>(smem + C::kOffW);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* k_full = bars;
  uint64_t* k_empty = bars + C::kStages;
  uint64_t* q_full = bars + 2 * C::kStages;       // [1]
  uint64_t* q_empty = q_full + 1;                 // [1]
  uint64_t* acc_full = q_empty + 1;               // [2]
  uint64_t* acc_empty = acc_full + 2;             // [2]
  uint64_t* w_full = acc_empty + 2;               // [2]
  uint64_t* w_empty = w_full + 2;                 // [2]
  uint64_t* mma_done = w_empty + 2;               // [1]
  uint64_t* unit_full = mma_done + 1;             // [kUnitRing]
  uint64_t* unit_empty = unit_full + C::kUnitRing;  // [kUnitRing]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
  volatile int* sUnit = reinterpret_cast<volatile int*>(smem + C::kOffUnit);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], C::kEpiWarps);
      mbar_init(&w_full[b], 32);
      mbar_init(&w_empty[b], C::kEpiWarps);
    }
    mbar_init(mma_done, 1);
    for (int r = 0; r < C::kUnitRing; ++r) {
      mbar_init(&unit_full[r], 1);
      mbar_init(&unit_empty[r], 1 + C::kEpiWarps);  // the MMA warp and the epilogue warps
    }
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tm_k);
    prefetch_tmap(&tm_q);
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    uint32_t it = 0, uq = 0;
    int q_parity_issued = -1;  // parity of the last q_full phase with copies in flight
    bool ok = true;
    for (uint32_t un = 0; ok; ++un) {
      // the next non-empty unit of the queue (-1 once it is exhausted), handed
      // to the MMA and epilogue warps through the unit ring
      int u = -1;
      for (;;) {
        int v = 0;
        if (lane == 0) v = static_cast<int>(atomicAdd(&p.ws->unit_next, 1u));
        v = __shfl_sync(0xffffffffu, v, 0);
        if (v >= p.n_units) break;
        int qb_, kt0_, kt1_;
        if (unit_range<C>(p, v, qb_, kt0_, kt1_)) {
          u = v;
          break;
        }
      }
      const int slot = static_cast<int>(un % C::kUnitRing);
      ok = __all_sync(0xffffffffu, mbar_wait(&unit_empty[slot], ((un / C::kUnitRing) & 1) ^ 1, abort_flag,
                                             p.ws, 9));
      if (!ok) break;
      if (lane == 0) {
        sUnit[slot] = u;
        mbar_arrive(&unit_full[slot]);
      }
      if (u < 0) break;
      int qb, kt0, kt1;
      unit_range<C>(p, u, qb, kt0, kt1);
      // head weights of the block -> sW[uq & 1] (all 32 lanes write and arrive)
      const int wb = uq & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&w_empty[wb], ((uq >> 1) & 1) ^ 1, abort_flag, p.ws, 1));
      if (!ok) break;
      for (int e = lane; e < C::kN; e += 32) {
        const int i = qb * C::kQB + e / HI;
        float wv = i < p.n_q ? __ldg(p.w_idx + static_cast<int64_t>(qb) * C::kN + e) : 0.f;
        // FP8: w * s_q (a power of two: exact); the key's scale comes in the epilogue
        if (FP8 && i < p.n_q) wv *= __ldg(p.q_scale + static_cast<int64_t>(qb) * C::kN + e);
        sW[wb * C::kN + e] = wv;
      }
      mbar_arrive(&w_full[wb]);
      // the block's q_idx rows
      ok = __all_sync(0xffffffffu, mbar_wait(q_empty, (uq & 1) ^ 1, abort_flag, p.ws, 2));
      if (!ok) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(q_full, C::kQBytes);
        for (int c = 0; c < C::kNChunk; ++c)
          tma_load_2d(sQ + c * C::kQChunkBytes, &tm_q, c * C::kChunk, qb * C::kN, q_full);
      }
      q_parity_issued = static_cast<int>(uq & 1);
      for (int kt = kt0; kt < kt1; ++kt, ++it) {
        const int st = it % C::kStages;
        ok = __all_sync(0xffffffffu,
                        mbar_wait(&k_empty[st], ((it / C::kStages) & 1) ^ 1, abort_flag, p.ws, 3));
        if (!ok) break;
        if (lane == 0) {
          mbar_arrive_expect_tx(&k_full[st], C::kKTileBytes);
          for (int c = 0; c < C::kNChunk; ++c)
            tma_load_2d(sK + st * C::kKTileBytes + c * C::kKChunkBytes, &tm_k, c * C::kChunk,
                        kt * C::kM, &k_full[st]);
        }
      }
      if (ok) ++uq;
    }
    if (!ok && lane == 0) {  // let every issued copy land before the CTA exits
      const uint32_t n_back = it < static_cast<uint32_t>(C::kStages) ? it : C::kStages;
      for (uint32_t b = 1; b <= n_back; ++b) {
        const uint32_t tile = it - b;
        drain_wait(&k_full[tile % C::kStages], (tile / C::kStages) & 1);
      }
      if (q_parity_issued >= 0) drain_wait(q_full, static_cast<uint32_t>(q_parity_issued));
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the loop with warp-uniform operands and one elected
    // lane issues: descriptors are a base plus compile-time offsets, so an
    // issue costs a few cycles (a single-thread loop with run-time
    // descriptors costs more than a 128-cycle MMA).
    uint32_t it = 0, uq = 0;
    bool ok = true;
    const uint64_t dk0 = smem_desc(smem_u32(sK), 16, C::kSbo, C::kSwzCode);
    const uint64_t dq0 = smem_desc(smem_u32(sQ), 16, C::kSbo, C::kSwzCode);
    for (uint32_t un = 0; ok; ++un) {
      const int u = take_unit<C>(unit_full, unit_empty, sUnit, un, abort_flag, p.ws, 10, ok);
      if (u < 0) break;
      int qb, kt0, kt1;
      unit_range<C>(p, u, qb, kt0, kt1);
      if (!(ok = __all_sync(0xffffffffu, mbar_wait(q_full, uq & 1, abort_flag, p.ws, 4)))) break;
      for (int kt = kt0; kt < kt1; ++kt, ++it) {
        const int st = it % C::kStages, buf = it & 1;
        if (!(ok = __all_sync(0xffffffffu,
                              mbar_wait(&acc_empty[buf], ((it >> 1) & 1) ^ 1, abort_flag, p.ws, 5))))
          break;
        if (!(ok = __all_sync(0xffffffffu,
                              mbar_wait(&k_full[st], (it / C::kStages) & 1, abort_flag, p.ws, 6))))
          break;
        tc_fence_after();
        const uint32_t d = tmem_base + buf * C::kN;
        const uint64_t dk = dk0 + static_cast<uint64_t>((st * C::kKTileBytes) >> 4);
#pragma unroll
        for (int ks = 0; ks < C::kKSteps; ++ks) {
          const int c = ks / C::kStepsPerChunk;
          const uint32_t off = (ks % C::kStepsPerChunk) * 32;
          const uint64_t a = dk + static_cast<uint64_t>((c * C::kKChunkBytes + off) >> 4);
          const uint64_t b = dq0 + static_cast<uint64_t>((c * C::kQChunkBytes + off) >> 4);
          if constexpr (FP8) mma_f8_ss_warp(d, a, b, C::kIdesc, ks > 0 ? 1u : 0u);
          else mma_bf16_ss_warp(d, a, b, C::kIdesc, ks > 0 ? 1u : 0u);
        }
        mma_commit_warp(&k_empty[st]);
        mma_commit_warp(&acc_full[buf]);
      }
      if (!ok) break;
      mma_commit_warp(q_empty);
      ++uq;
    }
    // every MMA issued must complete before TMEM is released
    mma_commit_warp(mma_done);
    drain_wait(mma_done, 0);
  } else {
    // ------------------------------------------------------------ epilogue
    const int wg = (warp - 2) >> 2;        // column range (kColsPerWg columns)
    const int quarter = warp & 3;          // TMEM lane quarter this warp may access
    const int key_local = quarter * 32 + lane;
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    uint32_t it = 0, uq = 0;
    bool ok = true;
    for (uint32_t un = 0; ok; ++un) {
      const int u = take_unit<C>(unit_full, unit_empty, sUnit, un, abort_flag, p.ws, 11, ok);
      if (u < 0) break;
      int qb, kt0, kt1;
      unit_range<C>(p, u, qb, kt0, kt1);
      const int wb = uq & 1;
      ok = __all_sync(0xffffffffu, mbar_wait(&w_full[wb], (uq >> 1) & 1, abort_flag, p.ws, 7));
      if (!ok) break;
      const float* w = sW + wb * C::kN;
      for (int kt = kt0; kt < kt1; ++kt, ++it) {
        const int buf = it & 1;
        ok = __all_sync(0xffffffffu,
                        mbar_wait(&acc_full[buf], (it >> 1) & 1, abort_flag, p.ws, 8));
        if (!ok) break;
        tc_fence_after();
        const int s = kt * C::kM + key_local;
        // FP8: the key row's scale, applied to the finished head sum (a power
        // of two: relu(s_k x) = s_k relu(x), and the product is exact)
        const float ks = FP8 ? (s < p.ctx_len ? __ldg(p.k_scale + s) : 0.f) : 1.f;
        // the warp's 32-column groups: all loaded, and the accumulator handed
        // back to the MMA warp as soon as they are in registers, so the next
        // tile but one accumulates there while this one is summed
        uint32_t v[C::kGroups][32];
#pragma unroll
        for (int h = 0; h < C::kGroups; ++h)
          tmem_ld_32x32b_x32(tmem_base + lane_addr + buf * C::kN + wg * C::kColsPerWg + h * 32, v[h]);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&acc_empty[buf]);
#pragma unroll
        for (int h = 0; h < C::kGroups; ++h) {
          const int col0 = wg * C::kColsPerWg + h * 32;
#pragma unroll
          for (int qq = 0; qq < 32 / HI; ++qq) {
            // the head sum in four interleaved partial sums (heads j mod 4),
            // so that consecutive multiply-adds do not wait on each other;
            // the weights are read as float4 broadcasts
            constexpr int kPart = HI >= 4 ? 4 : HI;
            float part[kPart];
#pragma unroll
            for (int u = 0; u < kPart; ++u) part[u] = 0.f;
#pragma unroll
            for (int j0 = 0; j0 < HI; j0 += 4) {
              float wv[4];
              if constexpr (HI >= 4) {
                const float4 w4 = *reinterpret_cast<const float4*>(w + col0 + qq * HI + j0);
                wv[0] = w4.x;
                wv[1] = w4.y;
                wv[2] = w4.z;
                wv[3] = w4.w;
              } else {
#pragma unroll
                for (int e = 0; e < HI; ++e) wv[e] = w[col0 + qq * HI + e];
              }
#pragma unroll
              for (int e = 0; e < 4 && j0 + e < HI; ++e) {
                const int j = j0 + e;
                part[j % kPart] = fmaf(wv[e], fmaxf(__uint_as_float(v[h][qq * HI + j]), 0.f),
                                       part[j % kPart]);
              }
            }
            float acc = part[0];
#pragma unroll
            for (int u = 1; u < kPart; ++u) acc += part[u];
            const int i = qb * C::kQB + (col0 + qq * HI) / HI;
            if (i < p.n_q && s <= p.q_pos0 + i && DSA_IN_BOUNDS(p.ws, s, p.ld, 20))
              p.scores[static_cast<int64_t>(i) * p.ld + s] = FP8 ? acc * ks : acc;
          }
        }
      }
      if (!ok) break;
      __syncwarp();
      if (lane == 0) mbar_arrive(&w_empty[wb]);
      ++uq;
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

constexpr int kOneCtaPerSmSmem = 120 * 1024;

int num_sms() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

template <int HI, int DI, bool FP8>
cudaError_t launch(const dsa_dims& d, const void* q_idx, const void* k_idx, const float* q_scale,
                   const float* k_scale, const float* w_idx, float* scores, int64_t ld,
                   WsHeader* ws, cudaStream_t st) {
  using C = IdxCfg<HI, DI, FP8>;
  CUtensorMap tm_k, tm_q;
  if (FP8) {
    if (!make_tmap_u8_2d(&tm_k, k_idx, DI, static_cast<uint64_t>(d.ctx_len), C::kChunk, C::kM,
                         C::kSwzMap) ||
        !make_tmap_u8_2d(&tm_q, q_idx, DI, static_cast<uint64_t>(d.n_q) * HI, C::kChunk, C::kN,
                         C::kSwzMap))
      return cudaErrorInvalidValue;
  } else if (!make_tmap_bf16_2d(&tm_k, k_idx, DI, static_cast<uint64_t>(d.ctx_len), C::kChunk,
                                C::kM, C::kSwzMap) ||
             !make_tmap_bf16_2d(&tm_q, q_idx, DI, static_cast<uint64_t>(d.n_q) * HI, C::kChunk,
                                C::kN, C::kSwzMap)) {
    return cudaErrorInvalidValue;
  }
  IdxParams p;
  p.w_idx = w_idx;
  p.q_scale = q_scale;
  p.k_scale = k_scale;
  p.ctx_len = d.ctx_len;
  p.scores = scores;
  p.ld = ld;
  p.n_q = d.n_q;
  p.q_pos0 = d.q_pos0;
  p.ws = ws;
  const int max_tiles = (d.q_pos0 + d.n_q - 1) / C::kM + 1;
  p.n_qb = (d.n_q + C::kQB - 1) / C::kQB;
  // 32 tiles per unit, or fewer when a small chunk (a decode step) would then
  // give fewer units than SMs; a score does not depend on the unit it is in
  p.tpu = C::kTilesPerUnit;
  const long long tiles_total = static_cast<long long>(p.n_qb) * max_tiles;
  if (tiles_total < static_cast<long long>(C::kTilesPerUnit) * num_sms())
    p.tpu = static_cast<int>((tiles_total + num_sms() - 1) / num_sms());
  if (p.tpu < 1) p.tpu = 1;
  const int slots = (max_tiles + p.tpu - 1) / p.tpu;
  p.n_units = p.n_qb * slots;
  // the work queue starts at unit 0 on every launch
  cudaError_t e0 = cudaMemsetAsync(&ws->unit_next, 0, sizeof(ws->unit_next), st);
  if (e0 != cudaSuccess) return e0;
  const int grid = p.n_units < num_sms() ? p.n_units : num_sms();
  // The CTA owns all 512 TMEM columns of its SM: ask for enough shared memory
  // that a second CTA can never be resident beside it.
  const int smem = C::kSmemBytes > kOneCtaPerSmSmem ? C::kSmemBytes : kOneCtaPerSmSmem;
  cudaError_t e = cudaFuncSetAttribute(index_scores_tc<HI, DI, FP8>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  index_scores_tc<HI, DI, FP8><<<grid, C::kThreads, smem, st>>>(tm_k, tm_q, p);
  return cudaGetLastError();
}

// e4m3 codes of bf16 rows (one warp per row of `cols` <= 128 values): the
// row's scale is the smallest power of two s with max|x| <= 448 s, the code
// is x / s rounded to the nearest e4m3 value (ties to even, the hardware
// conversion), and xhat = code * s as bf16 (exact).
__global__ void quantize_fp8_kernel(const uint16_t* __restrict__ x, int64_t rows, int cols,
                                    uint8_t* __restrict__ x8, float* __restrict__ scale,
                                    uint16_t* __restrict__ xhat) {
  const int64_t r = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  const uint16_t* xr = x + r * cols;
  float v[4];
  float amax = 0.f;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int c = lane * 4 + u;
    v[u] = c < cols ? bf16_to_f32(xr[c]) : 0.f;
    amax = fmaxf(amax, fabsf(v[u]));
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  // k: 448 * 2^k >= amax with k minimal; amax = m * 2^E, m in [1, 2):
  // k = E - 8 when m <= 1.75, else E - 7 (448 = 1.75 * 2^8)
  int k = 0;
  if (amax > 0.f) {
    int E;
    const float m = frexpf(amax, &E) * 2.f;  // amax = m * 2^(E-1)
    E -= 1;
    k = m <= 1.75f ? E - 8 : E - 7;
  }
  if (lane == 0) scale[r] = ldexpf(1.f, k);
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int c = lane * 4 + u;
    if (c >= cols) break;
    const float q = ldexpf(v[u], -k);  // exact
    const __nv_fp8_storage_t code = __nv_cvt_float_to_fp8(q, __NV_SATFINITE, __NV_E4M3);
    x8[r * cols + c] = static_cast<uint8_t>(code);
    const __half_raw hr = __nv_cvt_fp8_to_halfraw(code, __NV_E4M3);
    const float deq = ldexpf(__half2float(__half(hr)), k);
    xhat[r * cols + c] = static_cast<uint16_t>(__float_as_uint(deq) >> 16);
  }
}

}  // namespace

cudaError_t launch_index_scores(const dsa_dims& d, const uint16_t* q_idx, const uint16_t* k_idx,
                                const float* w_idx, float* scores, int64_t ld, WsHeader* ws,
                                cudaStream_t st) {
  if (d.n_idx_heads == 32 && d.d_idx == 128)
    return launch<32, 128, false>(d, q_idx, k_idx, nullptr, nullptr, w_idx, scores, ld, ws, st);
  if (d.n_idx_heads == 2 && d.d_idx == 32)
    return launch<2, 32, false>(d, q_idx, k_idx, nullptr, nullptr, w_idx, scores, ld, ws, st);
  return cudaErrorInvalidValue;
}

cudaError_t launch_index_scores_fp8(const dsa_dims& d, const uint8_t* q8, const float* q_scale,
                                    const uint8_t* k8, const float* k_scale, const float* w_idx,
                                    float* scores, int64_t ld, WsHeader* ws, cudaStream_t st) {
  if (d.n_idx_heads == 32 && d.d_idx == 128)
    return launch<32, 128, true>(d, q8, k8, q_scale, k_scale, w_idx, scores, ld, ws, st);
  if (d.n_idx_heads == 2 && d.d_idx == 32)
    return launch<2, 32, true>(d, q8, k8, q_scale, k_scale, w_idx, scores, ld, ws, st);
  return cudaErrorInvalidValue;
}

cudaError_t launch_quantize_fp8(const uint16_t* x, int64_t rows, int cols, uint8_t* x8,
                                float* scale, uint16_t* xhat, cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  if (cols < 1 || cols > 128) return cudaErrorInvalidValue;
  const int threads = 256;
  const int64_t blocks = (rows * 32 + threads - 1) / threads;
  quantize_fp8_kernel<<<static_cast<unsigned>(blocks), threads, 0, st>>>(x, rows, cols, x8, scale,
                                                                         xhat);
  return cudaGetLastError();
}

}  // namespace dsa
