// attention.cu -- sparse MLA-style attention over the selected keys on tcgen05
// tensor cores (component-table row "DSA sparse-attention core" of the
// feedman.me post feedman.me/posts/wy2HU).
//
//   z_s = scale * (q[h,:Dc] . latent[s] + q[h,Dc:] . rope[s]),  s in S_t
//   out[h] = sum_s softmax(z)_s * latent[s],   lse[h] = log sum_s exp(z_s)
//
// The page's own kernel takes one query per threadgroup and forms scalar dot
// products over the 2,048 gathered keys (paragraph "Two levers fell out of
// this"), and proposes sharing gathered keys across neighbouring queries. On
// B200 the gathered rows go through shared memory into tcgen05 MMAs instead;
// selections of neighbouring queries barely overlap on these workloads, so a
// CTA works on one query at a time and the 32 heads of that query are what
// share each gathered row.
//
// Per query, in tiles of 128 selected keys:
//   gather   latent (8 x 64-dim chunks) and rope rows of the tile into nine
//            16 KB shared-memory slots, 128-byte swizzled, one key per 128-byte
//            row, with TMA tile::gather4 loads (four selected rows each);
//   QK^T     S^T[key, head] = K_tile . Q^T: keys are the MMA's M (128), the
//            padded heads its N, K = Dc + Dr, both operands K-major; rope
//            chunk first so its slot is released earliest. A tcgen05.mma that
//            depends on the previous one's accumulator waits out its latency,
//            so the K steps feed four independent partial sums (summed by the
//            softmax) and the PV interleaves its four 128-dim output blocks;
//   softmax  one thread per key lane of S^T: the per-head tile maximum is found
//            with a warp transpose-reduction plus a four-warp exchange through
//            shared memory (mbarrier-synchronised), the running maximum is
//            raised only when a tile exceeds it by more than 2^8 (then O and
//            the partial sums are rescaled), and p = 2^(z log2e - m) is written
//            as bf16 into P [key, head] (one 16-byte-chunked row per key);
//   PV       O^T[dim, head] += latent_tile^T . P^T: the same latent slots read
//            MN-major as A (dims as M, four 128-dim blocks), P MN-major as B;
//            each block's two slots are released as soon as its MMAs finish,
//            so the next tile's gather overlaps the current PV.
// Accumulators live in TMEM (S^T double-buffered per tile, O^T per query);
// the epilogue divides by the row sum, rounds to bf16 and writes out / lse.
//
// Roles (288 threads, one CTA per SM, persistent over queries):
//   warps 0-3  producers: cp.async gathers and the query's q rows;
//   warp  4    TMEM owner and single-thread tcgen05.mma issuer;
//   warps 5-8  softmax and epilogue (TMEM lanes 0-127 = keys, then dims).
// Every wait is bounded; on a timeout the CTA records DSA_ERR_TIMEOUT, all
// roles stop, copies and MMAs in flight are drained and TMEM is freed.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "dsa_internal.cuh"
#include "sm100_primitives.cuh"

namespace dsa {
namespace {

using namespace sm100;

template <int H, int DC, int DR>
struct AttnCfg {
  static constexpr int kKeys = 128;                   // keys per tile (MMA M of QK^T)
  static constexpr int NH = H < 16 ? 16 : H;          // heads padded to a legal MMA N
  static constexpr int NL = DC / 64;                  // latent 64-dim chunks
  static constexpr int MB = (DC + 127) / 128;         // 128-dim blocks of the PV
  static constexpr int NLS = 2 * MB;                  // latent slots (zero-padded)
  static constexpr int kRope = NLS;                   // slot index of the rope chunk
  static constexpr int kSlots = NLS + 1;
  static constexpr int kRopeSteps = DR / 16;
  static constexpr int kSlotBytes = kKeys * 128;      // 16 KB
  static constexpr int kQChunks = NL + 1;             // latent chunks + rope chunk
  static constexpr int kQChunkBytes = NH * 128;
  // P: one row of NH bf16 per key (MN-major B operand of the PV), 64- or
  // 32-byte rows swizzled in 8-row atoms
  static constexpr int kPRowBytes = NH * 2;
  static constexpr int kPBytes = kKeys * kPRowBytes;
  static constexpr uint32_t kPSwz = NH == 32 ? 4u : 6u;  // descriptor code: 64B / 32B swizzle
  static constexpr int kThreads = 288;
  static constexpr int kGatherPositions = NL + 1;     // rope, L0..L(NL-1)
  static constexpr bool kRopeTma = DR == 64;          // a 128-byte rope row: TMA gather4
  static constexpr uint32_t kQBytes = H * 128 * kQChunks;  // q boxes (zero-filled past Dc+Dr)
  static constexpr uint32_t kIdescQK = idesc_bf16_f32(128, NH, false, false);
  static constexpr uint32_t kIdescPV = idesc_bf16_f32(128, NH, true, true);
  // TMEM columns: S^T[2 buffers][kChains partial sums] then O^T[2][MB]
  static constexpr int kChains = 4;                   // independent QK^T accumulators
  static constexpr int kTmemS = 0;
  static constexpr int kTmemO = 2 * kChains * NH;
  static constexpr int kTmemUsed = 2 * kChains * NH + 2 * MB * NH;
  static constexpr int kTmemCols = kTmemUsed <= 32 ? 32 : kTmemUsed <= 64 ? 64 : kTmemUsed <= 128 ? 128
                                   : kTmemUsed <= 256 ? 256 : 512;
  // shared memory carve (from a 1024-byte aligned base)
  static constexpr int kOffSlots = 0;
  static constexpr int kOffQ = kOffSlots + kSlots * kSlotBytes;
  static constexpr int kOffP = kOffQ + kQChunks * kQChunkBytes;
  static constexpr int kOffRed = kOffP + 2 * kPBytes;            // [2][4][32] floats
  static constexpr int kOffBar = kOffRed + 2 * 4 * 32 * 4;
  static constexpr int kNumBars = 2 * kSlots + 2 + 2 * 2 + 2 * 2 + 2 * 2 + 1 + 2 + 1;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;
  static_assert(DC % 64 == 0 && DR % 16 == 0 && DR <= 64 && (NH % 16) == 0 && NH <= 32 &&
                    (H & (H - 1)) == 0,
                "shape");
};

struct AttnParams {
  const uint16_t* q;
  const uint16_t* latent;
  const uint16_t* rope;
  const int32_t* idx;
  uint16_t* out;
  float* lse;
  int n_q, q_pos0, ctx_len, k;
  int prefix_valid;  // idx rows hold min(k, t+1) valid keys first (selections of this library)
  float scale_log2;  // softmax_scale * log2(e)
  WsHeader* ws;
};

__device__ __forceinline__ int n_tiles_of(const AttnParams& p, int i) {
  const int valid = p.prefix_valid ? min(p.k, p.q_pos0 + i + 1) : p.k;
  return (valid + 127) / 128;
}

__device__ __forceinline__ void drain_wait(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity))
    if (clock64() - t0 > kWaitLimitCycles) break;
}

// Reduces NV values across the 32 lanes of a warp; afterwards lane l holds the
// reduction of value (l % NV) over all lanes. NV is a power of two <= 32.
template <int NV, bool kMax>
__device__ __forceinline__ float warp_transpose_reduce(float (&v)[NV]) {
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

template <int NH>
__device__ __forceinline__ void tmem_ld_row(uint32_t taddr, float (&x)[NH]) {
  if constexpr (NH == 32) {
    uint32_t r[32];
    tmem_ld_32x32b_x32(taddr, r);
    tmem_ld_wait();
#pragma unroll
    for (int e = 0; e < 32; ++e) x[e] = __uint_as_float(r[e]);
  } else {
    uint32_t r[16];
    tmem_ld_32x32b_x16(taddr, r);
    tmem_ld_wait();
#pragma unroll
    for (int e = 0; e < 16; ++e) x[e] = __uint_as_float(r[e]);
  }
}

template <int NH>
__device__ __forceinline__ void tmem_st_row(uint32_t taddr, const float (&x)[NH]) {
  if constexpr (NH == 32) {
    uint32_t r[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(x[e]);
    tmem_st_32x32b_x32(taddr, r);
  } else {
    uint32_t r[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) r[e] = __float_as_uint(x[e]);
    tmem_st_32x32b_x16(taddr, r);
  }
}

template <int H, int DC, int DR>
__global__ void __launch_bounds__(AttnCfg<H, DC, DR>::kThreads, 1)
    sparse_attn_tc(const __grid_constant__ CUtensorMap tm_lat, const __grid_constant__ CUtensorMap tm_rope,
                   const __grid_constant__ CUtensorMap tm_q, const AttnParams p) {
  using C = AttnCfg<H, DC, DR>;
  constexpr int NH = C::NH;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* sSlots = smem + C::kOffSlots;
  unsigned char* sQ = smem + C::kOffQ;
  unsigned char* sP = smem + C::kOffP;
  float* sRed = reinterpret_cast<float*>(smem + C::kOffRed);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* slot_full = bars;                        // [kSlots]
  uint64_t* slot_empty = bars + C::kSlots;           // [kSlots]
  uint64_t* q_full = bars + 2 * C::kSlots;           // [1]
  uint64_t* q_empty = q_full + 1;                    // [1]
  uint64_t* s_full = q_empty + 1;                    // [2]
  uint64_t* s_empty = s_full + 2;                    // [2]
  uint64_t* p_full = s_empty + 2;                    // [2]
  uint64_t* p_empty = p_full + 2;                    // [2]
  uint64_t* o_full = p_empty + 2;                    // [2]
  uint64_t* o_empty = o_full + 2;                    // [2]
  uint64_t* o_step = o_empty + 2;                    // [1]
  uint64_t* exch = o_step + 1;                       // [2]
  uint64_t* mma_done = exch + 2;                     // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // zero every operand buffer once: padded heads, padded latent slots and the
  // unused part of a narrow rope chunk must read as zeros
  for (int e = threadIdx.x * 16; e < C::kOffRed; e += C::kThreads * 16)
    *reinterpret_cast<uint4*>(smem + e) = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kSlots; ++s) {
      // TMA slots complete on bytes after one arrive; a cp.async rope slot on
      // the 32 noinc arrivals of its warp
      mbar_init(&slot_full[s], (s == C::kRope && !C::kRopeTma) ? 32 : 1);
      mbar_init(&slot_empty[s], 1);
    }
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_empty[b], 128);
      mbar_init(&p_full[b], 128);
      mbar_init(&p_empty[b], 1);
      mbar_init(&o_full[b], 1);
      mbar_init(&o_empty[b], 128);
      mbar_init(&exch[b], 128);
    }
    mbar_init(o_step, 1);
    mbar_init(mma_done, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 4) tmem_alloc(tmem_slot, C::kTmemCols);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp < 4) {
    // -------------------------------------------------------------- producers
    // This warp fills gather positions w, w+4, ... of each tile (position 0 is
    // the rope chunk, position 1+c latent chunk c). A slot of 128 keys is 32
    // TMA gather4 loads, one per lane: lane l brings keys 4l..4l+3 (four
    // 128-byte rows, 512 swizzled bytes) and the slot's mbarrier completes on
    // its 16 KB of transactions. Warp 0 also loads the query's q rows with 2D
    // TMA boxes. A 16-dim rope chunk (too narrow for a 128-byte swizzled box)
    // is gathered with cp.async, each lane announcing its copies with
    // cp.async.mbarrier.arrive.noinc.
    if (warp == 0 && lane == 0) {
      prefetch_tmap(&tm_lat);
      prefetch_tmap(&tm_q);
      if (C::kRopeTma) prefetch_tmap(&tm_rope);
    }
    uint32_t tc = 0, qi = 0;
    bool ok = true;
    int last_slot_parity = -1;  // parity of this warp's last issued slot fills (for draining)
    int q_parity = -1;
    for (int i = blockIdx.x; i < p.n_q && ok; i += gridDim.x, ++qi) {
      if (warp == 0) {
        ok = __all_sync(0xffffffffu, mbar_wait(q_empty, (qi & 1) ^ 1, abort_flag, p.ws, 20));
        if (!ok) break;
        if (lane == 0) {
          mbar_arrive_expect_tx(q_full, C::kQBytes);
          for (int c = 0; c < C::kQChunks; ++c)
            tma_load_2d(sQ + c * C::kQChunkBytes, &tm_q, c * 64, i * H, q_full);
        }
        q_parity = qi & 1;
      }
      const int nt = n_tiles_of(p, i);
      const int32_t* irow = p.idx + static_cast<int64_t>(i) * p.k;
      for (int j = 0; j < nt && ok; ++j, ++tc) {
        // rows of keys 4*lane .. 4*lane+3 (masked or out-of-range keys read row 0;
        // their softmax weight is zero)
        int r4[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int sel = j * 128 + 4 * lane + e;
          int row = sel < p.k ? __ldg(irow + sel) : -1;
          if (row >= p.ctx_len) {
            report(p.ws, kDevRange, static_cast<unsigned>(i));
            row = -1;
          }
          r4[e] = row < 0 ? 0 : row;
        }
        for (int pos = warp; pos < C::kGatherPositions; pos += 4) {
          const int slot = pos == 0 ? C::kRope : pos - 1;
          ok = __all_sync(0xffffffffu,
                          mbar_wait(&slot_empty[slot], (tc & 1) ^ 1, abort_flag, p.ws, 21));
          if (!ok) break;
          unsigned char* dst = sSlots + slot * C::kSlotBytes;
          if (slot != C::kRope || C::kRopeTma) {
            if (lane == 0) mbar_arrive_expect_tx(&slot_full[slot], C::kSlotBytes);
            __syncwarp();
            if (slot == C::kRope)
              tma_gather4(dst + lane * 512, &tm_rope, 0, r4[0], r4[1], r4[2], r4[3], &slot_full[slot]);
            else
              tma_gather4(dst + lane * 512, &tm_lat, slot * 64, r4[0], r4[1], r4[2], r4[3],
                          &slot_full[slot]);
          } else {
            const int part = lane & 7;
            if (part < DR / 8) {
#pragma unroll 4
              for (int it = 0; it < 32; ++it) {
                const int key = (lane >> 3) + 4 * it;
                const int sel = j * 128 + key;
                int row = sel < p.k ? __ldg(irow + sel) : -1;
                if (row < 0 || row >= p.ctx_len) row = 0;
                cp_async_16(dst + key * 128 + ((part ^ (key & 7)) << 4),
                            p.rope + static_cast<int64_t>(row) * DR + part * 8);
              }
            }
            cp_async_arrive_noinc(&slot_full[slot]);
          }
          last_slot_parity = tc & 1;
        }
      }
    }
    cp_async_wait_all();  // every cp.async copy lands before the CTA can exit
    if (!ok && lane == 0) {  // and every TMA load this warp issued
      if (last_slot_parity >= 0)
        for (int pos = warp; pos < C::kGatherPositions; pos += 4) {
          const int slot = pos == 0 ? C::kRope : pos - 1;
          if (slot != C::kRope || C::kRopeTma) drain_wait(&slot_full[slot], last_slot_parity);
        }
      if (q_parity >= 0) drain_wait(q_full, q_parity);
    }
  } else if (warp == 4) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      uint32_t tc = 0, qi = 0;
      bool ok = true;
      const uint32_t slots_addr = smem_u32(sSlots);
      const uint32_t q_addr = smem_u32(sQ);
      const uint32_t p_addr = smem_u32(sP);
      for (int i = blockIdx.x; i < p.n_q && ok; i += gridDim.x, ++qi) {
        const int nt = n_tiles_of(p, i);
        const int ob = qi & 1;
        if (!(ok = mbar_wait(q_full, qi & 1, abort_flag, p.ws, 30))) break;
        fence_proxy_async_smem();
        for (int j = 0; j < nt; ++j, ++tc) {
          const int sb = tc & 1, pb = tc & 1;
          // ---- S^T = K_tile . Q^T
          if (!(ok = mbar_wait(&s_empty[sb], ((tc >> 1) & 1) ^ 1, abort_flag, p.ws, 31))) break;
          // S^T accumulates in kChains independent partial sums (K-step ks of
          // every chunk goes to chain ks), so consecutive MMAs never wait on
          // each other's accumulator; the softmax adds the partials.
          const uint32_t d_s = tmem_base + C::kTmemS + sb * C::kChains * NH;
          if (!(ok = mbar_wait(&slot_full[C::kRope], tc & 1, abort_flag, p.ws, 32))) break;
          fence_proxy_async_smem();
          tc_fence_after();
#pragma unroll
          for (int ks = 0; ks < C::kRopeSteps; ++ks) {
            const uint64_t a = smem_desc(slots_addr + C::kRope * C::kSlotBytes + ks * 32, 16, 1024, 2);
            const uint64_t b = smem_desc(q_addr + C::NL * C::kQChunkBytes + ks * 32, 16, 1024, 2);
            mma_bf16_ss(d_s + (ks % C::kChains) * NH, a, b, C::kIdescQK, ks >= C::kChains ? 1u : 0u);
          }
          mma_commit(&slot_empty[C::kRope]);
          for (int c = 0; c < C::NL && ok; ++c) {
            if (!(ok = mbar_wait(&slot_full[c], tc & 1, abort_flag, p.ws, 33))) break;
            fence_proxy_async_smem();
            tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
              const uint64_t a = smem_desc(slots_addr + c * C::kSlotBytes + ks * 32, 16, 1024, 2);
              const uint64_t b = smem_desc(q_addr + c * C::kQChunkBytes + ks * 32, 16, 1024, 2);
              const bool fresh = c == 0 && ks >= C::kRopeSteps;  // chain not yet written this tile
              mma_bf16_ss(d_s + ks * NH, a, b, C::kIdescQK, fresh ? 0u : 1u);
            }
          }
          if (!ok) break;
          mma_commit(&s_full[sb]);
          if (j == nt - 1) mma_commit(q_empty);
          // ---- O^T += latent_tile^T . P^T
          if (!(ok = mbar_wait(&p_full[pb], (tc >> 1) & 1, abort_flag, p.ws, 34))) break;
          if (j == 0 && !(ok = mbar_wait(&o_empty[ob], ((qi >> 1) & 1) ^ 1, abort_flag, p.ws, 35)))
            break;
          tc_fence_after();
          // the MB output blocks are independent accumulators: interleave them
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint64_t b = smem_desc(p_addr + pb * C::kPBytes + kk * 16 * C::kPRowBytes,
                                         8 * C::kPRowBytes, 8 * C::kPRowBytes, C::kPSwz);
#pragma unroll
            for (int mb = 0; mb < C::MB; ++mb) {
              const uint32_t d_o = tmem_base + C::kTmemO + (ob * C::MB + mb) * NH;
              const uint64_t a = smem_desc(slots_addr + (2 * mb) * C::kSlotBytes + kk * 2048,
                                           C::kSlotBytes, 1024, 2);
              mma_bf16_ss(d_o, a, b, C::kIdescPV, (j == 0 && kk == 0) ? 0u : 1u);
            }
          }
          for (int c = 0; c < C::NL; ++c) mma_commit(&slot_empty[c]);
          mma_commit(&p_empty[pb]);
          mma_commit(o_step);
          if (j == nt - 1) mma_commit(&o_full[ob]);
        }
      }
      mma_commit(mma_done);
      drain_wait(mma_done, 0);
    }
  } else {
    // ------------------------------------------------- softmax and epilogue
    const int quarter = warp & 3;               // TMEM lane quarter of this warp
    const int r = quarter * 32 + lane;          // key lane (and dim lane in the epilogue)
    const int sw = warp - 5;                    // softmax warp index 0..3
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    uint32_t tc = 0, qi = 0, xc = 0;
    bool ok = true;
    for (int i = blockIdx.x; i < p.n_q && ok; i += gridDim.x, ++qi) {
      const int nt = n_tiles_of(p, i);
      const int ob = qi & 1;
      const int32_t* irow = p.idx + static_cast<int64_t>(i) * p.k;
      float m_lane = -INFINITY;       // running max (log2 units) of head `lane`
      float mrep[NH];                 // running max of every head, replicated
      float lpart[NH];                // this key lane's share of the row sums
#pragma unroll
      for (int h = 0; h < NH; ++h) {
        mrep[h] = -INFINITY;
        lpart[h] = 0.f;
      }
      for (int j = 0; j < nt; ++j, ++tc) {
        const int sb = tc & 1, pb = tc & 1;
        const int sel = j * 128 + r;
        const int row = sel < p.k ? __ldg(irow + sel) : -1;  // issued before the wait
        ok = __all_sync(0xffffffffu, mbar_wait(&s_full[sb], (tc >> 1) & 1, abort_flag, p.ws, 40));
        if (!ok) break;
        tc_fence_after();
        float x[NH];
        tmem_ld_row<NH>(tmem_base + lane_addr + C::kTmemS + sb * C::kChains * NH, x);
#pragma unroll
        for (int ch = 1; ch < C::kChains; ++ch) {
          float y[NH];
          tmem_ld_row<NH>(tmem_base + lane_addr + C::kTmemS + (sb * C::kChains + ch) * NH, y);
#pragma unroll
          for (int h = 0; h < NH; ++h) x[h] += y[h];
        }
        tc_fence_before();
        mbar_arrive(&s_empty[sb]);
        const bool valid = row >= 0 && row < p.ctx_len;
#pragma unroll
        for (int h = 0; h < NH; ++h) x[h] = (valid && h < H) ? x[h] * p.scale_log2 : -INFINITY;
        // per-head maximum of this tile over all 128 keys
        float red[NH];
#pragma unroll
        for (int h = 0; h < NH; ++h) red[h] = x[h];
        const float wmax = warp_transpose_reduce<NH, true>(red);
        float* xbuf = sRed + (xc & 1) * 128;
        if (lane < NH) xbuf[sw * 32 + lane] = wmax;
        mbar_arrive(&exch[xc & 1]);
        ok = __all_sync(0xffffffffu, mbar_wait(&exch[xc & 1], (xc >> 1) & 1, abort_flag, p.ws, 41));
        ++xc;
        if (!ok) break;
        float tmax = -INFINITY;
        if (lane < NH)
          tmax = fmaxf(fmaxf(xbuf[lane], xbuf[32 + lane]), fmaxf(xbuf[64 + lane], xbuf[96 + lane]));
        const bool need = lane < H && tmax > -INFINITY && (m_lane == -INFINITY || tmax > m_lane + 8.f);
        if (__any_sync(0xffffffffu, need)) {
          const float m_new = fmaxf(m_lane, tmax);
          const float alpha_lane = m_lane == -INFINITY ? 0.f : ex2_approx(m_lane - m_new);
          m_lane = m_new;
          float alpha[NH];
#pragma unroll
          for (int h = 0; h < NH; ++h) {
            alpha[h] = __shfl_sync(0xffffffffu, alpha_lane, h);
            mrep[h] = __shfl_sync(0xffffffffu, m_lane, h);
            lpart[h] *= alpha[h];
          }
          if (j > 0) {  // rescale O^T once the previous tile's PV is complete
            ok = __all_sync(0xffffffffu, mbar_wait(o_step, (tc - 1) & 1, abort_flag, p.ws, 42));
            if (!ok) break;
            tc_fence_after();
#pragma unroll 1
            for (int mb = 0; mb < C::MB; ++mb) {
              const uint32_t ta = tmem_base + lane_addr + C::kTmemO + (ob * C::MB + mb) * NH;
              float o[NH];
              tmem_ld_row<NH>(ta, o);
#pragma unroll
              for (int h = 0; h < NH; ++h) o[h] *= alpha[h];
              tmem_st_row<NH>(ta, o);
            }
            tmem_st_wait();
          }
        }
        // probabilities of this key for every head, bf16, into P^T[pb][h][r]
        ok = __all_sync(0xffffffffu,
                        mbar_wait(&p_empty[pb], ((tc >> 1) & 1) ^ 1, abort_flag, p.ws, 43));
        if (!ok) break;
        // this key's row of P: NH bf16, written as 16-byte chunks at their
        // swizzled positions (chunk c ^ ((r >> 1) & 3) for 64-byte rows,
        // c ^ ((r >> 2) & 1) for 32-byte rows)
        uint32_t packed[NH / 2];
#pragma unroll
        for (int h2 = 0; h2 < NH / 2; ++h2) {
          float pv[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int h = 2 * h2 + e;
            pv[e] = 0.f;
            if (h < H && x[h] > -INFINITY && mrep[h] > -INFINITY) pv[e] = ex2_approx(x[h] - mrep[h]);
            lpart[h] += pv[e];
          }
          const __nv_bfloat162 b2 = __floats2bfloat162_rn(pv[0], pv[1]);
          packed[h2] = *reinterpret_cast<const uint32_t*>(&b2);
        }
        unsigned char* prow = sP + pb * C::kPBytes + r * C::kPRowBytes;
        const int swz = NH == 32 ? ((r >> 1) & 3) : ((r >> 2) & 1);
#pragma unroll
        for (int c = 0; c < NH / 8; ++c)
          *reinterpret_cast<uint4*>(prow + ((c ^ swz) << 4)) =
              make_uint4(packed[4 * c], packed[4 * c + 1], packed[4 * c + 2], packed[4 * c + 3]);
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&p_full[pb]);
      }
      if (!ok) break;
      // ---- epilogue of query i
      ok = __all_sync(0xffffffffu, mbar_wait(&o_full[ob], (qi >> 1) & 1, abort_flag, p.ws, 44));
      if (!ok) break;
      tc_fence_after();
      const float lsum = warp_transpose_reduce<NH, false>(lpart);
      float* xbuf = sRed + (xc & 1) * 128;
      if (lane < NH) xbuf[sw * 32 + lane] = lsum;
      mbar_arrive(&exch[xc & 1]);
      ok = __all_sync(0xffffffffu, mbar_wait(&exch[xc & 1], (xc >> 1) & 1, abort_flag, p.ws, 45));
      ++xc;
      if (!ok) break;
      float l_lane = 0.f;
      if (lane < NH) l_lane = xbuf[lane] + xbuf[32 + lane] + xbuf[64 + lane] + xbuf[96 + lane];
      const float inv_lane = l_lane > 0.f ? 1.f / l_lane : 0.f;
      if (sw == 0 && lane < H && p.lse)
        p.lse[static_cast<int64_t>(i) * H + lane] =
            l_lane > 0.f ? (m_lane + log2f(l_lane)) * 0.6931471805599453f : -INFINITY;
      float inv[NH];
#pragma unroll
      for (int h = 0; h < NH; ++h) inv[h] = __shfl_sync(0xffffffffu, inv_lane, h);
#pragma unroll 1
      for (int mb = 0; mb < C::MB; ++mb) {
        float o[NH];
        tmem_ld_row<NH>(tmem_base + lane_addr + C::kTmemO + (ob * C::MB + mb) * NH, o);
        const int d = mb * 128 + r;
        if (d < DC) {
          uint16_t* orow = p.out + static_cast<int64_t>(i) * H * DC + d;
#pragma unroll
          for (int h = 0; h < H; ++h) orow[h * DC] = f32_to_bf16_rne(o[h] * inv[h]);
        }
      }
      tc_fence_before();
      mbar_arrive(&o_empty[ob]);
    }
  }

  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

int num_sms() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

constexpr int kOneCtaPerSmSmem = 120 * 1024;

template <int H, int DC, int DR>
cudaError_t launch(const dsa_dims& d, const uint16_t* q, const uint16_t* latent,
                   const uint16_t* rope, const int32_t* idx, uint16_t* out, float* lse,
                   bool prefix_valid, WsHeader* ws, cudaStream_t st) {
  using C = AttnCfg<H, DC, DR>;
  AttnParams p;
  p.q = q;
  p.latent = latent;
  p.rope = rope;
  p.idx = idx;
  p.out = out;
  p.lse = lse;
  p.n_q = d.n_q;
  p.q_pos0 = d.q_pos0;
  p.ctx_len = d.ctx_len;
  p.k = d.top_k;
  p.prefix_valid = prefix_valid ? 1 : 0;
  p.scale_log2 = d.softmax_scale * 1.4426950408889634f;
  p.ws = ws;
  CUtensorMap tm_lat, tm_rope, tm_q;
  if (!make_tmap_bf16_2d(&tm_lat, latent, DC, static_cast<uint64_t>(d.ctx_len), 64, 1,
                         CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_tmap_bf16_2d(&tm_q, q, DC + DR, static_cast<uint64_t>(d.n_q) * H, 64, H,
                         CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (C::kRopeTma) {
    if (!make_tmap_bf16_2d(&tm_rope, rope, DR, static_cast<uint64_t>(d.ctx_len), 64, 1,
                           CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
  } else {
    tm_rope = tm_lat;  // unused
  }
  const int grid = d.n_q < num_sms() ? d.n_q : num_sms();
  const int smem = C::kSmemBytes > kOneCtaPerSmSmem ? C::kSmemBytes : kOneCtaPerSmSmem;
  cudaError_t e = cudaFuncSetAttribute(sparse_attn_tc<H, DC, DR>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  sparse_attn_tc<H, DC, DR><<<grid, C::kThreads, smem, st>>>(tm_lat, tm_rope, tm_q, p);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_sparse_attn(const dsa_dims& d, const uint16_t* q, const uint16_t* latent,
                               const uint16_t* rope, const int32_t* idx, uint16_t* out,
                               float* lse, bool prefix_valid, WsHeader* ws, cudaStream_t st) {
  if (d.n_heads == 32 && d.d_latent == 512 && d.d_rope == 64)
    return launch<32, 512, 64>(d, q, latent, rope, idx, out, lse, prefix_valid, ws, st);
  if (d.n_heads == 4 && d.d_latent == 64 && d.d_rope == 16)
    return launch<4, 64, 16>(d, q, latent, rope, idx, out, lse, prefix_valid, ws, st);
  return cudaErrorInvalidValue;
}

}  // namespace dsa
