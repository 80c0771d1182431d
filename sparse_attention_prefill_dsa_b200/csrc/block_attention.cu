// block_attention.cu -- the block-sparse form of the sparse attention: a group
// of QB neighbouring queries gathers the union of their selected keys once and
// runs QK^T and PV for all of the group's heads on that union, with a per-query
// mask (component-table row "DSA sparse-attention core" of the feedman.me post
// feedman.me/posts/wy2HU; the paragraph "Two levers fell out of this" proposes
// a block-sparse kernel that shares gathered keys across neighbouring queries
// and uses the matrix units).
//
// Per group g (queries QB*g .. QB*g + QB - 1):
//   union    a small kernel marks every selected key of the group's queries in
//            per-query bitmaps over the context and writes the union in
//            ascending key order with a QB-bit membership mask per key;
//   gather   each 128-key tile of the union (512 latent + 64 rope dims per
//            key) into shared memory with cp.async, 128-byte swizzled, as in
//            the per-query kernel;
//   QK^T     S^T[key, (query, head)] = K_tile . Q^T with N = 32 QB columns;
//   softmax  one thread per key lane; the tile maximum of every column, the
//            running maximum and the rescale of O when it grows; a key outside
//            a query's own selection (mask bit clear) gets p = 0 for that
//            query's columns;
//   PV       O^T[dim, (query, head)] += latent_tile^T . P^T.
// One CTA works on one group at a time and its steps run one after another:
// a tile (144 KB) and the group's q rows (36 KB per query) leave no room for
// a second tile, so the gather of a tile waits for the previous tile's PV.
// QB = 1 is the same kernel on single queries, the like-for-like baseline of
// the union. P is written into the tile's rope chunk once QK^T has consumed it.
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "dsa_internal.cuh"
#include "sm100_primitives.cuh"

namespace dsa {
namespace {

using namespace sm100;

// Shared-memory descriptor advanced by a byte offset (start address field, in
// 16-byte units; every operand lies below 256 KB).
__device__ __forceinline__ uint64_t blk_desc_add(uint64_t d, uint32_t bytes) {
  return d + static_cast<uint64_t>(bytes >> 4);
}

constexpr int kBlkThreads = 256;  // warps 0-3 softmax / epilogue, warp 4 MMA, all gather

template <int QB, int H, int DC, int DR>
struct BlkCfg {
  static constexpr int kKeys = 128;
  static constexpr int NQ = QB * H;                 // the group's (query, head) columns
  static constexpr int NH = NQ < 16 ? 16 : NQ;       // MMA N (columns past NQ are padding)
  static constexpr int NL = DC / 64;
  static constexpr int MB = (DC + 127) / 128;       // PV blocks (pairs of 64-dim chunks)
  static constexpr int kChunkBytes = kKeys * 128;   // 64 dims of 128 keys
  static constexpr int kTileChunks = NL + 1;        // latent chunks, then the rope chunk
  static constexpr int kQChunkBytes = NH * 128;
  static constexpr int kQChunks = NL + 1;
  static constexpr int kPRowBytes = NH * 2;
  static constexpr uint32_t kPSwz = NH == 64 ? 2u : (NH == 32 ? 4u : 6u);  // 128 / 64 / 32 B
  static constexpr uint32_t kIdescQK = idesc_bf16_f32(128, NH, false, false);
  static constexpr uint32_t kIdescPV = idesc_bf16_f32(128, NH, true, true);
  static constexpr int kTmemS = 0;
  static constexpr int kTmemO = NH;
  static constexpr int kTmemUsed = NH + MB * NH;
  static constexpr int kTmemCols = kTmemUsed <= 128 ? 128 : kTmemUsed <= 256 ? 256 : 512;
  static constexpr int kOffTile = 0;
  static constexpr int kOffRope = kOffTile + NL * kChunkBytes;   // also P after QK^T
  static constexpr int kOffQ = kOffTile + kTileChunks * kChunkBytes;
  static constexpr int kOffRed = kOffQ + kQChunks * kQChunkBytes;  // [4 warps][NH] floats
  static constexpr int kOffM = kOffRed + 4 * NH * 4;                // running max [NH]
  static constexpr int kOffInv = kOffM + NH * 4;                    // 1 / row sum [NH]
  static constexpr int kOffBar = kOffInv + NH * 4;
  static constexpr int kOffMisc = kOffBar + 4 * 8;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;
  static_assert(NH == 16 || NH == 32 || NH == 64, "group heads");
  static_assert(kKeys * kPRowBytes <= kChunkBytes, "P fits the rope chunk");
  static_assert(kSmemBytes <= 232448, "shared memory");
  static_assert(DC % 128 == 0 || DC == 64, "latent width");
};

struct BlkParams {
  const uint16_t* q;
  const uint16_t* latent;
  const uint16_t* rope;
  const int32_t* ukeys;   // [n_groups, QB * k]: union keys, ascending (count in ucount)
  const uint8_t* umask;   // [n_groups, QB * k]: bit b = key selected by query QB*g + b
  const int32_t* ucount;  // [n_groups]
  uint16_t* out;
  float* lse;
  int n_q, q_pos0, k, n_groups;
  float scale_log2;
  WsHeader* ws;
};

// ------------------------------------------------------------------ union

// One CTA per group: bitmaps of the group's selections, then the union in
// ascending key order with each key's membership mask. Entries < 0 are
// skipped; an entry past its query's position t is reported (DSA_ERR_RANGE)
// and skipped.
template <int QB>
__global__ void block_union_kernel(const int32_t* __restrict__ idx, int n_q, int q_pos0, int k,
                                   int n_words, int32_t* ukeys, uint8_t* umask, int32_t* ucount,
                                   WsHeader* ws) {
  extern __shared__ uint32_t bits[];  // [QB][n_words]
  __shared__ int wsum[kBlkThreads / 32];
  const int g = blockIdx.x;
  for (int e = threadIdx.x; e < QB * n_words; e += blockDim.x) bits[e] = 0u;
  __syncthreads();
  for (int b = 0; b < QB; ++b) {
    const int i = g * QB + b;
    if (i >= n_q) break;
    const int t = q_pos0 + i;
    for (int c = threadIdx.x; c < k; c += blockDim.x) {
      const int s = __ldg(idx + static_cast<int64_t>(i) * k + c);
      if (s < 0) continue;
      if (s > t) {
        report(ws, kDevRange, static_cast<unsigned>(i));
        continue;
      }
      atomicOr(&bits[b * n_words + (s >> 5)], 1u << (s & 31));
    }
  }
  __syncthreads();
  // each thread takes a contiguous run of words; a block scan of the runs'
  // key counts gives every run its output offset
  const int per = (n_words + blockDim.x - 1) / blockDim.x;
  const int w0 = min(static_cast<int>(threadIdx.x) * per, n_words), w1 = min(w0 + per, n_words);
  int cnt = 0;
  for (int w = w0; w < w1; ++w) {
    uint32_t u = 0;
#pragma unroll
    for (int b = 0; b < QB; ++b) u |= bits[b * n_words + w];
    cnt += __popc(u);
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[warp] = x;
  __syncthreads();
  int base = 0, total = 0;
  for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) {
    if (w < warp) base += wsum[w];
    total += wsum[w];
  }
  int pos = base + x - cnt;
  int32_t* uk = ukeys + static_cast<int64_t>(g) * QB * k;
  uint8_t* um = umask + static_cast<int64_t>(g) * QB * k;
  for (int w = w0; w < w1; ++w) {
    uint32_t pl[QB];
    uint32_t u = 0;
#pragma unroll
    for (int b = 0; b < QB; ++b) {
      pl[b] = bits[b * n_words + w];
      u |= pl[b];
    }
    while (u) {
      const int bit = __ffs(u) - 1;
      u &= u - 1;
      uint8_t m = 0;
#pragma unroll
      for (int b = 0; b < QB; ++b) m |= static_cast<uint8_t>(((pl[b] >> bit) & 1u) << b);
      if (DSA_IN_BOUNDS(ws, pos, QB * k, 30)) {
        uk[pos] = w * 32 + bit;
        um[pos] = m;
      }
      ++pos;
    }
  }
  if (threadIdx.x == 0) ucount[g] = total;
}

// ------------------------------------------------------------- attention

// Reduces NV (<= 32) values across a warp; lane l gets value l % NV's result.
template <int NV>
__device__ __forceinline__ float blk_warp_max(float (&v)[NV]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int s = 16; s >= NV; s >>= 1)
#pragma unroll
    for (int e = 0; e < NV; ++e) v[e] = fmaxf(v[e], __shfl_xor_sync(0xffffffffu, v[e], s));
#pragma unroll
  for (int s = NV / 2; s >= 1; s >>= 1) {
    const bool upper = (lane & s) != 0;
#pragma unroll
    for (int e = 0; e < s; ++e) {
      const float send = upper ? v[e] : v[e + s];
      const float keep = upper ? v[e + s] : v[e];
      v[e] = fmaxf(keep, __shfl_xor_sync(0xffffffffu, send, s));
    }
  }
  return v[0];
}

template <int NV>
__device__ __forceinline__ float blk_warp_sum(float (&v)[NV]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int s = 16; s >= NV; s >>= 1)
#pragma unroll
    for (int e = 0; e < NV; ++e) v[e] += __shfl_xor_sync(0xffffffffu, v[e], s);
#pragma unroll
  for (int s = NV / 2; s >= 1; s >>= 1) {
    const bool upper = (lane & s) != 0;
#pragma unroll
    for (int e = 0; e < s; ++e) {
      const float send = upper ? v[e] : v[e + s];
      const float keep = upper ? v[e + s] : v[e];
      v[e] = keep + __shfl_xor_sync(0xffffffffu, send, s);
    }
  }
  return v[0];
}

__device__ __forceinline__ void named_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

template <int NC>
__device__ __forceinline__ void blk_tmem_ld(uint32_t taddr, float (&x)[NC]) {
  uint32_t r[NC];
  if constexpr (NC == 32) tmem_ld_32x32b_x32(taddr, r);
  else if constexpr (NC == 16) tmem_ld_32x32b_x16(taddr, r);
  else tmem_ld_32x32b_x8(taddr, r);
  tmem_ld_wait();
#pragma unroll
  for (int e = 0; e < NC; ++e) x[e] = __uint_as_float(r[e]);
}

template <int NC>
__device__ __forceinline__ void blk_tmem_st(uint32_t taddr, const float (&x)[NC]) {
  uint32_t r[NC];
#pragma unroll
  for (int e = 0; e < NC; ++e) r[e] = __float_as_uint(x[e]);
  if constexpr (NC == 32) tmem_st_32x32b_x32(taddr, r);
  else if constexpr (NC == 16) tmem_st_32x32b_x16(taddr, r);
  else tmem_st_32x32b_x8(taddr, r);
}

template <int QB, int H, int DC, int DR>
__global__ void __launch_bounds__(kBlkThreads, 1)
    block_attn_tc(const __grid_constant__ CUtensorMap tm_q, const BlkParams p) {
  using C = BlkCfg<QB, H, DC, DR>;
  constexpr int NH = C::NH;
  constexpr int CW = NH < 32 ? NH : 32;  // columns per TMEM load
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* sTile = smem + C::kOffTile;
  unsigned char* sRope = smem + C::kOffRope;
  unsigned char* sP = sRope;
  unsigned char* sQ = smem + C::kOffQ;
  float* sRed = reinterpret_cast<float*>(smem + C::kOffRed);
  float* sM = reinterpret_cast<float*>(smem + C::kOffM);
  float* sInv = reinterpret_cast<float*>(smem + C::kOffInv);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  uint64_t* q_full = bars;
  uint64_t* s_full = bars + 1;
  uint64_t* o_step = bars + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  for (int e = threadIdx.x * 16; e < C::kOffRed; e += kBlkThreads * 16)
    *reinterpret_cast<uint4*>(smem + e) = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(s_full, 1);
    mbar_init(o_step, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 4) tmem_alloc(tmem_slot, C::kTmemCols);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const uint64_t dq = smem_desc(smem_u32(sQ), 16, 1024, 2);
  const uint64_t dtile_k = smem_desc(smem_u32(sTile), 16, 1024, 2);
  const uint64_t dtile_mn = smem_desc(smem_u32(sTile), C::kChunkBytes, 1024, 2);
  const uint64_t dp = smem_desc(smem_u32(sP), 8 * C::kPRowBytes, 8 * C::kPRowBytes, C::kPSwz);
  const uint64_t drope = smem_desc(smem_u32(sRope), 16, 1024, 2);

  uint32_t n_q_loads = 0, n_s = 0, n_o = 0;
  bool ok = true;
  for (int g = blockIdx.x; g < p.n_groups && ok; g += gridDim.x) {
    const int n_u = p.ucount[g];
    const int nt = (n_u + 127) / 128;
    const int32_t* uk = p.ukeys + static_cast<int64_t>(g) * QB * p.k;
    const uint8_t* um = p.umask + static_cast<int64_t>(g) * QB * p.k;
    if (threadIdx.x == 0) {
      mbar_arrive_expect_tx(q_full, static_cast<uint32_t>(C::kQChunks * C::kQChunkBytes));
      for (int c = 0; c < C::kQChunks; ++c)
        tma_load_2d(sQ + c * C::kQChunkBytes, &tm_q, c * 64, g * C::NQ, q_full);
    }
    ++n_q_loads;
    // every group's q load is waited for, even a group without keys, so the
    // barrier's phases stay in step
    if (warp == 4) ok = __all_sync(0xffffffffu, mbar_wait(q_full, (n_q_loads - 1) & 1, abort_flag, p.ws, 50));
    ok = __syncthreads_and(ok);
    if (!ok) break;
    // softmax state of this thread's key lane (warps 0-3); heads of column
    // lane and lane + 32 (NH = 64) for the running maxima
    float lpart[NH];
#pragma unroll
    for (int h = 0; h < NH; ++h) lpart[h] = 0.f;
    if (threadIdx.x < NH) sM[threadIdx.x] = -INFINITY;
    for (int j = 0; j < nt && ok; ++j) {
      // ---- gather: thread (w, l) copies 16-byte part l % 8 of keys 4w' + l / 8
      // (w' < 64 over the 256 threads, four rounds of 32 keys)
      const int part = threadIdx.x & 7;
      for (int kr = threadIdx.x >> 3; kr < 128; kr += kBlkThreads / 8) {
        const int sel = j * 128 + kr;
        int row = sel < n_u ? __ldg(uk + sel) : 0;
        if (!DSA_IN_BOUNDS(p.ws, row, p.q_pos0 + p.n_q, 31)) row = 0;
        const uint32_t doff = kr * 128 + ((part ^ (kr & 7)) << 4);
        const uint16_t* lsrc = p.latent + static_cast<int64_t>(row) * DC + part * 8;
#pragma unroll
        for (int c = 0; c < C::NL; ++c) cp_async_16(sTile + c * C::kChunkBytes + doff, lsrc + c * 64);
        if (part < DR / 8) cp_async_16(sRope + doff, p.rope + static_cast<int64_t>(row) * DR + part * 8);
      }
      cp_async_wait_all();
      fence_proxy_async_smem();
      __syncthreads();
      // ---- QK^T (warp 4)
      if (warp == 4) {
        tc_fence_after();
        const uint32_t d_s = tmem_base + C::kTmemS;
#pragma unroll
        for (int ks = 0; ks < DR / 16; ++ks)
          mma_bf16_ss_warp(d_s, blk_desc_add(drope, ks * 32),
                           blk_desc_add(dq, C::NL * C::kQChunkBytes + ks * 32), C::kIdescQK,
                           ks > 0 ? 1u : 0u);
#pragma unroll 1
        for (int c = 0; c < C::NL; ++c)
#pragma unroll
          for (int ks = 0; ks < 4; ++ks)
            mma_bf16_ss_warp(d_s, blk_desc_add(dtile_k, c * C::kChunkBytes + ks * 32),
                             blk_desc_add(dq, c * C::kQChunkBytes + ks * 32), C::kIdescQK, 1u);
        mma_commit_warp(s_full);
      }
      ok = __syncthreads_and(ok);
      if (!ok) break;
      // ---- softmax (warps 0-3): key lane r
      if (warp < 4) {
        ok = __all_sync(0xffffffffu, mbar_wait(s_full, n_s & 1, abort_flag, p.ws, 51));
      }
      ++n_s;
      ok = __syncthreads_and(ok);
      if (!ok) break;
      if (warp < 4) {
        tc_fence_after();
        const int r = warp * 32 + lane;
        const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
        const int sel = j * 128 + r;
        const int row = sel < n_u ? __ldg(uk + sel) : -1;
        const uint32_t mask = sel < n_u ? __ldg(um + sel) : 0u;
        // masked logits (log2 units) of columns c0 .. c0 + CW - 1 of this key
        auto logits = [&](int c0, float (&z)[CW]) {
          float x[CW];
          blk_tmem_ld<CW>(tmem_base + lane_addr + C::kTmemS + c0, x);
#pragma unroll
          for (int e = 0; e < CW; ++e) {
            const int col = c0 + e, qq = col / H;
            const bool valid = row >= 0 && col < C::NQ && ((mask >> qq) & 1u);
            z[e] = valid ? x[e] * p.scale_log2 : -INFINITY;
          }
        };
        // tile maximum of every column over the 128 keys
#pragma unroll 1
        for (int c0 = 0; c0 < NH; c0 += CW) {
          float v[CW];
          logits(c0, v);
          const float wm = blk_warp_max<CW>(v);
          if (lane < CW) sRed[warp * NH + c0 + lane] = wm;
        }
        named_sync(1, 128);
        // new running maxima (thread c < NH owns column c), alpha into sRed[4 * NH ..)
        float* sAlpha = sRed;  // reused after the reduction is read
        float alpha_c = 1.f, m_c = -INFINITY;
        if (threadIdx.x < NH) {
          const int c = threadIdx.x;
          const float tmax = fmaxf(fmaxf(sRed[c], sRed[NH + c]), fmaxf(sRed[2 * NH + c], sRed[3 * NH + c]));
          const float m_old = sM[c];
          m_c = fmaxf(m_old, tmax);
          alpha_c = (m_old == -INFINITY || m_c == -INFINITY) ? (m_old == -INFINITY ? 0.f : 1.f)
                                                             : ex2_approx(m_old - m_c);
        }
        named_sync(1, 128);
        if (threadIdx.x < NH) {
          sM[threadIdx.x] = m_c;
          sAlpha[threadIdx.x] = alpha_c;
        }
        named_sync(1, 128);
        // rescale the row sums and (after the previous PV) O^T
        bool any_rescale = false;
#pragma unroll
        for (int h = 0; h < NH; ++h) {
          const float a = sAlpha[h];
          lpart[h] *= a;
          any_rescale |= a != 1.f;
        }
        if (j > 0 && any_rescale) {
#pragma unroll 1
          for (int mb = 0; mb < C::MB; ++mb) {
#pragma unroll
            for (int c0 = 0; c0 < NH; c0 += CW) {
              const uint32_t ta = tmem_base + lane_addr + C::kTmemO + mb * NH + c0;
              float o[CW];
              blk_tmem_ld<CW>(ta, o);
#pragma unroll
              for (int e = 0; e < CW; ++e) o[e] *= sAlpha[c0 + e];
              blk_tmem_st<CW>(ta, o);
            }
          }
          tmem_st_wait();
        }
        // P: this key's row of NH bf16, 16-byte chunks of eight columns at
        // their swizzled positions
        unsigned char* prow = sP + r * C::kPRowBytes;
#pragma unroll
        for (int c0 = 0; c0 < NH; c0 += CW) {
          float z[CW];
          logits(c0, z);
#pragma unroll
          for (int c8 = 0; c8 < CW / 8; ++c8) {
            uint32_t w4[4];
#pragma unroll
            for (int e2 = 0; e2 < 4; ++e2) {
              float pv[2];
#pragma unroll
              for (int e = 0; e < 2; ++e) {
                const int ce = 8 * c8 + 2 * e2 + e, col = c0 + ce;
                const float m = sM[col];
                pv[e] = (z[ce] > -INFINITY && m > -INFINITY) ? ex2_approx(z[ce] - m) : 0.f;
                lpart[col] += pv[e];
              }
              const __nv_bfloat162 b2 = __floats2bfloat162_rn(pv[0], pv[1]);
              w4[e2] = *reinterpret_cast<const uint32_t*>(&b2);
            }
            const int ch = c0 / 8 + c8;  // 16-byte chunk of the row
            int swz;
            if constexpr (NH == 64) swz = ch ^ (r & 7);
            else if constexpr (NH == 32) swz = ch ^ ((r >> 1) & 3);
            else swz = ch ^ ((r >> 2) & 1);
            *reinterpret_cast<uint4*>(prow + (swz << 4)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
      }
      __syncthreads();
      // ---- PV (warp 4)
      if (warp == 4) {
        tc_fence_after();
#pragma unroll
        for (int mb = 0; mb < C::MB; ++mb)
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_bf16_ss_warp(tmem_base + C::kTmemO + mb * NH,
                             blk_desc_add(dtile_mn, mb * 2 * C::kChunkBytes + kk * 2048),
                             blk_desc_add(dp, kk * 16 * C::kPRowBytes), C::kIdescPV,
                             (j == 0 && kk == 0) ? 0u : 1u);
        mma_commit_warp(o_step);
        ok = __all_sync(0xffffffffu, mbar_wait(o_step, n_o & 1, abort_flag, p.ws, 52));
      }
      ++n_o;
      ok = __syncthreads_and(ok);
    }
    if (!ok) break;
    // ---- epilogue (warps 0-3): row sums, O^T / l, lse
    if (warp < 4) {
      tc_fence_after();
#pragma unroll
      for (int c0 = 0; c0 < NH; c0 += CW) {
        float v[CW];
#pragma unroll
        for (int e = 0; e < CW; ++e) v[e] = lpart[c0 + e];
        const float ws_ = blk_warp_sum<CW>(v);
        if (lane < CW) sRed[warp * NH + c0 + lane] = ws_;
      }
      named_sync(1, 128);
      const int r = warp * 32 + lane;
      const uint32_t lane_addr = static_cast<uint32_t>(warp * 32) << 16;
      if (threadIdx.x < NH) {
        const int c = threadIdx.x, qq = c / H, h = c % H;
        const int i = g * QB + qq;
        const float l = sRed[c] + sRed[NH + c] + sRed[2 * NH + c] + sRed[3 * NH + c];
        if (c < C::NQ && i < p.n_q && p.lse)
          p.lse[static_cast<int64_t>(i) * H + h] =
              l > 0.f ? (sM[c] + log2f(l)) * 0.6931471805599453f : -INFINITY;
        sInv[c] = l > 0.f ? 1.f / l : 0.f;
      }
      named_sync(1, 128);
#pragma unroll 1
      for (int mb = 0; mb < C::MB; ++mb) {
#pragma unroll
        for (int c0 = 0; c0 < NH; c0 += CW) {
          float o[CW];
          blk_tmem_ld<CW>(tmem_base + lane_addr + C::kTmemO + mb * NH + c0, o);
          const int d = mb * 128 + r;
#pragma unroll
          for (int e = 0; e < CW; ++e) {
            const int c = c0 + e, qq = c / H, h = c % H;
            const int i = g * QB + qq;
            // a column without a valid key (or a group without tiles) never
            // had O written: its output is 0
            if (d < DC && c < C::NQ && i < p.n_q)
              p.out[(static_cast<int64_t>(i) * H + h) * DC + d] =
                  sInv[c] > 0.f && nt > 0 ? f32_to_bf16_rne(o[e] * sInv[c]) : 0;
          }
        }
      }
      tc_fence_before();
    }
    __syncthreads();
  }
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

int blk_num_sms() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

template <int QB, int H, int DC, int DR>
cudaError_t launch_block(const dsa_dims& d, const uint16_t* q, const uint16_t* latent,
                         const uint16_t* rope, const int32_t* idx, uint16_t* out, float* lse,
                         WsHeader* ws, void* scratch, cudaStream_t st) {
  using C = BlkCfg<QB, H, DC, DR>;
  const int n_groups = (d.n_q + QB - 1) / QB;
  int32_t* ukeys = static_cast<int32_t*>(scratch);
  uint8_t* umask = reinterpret_cast<uint8_t*>(ukeys + static_cast<int64_t>(n_groups) * QB * d.top_k);
  int32_t* ucount = reinterpret_cast<int32_t*>(
      (reinterpret_cast<uintptr_t>(umask + static_cast<int64_t>(n_groups) * QB * d.top_k) + 15) &
      ~static_cast<uintptr_t>(15));
  const int n_words = (d.q_pos0 + d.n_q + 31) / 32;
  block_union_kernel<QB><<<n_groups, kBlkThreads, QB * n_words * 4, st>>>(
      idx, d.n_q, d.q_pos0, d.top_k, n_words, ukeys, umask, ucount, ws);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  BlkParams p;
  p.q = q;
  p.latent = latent;
  p.rope = rope;
  p.ukeys = ukeys;
  p.umask = umask;
  p.ucount = ucount;
  p.out = out;
  p.lse = lse;
  p.n_q = d.n_q;
  p.q_pos0 = d.q_pos0;
  p.k = d.top_k;
  p.n_groups = n_groups;
  p.scale_log2 = d.softmax_scale * 1.4426950408889634f;
  p.ws = ws;
  CUtensorMap tm_q;
  if (!make_tmap_bf16_2d(&tm_q, q, DC + DR, static_cast<uint64_t>(d.n_q) * H, 64, C::NH,
                         CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  const int grid = n_groups < blk_num_sms() ? n_groups : blk_num_sms();
  const int smem = C::kSmemBytes > 120 * 1024 ? C::kSmemBytes : 120 * 1024;
  e = cudaFuncSetAttribute(block_attn_tc<QB, H, DC, DR>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           smem);
  if (e != cudaSuccess) return e;
  block_attn_tc<QB, H, DC, DR><<<grid, kBlkThreads, smem, st>>>(tm_q, p);
  return cudaGetLastError();
}

}  // namespace

size_t block_attn_scratch_bytes(const dsa_dims& d, int qb) {
  const size_t n_groups = (static_cast<size_t>(d.n_q) + qb - 1) / qb;
  const size_t lists = n_groups * qb * d.top_k;
  return (lists * 4 + lists + 15) / 16 * 16 + n_groups * 4;
}

cudaError_t launch_block_attn(const dsa_dims& d, const uint16_t* q, const uint16_t* latent,
                              const uint16_t* rope, const int32_t* idx, uint16_t* out, float* lse,
                              int qb, WsHeader* ws, void* scratch, cudaStream_t st) {
  if (d.n_heads == 32 && d.d_latent == 512 && d.d_rope == 64) {
    if (qb == 1) return launch_block<1, 32, 512, 64>(d, q, latent, rope, idx, out, lse, ws, scratch, st);
    if (qb == 2) return launch_block<2, 32, 512, 64>(d, q, latent, rope, idx, out, lse, ws, scratch, st);
  }
  if (d.n_heads == 4 && d.d_latent == 64 && d.d_rope == 16) {
    if (qb == 1) return launch_block<1, 4, 64, 16>(d, q, latent, rope, idx, out, lse, ws, scratch, st);
    if (qb == 2) return launch_block<2, 4, 64, 16>(d, q, latent, rope, idx, out, lse, ws, scratch, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace dsa
