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
//   gather   the tile's rope chunk and its latent rows, as 128-dim pairs of
//            64-dim chunks (one 32 KB pair per PV output block), into
//            shared memory with cp.async: one key per 128-byte row, 128-byte
//            swizzled, eight threads per row so every request is a full
//            128-byte line. Pairs form a ring one pair deeper than a tile, so
//            the next tile's rope and first pair arrive during the softmax;
//   QK^T     S^T[key, head] = K_tile . Q^T: keys are the MMA's M (128), the
//            padded heads its N, K = Dc + Dr, both operands K-major;
//   softmax  one thread per key lane of S^T, p = 2^(z log2e - m) written as
//            bf16 into P [key, head] (one 16-byte-chunked row per key). The
//            reference m is a running maximum. On a query's first tile it is
//            the tile maximum (a warp transpose-reduction plus a four-warp
//            exchange through shared memory, mbarrier-synchronised). Every
//            score of head h is at most B_h = |scale| log2e ||q_h|| max_s ||k_s||
//            (Cauchy-Schwarz), so while B_h <= m_h + 64 for every head, p stays
//            below 2^64 and no later tile can overflow fp32 or bf16: such
//            tiles keep m as it is and skip the reduction and the exchange.
//            Otherwise a tile takes the exact path, and m is raised only when
//            the tile maximum exceeds it by more than 2^8 (then O is rescaled
//            in TMEM). max_s ||k_s|| comes from a small pass over the keys
//            before the attention kernel, ||q_h|| from the q rows in shared
//            memory on the first tile;
//   PV       O^T[dim, head] += latent_tile^T . P^T: the latent pairs read
//            MN-major as A (dims as M, one 128-dim block per pair), P MN-major
//            as B. Each pair is released the moment its block's MMAs finish,
//            so the next tile's gather runs under the current PV.
// The MMA issuer orders its work as QK^T(t) on the rope and first pair,
// PV(t-1), then QK^T(t) on the rest, so the tensor pipe works while the
// gather of tile t completes. Accumulators live in TMEM (S^T double-buffered
// per tile, O^T per query); the epilogue divides by the row sum, rounds to
// bf16 and writes out / lse.
//
// Roles (416 threads, one CTA per SM, persistent over queries):
//   warps 0-3  producers: cp.async gathers of every tile;
//   warp  4    TMEM owner and tcgen05.mma issuer (warp-collective, one
//              elected lane issues);
//   warps 5-12 softmax and epilogue, two warps per TMEM lane quarter (lanes
//              = keys, then dims), each on half of the heads; every softmax
//              warp tracks the running maxima of all heads, so the decisions
//              that need all of them are made alike without exchange. One
//              lane also loads each query's q rows with 2D TMA once the
//              previous query's last QK^T has completed.
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
  static constexpr int MB = (DC + 127) / 128;         // 128-dim PV blocks = latent pairs per tile
  static constexpr int kRopeSteps = DR / 16;
  static constexpr int kChunkBytes = kKeys * 128;     // 16 KB: 64 dims of 128 keys
  static constexpr int kPairBytes = 2 * kChunkBytes;  // one PV block (upper half zero if DC < 128)
  static constexpr int kPairs = MB + 1 > 3 ? MB + 1 : 3;  // ring: one tile plus one pair
  static constexpr int kQChunks = NL + 1;             // latent chunks + rope chunk
  static constexpr int kQChunkBytes = NH * 128;
  // P: one row of NH bf16 per key (MN-major B operand of the PV), 64- or
  // 32-byte rows swizzled in 8-row atoms
  static constexpr int kPRowBytes = NH * 2;
  static constexpr int kPBytes = kKeys * kPRowBytes;
  static constexpr uint32_t kPSwz = NH == 32 ? 4u : 6u;  // descriptor code: 64B / 32B swizzle
  static constexpr int kProducerThreads = 128;        // warps 0-3
  static constexpr int kSoftmaxWarps = 8;            // two per TMEM lane quarter, half the heads each
  static constexpr int HH = NH / 2;                   // heads per softmax warp
  static constexpr int kSoftmaxThreads = 32 * kSoftmaxWarps;
  static constexpr int kThreads = 32 * (5 + kSoftmaxWarps);
  static constexpr int kRowsPerThread = kKeys / 16;   // keys 32w + lane/8 + 4i, i < 8
  static constexpr uint32_t kQBytes = H * 128 * kQChunks;  // q boxes (zero-filled past Dc+Dr)
  static constexpr uint32_t kIdescQK = idesc_bf16_f32(128, NH, false, false);
  static constexpr uint32_t kIdescPV = idesc_bf16_f32(128, NH, true, true);
  // TMEM columns: S^T[2] then O^T[2 queries][MB]
  static constexpr int kTmemS = 0;
  static constexpr int kTmemO = 2 * NH;
  static constexpr int kTmemUsed = 2 * NH + 2 * MB * NH;
  static constexpr int kTmemCols = kTmemUsed <= 32 ? 32 : kTmemUsed <= 64 ? 64 : kTmemUsed <= 128 ? 128
                                   : kTmemUsed <= 256 ? 256 : 512;
  // shared memory carve (from a 1024-byte aligned base)
  static constexpr int kOffPairs = 0;
  static constexpr int kOffRope = kOffPairs + kPairs * kPairBytes;
  static constexpr int kOffQ = kOffRope + kChunkBytes;
  static constexpr int kOffP = kOffQ + kQChunks * kQChunkBytes;
  static constexpr int kOffRed = kOffP + kPBytes;                // [2][8 warps][16] floats
  static constexpr int kOffNorm = kOffRed + 2 * 8 * 16 * 4;      // [8 warps][32] floats
  static constexpr int kOffM = kOffNorm + 8 * 32 * 4;            // [8 warps][32] floats
  static constexpr int kOffBar = kOffM + 8 * 32 * 4;
  static constexpr int kNumBars = 3 * kPairs + 17;
  static constexpr int kOffMisc = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffMisc + 16 + 1024;
  static_assert(DC % 64 == 0 && DR % 16 == 0 && DR <= 64 && (NH % 16) == 0 && NH <= 32 &&
                    (H & (H - 1)) == 0,
                "shape");
  static_assert(kOffQ % 1024 == 0 && kOffP % 1024 == 0, "operand alignment");
  static_assert(kSmemBytes <= 232448, "shared memory");
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
  // Work items: item w is query w / n_split and the key tiles [j * tps,
  // (j + 1) * tps) of its selection, j = w % n_split. n_split = 1 (one item
  // per query) writes out / lse directly; n_split > 1 (decode: few queries,
  // their tiles spread over SMs) writes each item's unnormalised partial O,
  // running maximum (log2 units) and row sum to part_o / part_ml for the
  // combine pass.
  int n_split, tps, n_items;
  float* part_o;   // [n_items, H, DC]
  float2* part_ml; // [n_items, H]: (m, l)
};

__device__ __forceinline__ int n_valid_of(const AttnParams& p, int i) {
  return p.prefix_valid ? min(p.k, p.q_pos0 + i + 1) : p.k;
}

__device__ __forceinline__ int n_tiles_of(const AttnParams& p, int i) {
  return (n_valid_of(p, i) + 127) / 128;
}

// Selected key `sel` of query i, or -1 past the query's selection.
__device__ __forceinline__ int selected_row(const AttnParams& p, int i, int sel) {
  return sel < n_valid_of(p, i) ? __ldg(p.idx + static_cast<int64_t>(i) * p.k + sel) : -1;
}

// Query and key-tile range [t0, t1) of item w.
__device__ __forceinline__ void item_range(const AttnParams& p, int w, int& i, int& t0, int& t1) {
  i = w / p.n_split;
  t0 = (w - i * p.n_split) * p.tps;
  t1 = min(n_tiles_of(p, i), t0 + p.tps);
}

// This CTA's first item at or after w (w, w + grid, ...) with at least one
// key tile, or n_items. Every role walks the same sequence.
__device__ __forceinline__ int next_item(const AttnParams& p, int w) {
  for (; w < p.n_items; w += gridDim.x) {
    int i, t0, t1;
    item_range(p, w, i, t0, t1);
    if (t0 < t1) return w;
  }
  return p.n_items;
}

// The tile after tile j of item w (query i, tiles up to t1): (i, j + 1), or
// the first tile of this CTA's next item; ni = -1 when there is none.
__device__ __forceinline__ void tile_after(const AttnParams& p, int w, int i, int j, int t1, int& ni,
                                           int& nj) {
  if (j + 1 < t1) {
    ni = i;
    nj = j + 1;
    return;
  }
  const int nw = next_item(p, w + static_cast<int>(gridDim.x));
  ni = -1;
  nj = 0;
  if (nw < p.n_items) {
    int e1;
    item_range(p, nw, ni, nj, e1);
  }
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

// A warp's 32 TMEM lanes x NC consecutive 32-bit columns (NC = 8, 16 or 32).
template <int NC>
__device__ __forceinline__ void tmem_ld_row(uint32_t taddr, float (&x)[NC]) {
  uint32_t r[NC];
  if constexpr (NC == 32) tmem_ld_32x32b_x32(taddr, r);
  else if constexpr (NC == 16) tmem_ld_32x32b_x16(taddr, r);
  else tmem_ld_32x32b_x8(taddr, r);
  tmem_ld_wait();
#pragma unroll
  for (int e = 0; e < NC; ++e) x[e] = __uint_as_float(r[e]);
}

template <int NC>
__device__ __forceinline__ void tmem_st_row(uint32_t taddr, const float (&x)[NC]) {
  uint32_t r[NC];
#pragma unroll
  for (int e = 0; e < NC; ++e) r[e] = __float_as_uint(x[e]);
  if constexpr (NC == 32) tmem_st_32x32b_x32(taddr, r);
  else if constexpr (NC == 16) tmem_st_32x32b_x16(taddr, r);
  else tmem_st_32x32b_x8(taddr, r);
}

// Shared-memory descriptor advanced by a byte offset (the start address is
// the low field, in 16-byte units; every operand lies below 256 KB).
__device__ __forceinline__ uint64_t desc_add(uint64_t d, uint32_t bytes) {
  return d + static_cast<uint64_t>(bytes >> 4);
}

// mbarrier layout (all in shared memory, after the operand buffers)
template <class C>
struct AttnBars {
  static constexpr int kPairFull = 0;                  // [kPairs][2] (one per 64-dim chunk)
  static constexpr int kPairEmpty = 2 * C::kPairs;     // [kPairs]
  static constexpr int kRopeFull = 3 * C::kPairs;
  static constexpr int kRopeEmpty = kRopeFull + 1;
  static constexpr int kQFull = kRopeEmpty + 1;
  static constexpr int kSFull = kQFull + 1;            // [2]
  static constexpr int kSEmpty = kSFull + 2;           // [2]
  static constexpr int kPFull = kSEmpty + 2;
  static constexpr int kPEmpty = kPFull + 1;
  static constexpr int kOFull = kPEmpty + 1;           // [2]
  static constexpr int kOEmpty = kOFull + 2;           // [2]
  static constexpr int kOStep = kOEmpty + 2;
  static constexpr int kExch = kOStep + 1;             // [2]
  static constexpr int kMmaDone = kExch + 2;
  static constexpr int kCount = kMmaDone + 1;
  static_assert(kCount == C::kNumBars, "barrier count");
};

// A wait by every lane of a warp, with one outcome for the whole warp.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          WsHeader* ws, unsigned site) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, ws, site));
}

// QK^T on latent pair mb of tile tc, each chunk as soon as it lands
// (warp-collective).
template <class C>
__device__ __forceinline__ bool attn_qk_pair(const AttnParams& p, volatile int* abort_flag, uint64_t* bars,
                                             uint64_t dpair_k, uint64_t dq, uint32_t tc, int mb,
                                             uint32_t d_s) {
  using B = AttnBars<C>;
  const uint32_t seq = C::MB * tc + mb;
  const uint32_t pi = seq % C::kPairs;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int c = 2 * mb + half;
    if (c >= C::NL) break;
    if (!warp_wait(&bars[B::kPairFull + 2 * pi + half], (seq / C::kPairs) & 1, abort_flag, p.ws, 33))
      return false;
    fence_proxy_async_smem();
    tc_fence_after();
    const uint64_t a = desc_add(dpair_k, pi * C::kPairBytes + half * C::kChunkBytes);
    const uint64_t b = desc_add(dq, c * C::kQChunkBytes);
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
      mma_bf16_ss_warp(d_s, desc_add(a, ks * 32), desc_add(b, ks * 32), C::kIdescQK, 1u);
  }
  return true;
}

// O^T += latent_tile^T . P^T for tile tc of the qi-th query of this CTA,
// releasing each latent pair as its block's MMAs complete (warp-collective).
template <class C>
__device__ __forceinline__ bool attn_pv(const AttnParams& p, volatile int* abort_flag, uint64_t* bars,
                                        uint32_t tmem_base, uint64_t dpair_mn, uint64_t dp, uint32_t tc,
                                        uint32_t qi, bool first, bool last) {
  using B = AttnBars<C>;
  constexpr int NH = C::NH;
  if (!warp_wait(&bars[B::kPFull], tc & 1, abort_flag, p.ws, 34)) return false;
  if (first && !warp_wait(&bars[B::kOEmpty + (qi & 1)], ((qi >> 1) & 1) ^ 1, abort_flag, p.ws, 35))
    return false;
  tc_fence_after();
  const uint32_t d_o = tmem_base + C::kTmemO + (qi & 1) * C::MB * NH;
#pragma unroll
  for (int mb = 0; mb < C::MB; ++mb) {
    const uint32_t pi = (C::MB * tc + mb) % C::kPairs;
    const uint64_t a = desc_add(dpair_mn, pi * C::kPairBytes);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
      mma_bf16_ss_warp(d_o + mb * NH, desc_add(a, kk * 2048), desc_add(dp, kk * 16 * C::kPRowBytes),
                       C::kIdescPV, (first && kk == 0) ? 0u : 1u);
    mma_commit_warp(&bars[B::kPairEmpty + pi]);
  }
  mma_commit_warp(&bars[B::kPEmpty]);
  mma_commit_warp(&bars[B::kOStep]);
  if (last) mma_commit_warp(&bars[B::kOFull + (qi & 1)]);
  return true;
}

template <int H, int DC, int DR>
__global__ void __launch_bounds__(AttnCfg<H, DC, DR>::kThreads, 1)
    sparse_attn_tc(const __grid_constant__ CUtensorMap tm_q, const AttnParams p) {
  using C = AttnCfg<H, DC, DR>;
  constexpr int NH = C::NH;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* sPairs = smem + C::kOffPairs;
  unsigned char* sRope = smem + C::kOffRope;
  unsigned char* sQ = smem + C::kOffQ;
  unsigned char* sP = smem + C::kOffP;
  float* sRed = reinterpret_cast<float*>(smem + C::kOffRed);
  float* sNorm = reinterpret_cast<float*>(smem + C::kOffNorm);
  float* sM = reinterpret_cast<float*>(smem + C::kOffM);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kOffBar);
  using B = AttnBars<C>;
  uint64_t* pair_full = bars + B::kPairFull;
  uint64_t* pair_empty = bars + B::kPairEmpty;
  uint64_t* rope_full = bars + B::kRopeFull;
  uint64_t* rope_empty = bars + B::kRopeEmpty;
  uint64_t* q_full = bars + B::kQFull;
  uint64_t* s_full = bars + B::kSFull;
  uint64_t* s_empty = bars + B::kSEmpty;
  uint64_t* p_full = bars + B::kPFull;
  uint64_t* p_empty = bars + B::kPEmpty;
  uint64_t* o_full = bars + B::kOFull;
  uint64_t* o_empty = bars + B::kOEmpty;
  uint64_t* o_step = bars + B::kOStep;
  uint64_t* exch = bars + B::kExch;
  uint64_t* mma_done = bars + B::kMmaDone;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::kOffMisc + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // zero every operand buffer once: padded heads, the upper half of a pair
  // when Dc < 128 and the unused part of a narrow rope chunk read as zeros
  for (int e = threadIdx.x * 16; e < C::kOffRed; e += C::kThreads * 16)
    *reinterpret_cast<uint4*>(smem + e) = make_uint4(0u, 0u, 0u, 0u);
  fence_proxy_async_smem();
  if (threadIdx.x == 0) {
    for (int s = 0; s < 2 * C::kPairs; ++s) mbar_init(&pair_full[s], C::kProducerThreads);
    for (int s = 0; s < C::kPairs; ++s) mbar_init(&pair_empty[s], 1);
    mbar_init(rope_full, C::kProducerThreads);
    mbar_init(rope_empty, 1);
    mbar_init(q_full, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_empty[b], C::kSoftmaxThreads);
      mbar_init(&o_full[b], 1);
      mbar_init(&o_empty[b], C::kSoftmaxThreads);
      mbar_init(&exch[b], C::kSoftmaxThreads);
    }
    mbar_init(p_full, C::kSoftmaxThreads);
    mbar_init(p_empty, 1);
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
    // Thread (warp w, lane l) copies 16-byte part l%8 of keys 32w + l/8 + 4i
    // (i < 8) of every chunk: each warp-wide cp.async moves four full
    // 128-byte rows. A chunk's mbarrier completes on the noinc arrivals of all
    // 128 producer threads. Row indices of the next tile are loaded while the
    // current tile's copies are issued.
    constexpr int R = C::kRowsPerThread;
    const int kbase = 32 * warp + (lane >> 3);
    const int part = lane & 7;
    uint32_t doff[R];  // swizzled destination of each key's part in a chunk
#pragma unroll
    for (int e = 0; e < R; ++e) {
      const int key = kbase + 4 * e;
      doff[e] = key * 128 + ((part ^ (key & 7)) << 4);
    }
    int cur[R], nxt[R];
    const int w0 = next_item(p, blockIdx.x);
    if (w0 < p.n_items) {
      int i0, a0, b0;
      item_range(p, w0, i0, a0, b0);
#pragma unroll
      for (int e = 0; e < R; ++e) cur[e] = selected_row(p, i0, a0 * 128 + kbase + 4 * e);
    }
    uint32_t tc = 0;
    bool ok = true;
    for (int w = w0; w < p.n_items && ok; w = next_item(p, w + gridDim.x)) {
      int i, t0, t1;
      item_range(p, w, i, t0, t1);
      for (int j = t0; j < t1 && ok; ++j, ++tc) {
        int ni, nj;
        tile_after(p, w, i, j, t1, ni, nj);
        if (ni >= 0) {
#pragma unroll
          for (int e = 0; e < R; ++e) nxt[e] = selected_row(p, ni, nj * 128 + kbase + 4 * e);
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
          if (!DSA_IN_BOUNDS(p.ws, row, p.ctx_len, 13)) row = 0;
          lsrc[e] = p.latent + static_cast<int64_t>(row) * DC + part * 8;
          rsrc[e] = p.rope + static_cast<int64_t>(row) * DR + part * 8;
        }
        ok = __all_sync(0xffffffffu, mbar_wait(rope_empty, (tc & 1) ^ 1, abort_flag, p.ws, 20));
        if (!ok) break;
        if (part < DR / 8) {
#pragma unroll
          for (int e = 0; e < R; ++e)
            if (DSA_IN_BOUNDS(p.ws, doff[e] + 16, C::kChunkBytes + 1, 10)) cp_async_16(sRope + doff[e], rsrc[e]);
        }
        cp_async_arrive_noinc(rope_full);
#pragma unroll
        for (int mb = 0; mb < C::MB; ++mb) {
          const uint32_t seq = C::MB * tc + mb;
          const uint32_t pi = seq % C::kPairs;
          ok = __all_sync(0xffffffffu, mbar_wait(&pair_empty[pi], ((seq / C::kPairs) & 1) ^ 1,
                                                 abort_flag, p.ws, 21));
          if (!ok) break;
          unsigned char* dst = sPairs + pi * C::kPairBytes;
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            const int c = 2 * mb + half;
            if (c < C::NL) {
#pragma unroll
              for (int e = 0; e < R; ++e)
                if (DSA_IN_BOUNDS(p.ws, pi * C::kPairBytes + half * C::kChunkBytes + doff[e] + 16,
                                  C::kPairs * C::kPairBytes + 1, 14))
                  cp_async_16(dst + half * C::kChunkBytes + doff[e], lsrc[e] + c * 64);
              cp_async_arrive_noinc(&pair_full[2 * pi + half]);
            }
          }
        }
#pragma unroll
        for (int e = 0; e < R; ++e) cur[e] = nxt[e];
      }
    }
    cp_async_wait_all();  // every copy lands before the CTA can exit
  } else if (warp == 4) {
    // ------------------------------------------------------------ MMA issuer
    const uint64_t dq = smem_desc(smem_u32(sQ), 16, 1024, 2);
    const uint64_t drope = smem_desc(smem_u32(sRope), 16, 1024, 2);
    const uint64_t dpair_k = smem_desc(smem_u32(sPairs), 16, 1024, 2);
    const uint64_t dpair_mn = smem_desc(smem_u32(sPairs), C::kChunkBytes, 1024, 2);
    const uint64_t dp = smem_desc(smem_u32(sP), 8 * C::kPRowBytes, 8 * C::kPRowBytes, C::kPSwz);
    // the PV of a finished tile (pend_*), issued once the next tile's first
    // chunks are in
    bool pend = false, pend_first = false, pend_last = false;
    uint32_t pend_tc = 0, pend_qi = 0;
    uint32_t tc = 0, qi = 0;
    bool ok = true;
    for (int w = next_item(p, blockIdx.x); w < p.n_items && ok; w = next_item(p, w + gridDim.x), ++qi) {
      int i, t0, t1;
      item_range(p, w, i, t0, t1);
      for (int j = t0; j < t1; ++j, ++tc) {
        const int sb = tc & 1;
        const uint32_t d_s = tmem_base + C::kTmemS + sb * NH;
        if (j == t0) {
          // a new query: the previous query's last PV goes first, then q
          if (pend && !(ok = attn_pv<C>(p, abort_flag, bars, tmem_base, dpair_mn, dp, pend_tc, pend_qi,
                                        pend_first, pend_last)))
            break;
          pend = false;
          if (!(ok = warp_wait(q_full, qi & 1, abort_flag, p.ws, 30))) break;
          tc_fence_after();
        }
        if (!(ok = warp_wait(&s_empty[sb], ((tc >> 1) & 1) ^ 1, abort_flag, p.ws, 31))) break;
        if (!(ok = warp_wait(rope_full, tc & 1, abort_flag, p.ws, 32))) break;
        fence_proxy_async_smem();
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < C::kRopeSteps; ++ks)
          mma_bf16_ss_warp(d_s, desc_add(drope, ks * 32), desc_add(dq, C::NL * C::kQChunkBytes + ks * 32),
                           C::kIdescQK, ks > 0 ? 1u : 0u);
        mma_commit_warp(rope_empty);
        if (!(ok = attn_qk_pair<C>(p, abort_flag, bars, dpair_k, dq, tc, 0, d_s))) break;
        if (pend && !(ok = attn_pv<C>(p, abort_flag, bars, tmem_base, dpair_mn, dp, pend_tc, pend_qi,
                                      pend_first, pend_last)))
          break;
        pend = false;
        for (int mb = 1; mb < C::MB && ok; ++mb)
          ok = attn_qk_pair<C>(p, abort_flag, bars, dpair_k, dq, tc, mb, d_s);
        if (!ok) break;
        mma_commit_warp(&s_full[sb]);
        pend = true;
        pend_tc = tc;
        pend_qi = qi;
        pend_first = j == t0;
        pend_last = j == t1 - 1;
      }
    }
    if (ok && pend)
      ok = attn_pv<C>(p, abort_flag, bars, tmem_base, dpair_mn, dp, pend_tc, pend_qi, pend_first, pend_last);
    mma_commit_warp(mma_done);
    drain_wait(mma_done, 0);
  } else {
    // ------------------------------------------------- softmax and epilogue
    constexpr int HH = C::HH;
    const int quarter = warp & 3;               // TMEM lane quarter of this warp
    const int r = quarter * 32 + lane;          // key lane (and dim lane in the epilogue)
    const int sw = warp - 5;                    // softmax warp index 0..7
    const int hh = sw >> 2;                     // this warp's heads: hh*HH .. hh*HH+HH-1
    const uint32_t lane_addr = static_cast<uint32_t>(quarter * 32) << 16;
    const bool q_loader = warp == 5 && lane == 0;
    int q_loads = 0;
    const int w_first = next_item(p, blockIdx.x);
    int row_next = -1;
    if (w_first < p.n_items) {
      int i0, a0, b0;
      item_range(p, w_first, i0, a0, b0);
      row_next = selected_row(p, i0, a0 * 128 + r);
      if (q_loader) {
        prefetch_tmap(&tm_q);
        mbar_arrive_expect_tx(q_full, C::kQBytes);
        for (int c = 0; c < C::kQChunks; ++c)
          tma_load_2d(sQ + c * C::kQChunkBytes, &tm_q, c * 64, i0 * H, q_full);
        q_loads = 1;
      }
    }
    uint32_t tc = 0, qi = 0, xc = 0;
    bool ok = true;
    // max_s ||k_s|| of the context, with the rounding slack of its float32 sum
    const float kmax = __uint_as_float(*reinterpret_cast<volatile unsigned int*>(&p.ws->akmax_bits));
    const float bound_scale = fabsf(p.scale_log2) * kmax;
    // the exchange slot of head h (lane) from the warp of quarter-rank qq of
    // h's half: warps hh*4 .. hh*4+3 hold the halves' partial values
    const int xslot = (lane / HH) * 4 * 16 + (lane % HH);
    for (int w = w_first; w < p.n_items && ok; w = next_item(p, w + gridDim.x), ++qi) {
      int i, t0, t1;
      item_range(p, w, i, t0, t1);
      const int ob = qi & 1;
      const int w_next = next_item(p, w + gridDim.x);
      const bool next_q = w_next < p.n_items;
      float m_lane = -INFINITY;       // running max (log2 units) of head `lane` (all heads)
      float bound_lane = INFINITY;    // B_lane: bound on every score of head `lane`
      bool fixed_m = false;           // B_h <= m_h + 64 for every head: keep m as it is
      float* mrep = sM + sw * 32;     // running max of every head (this warp's copy)
      float lpart[HH];                // this key lane's share of the row sums of its heads
      mrep[lane] = -INFINITY;
      __syncwarp();
#pragma unroll
      for (int h = 0; h < HH; ++h) lpart[h] = 0.f;
      for (int j = t0; j < t1; ++j, ++tc) {
        const int sb = tc & 1;
        const int row = row_next;
        {
          int ni, nj;
          tile_after(p, w, i, j, t1, ni, nj);
          row_next = ni >= 0 ? selected_row(p, ni, nj * 128 + r) : -1;
        }
        ok = __all_sync(0xffffffffu, mbar_wait(&s_full[sb], (tc >> 1) & 1, abort_flag, p.ws, 40));
        if (!ok) break;
        tc_fence_after();
        float x[HH];
        tmem_ld_row<HH>(tmem_base + lane_addr + C::kTmemS + sb * NH + hh * HH, x);
        tc_fence_before();
        mbar_arrive(&s_empty[sb]);
        if (j == t0) {
          // this warp's share of ||q_h||^2 for every head (q chunks sw, sw+8;
          // lane = head), reading a row's 16-byte units in a lane-rotated order
          ok = __all_sync(0xffffffffu, mbar_wait(q_full, qi & 1, abort_flag, p.ws, 46));
          if (!ok) break;
          float qn2 = 0.f;
          if (lane < NH) {
            for (int c = sw; c < C::kQChunks; c += C::kSoftmaxWarps) {
              const unsigned char* qrow = sQ + c * C::kQChunkBytes + lane * 128;
#pragma unroll
              for (int u = 0; u < 8; ++u) {
                const uint4 v = *reinterpret_cast<const uint4*>(qrow + (((u + lane) & 7) << 4));
                const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                  const float a = __uint_as_float(w[e] << 16), b = __uint_as_float(w[e] & 0xFFFF0000u);
                  qn2 = fmaf(a, a, fmaf(b, b, qn2));
                }
              }
            }
          }
          sNorm[sw * 32 + lane] = qn2;
        }
        const bool issue_q = j == t1 - 1 && q_loader && next_q;
        const bool valid = row >= 0 && row <= p.q_pos0 + i;
        if (!fixed_m) {
          // per-head maximum of this tile over all 128 keys (log2 units)
          float red[HH];
#pragma unroll
          for (int h = 0; h < HH; ++h)
            red[h] = (valid && hh * HH + h < H) ? x[h] * p.scale_log2 : -INFINITY;
          const float wmax = warp_transpose_reduce<HH, true>(red);
          float* xbuf = sRed + (xc & 1) * 128;
          if (lane < HH) xbuf[sw * 16 + lane] = wmax;
          mbar_arrive(&exch[xc & 1]);
          ok = __all_sync(0xffffffffu, mbar_wait(&exch[xc & 1], (xc >> 1) & 1, abort_flag, p.ws, 41));
          ++xc;
          if (!ok) break;
          float tmax = -INFINITY;
          if (lane < NH)
            tmax = fmaxf(fmaxf(xbuf[xslot], xbuf[xslot + 16]), fmaxf(xbuf[xslot + 32], xbuf[xslot + 48]));
          if (j == t0 && lane < NH) {
            float qn2 = 0.f;
#pragma unroll
            for (int w = 0; w < C::kSoftmaxWarps; ++w) qn2 += sNorm[w * 32 + lane];
            // the float32 sums are within 2^-8 of exact; the slack covers them
            bound_lane = bound_scale * sqrtf(qn2) * (1.f + 0.00390625f);
          }
          const bool need = lane < H && tmax > -INFINITY && (m_lane == -INFINITY || tmax > m_lane + 8.f);
          if (__any_sync(0xffffffffu, need)) {
            const float m_new = fmaxf(m_lane, tmax);
            const float alpha_lane = m_lane == -INFINITY ? 0.f : ex2_approx(m_lane - m_new);
            m_lane = m_new;
            float alpha[HH];
#pragma unroll
            for (int h = 0; h < HH; ++h) {
              alpha[h] = __shfl_sync(0xffffffffu, alpha_lane, hh * HH + h);
              lpart[h] *= alpha[h];
            }
            mrep[lane] = m_lane;
            __syncwarp();
            if (j > t0) {  // rescale this warp's O^T columns once the previous tile's PV is complete
              ok = __all_sync(0xffffffffu, mbar_wait(o_step, (tc - 1) & 1, abort_flag, p.ws, 42));
              if (!ok) break;
              tc_fence_after();
#pragma unroll 1
              for (int mb = 0; mb < C::MB; ++mb) {
                const uint32_t ta = tmem_base + lane_addr + C::kTmemO + (ob * C::MB + mb) * NH + hh * HH;
                float o[HH];
                tmem_ld_row<HH>(ta, o);
#pragma unroll
                for (int h = 0; h < HH; ++h) o[h] *= alpha[h];
                tmem_st_row<HH>(ta, o);
              }
              tmem_st_wait();
            }
          }
          // B_h <= m_h + 64 for every head: 2^(z - m) < 2^64 on every later tile
          fixed_m = __all_sync(0xffffffffu, lane >= H || bound_lane <= m_lane + 64.f);
        }
        if (issue_q) {
          // every QK^T of query i has completed and every warp has read its q
          // rows (the first tile's exchange): bring in the next query's q
          mbar_arrive_expect_tx(q_full, C::kQBytes);
          int i_next, a1, b1;
          item_range(p, w_next, i_next, a1, b1);
          for (int c = 0; c < C::kQChunks; ++c)
            tma_load_2d(sQ + c * C::kQChunkBytes, &tm_q, c * 64, i_next * H, q_full);
          ++q_loads;
        }
        // the previous tile's PV has finished reading P
        ok = __all_sync(0xffffffffu, mbar_wait(p_empty, (tc & 1) ^ 1, abort_flag, p.ws, 43));
        if (!ok) break;
        // this key's P for this warp's heads: p = 2^(z scale log2e - m) as bf16,
        // written as 16-byte chunks of eight heads at their swizzled positions
        // (chunk c ^ ((r >> 1) & 3) for 64-byte rows, c ^ ((r >> 2) & 1) for
        // 32-byte rows); a masked key's row is zero
        unsigned char* prow = sP + r * C::kPRowBytes;
        const int swz = NH == 32 ? ((r >> 1) & 3) : ((r >> 2) & 1);
#pragma unroll
        for (int cl = 0; cl < HH / 8; ++cl) {
          const int c = hh * (HH / 8) + cl;  // chunk of heads 8c .. 8c+7
          const float4 ma = *reinterpret_cast<const float4*>(mrep + 8 * c);
          const float4 mb = *reinterpret_cast<const float4*>(mrep + 8 * c + 4);
          const float m8[8] = {ma.x, ma.y, ma.z, ma.w, mb.x, mb.y, mb.z, mb.w};
          uint32_t w4[4];
#pragma unroll
          for (int e2 = 0; e2 < 4; ++e2) {
            float pv[2];
#pragma unroll
            for (int e = 0; e < 2; ++e) {
              const int hl = 8 * cl + 2 * e2 + e;  // local head
              const float mh = m8[2 * e2 + e];
              pv[e] = 0.f;
              if (8 * c + 2 * e2 + e < H && valid && mh > -INFINITY)
                pv[e] = ex2_approx(fmaf(x[hl], p.scale_log2, -mh));
              lpart[hl] += pv[e];
            }
            const __nv_bfloat162 b2 = __floats2bfloat162_rn(pv[0], pv[1]);
            w4[e2] = *reinterpret_cast<const uint32_t*>(&b2);
          }
          if (DSA_IN_BOUNDS(p.ws, r * C::kPRowBytes + ((c ^ swz) << 4) + 16, C::kPBytes + 1, 11))
          *reinterpret_cast<uint4*>(prow + ((c ^ swz) << 4)) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(p_full);
      }
      if (!ok) break;
      // ---- epilogue of query i
      ok = __all_sync(0xffffffffu, mbar_wait(&o_full[ob], (qi >> 1) & 1, abort_flag, p.ws, 44));
      if (!ok) break;
      tc_fence_after();
      const float lsum = warp_transpose_reduce<HH, false>(lpart);
      float* xbuf = sRed + (xc & 1) * 128;
      if (lane < HH) xbuf[sw * 16 + lane] = lsum;
      mbar_arrive(&exch[xc & 1]);
      ok = __all_sync(0xffffffffu, mbar_wait(&exch[xc & 1], (xc >> 1) & 1, abort_flag, p.ws, 45));
      ++xc;
      if (!ok) break;
      float l_lane = 0.f;
      if (lane < NH) l_lane = xbuf[xslot] + xbuf[xslot + 16] + xbuf[xslot + 32] + xbuf[xslot + 48];
      if (p.n_split > 1) {
        // a partial of a split query: unnormalised O, the reference maximum
        // (log2 units) and the row sum, merged by the combine pass
        if (sw == 0 && lane < H)
          p.part_ml[static_cast<int64_t>(w) * H + lane] = make_float2(m_lane, l_lane);
#pragma unroll 1
        for (int mb = 0; mb < C::MB; ++mb) {
          float o[HH];
          tmem_ld_row<HH>(tmem_base + lane_addr + C::kTmemO + (ob * C::MB + mb) * NH + hh * HH, o);
          const int d = mb * 128 + r;
          if (d < DC) {
            float* orow = p.part_o + (static_cast<int64_t>(w) * H + hh * HH) * DC + d;
#pragma unroll
            for (int h = 0; h < HH; ++h)
              if (hh * HH + h < H &&
                  DSA_IN_BOUNDS(p.ws, (static_cast<int64_t>(w) * H + hh * HH + h) * DC + d,
                                static_cast<int64_t>(p.n_items) * H * DC, 15))
                orow[h * DC] = o[h];
          }
        }
        tc_fence_before();
        mbar_arrive(&o_empty[ob]);
        continue;
      }
      const float inv_lane = l_lane > 0.f ? 1.f / l_lane : 0.f;
      if (sw == 0 && lane < H && p.lse)
        p.lse[static_cast<int64_t>(i) * H + lane] =
            l_lane > 0.f ? (m_lane + log2f(l_lane)) * 0.6931471805599453f : -INFINITY;
      float inv[HH];
#pragma unroll
      for (int h = 0; h < HH; ++h) inv[h] = __shfl_sync(0xffffffffu, inv_lane, hh * HH + h);
#pragma unroll 1
      for (int mb = 0; mb < C::MB; ++mb) {
        float o[HH];
        tmem_ld_row<HH>(tmem_base + lane_addr + C::kTmemO + (ob * C::MB + mb) * NH + hh * HH, o);
        const int d = mb * 128 + r;
        if (d < DC) {
          uint16_t* orow = p.out + (static_cast<int64_t>(i) * H + hh * HH) * DC + d;
#pragma unroll
          for (int h = 0; h < HH; ++h)
            if (hh * HH + h < H &&
                DSA_IN_BOUNDS(p.ws, (static_cast<int64_t>(i) * H + hh * HH + h) * DC + d,
                              static_cast<int64_t>(p.n_q) * H * DC, 12))
              orow[h * DC] = f32_to_bf16_rne(o[h] * inv[h]);
        }
      }
      tc_fence_before();
      mbar_arrive(&o_empty[ob]);
    }
    // a q load that nobody consumed lands before the CTA exits
    if (!ok && q_loader && q_loads > 0) drain_wait(q_full, (q_loads - 1) & 1);
  }

  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::kTmemCols);
  }
}

// max_s ||[latent_s, rope_s]||_2 over the context, one warp per key, as a
// float32 bit pattern in the workspace header (non-negative floats order like
// their bit patterns). Scaled up by 2^-8 to cover the float32 sums.
template <int DC, int DR>
__global__ void attn_key_norm_max_kernel(const uint16_t* __restrict__ latent,
                                         const uint16_t* __restrict__ rope, int T, WsHeader* ws) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  float best = 0.f;
  for (int s = warp; s < T; s += nwarps) {
    float ss = 0.f;
    const uint4* lr = reinterpret_cast<const uint4*>(latent + static_cast<int64_t>(s) * DC);
    const uint4* rr = reinterpret_cast<const uint4*>(rope + static_cast<int64_t>(s) * DR);
    for (int v = lane; v < (DC + DR) / 8; v += 32) {
      const uint4 u = v < DC / 8 ? __ldg(lr + v) : __ldg(rr + (v - DC / 8));
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float a = __uint_as_float(w[e] << 16), b = __uint_as_float(w[e] & 0xFFFF0000u);
        ss = fmaf(a, a, fmaf(b, b, ss));
      }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    best = fmaxf(best, ss);
  }
  if (lane == 0 && best > 0.f)
    atomicMax(&ws->akmax_bits, __float_as_uint(sqrtf(best) * (1.f + 0.00390625f)));
}

int num_sms() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

constexpr int kOneCtaPerSmSmem = 120 * 1024;

// Merges the partials of a split query, one CTA per (query, head), a thread
// per 4 dims: with M the largest reference maximum of the query's items and
// a_j = 2^(m_j - M), out = sum_j a_j O_j / sum_j a_j l_j and
// lse = (M + log2 sum_j a_j l_j) ln 2. Items without tiles were never
// written and are skipped, as are items whose keys were all masked (l = 0).
template <int H, int DC>
__global__ void attn_split_combine(const AttnParams p) {
  const int i = blockIdx.x / H, h = blockIdx.x % H;
  const int nt = n_tiles_of(p, i);
  float M = -INFINITY;
  for (int j = 0; j < p.n_split && j * p.tps < nt; ++j) {
    const float2 ml = p.part_ml[(static_cast<int64_t>(i) * p.n_split + j) * H + h];
    if (ml.y > 0.f) M = fmaxf(M, ml.x);
  }
  float L = 0.f;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  const int d0 = threadIdx.x * 4;
  for (int j = 0; j < p.n_split && j * p.tps < nt; ++j) {
    const int64_t w = static_cast<int64_t>(i) * p.n_split + j;
    const float2 ml = p.part_ml[w * H + h];
    if (!(ml.y > 0.f)) continue;
    const float a = exp2f(ml.x - M);
    L = fmaf(a, ml.y, L);
    if (d0 < DC) {
      const float4 o = *reinterpret_cast<const float4*>(p.part_o + (w * H + h) * DC + d0);
      acc[0] = fmaf(a, o.x, acc[0]);
      acc[1] = fmaf(a, o.y, acc[1]);
      acc[2] = fmaf(a, o.z, acc[2]);
      acc[3] = fmaf(a, o.w, acc[3]);
    }
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  if (d0 < DC) {
    uint16_t* orow = p.out + (static_cast<int64_t>(i) * H + h) * DC + d0;
    const uint32_t lo = f32_to_bf16_rne(acc[0] * inv) | (static_cast<uint32_t>(f32_to_bf16_rne(acc[1] * inv)) << 16);
    const uint32_t hi = f32_to_bf16_rne(acc[2] * inv) | (static_cast<uint32_t>(f32_to_bf16_rne(acc[3] * inv)) << 16);
    *reinterpret_cast<uint2*>(orow) = make_uint2(lo, hi);
  }
  if (threadIdx.x == 0 && p.lse)
    p.lse[static_cast<int64_t>(i) * H + h] = L > 0.f ? (M + log2f(L)) * 0.6931471805599453f : -INFINITY;
}

template <int H, int DC, int DR>
cudaError_t launch(const dsa_dims& d, const uint16_t* q, const uint16_t* latent,
                   const uint16_t* rope, const int32_t* idx, uint16_t* out, float* lse,
                   bool prefix_valid, WsHeader* ws, int n_split, void* part, cudaStream_t st) {
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
  const int max_tiles = (d.top_k + 127) / 128;
  p.n_split = n_split < 1 ? 1 : (n_split > max_tiles ? max_tiles : n_split);
  p.tps = (max_tiles + p.n_split - 1) / p.n_split;
  p.n_items = d.n_q * p.n_split;
  p.part_ml = static_cast<float2*>(part);
  p.part_o = part ? reinterpret_cast<float*>(static_cast<char*>(part) +
                                              attn_split_ml_bytes(d.n_q, p.n_split, H))
                  : nullptr;
  if (p.n_split > 1 && !part) return cudaErrorInvalidValue;
  CUtensorMap tm_q;
  if (!make_tmap_bf16_2d(&tm_q, q, DC + DR, static_cast<uint64_t>(d.n_q) * H, 64, H,
                         CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  const int grid = p.n_items < num_sms() ? p.n_items : num_sms();
  const int smem = C::kSmemBytes > kOneCtaPerSmSmem ? C::kSmemBytes : kOneCtaPerSmSmem;
  cudaError_t e = cudaFuncSetAttribute(sparse_attn_tc<H, DC, DR>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  sparse_attn_tc<H, DC, DR><<<grid, C::kThreads, smem, st>>>(tm_q, p);
  if (p.n_split > 1) {
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    attn_split_combine<H, DC><<<d.n_q * H, (DC / 4 + 31) / 32 * 32, 0, st>>>(p);
  }
  return cudaGetLastError();
}

template <int DC, int DR>
cudaError_t launch_norm(const dsa_dims& d, const uint16_t* latent, const uint16_t* rope, WsHeader* ws,
                        cudaStream_t st) {
  const int threads = 256;
  int blocks = (d.ctx_len * 32 + threads - 1) / threads;
  if (blocks > num_sms() * 8) blocks = num_sms() * 8;
  attn_key_norm_max_kernel<DC, DR><<<blocks, threads, 0, st>>>(latent, rope, d.ctx_len, ws);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_key_norm_max(const dsa_dims& d, const uint16_t* latent, const uint16_t* rope,
                                     WsHeader* ws, cudaStream_t st) {
  if (d.d_latent == 512 && d.d_rope == 64) return launch_norm<512, 64>(d, latent, rope, ws, st);
  if (d.d_latent == 64 && d.d_rope == 16) return launch_norm<64, 16>(d, latent, rope, ws, st);
  return cudaErrorInvalidValue;
}

cudaError_t launch_sparse_attn(const dsa_dims& d, const uint16_t* q, const uint16_t* latent,
                               const uint16_t* rope, const int32_t* idx, uint16_t* out,
                               float* lse, bool prefix_valid, WsHeader* ws, cudaStream_t st,
                               int n_split, void* part) {
  if (d.n_heads == 32 && d.d_latent == 512 && d.d_rope == 64)
    return launch<32, 512, 64>(d, q, latent, rope, idx, out, lse, prefix_valid, ws, n_split, part, st);
  if (d.n_heads == 4 && d.d_latent == 64 && d.d_rope == 16)
    return launch<4, 64, 16>(d, q, latent, rope, idx, out, lse, prefix_valid, ws, n_split, part, st);
  return cudaErrorInvalidValue;
}

int attn_decode_split(const dsa_dims& d) {
  const int max_tiles = (d.top_k + 127) / 128;
  if (d.n_q <= 0) return 1;
  int n = num_sms() / d.n_q;
  if (n > max_tiles) n = max_tiles;
  return n < 1 ? 1 : n;
}

}  // namespace dsa
