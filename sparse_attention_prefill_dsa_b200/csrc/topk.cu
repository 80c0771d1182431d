// topk.cu -- per-query top-k selection over indexer scores (sm_100a).
//
// The feedman.me post (feedman.me/posts/wy2HU), paragraph after its component
// table, names a "per-query top-2048" step in front of the sparse-attention
// gather; the tie policy (score descending, then key index ascending) is the
// reading this library fixes, in the spirit of the TensorFold issue #743
// thread, whose maintainers grant no tie exception between chunkings.
//
// One CTA per query row. The row's float32 scores s = 0..t are staged once in
// shared memory (t + 1 <= 49152 -> at most 192 KB) as order-preserving uint32
// keys. A three-pass radix select (11 + 11 + 10 bits, shared-memory
// histograms, warp-shuffle and shared-memory block scans) finds the k-th
// largest key exactly. The output pass walks the row in tiles of 512 keys
// and compacts the kept keys in ascending index order with ballot/popc-style
// block scans, so no sort is needed.
//
// Exact float64 order (indexer inputs given). Let X be the float64 score of
// the contract (sequential float64 dot per head, ReLU, sequential float64
// head sum, no fused multiply-add on the head sum) and F the float32 score.
// For every key,
//   |F - X| <= delta_t = kBoundRel * A_t * Kmax,
//   A_t  = sum_j |w_tj| * ||qI_tj||_2,   Kmax = max_s ||kI_s||_2,
// because each float32 head dot is within kDotRel * ||q|| * ||k|| of the exact
// dot (Cauchy-Schwarz on the accumulation bound), ReLU is 1-Lipschitz, the
// float32 head sum adds at most 64 * 2^-24 of sum_j |w_j| r_j, and the float64
// contract is itself within ~2^-45 of the exact value. With v = the k-th
// largest F: a key with F > v + 2 delta is certainly kept, F < v - 2 delta is
// certainly dropped, and only the band in between is re-scored in float64 in
// the contract's exact operation order; the band is then ranked by
// (X descending, index ascending). The dot is a float64 chain of exact
// products (bf16 x bf16 fits in 16 bits), so a fused multiply-add there
// rounds exactly like the separate multiply and add of the contract; the head
// sum multiplies a float32 weight by a float64 value, which is not exact, so
// it uses explicitly unfused __dmul_rn / __dadd_rn.
#include <cuda_runtime.h>
#include <stdint.h>

#include "dsa_internal.cuh"

namespace dsa {
namespace {

constexpr int kThreads = 512;
constexpr int kWarps = kThreads / 32;
constexpr int kTile = kThreads;
constexpr int kHistBins = 2048;

// Error-bound constants (see the header comment). kDotRel bounds a 128-term
// bf16 dot product accumulated in float32 (tensor-core blocks or a sequential
// FMA chain) relative to ||q|| * ||k||; kBoundRel adds the float32 head sum
// (<= 64 roundings of 2^-24) and slack for the float64 contract.
constexpr double kDotRel = 1.0 / 16384.0;        // 2^-14
constexpr double kBoundRel = kDotRel + 1.0 / 131072.0;  // + 2^-17
constexpr double kNormSlack = 1.0 + 1.0 / 1073741824.0;  // 1 + 2^-30

__device__ __forceinline__ uint32_t f2key(float f) {
  uint32_t b = __float_as_uint(f);
  if (b == 0x80000000u) b = 0u;  // -0 and +0 compare equal: one key
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ float key2f(uint32_t u) {
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7FFFFFFFu) : ~u);
}

// Order-preserving map of a finite double to uint64.
__device__ __forceinline__ unsigned long long d2key(double x) {
  unsigned long long b = static_cast<unsigned long long>(__double_as_longlong(x));
  if (b == 0x8000000000000000ull) b = 0ull;
  return (b & 0x8000000000000000ull) ? ~b : (b | 0x8000000000000000ull);
}

struct Scratch {          // static part of shared memory
  int warp_tot[kWarps];
  int bcast[4];
  unsigned long long bcast64;
  double dbl[kWarps];
};

// Block-wide exclusive prefix sum of one int per thread; returns the prefix,
// writes the block total to *total. Two __syncthreads.
__device__ __forceinline__ int block_excl_scan(int v, int* total, Scratch& sc) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sc.warp_tot[warp] = x;
  __syncthreads();
  if (warp == 0) {
    int w = lane < kWarps ? sc.warp_tot[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      int y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < kWarps) sc.warp_tot[lane] = w;  // inclusive per warp
  }
  __syncthreads();
  const int warp_base = warp ? sc.warp_tot[warp - 1] : 0;
  *total = sc.warp_tot[kWarps - 1];
  __syncthreads();  // warp_tot is reused by the next scan
  return warp_base + x - v;
}

// Given per-bin counts hist[0..nbins) (nbins = 4 * kThreads or fewer) and a
// rank kr >= 1 counted from the top, finds bin b with
//   sum(hist[b+1..]) < kr <= sum(hist[b..]).
// Returns b and writes the count strictly above b to *above.
__device__ int find_bin_from_top(const int* hist, int nbins, int kr, int* above,
                                 Scratch& sc) {
  const int per = (nbins + kThreads - 1) / kThreads;  // bins per thread (<= 4)
  // thread t owns bins counted from the top: top index r = t*per .. t*per+per-1,
  // bin = nbins-1-r
  int local = 0;
  for (int r = threadIdx.x * per; r < threadIdx.x * per + per; ++r)
    if (r < nbins) local += hist[nbins - 1 - r];
  int tot;
  int before = block_excl_scan(local, &tot, sc);  // count in bins above this thread's
  if (before < kr && before + local >= kr) {
    int acc = before;
    for (int r = threadIdx.x * per; r < threadIdx.x * per + per; ++r) {
      const int c = hist[nbins - 1 - r];
      if (acc + c >= kr) {
        sc.bcast[0] = nbins - 1 - r;
        sc.bcast[1] = acc;
        break;
      }
      acc += c;
    }
  }
  __syncthreads();
  const int b = sc.bcast[0];
  *above = sc.bcast[1];
  __syncthreads();
  return b;
}

// float64 score of the contract for key s, computed by one warp. Lane j < HI
// forms head j's dot product; lane 0..31 all return the head sum.
__device__ __forceinline__ double rescore_warp(const uint16_t* __restrict__ qT,  // [DI][HI]
                                               const float* __restrict__ w_s,    // [HI]
                                               const uint16_t* __restrict__ krow_g,
                                               uint16_t* __restrict__ kst,       // [DI] per warp
                                               int HI, int DI) {
  const int lane = threadIdx.x & 31;
  for (int c = lane * 8; c < DI; c += 256)
    *reinterpret_cast<uint4*>(kst + c) = __ldg(reinterpret_cast<const uint4*>(krow_g + c));
  __syncwarp();
  double r = 0.0;
  if (lane < HI) {
    double acc = 0.0;
    for (int c = 0; c < DI; ++c)  // exact products: fma == mul-then-add here
      acc = fma(bf16_to_f64(qT[c * HI + lane]), bf16_to_f64(kst[c]), acc);
    r = acc > 0.0 ? acc : 0.0;
  }
  double x = 0.0;
  for (int j = 0; j < HI; ++j) {
    const double rj = __shfl_sync(0xffffffffu, r, j);
    x = __dadd_rn(x, __dmul_rn(static_cast<double>(w_s[j]), rj));
  }
  __syncwarp();
  return x;
}

struct TopkArgs {
  const float* scores;
  int64_t ld;
  int n_q, q_pos0, k;
  const uint16_t* q_idx;
  const uint16_t* k_idx;
  const float* w_idx;
  int HI, DI;
  int32_t* idx;
  WsHeader* ws;
  int n_cap;  // capacity of the key array (max row length, multiple of 4)
  int bcap;   // band cache capacity (refine only)
};

// Classes for the output pass.
constexpr int kBelow = 0, kAbove = 1, kTie = 2;

// Output pass: keeps every kAbove key and the first `need_ties` kTie keys in
// index order, writing them in ascending index order. cls(s) is evaluated per
// key by each thread; `prep(base)` runs (block-uniform) before each tile.
template <class Classify, class Prep>
__device__ void emit_selection(int n, int need_ties, int32_t* __restrict__ out, Scratch& sc,
                               Classify cls, Prep prep, WsHeader* ws, int row, int expect) {
  int out_base = 0, tie_base = 0;
  for (int base = 0; base < n; base += kTile) {
    prep(base);
    const int s = base + threadIdx.x;
    const int c = s < n ? cls(s) : kBelow;
    const int packed = (c == kAbove ? 1 : 0) | (c == kTie ? (1 << 16) : 0);
    int tot;
    const int ex = block_excl_scan(packed, &tot, sc);
    const int above_before = ex & 0xFFFF, ties_before = ex >> 16;
    const int tot_above = tot & 0xFFFF, tot_ties = tot >> 16;
    int take = need_ties - tie_base;
    take = take < 0 ? 0 : take;
    const bool keep = c == kAbove || (c == kTie && ties_before < take);
    const int pos = out_base + above_before + min(ties_before, take);
    if (keep && pos < expect) out[pos] = s;  // never write past the row
    out_base += tot_above + min(tot_ties, take);
    tie_base += tot_ties;
  }
  // Every caller keeps exactly min(k, n) keys; anything else is a defect.
  if (threadIdx.x == 0 && out_base != expect) report(ws, kDevInternal, static_cast<unsigned>(row));
}

template <bool kRefine>
__global__ void __launch_bounds__(kThreads, 1) topk_kernel(TopkArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ Scratch sc;
  const int row = blockIdx.x;
  const int t = a.q_pos0 + row;
  const int n = t + 1;
  const int k = a.k;
  int32_t* out = a.idx + static_cast<int64_t>(row) * k;

  if (n <= k) {  // every causal key is kept
    for (int c = threadIdx.x; c < k; c += kThreads) out[c] = c < n ? c : -1;
    return;
  }

  uint32_t* keys = reinterpret_cast<uint32_t*>(smem);
  int* hist = reinterpret_cast<int*>(smem + sizeof(uint32_t) * a.n_cap);

  // ---- stage the row as keys and build the first histogram (bits 31..21)
  for (int b = threadIdx.x; b < kHistBins; b += kThreads) hist[b] = 0;
  __syncthreads();
  const float* srow = a.scores + static_cast<int64_t>(row) * a.ld;
  const int n4 = n & ~3;
  for (int s = threadIdx.x * 4; s < n4; s += kThreads * 4) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(srow + s));
    const uint32_t u0 = f2key(v.x), u1 = f2key(v.y), u2 = f2key(v.z), u3 = f2key(v.w);
    *reinterpret_cast<uint4*>(keys + s) = make_uint4(u0, u1, u2, u3);
    atomicAdd(&hist[u0 >> 21], 1);
    atomicAdd(&hist[u1 >> 21], 1);
    atomicAdd(&hist[u2 >> 21], 1);
    atomicAdd(&hist[u3 >> 21], 1);
  }
  for (int s = n4 + threadIdx.x; s < n; s += kThreads) {
    const uint32_t u = f2key(__ldg(srow + s));
    keys[s] = u;
    atomicAdd(&hist[u >> 21], 1);
  }
  __syncthreads();

  // ---- radix select: 11 + 11 + 10 bits
  int kr = k, above;
  uint32_t prefix = static_cast<uint32_t>(find_bin_from_top(hist, 2048, kr, &above, sc)) << 21;
  kr -= above;
  uint32_t mask = 0xFFE00000u;
  {
    for (int b = threadIdx.x; b < kHistBins; b += kThreads) hist[b] = 0;
    __syncthreads();
    for (int s = threadIdx.x; s < n; s += kThreads) {
      const uint32_t u = keys[s];
      if ((u & mask) == prefix) atomicAdd(&hist[(u >> 10) & 0x7FFu], 1);
    }
    __syncthreads();
    prefix |= static_cast<uint32_t>(find_bin_from_top(hist, 2048, kr, &above, sc)) << 10;
    kr -= above;
    mask = 0xFFFFFC00u;
    for (int b = threadIdx.x; b < 1024; b += kThreads) hist[b] = 0;
    __syncthreads();
    for (int s = threadIdx.x; s < n; s += kThreads) {
      const uint32_t u = keys[s];
      if ((u & mask) == prefix) atomicAdd(&hist[u & 0x3FFu], 1);
    }
    __syncthreads();
    prefix |= static_cast<uint32_t>(find_bin_from_top(hist, 1024, kr, &above, sc));
    kr -= above;
  }
  const uint32_t uk = prefix;  // key of the k-th largest score; kr ties at uk are kept

  if (!kRefine) {
    emit_selection(
        n, kr, out, sc,
        [&](int s) {
          const uint32_t u = keys[s];
          return u > uk ? kAbove : (u == uk ? kTie : kBelow);
        },
        [](int) {}, a.ws, row, k);
    return;
  }

  // ---------------- exact float64 order: certified band + float64 re-score
  const int HI = a.HI, DI = a.DI;
  unsigned char* p = smem + sizeof(uint32_t) * a.n_cap + sizeof(int) * kHistBins;
  uint16_t* qT = reinterpret_cast<uint16_t*>(p);  p += sizeof(uint16_t) * 32 * 128;
  float* w_s = reinterpret_cast<float*>(p);       p += sizeof(float) * 32;
  uint16_t* kst = reinterpret_cast<uint16_t*>(p); p += sizeof(uint16_t) * kWarps * 128;
  int* tile_s = reinterpret_cast<int*>(p);        p += sizeof(int) * kTile;
  double* tile_x = reinterpret_cast<double*>(p);  p += sizeof(double) * kTile;
  unsigned long long* bx = reinterpret_cast<unsigned long long*>(p);
  p += sizeof(unsigned long long) * a.bcap;
  unsigned char* bsel = p;

  // query row of the indexer, transposed to [c][j] so that lane j reads
  // consecutive halves; weights; A_t = sum_j |w_j| ||q_j||
  const uint16_t* qrow = a.q_idx + static_cast<int64_t>(row) * HI * DI;
  for (int e = threadIdx.x; e < HI * DI; e += kThreads) {
    const int j = e / DI, c = e - j * DI;
    qT[c * HI + j] = qrow[e];
  }
  if (threadIdx.x < HI) w_s[threadIdx.x] = a.w_idx[static_cast<int64_t>(row) * HI + threadIdx.x];
  {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    double acc = 0.0;
    for (int j = warp; j < HI; j += kWarps) {
      double ss = 0.0;
      for (int c = lane; c < DI; c += 32) {
        const double v = bf16_to_f64(qrow[j * DI + c]);
        ss += v * v;
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      acc += fabs(static_cast<double>(a.w_idx[static_cast<int64_t>(row) * HI + j])) * sqrt(ss);
    }
    if (lane == 0) sc.dbl[warp] = acc;
  }
  __syncthreads();
  double A = 0.0;
  for (int w = 0; w < kWarps; ++w) A += sc.dbl[w];
  A *= kNormSlack;
  const double kmax = __longlong_as_double(static_cast<long long>(a.ws->kmax_bits));
  const double delta = kBoundRel * A * kmax;
  const double vk = static_cast<double>(key2f(uk));
  const double lo = vk - 2.0 * delta, hi = vk + 2.0 * delta;

  // counts: certainly kept (F > hi) and band (lo <= F <= hi)
  int c_in = 0, c_band = 0;
  for (int s = threadIdx.x; s < n; s += kThreads) {
    const double f = static_cast<double>(key2f(keys[s]));
    c_in += f > hi;
    c_band += (f >= lo && f <= hi);
  }
  int tot_in, tot_band;
  block_excl_scan(c_in, &tot_in, sc);
  block_excl_scan(c_band, &tot_band, sc);
  const int r = k - tot_in;  // band keys still to take, 1 <= r <= tot_band

  auto is_band = [&](int s) {
    const double f = static_cast<double>(key2f(keys[s]));
    return f >= lo && f <= hi;
  };
  auto is_in = [&](int s) { return static_cast<double>(key2f(keys[s])) > hi; };

  if (r == tot_band) {  // the whole band is kept: no re-score needed
    emit_selection(
        n, 0, out, sc, [&](int s) { return (is_in(s) || is_band(s)) ? kAbove : kBelow; },
        [](int) {}, a.ws, row, k);
    return;
  }

  const int warp = threadIdx.x >> 5;
  uint16_t* my_kst = kst + warp * 128;
  // Re-scores the band keys of tile [base, base+512): afterwards tile_s[j] and
  // tile_x[j], j < returned count, hold them in index order. With fill_cache,
  // the float64 keys also go to bx[pos0 + j] (positions < bcap).
  auto band_tile = [&](int base, int pos0, bool fill_cache) -> int {
    const int s = base + threadIdx.x;
    const int flag = (s < n && is_band(s)) ? 1 : 0;
    int nb;
    const int j = block_excl_scan(flag, &nb, sc);
    if (flag) tile_s[j] = s;
    __syncthreads();
    for (int jj = warp; jj < nb; jj += kWarps) {
      const double x = rescore_warp(qT, w_s, a.k_idx + static_cast<int64_t>(tile_s[jj]) * DI,
                                    my_kst, HI, DI);
      if ((threadIdx.x & 31) == 0) {
        tile_x[jj] = x;
        if (fill_cache && pos0 + jj < a.bcap) bx[pos0 + jj] = d2key(x);
      }
    }
    __syncthreads();
    return nb;
  };

  if (tot_band <= a.bcap) {
    // one sweep fills the cache with the band's float64 keys (in index order)
    int pos0 = 0;
    for (int base = 0; base < n; base += kTile) pos0 += band_tile(base, pos0, true);
    // rank within the band by (X desc, position asc); keep rank < r
    for (int b = threadIdx.x; b < tot_band; b += kThreads) {
      const unsigned long long xb = bx[b];
      int rank = 0;
      for (int o = 0; o < tot_band; ++o) {
        const unsigned long long xo = bx[o];
        rank += (xo > xb) || (xo == xb && o < b);
      }
      bsel[b] = rank < r ? 1 : 0;
    }
    __syncthreads();
    // output: band position of s = running band count before s
    int band_base = 0;
    int* tile_pos = tile_s;  // reuse: band position of each tile key
    emit_selection(
        n, 0, out, sc,
        [&](int s) {
          if (is_in(s)) return kAbove;
          const int pos = tile_pos[s & (kTile - 1)];
          return (pos >= 0 && bsel[pos]) ? kAbove : kBelow;
        },
        [&](int base) {
          const int s = base + threadIdx.x;
          const int flag = (s < n && is_band(s)) ? 1 : 0;
          int nb;
          const int j = block_excl_scan(flag, &nb, sc);
          tile_pos[threadIdx.x] = flag ? band_base + j : -1;
          band_base += nb;
          __syncthreads();
        },
        a.ws, row, k);
    return;
  }

  // ---- band larger than the cache (degenerate inputs): 64-bit radix select
  // over the band's float64 keys, re-scoring the band in every pass.
  int* hist256 = hist;
  unsigned long long pre = 0ull, msk = 0ull;
  int rr = r;
  for (int shift = 56; shift >= 0; shift -= 8) {
    for (int b = threadIdx.x; b < 256; b += kThreads) hist256[b] = 0;
    __syncthreads();
    for (int base = 0; base < n; base += kTile) {
      const int nb = band_tile(base, 0, false);
      if (threadIdx.x < nb) {
        const unsigned long long key = d2key(tile_x[threadIdx.x]);
        if ((key & msk) == pre) atomicAdd(&hist256[(key >> shift) & 0xFFull], 1);
      }
      __syncthreads();
    }
    int ab;
    const int bsel_bin = find_bin_from_top(hist256, 256, rr, &ab, sc);
    rr -= ab;
    pre |= static_cast<unsigned long long>(bsel_bin) << shift;
    msk |= 0xFFull << shift;
  }
  const unsigned long long xr = pre;  // key of the r-th largest band score; rr ties kept
  emit_selection(
      n, rr, out, sc,
      [&](int s) {
        if (is_in(s)) return kAbove;
        const int j = tile_s[s & (kTile - 1)];
        if (j < 0) return kBelow;
        const unsigned long long key = d2key(tile_x[j]);
        return key > xr ? kAbove : (key == xr ? kTie : kBelow);
      },
      [&](int base) {
        // re-score this tile's band keys, then map each tile slot to its list entry
        const int nb = band_tile(base, 0, false);
        const int s = base + threadIdx.x;
        // tile_s holds key indices of band entries; invert into a slot map
        // stored in the upper half of tile_x's storage is not possible (doubles
        // in use), so search: the list is sorted, nb <= 512.
        int found = -1;
        if (s < n && is_band(s)) {
          int lo_i = 0, hi_i = nb - 1;
          while (lo_i <= hi_i) {
            const int mid = (lo_i + hi_i) >> 1;
            const int v = tile_s[mid];
            if (v == s) { found = mid; break; }
            if (v < s) lo_i = mid + 1; else hi_i = mid - 1;
          }
        }
        __syncthreads();
        tile_s[threadIdx.x] = found;  // slot -> list index (or -1)
        __syncthreads();
      },
      a.ws, row, k);
}

__global__ void key_norm_max_kernel(const uint16_t* __restrict__ k_idx, int T, int DI,
                                    WsHeader* ws) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int nwarps = (gridDim.x * blockDim.x) >> 5;
  double best = 0.0;
  for (int s = warp; s < T; s += nwarps) {
    double ss = 0.0;
    for (int c = lane; c < DI; c += 32) {
      const double v = bf16_to_f64(k_idx[static_cast<int64_t>(s) * DI + c]);
      ss += v * v;
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
    best = fmax(best, sqrt(ss) * kNormSlack);
  }
  if (lane == 0 && best > 0.0)
    atomicMax(&ws->kmax_bits, static_cast<unsigned long long>(__double_as_longlong(best)));
}

}  // namespace

cudaError_t launch_key_norm_max(const dsa_dims& d, const uint16_t* k_idx, WsHeader* ws,
                                cudaStream_t st) {
  const int threads = 256;
  int blocks = (d.ctx_len * 32 + threads - 1) / threads;
  if (blocks > 148 * 8) blocks = 148 * 8;
  key_norm_max_kernel<<<blocks, threads, 0, st>>>(k_idx, d.ctx_len, d.d_idx, ws);
  return cudaGetLastError();
}

cudaError_t launch_topk(const dsa_dims& d, const float* scores, int64_t ld, const uint16_t* q_idx,
                        const uint16_t* k_idx, const float* w_idx, int32_t* idx, WsHeader* ws,
                        cudaStream_t st) {
  TopkArgs a;
  a.scores = scores;
  a.ld = ld;
  a.n_q = d.n_q;
  a.q_pos0 = d.q_pos0;
  a.k = d.top_k;
  a.q_idx = q_idx;
  a.k_idx = k_idx;
  a.w_idx = w_idx;
  a.HI = d.n_idx_heads;
  a.DI = d.d_idx;
  a.idx = idx;
  a.ws = ws;
  a.n_cap = ((d.q_pos0 + d.n_q) + 3) & ~3;
  const bool refine = q_idx != nullptr;
  size_t base = sizeof(uint32_t) * a.n_cap + sizeof(int) * kHistBins;
  int max_smem = 0, dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  const size_t static_bytes = sizeof(Scratch) + 64;
  size_t bytes = base;
  if (refine) {
    base += sizeof(uint16_t) * 32 * 128 + sizeof(float) * 32 + sizeof(uint16_t) * kWarps * 128 +
            sizeof(int) * kTile + sizeof(double) * kTile;
    const size_t avail = static_cast<size_t>(max_smem) - static_bytes;
    if (avail < base) return cudaErrorInvalidConfiguration;
    size_t bc = (avail - base) / (sizeof(unsigned long long) + 1);
    if (bc > 4096) bc = 4096;
    a.bcap = static_cast<int>(bc);
    bytes = base + a.bcap * (sizeof(unsigned long long) + 1);
  } else {
    a.bcap = 0;
    if (static_cast<size_t>(max_smem) < base + static_bytes) return cudaErrorInvalidConfiguration;
  }
  if (refine) {
    cudaFuncSetAttribute(topk_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(bytes));
    topk_kernel<true><<<d.n_q, kThreads, bytes, st>>>(a);
  } else {
    cudaFuncSetAttribute(topk_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         static_cast<int>(bytes));
    topk_kernel<false><<<d.n_q, kThreads, bytes, st>>>(a);
  }
  return cudaGetLastError();
}

}  // namespace dsa
