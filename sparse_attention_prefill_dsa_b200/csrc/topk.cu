// topk.cu -- per-query top-k selection over indexer scores (sm_100a).
//
// The feedman.me post (feedman.me/posts/wy2HU), paragraph after its component
// table, names a "per-query top-2048" step in front of the sparse-attention
// gather. The tie policy (score descending, then key index ascending) is the
// reading this library fixes, in the spirit of the TensorFold issue #743
// thread, whose maintainers grant no tie exception between chunkings.
//
// Two kernels. With the indexer inputs given (the exact mode of every layer
// call) topk_window_kernel, the window select described further down, runs
// first: a 192-thread CTA per row that keeps only a window of the row around
// its k-th value, four rows per SM. Rows it hands back (heavy ties, a
// degenerate range), and the float32-only mode, run topk_kernel, the bucket
// select described here:
//
// One CTA (384 threads) per query row; the row's float32 scores s = 0..t are
// staged once in shared memory (t + 1 <= 49152 -> at most 192 KB). Longer
// rows take two levels: pass 1 selects the top-k of every segment of at most
// 32,768 keys of a row (one CTA per segment), pass 2 the top-k among the
// segments' winners. The whole row's top-k is a subset of its segments'
// top-k sets (a key beaten by k keys of its own segment is beaten by them in
// the row), and both passes use the same exact order, so the result is the
// one-level selection's.
//
// k-th largest value, exactly: a bucket select. The value range [L, U] of the
// candidates is cut into 2,048 equal buckets, bucket(v) = floor((v - L) * 2048 /
// (U - L)) computed in float64 -- a monotone map, so buckets are ordered and
// every key in a higher bucket is strictly larger. One shared-memory histogram
// (low atomic contention because the buckets follow the values, not their bit
// patterns) locates the bucket that holds the k-th largest; its few members are
// ranked directly. A bucket with more than 1,024 members (heavy ties) is
// re-bucketed over its own value range; a range of one value ends the search.
//
// Output: each thread owns one contiguous segment of the row (odd length, so a
// warp's reads hit distinct banks); one block-wide scan of packed counters
// gives every segment its output offset, and the kept keys are written in
// ascending index order with no sort.
//
// Exact float64 order (indexer inputs given). Let X be the float64 score of
// the contract (sequential float64 dot per head, ReLU, sequential float64
// head sum) and F the float32 score. For every key,
//   |F - X| <= delta_t = kBoundRel * A_t * Kmax,
//   A_t  = sum_j |w_tj| * ||qI_tj||_2,   Kmax = max_s ||kI_s||_2.
// Each float32 head dot sums 128 exact bf16 products in 8 tensor-core blocks of
// 16; even if every one of the <= 136 additions (16 products and the running
// sum per block) truncated at float32 precision, the error stays below
// 136 * 2^-23 * sum|q*k| < 2^-15 * ||q|| * ||k|| (Cauchy-Schwarz). ReLU is
// 1-Lipschitz, the float32 head sum adds at most 64 * 2^-24 of
// sum_j |w_j| r_j, and the float64 contract itself is within ~2^-45 of the
// exact value. With v = the k-th largest F: a key with F > v + 2 delta is
// certainly kept, F < v - 2 delta is certainly dropped, and only the band in
// between is re-scored in float64 in the contract's operation order and
// ranked by (X descending, index ascending). The head dots are float64 chains
// of exact products (bf16 x bf16 fits in 16 bits), so a fused multiply-add
// rounds there exactly like the contract's separate multiply and add; the head
// sum multiplies a float32 weight by a float64 value, which is not exact, so
// it uses explicitly unfused __dmul_rn / __dadd_rn.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "dsa_internal.cuh"

namespace dsa {
namespace {

constexpr int kThreads = 384;
// first index of a row the window select hands back to topk_kernel
constexpr int32_t kRedoMarker = static_cast<int32_t>(0x80000000u);
constexpr int kWarps = kThreads / 32;
constexpr int kRescoreWarps = 8;  // warps that re-score band keys (their staging fits hist + cand + extra)
constexpr int kBins = 2048;
constexpr int kCandCap = 1024;
constexpr int kMaxRounds = 48;
// refine scratch: extra room that makes hist + cand + extra the key staging of
// the re-score (four keys of 128 dims as float64 high words, 2 KB per warp);
// the query's indexer row (at most 32 x 128) as the high 32-bit words of its
// float64 values (the low word of a widened bf16 is always zero), rows padded
// to DI + 4 words so that the 16-byte loads of lanes j .. j+7 (row j, same
// column) cover all 32 banks; the radix histogram of the slow path
constexpr int kKstStageBytes = 4 * 128 * 4;
constexpr int kKstExtraBytes = kRescoreWarps * kKstStageBytes - kBins * 4 - kCandCap * 4;
constexpr int kQRowBytes = 32 * (128 + 4) * 4;
constexpr int kHist256Bytes = 256 * 4;
// the slow path's scratch (radix histogram, window keys and scores) overlays
// the band cache, which that path does not use
constexpr int kSlowScratchBytes = kHist256Bytes + 4 * kThreads + 8 * kThreads;
static_assert(kKstExtraBytes >= 0 && kKstExtraBytes % 16 == 0, "key staging");
static_assert(kBins >= 2048, "the selection of the emit (top_k <= 2048) is staged in hist");

constexpr double kDotRel = 1.0 / 32768.0;                  // 2^-15
constexpr double kBoundRel = kDotRel + 1.0 / 131072.0;      // + 2^-17
constexpr double kNormSlack = 1.0 + 1.0 / 1073741824.0;     // 1 + 2^-30

// Classes for the output pass.
constexpr int kBelow = 0, kAbove = 1, kTie = 2;

struct Scratch {
  unsigned long long w64[kWarps];
  float wf0[kWarps], wf1[kWarps];
  double wd[kWarps];
  int bc[4];
  float bf[4];
};

__device__ __forceinline__ float canon(float f) { return f == 0.f ? 0.f : f; }  // -0 -> +0

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                   static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst))),
               "l"(gsrc)
               : "memory");
}

__device__ __forceinline__ unsigned long long d2key(double x) {
  unsigned long long b = static_cast<unsigned long long>(__double_as_longlong(x));
  if (b == 0x8000000000000000ull) b = 0ull;
  return (b & 0x8000000000000000ull) ? ~b : (b | 0x8000000000000000ull);
}

// ------------------------------------------------------------ block helpers

template <int NT = kThreads>
__device__ __forceinline__ void block_minmax(float& mn, float& mx, Scratch& sc) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
  if (lane == 0) {
    sc.wf0[warp] = mn;
    sc.wf1[warp] = mx;
  }
  __syncthreads();
  mn = sc.wf0[0];
  mx = sc.wf1[0];
#pragma unroll
  for (int w = 1; w < NT / 32; ++w) {
    mn = fminf(mn, sc.wf0[w]);
    mx = fmaxf(mx, sc.wf1[w]);
  }
  __syncthreads();
}

// Exclusive prefix sum of a packed pair of 32-bit counters; *total gets the sum.
template <int NT = kThreads>
__device__ __forceinline__ unsigned long long block_excl_scan64(unsigned long long v,
                                                                unsigned long long* total,
                                                                Scratch& sc) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned long long x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) sc.w64[warp] = x;
  __syncthreads();
  unsigned long long base = 0, tot = 0;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) {
    const unsigned long long t = sc.w64[w];
    if (w < warp) base += t;
    tot += t;
  }
  __syncthreads();
  *total = tot;
  return base + x - v;
}

// hist[0..NB) counts; finds bin b with sum(hist[b+1..]) < kr <= sum(hist[b..]).
template <int NB, int NT = kThreads>
__device__ int find_bin_from_top(const int* hist, int kr, int* above, Scratch& sc) {
  constexpr int per = (NB + NT - 1) / NT;  // bins per thread, counted from the top
  const int r0 = threadIdx.x * per;
  int local = 0;
#pragma unroll
  for (int e = 0; e < per; ++e)
    if (r0 + e < NB) local += hist[NB - 1 - (r0 + e)];
  unsigned long long tot;
  const int before =
      static_cast<int>(block_excl_scan64<NT>(static_cast<unsigned long long>(local), &tot, sc));
  if (before < kr && before + local >= kr) {
    int acc = before;
    for (int e = 0; e < per && r0 + e < NB; ++e) {
      const int c = hist[NB - 1 - (r0 + e)];
      if (acc + c >= kr) {
        sc.bc[0] = NB - 1 - (r0 + e);
        sc.bc[1] = acc;
        break;
      }
      acc += c;
    }
  }
  __syncthreads();
  const int b = sc.bc[0];
  *above = sc.bc[1];
  __syncthreads();
  return b;
}

// This thread's contiguous segment of [0, n): odd length, so the 32 threads
// of a warp start on 32 different shared-memory banks.
__device__ __forceinline__ void my_segment(int n, int& beg, int& end) {
  int len = (n + kThreads - 1) / kThreads;
  len |= 1;
  beg = min(static_cast<int>(threadIdx.x) * len, n);
  end = min(beg + len, n);
}

// Calls f(s, sc[s]) for s = beg .. end-1 in order. Eight values are loaded
// before their calls: f writes shared memory, which the compiler must assume
// may alias sc, so loads issued one per call would each wait for the previous
// call's writes.
template <class F>
__device__ __forceinline__ void for_segment(const float* sc, int beg, int end, F f) {
  int s = beg;
  for (; s + 8 <= end; s += 8) {
    float v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = sc[s + u];
#pragma unroll
    for (int u = 0; u < 8; ++u) f(s + u, v[u]);
  }
  for (; s < end; ++s) f(s, sc[s]);
}

// Bucket of v in [L, U]: (v - L) * scale rounded to an integer, clamped to the
// last bucket. Rounded float arithmetic is monotone in v, which is all the
// select needs; ranges too narrow for a finite float scale use float64.
struct Bucketer {
  float Lf, scalef;
  double Ld, scaled;
  bool wide;
  __device__ __forceinline__ Bucketer(float L, float U) {
    const float range = U - L;
    wide = range > 1e-30f && range < 1e30f;
    Lf = L;
    scalef = wide ? static_cast<float>(kBins) / range : 0.f;
    Ld = L;
    scaled = static_cast<double>(kBins) / (static_cast<double>(U) - static_cast<double>(L));
  }
  __device__ __forceinline__ int operator()(float v) const {
    if (wide) {
      // round((v - L) * scale) read from the mantissa of x + 2^23 (x is in
      // [0, kBins] up to rounding): FMA and integer pipes, no conversion
      const float y = fmaf(v - Lf, scalef, 8388608.f);
      const int b = __float_as_int(y) - 0x4B000000;
      return b > kBins - 1 ? kBins - 1 : b;
    }
    const double x = (static_cast<double>(v) - Ld) * scaled;
    return x >= static_cast<double>(kBins - 1) ? kBins - 1 : static_cast<int>(x);
  }
};

// Exact k-th largest of sc[0..n) (n > k). *n_above gets the number of values
// strictly larger. Uses hist[kBins] and cand[kCandCap]. Returns false if the
// search did not settle (not expected; reported by the caller).
__device__ bool kth_largest(const float* sc, int n, int k, float vmin, float vmax, int* hist,
                            float* cand, Scratch& sm, float* vk_out, int* n_above, WsHeader* ws) {
  float L = vmin, U = vmax;
  int kr = k, above = 0;
  int beg, end;
  my_segment(n, beg, end);
  for (int round = 0; round < kMaxRounds; ++round) {
    if (L == U) {  // every remaining candidate has the same value
      *vk_out = L;
      *n_above = above;
      return true;
    }
    for (int b = threadIdx.x; b < kBins; b += kThreads) hist[b] = 0;
    if (threadIdx.x == 0) sm.bc[2] = 0;
    __syncthreads();
    const Bucketer bucket(L, U);
    for_segment(sc, beg, end, [&](int, float v) {
      if (v >= L && v <= U) {
        const int b = bucket(v);
        if (DSA_IN_BOUNDS(ws, b, kBins, 1)) atomicAdd(&hist[b], 1);
      }
    });
    __syncthreads();
    int ab;
    const int bstar = find_bin_from_top<kBins>(hist, kr, &ab, sm);
    kr -= ab;
    above += ab;
    const int c = hist[bstar];
    float mn = INFINITY, mx = -INFINITY;
    if (c <= kCandCap) {
      // the bucket's members into cand[] (complete after the barrier)
      for_segment(sc, beg, end, [&](int, float v) {
        if (v >= L && v <= U && bucket(v) == bstar) {
          const int pos = atomicAdd(&sm.bc[2], 1);
          if (DSA_IN_BOUNDS(ws, pos, kCandCap, 2)) cand[pos] = v;
        }
      });
      __syncthreads();
    } else {
      // the bucket's value range, re-bucketed in the next round
      for_segment(sc, beg, end, [&](int, float v) {
        if (v >= L && v <= U && bucket(v) == bstar) {
          mn = fminf(mn, v);
          mx = fmaxf(mx, v);
        }
      });
      block_minmax(mn, mx, sm);
    }
    if (c <= kCandCap) {
      // rank the bucket's members: the kr-th largest value
      for (int e = threadIdx.x; e < c; e += kThreads) {
        const float v = cand[e];
        int gt = 0, ge = 0;
        for (int o = 0; o < c; ++o) {
          const float u = cand[o];
          gt += u > v;
          ge += u >= v;
        }
        if (gt < kr && kr <= ge) {
          sm.bf[0] = v;
          sm.bc[3] = gt;
        }
      }
      __syncthreads();
      *vk_out = sm.bf[0];
      *n_above = above + sm.bc[3];
      __syncthreads();
      return true;
    }
    L = mn;
    U = mx;
  }
  return false;
}

// Writes the selection to out[0..k): every kAbove key and the first need_ties
// kTie keys, in ascending index order. cls(v) classifies key s by v = sc[s].
// a_known >= 0 is the number of kAbove keys in this thread's segment (which
// then holds no kTie key), known to the caller; the counting pass is skipped.
// The selection is assembled in stage[0..k) (shared memory, 16-byte aligned)
// and then written out in coalesced pieces.
template <class Cls>
__device__ void emit_selection(const float* sc, int n, int need_ties, int k, int32_t* __restrict__ out,
                               int32_t* __restrict__ stage, Cls cls, Scratch& sm, WsHeader* ws, int row,
                               int a_known = -1, int key_off = 0, const int32_t* kmap = nullptr) {
  int beg, end;
  my_segment(n, beg, end);
  unsigned int a = 0, t = 0;
  if (a_known >= 0) {
    a = static_cast<unsigned int>(a_known);
  } else {
    for_segment(sc, beg, end, [&](int, float v) {
      const int c = cls(v);
      a += c == kAbove;
      t += c == kTie;
    });
  }
  unsigned long long tot;
  const unsigned long long ex = block_excl_scan64(
      static_cast<unsigned long long>(a) | (static_cast<unsigned long long>(t) << 32), &tot, sm);
  int ties_before = static_cast<int>(ex >> 32);
  int pos = static_cast<int>(ex & 0xffffffffu) + min(ties_before, need_ties);
  for_segment(sc, beg, end, [&](int s, float v) {
    const int c = cls(v);
    bool keep = c == kAbove;
    if (c == kTie) keep = ties_before++ < need_ties;
    if (keep) {
      // never write past the row (a count mismatch is reported below)
      if (pos < k) stage[pos] = kmap ? __ldg(kmap + s) : s + key_off;
      ++pos;
    }
  });
  const int total =
      static_cast<int>(tot & 0xffffffffu) + min(static_cast<int>(tot >> 32), need_ties);
  if (threadIdx.x == 0 && total != k) report(ws, kDevInternal, static_cast<unsigned>(row));
  __syncthreads();
  const int nw = min(total, k);
  if ((k & 3) == 0 && nw == k) {
    for (int i = threadIdx.x; i < k / 4; i += kThreads)
      reinterpret_cast<int4*>(out)[i] = reinterpret_cast<const int4*>(stage)[i];
  } else {
    for (int i = threadIdx.x; i < nw; i += kThreads) out[i] = stage[i];
  }
}

// Row data of a key for the float64 re-score: lane l holds dims 4l..4l+3.
__device__ __forceinline__ uint2 load_key_part(const uint16_t* __restrict__ k_idx, int key, int DI) {
  const int lane = threadIdx.x & 31;
  if (lane * 4 >= DI) return make_uint2(0u, 0u);
  return __ldg(reinterpret_cast<const uint2*>(k_idx + static_cast<int64_t>(key) * DI + lane * 4));
}

// float64 scores of the contract for four keys (one warp). raw[e] is key e's
// row part (load_key_part); lanes widen it once into this warp's kst as the
// high 32-bit words of the float64 values ([4][128] words; the low word of a
// widened bf16 is zero). Lane j < HI forms head j's four dot products, each a
// sequential float64 chain over the dims (fully unrolled; four dims per
// 16-byte load of the q row's high words, rows DI + 4 words apart, and four
// per broadcast load of each key), and p = w_j * relu(dot). The products go
// back through kst ([4][34] doubles) and lane e < 4 adds key e's in head
// order and returns that sum (other lanes return 0).
template <int DI>
__device__ __forceinline__ double rescore4(const uint32_t* __restrict__ qhi, double w_lane,
                                           const uint2 (&raw)[4], uint32_t* __restrict__ kst, int HI) {
  const int lane = threadIdx.x & 31;
  if (lane * 4 < DI) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t w[2] = {raw[e].x, raw[e].y};
      uint32_t h[4];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        h[2 * u] = static_cast<uint32_t>(__double2hiint(bf16_to_f64(static_cast<uint16_t>(w[u] & 0xFFFFu))));
        h[2 * u + 1] = static_cast<uint32_t>(__double2hiint(bf16_to_f64(static_cast<uint16_t>(w[u] >> 16))));
      }
      *reinterpret_cast<uint4*>(kst + e * 128 + lane * 4) = make_uint4(h[0], h[1], h[2], h[3]);
    }
  }
  __syncwarp();
  double pr[4] = {0.0, 0.0, 0.0, 0.0};
  if (lane < HI) {
    const uint4* q4 = reinterpret_cast<const uint4*>(qhi + lane * (DI + 4));
    double acc[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
    for (int c4 = 0; c4 < DI / 4; ++c4) {
      const uint4 qq = q4[c4];
      const double qd[4] = {__hiloint2double(static_cast<int>(qq.x), 0), __hiloint2double(static_cast<int>(qq.y), 0),
                            __hiloint2double(static_cast<int>(qq.z), 0), __hiloint2double(static_cast<int>(qq.w), 0)};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint4 kk = reinterpret_cast<const uint4*>(kst + e * 128)[c4];
        acc[e] = fma(qd[0], __hiloint2double(static_cast<int>(kk.x), 0), acc[e]);
        acc[e] = fma(qd[1], __hiloint2double(static_cast<int>(kk.y), 0), acc[e]);
        acc[e] = fma(qd[2], __hiloint2double(static_cast<int>(kk.z), 0), acc[e]);
        acc[e] = fma(qd[3], __hiloint2double(static_cast<int>(kk.w), 0), acc[e]);
      }
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) pr[e] = __dmul_rn(w_lane, acc[e] > 0.0 ? acc[e] : 0.0);
  }
  __syncwarp();
  double* prod = reinterpret_cast<double*>(kst);
  if (lane < HI) {
#pragma unroll
    for (int e = 0; e < 4; ++e) prod[e * 34 + lane] = pr[e];
  }
  __syncwarp();
  double sum = 0.0;
  if (lane < 4) {
    const double2* pe = reinterpret_cast<const double2*>(prod + lane * 34);
#pragma unroll
    for (int j2 = 0; j2 < 16; ++j2) {
      if (2 * j2 < HI) {
        const double2 v = pe[j2];
        sum = __dadd_rn(sum, v.x);
        sum = __dadd_rn(sum, v.y);  // HI is even
      }
    }
  }
  __syncwarp();
  return sum;
}

// rescore4 for eight keys per call (eight independent float64 chains per
// lane instead of four), the keys staged as float64 high words (8 x DI
// words). The same operation order as rescore4. Lane e < 8 returns key e's
// score; kst afterwards holds the [8][34] products of the head sum.
template <int DI>
__device__ __forceinline__ double rescore8h(const uint32_t* __restrict__ qhi, double w_lane,
                                            const uint2 (&raw)[8], uint32_t* __restrict__ kst, int HI) {
  const int lane = threadIdx.x & 31;
  if (lane * 4 < DI) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const uint32_t w[2] = {raw[e].x, raw[e].y};
      uint32_t h[4];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        h[2 * u] = static_cast<uint32_t>(__double2hiint(bf16_to_f64(static_cast<uint16_t>(w[u] & 0xFFFFu))));
        h[2 * u + 1] = static_cast<uint32_t>(__double2hiint(bf16_to_f64(static_cast<uint16_t>(w[u] >> 16))));
      }
      *reinterpret_cast<uint4*>(kst + e * DI + lane * 4) = make_uint4(h[0], h[1], h[2], h[3]);
    }
  }
  __syncwarp();
  double pr[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) pr[e] = 0.0;
  if (lane < HI) {
    const uint4* q4 = reinterpret_cast<const uint4*>(qhi + lane * (DI + 4));
    double acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.0;
#pragma unroll 2
    for (int c4 = 0; c4 < DI / 4; ++c4) {
      const uint4 qq = q4[c4];
      const double qd[4] = {__hiloint2double(static_cast<int>(qq.x), 0), __hiloint2double(static_cast<int>(qq.y), 0),
                            __hiloint2double(static_cast<int>(qq.z), 0), __hiloint2double(static_cast<int>(qq.w), 0)};
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const uint4 kk = reinterpret_cast<const uint4*>(kst + e * DI)[c4];
        acc[e] = fma(qd[0], __hiloint2double(static_cast<int>(kk.x), 0), acc[e]);
        acc[e] = fma(qd[1], __hiloint2double(static_cast<int>(kk.y), 0), acc[e]);
        acc[e] = fma(qd[2], __hiloint2double(static_cast<int>(kk.z), 0), acc[e]);
        acc[e] = fma(qd[3], __hiloint2double(static_cast<int>(kk.w), 0), acc[e]);
      }
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) pr[e] = __dmul_rn(w_lane, acc[e] > 0.0 ? acc[e] : 0.0);
  }
  __syncwarp();
  double* prod = reinterpret_cast<double*>(kst);
  if (lane < HI) {
#pragma unroll
    for (int e = 0; e < 8; ++e) prod[e * 34 + lane] = pr[e];
  }
  __syncwarp();
  double sum = 0.0;
  if (lane < 8) {
    const double2* pe = reinterpret_cast<const double2*>(prod + lane * 34);
#pragma unroll
    for (int j2 = 0; j2 < 16; ++j2) {
      if (2 * j2 < HI) {
        const double2 v = pe[j2];
        sum = __dadd_rn(sum, v.x);
        sum = __dadd_rn(sum, v.y);  // HI is even
      }
    }
  }
  __syncwarp();
  return sum;
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
  int n_cap;  // capacity of the score row (max row length, multiple of 4)
  int bcap;   // band cache capacity (refine only)
  int kst_extra;  // bytes of key staging after cand: kKstExtraBytes (8 re-score warps) or 0 (4)
  int kst_warps;  // warps that re-score band keys (8, or 4 when shared memory is short)
  // Two-level select for rows longer than one CTA's shared memory holds.
  // pass 1 takes each row's keys in segments of seg_len and writes every
  // segment's own top-k (ascending keys) to cand [n_q][n_seg][k]; pass 2
  // selects each row's top-k among those candidates. Every segment before a
  // row's last non-empty one holds seg_len >= k keys and gives exactly k
  // candidates, so a row's candidates are ascending keys with -1 only at the
  // end, and the (score, key) order among them is the order of positions.
  // pass 0 is the one-level select.
  int pass, seg_len, n_seg;
  int32_t* cand;
  // the window select (topk_window_kernel): words of its kept-key bitmap;
  // only_marked makes topk_kernel redo only the rows the window select
  // handed back
  int fw_words;
  int only_marked;
};

// kPass: 0 the one-level select, 1 and 2 the two passes of the long-row
// select (a template parameter, so that the one-level kernel carries none of
// the other passes' key mapping)
template <bool kRefine, int kPass>
__device__ __forceinline__ void topk_row(const TopkArgs& a, int blk, unsigned char* smem, Scratch& sm) {
  const int k = a.k;
  int row, n, key_off = 0;
  const int32_t* kmap = nullptr;  // pass 2: key of each position of the candidate row
  int32_t* out;
  if (kPass == 1) {  // segment seg of the row
    row = blk / a.n_seg;
    const int seg = blk - row * a.n_seg;
    key_off = seg * a.seg_len;
    n = min(a.seg_len, a.q_pos0 + row + 1 - key_off);
    out = a.cand + (static_cast<int64_t>(row) * a.n_seg + seg) * k;
    if (n <= 0) {  // a segment past the query's position
      for (int c = threadIdx.x; c < k; c += kThreads) out[c] = -1;
      return;
    }
  } else if (kPass == 2) {  // the row's candidates
    row = blk;
    const int t = a.q_pos0 + row;
    const int nv = t / a.seg_len + 1;  // non-empty segments
    n = (nv - 1) * k + min(k, t + 1 - (nv - 1) * a.seg_len);
    kmap = a.cand + static_cast<int64_t>(row) * a.n_seg * k;
    out = a.idx + static_cast<int64_t>(row) * k;
  } else {
    row = blk;
    n = a.q_pos0 + row + 1;
    out = a.idx + static_cast<int64_t>(row) * k;
  }

  if (n <= k) {  // every key of the row (or segment, or candidate list) is kept
    for (int c = threadIdx.x; c < k; c += kThreads)
      out[c] = c < n ? (kmap ? __ldg(kmap + c) : c + key_off) : -1;
    return;
  }

  float* sc = reinterpret_cast<float*>(smem);
  int* hist = reinterpret_cast<int*>(smem + sizeof(float) * a.n_cap);
  float* cand = reinterpret_cast<float*>(hist + kBins);
  // refine scratch after cand (see kKstExtraBytes / kQRowBytes): the q row as
  // float64 high words in padded rows of DI + 4 words
  uint32_t* qhi = reinterpret_cast<uint32_t*>(reinterpret_cast<unsigned char*>(cand + kCandCap) +
                                              (kRefine ? a.kst_extra : 0));
  const int qstride = a.DI + 4;
  const uint16_t* qrow = kRefine ? a.q_idx + static_cast<int64_t>(row) * a.HI * a.DI : nullptr;

  // head weight of head `lane` and max ||k_idx||, loaded now and used after the
  // select, so that their latency hides under it
  float w_pre = 0.f;
  unsigned long long kmax_pre = 0ull;
  if (kRefine) {
    const int lane0 = threadIdx.x & 31;
    if (lane0 < a.HI) w_pre = __ldg(a.w_idx + static_cast<int64_t>(row) * a.HI + lane0);
    kmax_pre = *reinterpret_cast<volatile unsigned long long*>(&a.ws->kmax_bits);
  }

  // ---- stage the row (and the query's indexer row) with asynchronous copies
  const float* srow = a.scores + static_cast<int64_t>(row) * a.ld + key_off;
  const int n4 = kmap ? 0 : n & ~3;  // pass 2 gathers its candidates' scores below
  for (int s = threadIdx.x * 4; s < n4; s += kThreads * 4) cp_async16(sc + s, srow + s);
  // the q row, widened to float64 once while the copies fly (only the high
  // words are kept), and this warp's share of A_t = sum_j |w_j| ||q_j||
  // (heads warp, warp + 12, ...; float64 from the widened values)
  if (kRefine) {
    constexpr int kHeadsPerWarp = (32 + kWarps - 1) / kWarps;
    const int wpr = a.DI / 2;  // bf16 pairs per row
    const uint32_t* q32 = reinterpret_cast<const uint32_t*>(qrow);
    const int w0 = threadIdx.x >> 5, l0 = threadIdx.x & 31;
    // every bf16 pair this lane widens (at most two per head: DI <= 128) is
    // loaded before the first is used, so the loads overlap
    uint32_t qv[kHeadsPerWarp][2];
#pragma unroll
    for (int u = 0; u < kHeadsPerWarp; ++u) {
      const int j = w0 + u * kWarps;
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const int pr = l0 + 32 * t;
        qv[u][t] = (j < a.HI && pr < wpr) ? __ldg(q32 + j * wpr + pr) : 0u;
      }
    }
    double acc = 0.0;
#pragma unroll
    for (int u = 0; u < kHeadsPerWarp; ++u) {
      const int j = w0 + u * kWarps;
      double ss = 0.0;
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const int pr = l0 + 32 * t;
        if (j < a.HI && pr < wpr && DSA_IN_BOUNDS(a.ws, j * qstride + 2 * pr + 1, kQRowBytes / 4, 3)) {
          const uint32_t v = qv[u][t];
          const double lo = static_cast<double>(__uint_as_float(v << 16));
          const double hi = static_cast<double>(__uint_as_float(v & 0xFFFF0000u));
          qhi[j * qstride + 2 * pr] = static_cast<uint32_t>(__double2hiint(lo));
          qhi[j * qstride + 2 * pr + 1] = static_cast<uint32_t>(__double2hiint(hi));
          ss += lo * lo;
          ss += hi * hi;
        }
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      const float wj = __shfl_sync(0xffffffffu, w_pre, j & 31);
      if (j < a.HI) acc += fabs(static_cast<double>(wj)) * sqrt(ss);
    }
    if (l0 == 0) sm.wd[w0] = acc;
  }
  for (int s = n4 + threadIdx.x; s < n; s += kThreads) {
    int key = s;
    if (kmap) {
      key = __ldg(kmap + s);
      if (key < 0 || key > a.q_pos0 + row) {  // pass 1 wrote no such candidate
        report(a.ws, kDevInternal, static_cast<unsigned>(row));
        key = 0;
      }
    }
    sc[s] = __ldg(srow + key);
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncthreads();
  // canonicalise -0 and find the row's range
  float mn = INFINITY, mx = -INFINITY;
  for (int s = threadIdx.x * 4; s < n4; s += kThreads * 4) {
    float4 v = *reinterpret_cast<const float4*>(sc + s);
    v.x = canon(v.x);
    v.y = canon(v.y);
    v.z = canon(v.z);
    v.w = canon(v.w);
    *reinterpret_cast<float4*>(sc + s) = v;
    mn = fminf(fminf(mn, v.x), fminf(fminf(v.y, v.z), v.w));
    mx = fmaxf(fmaxf(mx, v.x), fmaxf(fmaxf(v.y, v.z), v.w));
  }
  for (int s = n4 + threadIdx.x; s < n; s += kThreads) {
    const float v = canon(sc[s]);
    sc[s] = v;
    mn = fminf(mn, v);
    mx = fmaxf(mx, v);
  }
  block_minmax(mn, mx, sm);  // also makes sc[] visible to all threads

  float vk;
  int n_above;
  if (!kth_largest(sc, n, k, mn, mx, hist, cand, sm, &vk, &n_above, a.ws)) {
    if (threadIdx.x == 0) report(a.ws, kDevInternal, static_cast<unsigned>(row));
    return;
  }

  if (!kRefine) {
    emit_selection(
        sc, n, k - n_above, k, out, hist,
        [&](float v) { return v > vk ? kAbove : (v == vk ? kTie : kBelow); }, sm, a.ws, row, -1, key_off, kmap);
    return;
  }

  // ---------------- exact float64 order: certified band + float64 re-score
  const int HI = a.HI, DI = a.DI;
  // the key (cache row) at position s of the staged row
  auto key_of = [&](int s) { return kmap ? __ldg(kmap + s) : s + key_off; };
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  unsigned char* p = reinterpret_cast<unsigned char*>(qhi) + kQRowBytes;
  unsigned long long* bx = reinterpret_cast<unsigned long long*>(p);   // band cache
  int* bidx = reinterpret_cast<int*>(p + sizeof(unsigned long long) * a.bcap);
  int* hist256 = reinterpret_cast<int*>(p);                            // slow path only
  int* tile_s = hist256 + 256;
  double* tile_x = reinterpret_cast<double*>(tile_s + kThreads);
  // after the select: hist (+ cand + extra) hold the re-score's key staging,
  // 2 KB per re-scoring warp
  uint32_t* kst_all = reinterpret_cast<uint32_t*>(hist);
  const int kw = a.kst_warps;

  // A_t from the warps' shares formed while the row was staged (visible
  // since the select's block barriers), rounded up by a relative slack
  double A = 0.0;
  for (int w = 0; w < kWarps; ++w) A += sm.wd[w];
  A *= kNormSlack;
  const double kmax = __longlong_as_double(static_cast<long long>(kmax_pre));
  const double delta = kBoundRel * A * kmax;
  const double lo = static_cast<double>(vk) - 2.0 * delta;
  const double hi = static_cast<double>(vk) + 2.0 * delta;
  // the same tests on float scores: f >= lo <=> f >= RU(lo), f > hi <=> f > RD(hi)
  const float lo_f = __double2float_ru(lo);
  const float hi_f = __double2float_rd(hi);

  int beg, end;
  my_segment(n, beg, end);
  // one pass: count the certainly-kept keys and the band, collecting band keys
  // (any order) while they fit the cache
  if (threadIdx.x == 0) sm.bc[2] = 0;
  __syncthreads();
  // (the first two band keys of the segment are noted, so that the emit can
  // count the kept keys of the segment without a pass over it)
  int c_in = 0, c_band = 0, bk0 = -1, bk1 = -1;
  for_segment(sc, beg, end, [&](int s, float f) {
    c_in += f > hi_f;
    if (f >= lo_f && f <= hi_f) {
      if (c_band == 0) bk0 = s;
      if (c_band == 1) bk1 = s;
      ++c_band;
      const int pos = atomicAdd(&sm.bc[2], 1);
      if (pos < a.bcap) bidx[pos] = s;
    }
  });
  unsigned long long tot;
  block_excl_scan64(
      static_cast<unsigned long long>(c_in) | (static_cast<unsigned long long>(c_band) << 32),
      &tot, sm);
  const int tot_in = static_cast<int>(tot & 0xffffffffu);
  const int tot_band = static_cast<int>(tot >> 32);
  const int r = k - tot_in;  // band keys still to keep, 1 <= r <= tot_band

  if (r == tot_band) {  // the whole band is kept: no re-score needed
    emit_selection(
        sc, n, 0, k, out, hist, [&](float v) { return v >= lo_f ? kAbove : kBelow; }, sm, a.ws, row,
        c_in + c_band, key_off, kmap);
    return;
  }

  const double w_lane = lane < HI ? static_cast<double>(w_pre) : 0.0;
  uint32_t* my_kst = kst_all + warp * 512;

  if (tot_band <= a.bcap) {
    // re-score the collected band four keys per warp call (the next four rows
    // are loaded while the current ones are scored), rank it by (X desc,
    // index asc), and mark the row: kept band keys -> +inf, dropped -> -inf
    int b = warp < kw ? 4 * warp : tot_band;
    uint2 raw[4];
#pragma unroll
    for (int e = 0; e < 4; ++e)
      raw[e] = b < tot_band ? load_key_part(a.k_idx, key_of(bidx[min(b + e, tot_band - 1)]), DI) : make_uint2(0u, 0u);
    for (; b < tot_band; b += 4 * kw) {
      const int bn = b + 4 * kw;
      uint2 nraw[4];
#pragma unroll
      for (int e = 0; e < 4; ++e)
        nraw[e] = bn < tot_band ? load_key_part(a.k_idx, key_of(bidx[min(bn + e, tot_band - 1)]), DI)
                                : make_uint2(0u, 0u);
      const double xl = DI == 128 ? rescore4<128>(qhi, w_lane, raw, my_kst, HI)
                                  : rescore4<32>(qhi, w_lane, raw, my_kst, HI);
      if (lane < 4 && b + lane < tot_band && DSA_IN_BOUNDS(a.ws, b + lane, a.bcap, 4))
        bx[b + lane] = d2key(xl);
#pragma unroll
      for (int e = 0; e < 4; ++e) raw[e] = nraw[e];
    }
    __syncthreads();
    // rank of each band key by (X desc, index asc): a warp takes four keys at
    // a time, its lanes counting over the band for all four at once
    for (int b0 = 4 * warp; b0 < tot_band; b0 += 4 * kWarps) {
      unsigned long long xb[4];
      int sb[4], rank[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int b = min(b0 + e, tot_band - 1);
        xb[e] = bx[b];
        sb[e] = bidx[b];
        rank[e] = 0;
      }
      for (int o = lane; o < tot_band; o += 32) {
        const unsigned long long xo = bx[o];
        const int so = bidx[o];
#pragma unroll
        for (int e = 0; e < 4; ++e) rank[e] += (xo > xb[e]) || (xo == xb[e] && so < sb[e]);
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) rank[e] = __reduce_add_sync(0xffffffffu, rank[e]);
      const int my_rank = lane == 0 ? rank[0] : lane == 1 ? rank[1] : lane == 2 ? rank[2] : rank[3];
      const int my_s = lane == 0 ? sb[0] : lane == 1 ? sb[1] : lane == 2 ? sb[2] : sb[3];
      if (lane < 4 && b0 + lane < tot_band && DSA_IN_BOUNDS(a.ws, my_s, n, 5))
        sc[my_s] = my_rank < r ? INFINITY : -INFINITY;
    }
    const bool counted = __syncthreads_or(c_band > 2) == 0;
    const int kept = c_in + (bk0 >= 0 && sc[bk0] > hi_f) + (bk1 >= 0 && sc[bk1] > hi_f);
    emit_selection(
        sc, n, 0, k, out, hist, [&](float v) { return v > hi_f ? kAbove : kBelow; }, sm, a.ws, row,
        counted ? kept : -1, key_off, kmap);
    return;
  }

  // ---- band larger than the cache (degenerate inputs): radix select over the
  // band's float64 keys, 8 bits per pass, re-scoring the band in every pass in
  // windows of kThreads consecutive keys.
  auto band_window = [&](int base) -> int {  // tile_s/tile_x[0..nb) = band keys of the window
    const int s = base + threadIdx.x;
    int flag = 0;
    if (s < n) {
      const float f = sc[s];
      flag = (f >= lo_f && f <= hi_f) ? 1 : 0;
    }
    unsigned long long nb64;
    const int j = static_cast<int>(block_excl_scan64(static_cast<unsigned long long>(flag), &nb64, sm));
    const int nb = static_cast<int>(nb64);
    if (flag && DSA_IN_BOUNDS(a.ws, j, kThreads, 6)) tile_s[j] = s;
    __syncthreads();
    for (int jj = warp < kw ? 4 * warp : nb; jj < nb; jj += 4 * kw) {
      uint2 raw[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) raw[e] = load_key_part(a.k_idx, key_of(tile_s[min(jj + e, nb - 1)]), DI);
      const double xl = DI == 128 ? rescore4<128>(qhi, w_lane, raw, my_kst, HI)
                                  : rescore4<32>(qhi, w_lane, raw, my_kst, HI);
      if (lane < 4 && jj + lane < nb) tile_x[jj + lane] = xl;
    }
    __syncthreads();
    return nb;
  };
  unsigned long long pre = 0ull, msk = 0ull;
  int rr = r;
  for (int shift = 56; shift >= 0; shift -= 8) {
    for (int b = threadIdx.x; b < 256; b += kThreads) hist256[b] = 0;
    __syncthreads();
    for (int base = 0; base < n; base += kThreads) {
      const int nb = band_window(base);
      if (static_cast<int>(threadIdx.x) < nb) {
        const unsigned long long key = d2key(tile_x[threadIdx.x]);
        const int hb = static_cast<int>((key >> shift) & 0xFFull);
        if ((key & msk) == pre && DSA_IN_BOUNDS(a.ws, hb, 256, 7)) atomicAdd(&hist256[hb], 1);
      }
      __syncthreads();
    }
    int ab;
    const int bin = find_bin_from_top<256>(hist256, rr, &ab, sm);
    rr -= ab;
    pre |= static_cast<unsigned long long>(bin) << shift;
    msk |= 0xFFull << shift;
  }
  // mark the band: above the r-th largest -> +inf, equal -> NaN (a tie), below -> -inf
  for (int base = 0; base < n; base += kThreads) {
    const int nb = band_window(base);
    if (static_cast<int>(threadIdx.x) < nb) {
      const unsigned long long key = d2key(tile_x[threadIdx.x]);
      sc[tile_s[threadIdx.x]] = key > pre ? INFINITY : (key == pre ? NAN : -INFINITY);
    }
    __syncthreads();
  }
  emit_selection(
      sc, n, rr, k, out, hist,
      [&](float v) {
        if (isnan(v)) return kTie;
        return v > hi_f ? kAbove : kBelow;
      },
      sm, a.ws, row, -1, key_off, kmap);
}


// One CTA per row (or row segment, or candidate list); with only_marked a
// grid of a few CTAs per SM scans for the rows (pass 0) or row segments
// (pass 1) the window select handed back and redoes those alone.
template <bool kRefine, int kPass>
__global__ void __launch_bounds__(kThreads, 2) topk_kernel(TopkArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ Scratch sm;
  if (!a.only_marked) {
    topk_row<kRefine, kPass>(a, blockIdx.x, smem, sm);
    return;
  }
  if (*reinterpret_cast<volatile unsigned int*>(&a.ws->topk_redo) == 0u) return;
  __shared__ unsigned int s_mask[kWarps];  // per warp: which of its 32 rows are marked
  const int n_blk = kPass == 1 ? a.n_q * a.n_seg : a.n_q;
  int32_t* const base_out = kPass == 1 ? a.cand : a.idx;
  for (int base = blockIdx.x * kThreads; base < n_blk; base += gridDim.x * kThreads) {
    const int b = base + static_cast<int>(threadIdx.x);
    const bool marked =
        b < n_blk &&
        *reinterpret_cast<volatile int32_t*>(base_out + static_cast<int64_t>(b) * a.k) == kRedoMarker;
    const unsigned int m = __ballot_sync(0xffffffffu, marked);
    if ((threadIdx.x & 31) == 0) s_mask[threadIdx.x >> 5] = m;
    __syncthreads();
    for (int w = 0; w < kWarps; ++w) {
      unsigned int mw = s_mask[w];
      while (mw) {
        const int bit = __ffs(mw) - 1;
        mw &= mw - 1u;
        topk_row<kRefine, kPass>(a, base + 32 * w + bit, smem, sm);
        __syncthreads();
      }
    }
  }
}

// ---------------------------------------------------------------------------
// The one-level exact select without the row in shared memory: the window
// select. One CTA of 192 threads per row and about 50 KB of shared memory, so
// four rows share an SM (topk_kernel, which stages the row, fits two). The
// row is read from global memory (from L2 after its first pass) in coalesced
// chunks of 128 keys, a warp per chunk:
//   1. the row's range [L, U];
//   2. a histogram over 2,048 buckets of the range, and the bucket b* that
//      holds the k-th largest float score v;
//   3. the window pass: the keys above a window around b*, widened by
//      2 delta on either side (delta as in topk_kernel), go into a bitmap of
//      the row, and the window's keys are collected with their scores. Every
//      key within 2 delta of v is in the window, so v, the keys certainly
//      kept (above v + 2 delta) and the band [v - 2 delta, v + 2 delta] follow
//      from the window alone;
//   4. the band re-scored in float64 in the contract's order and ranked by
//      (X desc, key asc), exactly as in topk_kernel; the window's kept keys
//      are added to the bitmap;
//   5. the emit: a scan of the bitmap words' populations places the kept
//      keys in ascending order.
// A row whose range is a single value or too wide for a float bucket scale,
// or whose window holds more than kWinCap keys (heavy ties), is handed back:
// its first index is set to kRedoMarker and counted in the workspace header,
// and a second launch of topk_kernel redoes those rows alone.
constexpr int kFThreads = 192;
constexpr int kFWarps = kFThreads / 32;
constexpr int kFChunk = 128;
constexpr int kWinCap = 256;
// hist (2,048 ints), or the re-score's key staging: per warp 1,024 words,
// eight keys of up to 128 dims as float64 high words and then the head sum's
// [8][34] float64 products
constexpr int kFKstWords = 1024;
static_assert(kFKstWords >= 8 * 128 && kFKstWords * 4 >= 8 * 34 * 8, "window select key staging");
constexpr int kFRegionBytes = (kBins * 4 > kFWarps * kFKstWords * 4) ? kBins * 4 : kFWarps * kFKstWords * 4;

// kSeg: pass 1 of the long-row select (topk_kernel's pass 1): CTA (row,
// segment) selects among the segment's keys key_off .. key_off + n - 1 and
// writes them to the candidate buffer.
template <int DI, bool kSeg>
__global__ void __launch_bounds__(kFThreads, 4) topk_window_kernel(TopkArgs a) {
  extern __shared__ __align__(16) unsigned char smem[];
  __shared__ Scratch sm;
  __shared__ int s_ncand, s_chi;
  const int k = a.k;
  int row, n, key_off = 0;
  int32_t* out;
  if (kSeg) {
    row = blockIdx.x / a.n_seg;
    const int seg = blockIdx.x - row * a.n_seg;
    key_off = seg * a.seg_len;
    n = min(a.seg_len, a.q_pos0 + row + 1 - key_off);
    out = a.cand + (static_cast<int64_t>(row) * a.n_seg + seg) * k;
    if (n <= 0) {  // a segment past the query's position
      for (int c = threadIdx.x; c < k; c += kFThreads) out[c] = -1;
      return;
    }
  } else {
    row = blockIdx.x;
    n = a.q_pos0 + row + 1;
    out = a.idx + static_cast<int64_t>(row) * k;
  }
  if (n <= k) {  // every key is kept
    for (int c = threadIdx.x; c < k; c += kFThreads) out[c] = c < n ? c + key_off : -1;
    return;
  }
  const int HI = a.HI;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_chunks = (n + kFChunk - 1) / kFChunk;
  // shared memory: hist (later the emit's staging; the re-score's key
  // staging in between) | q row (float64 high words) | band cache |
  // kept-key bitmap | window keys and scores
  int* hist = reinterpret_cast<int*>(smem);
  // (the re-score's float64 key staging overlays hist, idle in that phase)
  double* kst_all = reinterpret_cast<double*>(smem);
  uint32_t* qhi = reinterpret_cast<uint32_t*>(smem + kFRegionBytes);
  unsigned long long* bx = reinterpret_cast<unsigned long long*>(
      reinterpret_cast<unsigned char*>(qhi) + kQRowBytes);
  int* bidx = reinterpret_cast<int*>(bx + kWinCap);
  uint32_t* bits = reinterpret_cast<uint32_t*>(bidx + kWinCap);
  int* cand_pos = reinterpret_cast<int*>(bits + a.fw_words);
  float* cand_val = reinterpret_cast<float*>(cand_pos + kWinCap);
  const int qstride = DI + 4;

  const float w_pre = lane < HI ? __ldg(a.w_idx + static_cast<int64_t>(row) * HI + lane) : 0.f;
  const unsigned long long kmax_bits = *reinterpret_cast<volatile unsigned long long*>(&a.ws->kmax_bits);
  for (int b = threadIdx.x; b < kBins; b += kFThreads) hist[b] = 0;
  if (threadIdx.x == 0) {
    s_ncand = 0;
    s_chi = 0;
  }
  // the q row widened to float64 high words, and this warp's share of
  // A_t = sum_j |w_j| ||q_j|| (heads warp, warp + 6, ...)
  {
    constexpr int kHeadsPerWarp = (32 + kFWarps - 1) / kFWarps;
    const int wpr = DI / 2;
    const uint32_t* q32 = reinterpret_cast<const uint32_t*>(a.q_idx + static_cast<int64_t>(row) * HI * DI);
    uint32_t qv[kHeadsPerWarp][2];
#pragma unroll
    for (int u = 0; u < kHeadsPerWarp; ++u) {
      const int j = warp + u * kFWarps;
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const int pr = lane + 32 * t;
        qv[u][t] = (j < HI && pr < wpr) ? __ldg(q32 + j * wpr + pr) : 0u;
      }
    }
    double acc = 0.0;
#pragma unroll
    for (int u = 0; u < kHeadsPerWarp; ++u) {
      const int j = warp + u * kFWarps;
      double ss = 0.0;
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        const int pr = lane + 32 * t;
        if (j < HI && pr < wpr && DSA_IN_BOUNDS(a.ws, j * qstride + 2 * pr + 1, kQRowBytes / 4, 50)) {
          const uint32_t v = qv[u][t];
          const double lo = static_cast<double>(__uint_as_float(v << 16));
          const double hi = static_cast<double>(__uint_as_float(v & 0xFFFF0000u));
          qhi[j * qstride + 2 * pr] = static_cast<uint32_t>(__double2hiint(lo));
          qhi[j * qstride + 2 * pr + 1] = static_cast<uint32_t>(__double2hiint(hi));
          ss += lo * lo;
          ss += hi * hi;
        }
      }
#pragma unroll
      for (int o = 16; o; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
      const float wj = __shfl_sync(0xffffffffu, w_pre, j & 31);
      if (j < HI) acc += fabs(static_cast<double>(wj)) * sqrt(ss);
    }
    if (lane == 0) sm.wd[warp] = acc;
  }

  // ---- 1. the row's range
  const float* srow = a.scores + static_cast<int64_t>(row) * a.ld + key_off;  // (key_off % 4 == 0)
  const float4* s4 = reinterpret_cast<const float4*>(srow);
  const int n4 = n >> 2;
  float mn = INFINITY, mx = -INFINITY;
  for (int i = threadIdx.x; i < n4; i += kFThreads) {
    const float4 v = __ldg(s4 + i);
    mn = fminf(fminf(mn, v.x), fminf(fminf(v.y, v.z), v.w));
    mx = fmaxf(fmaxf(mx, v.x), fmaxf(fmaxf(v.y, v.z), v.w));
  }
  for (int s = 4 * n4 + threadIdx.x; s < n; s += kFThreads) {
    const float v = __ldg(srow + s);
    mn = fminf(mn, v);
    mx = fmaxf(mx, v);
  }
  block_minmax<kFThreads>(mn, mx, sm);  // (also orders the zeroing above before its use)
  double A = 0.0;
  for (int w = 0; w < kFWarps; ++w) A += sm.wd[w];
  A *= kNormSlack;
  const double delta = kBoundRel * A * __longlong_as_double(static_cast<long long>(kmax_bits));
  const Bucketer bucket(mn, mx);
  bool redo = !(mn < mx) || !bucket.wide || !(delta < 1e30);

  float whi_f = 0.f, lo_f = 0.f, hi_f = 0.f;
  int c_hi_tot = 0;
  if (!redo) {
    // ---- 2. histogram and the bucket of the k-th largest
    for (int i = threadIdx.x; i < n4; i += kFThreads) {
      const float4 v = __ldg(s4 + i);
      atomicAdd(&hist[bucket(v.x)], 1);
      atomicAdd(&hist[bucket(v.y)], 1);
      atomicAdd(&hist[bucket(v.z)], 1);
      atomicAdd(&hist[bucket(v.w)], 1);
    }
    for (int s = 4 * n4 + threadIdx.x; s < n; s += kFThreads) atomicAdd(&hist[bucket(__ldg(srow + s))], 1);
    __syncthreads();
    int ab;
    const int bstar = find_bin_from_top<kBins, kFThreads>(hist, k, &ab, sm);
    // a value in bucket b lies within (b +- 0.5) bucket widths of L up to
    // float rounding (relative 2^-21 of at most 2048 widths); the window
    // allows 1.5 widths and 2 delta on either side
    const double width = (static_cast<double>(mx) - static_cast<double>(mn)) / kBins;
    const float wlo_f = __double2float_rd(static_cast<double>(mn) + (bstar - 1.5) * width - 2.0 * delta);
    whi_f = __double2float_ru(static_cast<double>(mn) + (bstar + 1.5) * width + 2.0 * delta);

    // ---- 3. the window pass
    int c_hi = 0;
    for (int c = warp; c < n_chunks; c += kFWarps) {
      const int s0 = c * kFChunk + 4 * lane;
      float v[4];
      if (s0 + 3 < n) {
        const float4 f4 = __ldg(reinterpret_cast<const float4*>(srow + s0));
        v[0] = f4.x; v[1] = f4.y; v[2] = f4.z; v[3] = f4.w;
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) v[e] = s0 + e < n ? __ldg(srow + s0 + e) : -INFINITY;
      }
      int above = 0;
      uint32_t mine = 0u;  // this lane's keys above the window, as bits of its chunk word
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float f = v[e];
        const bool up = f > whi_f;
        above += up;
        mine |= static_cast<uint32_t>(up) << (4 * (lane & 7) + e);
        if (s0 + e < n && f >= wlo_f && f <= whi_f) {
          const int pos = atomicAdd(&s_ncand, 1);
          if (pos < kWinCap) {
            cand_pos[pos] = s0 + e;
            cand_val[pos] = f;
          }
        }
      }
      // the chunk's four bitmap words (keys c * 128 + 32 g .. + 31 from lanes
      // 8 g .. 8 g + 7), written by one lane each; the window's kept keys are
      // added after this pass
      mine |= __shfl_xor_sync(0xffffffffu, mine, 1);
      mine |= __shfl_xor_sync(0xffffffffu, mine, 2);
      mine |= __shfl_xor_sync(0xffffffffu, mine, 4);
      if ((lane & 7) == 0 && DSA_IN_BOUNDS(a.ws, c * 4 + (lane >> 3), a.fw_words, 51))
        bits[c * 4 + (lane >> 3)] = mine;
      c_hi += __reduce_add_sync(0xffffffffu, above);
    }
    if (lane == 0) atomicAdd(&s_chi, c_hi);
    __syncthreads();
    const int n_cand = s_ncand;
    c_hi_tot = s_chi;
    redo = !(n_cand <= kWinCap && c_hi_tot < k && c_hi_tot + n_cand >= k);
    if (!redo) {
      // ---- 4. v, the certainly kept keys and the band, from the window
      const int kr = k - c_hi_tot;
      for (int i = threadIdx.x; i < n_cand; i += kFThreads) {
        const float vi = cand_val[i];
        int gt = 0, ge = 0;
        for (int o = 0; o < n_cand; ++o) {
          const float u = cand_val[o];
          gt += u > vi;
          ge += u >= vi;
        }
        if (gt < kr && kr <= ge) sm.bf[0] = vi;
      }
      __syncthreads();
      const float vk = sm.bf[0];
      lo_f = __double2float_ru(static_cast<double>(vk) - 2.0 * delta);
      hi_f = __double2float_rd(static_cast<double>(vk) + 2.0 * delta);
      if (warp == 0) {  // kept above hi_f; the band in window order
        int nb = 0, nin = 0;
        for (int i0 = 0; i0 < n_cand; i0 += 32) {
          const int i = i0 + lane;
          const bool valid = i < n_cand;
          const int s2 = valid ? cand_pos[i] : 0;
          const float f = valid ? cand_val[i] : 0.f;
          const bool in_band = valid && f >= lo_f && f <= hi_f;
          const bool above2 = valid && f > hi_f;
          const unsigned mb = __ballot_sync(0xffffffffu, in_band);
          nin += __popc(__ballot_sync(0xffffffffu, above2));
          if (in_band) bidx[nb + __popc(mb & ((1u << lane) - 1u))] = s2;
          if (above2) atomicOr(&bits[s2 >> 5], 1u << (s2 & 31));
          nb += __popc(mb);
        }
        if (lane == 0) {
          sm.bc[0] = nb;
          sm.bc[1] = nin;
        }
      }
      __syncthreads();
      const int tot_band = sm.bc[0];
      const int r = k - (c_hi_tot + sm.bc[1]);  // band keys still to keep, 1 <= r <= tot_band
      if (r == tot_band) {  // the whole band is kept
        for (int i = threadIdx.x; i < tot_band; i += kFThreads) {
          const int s2 = bidx[i];
          atomicOr(&bits[s2 >> 5], 1u << (s2 & 31));
        }
      } else {
        // re-score the band four keys per warp call (the next four key rows
        // are loaded while the current ones are scored)
        const double w_lane = lane < HI ? static_cast<double>(w_pre) : 0.0;
        // (4 KB per warp: eight 128-dim keys, or the [8][34] float64 products)
        uint32_t* my_kst = reinterpret_cast<uint32_t*>(kst_all) + warp * kFKstWords;
        for (int b = 8 * warp; b < tot_band; b += 8 * kFWarps) {
          uint2 raw[8];
#pragma unroll
          for (int e = 0; e < 8; ++e)
            raw[e] = load_key_part(a.k_idx, bidx[min(b + e, tot_band - 1)] + key_off, DI);
          const double xl = rescore8h<DI>(qhi, w_lane, raw, my_kst, HI);
          if (lane < 8 && b + lane < tot_band && DSA_IN_BOUNDS(a.ws, b + lane, kWinCap, 52))
            bx[b + lane] = d2key(xl);
        }
        __syncthreads();
        // rank by (X desc, key asc): a warp takes four band keys at a time
        for (int b0 = 4 * warp; b0 < tot_band; b0 += 4 * kFWarps) {
          unsigned long long xb[4];
          int sb[4], rank[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int bb = min(b0 + e, tot_band - 1);
            xb[e] = bx[bb];
            sb[e] = bidx[bb];
            rank[e] = 0;
          }
          for (int o = lane; o < tot_band; o += 32) {
            const unsigned long long xo = bx[o];
            const int so = bidx[o];
#pragma unroll
            for (int e = 0; e < 4; ++e) rank[e] += (xo > xb[e]) || (xo == xb[e] && so < sb[e]);
          }
#pragma unroll
          for (int e = 0; e < 4; ++e) rank[e] = __reduce_add_sync(0xffffffffu, rank[e]);
          const int my_rank = lane == 0 ? rank[0] : lane == 1 ? rank[1] : lane == 2 ? rank[2] : rank[3];
          const int my_s = lane == 0 ? sb[0] : lane == 1 ? sb[1] : lane == 2 ? sb[2] : sb[3];
          if (lane < 4 && b0 + lane < tot_band && my_rank < r && DSA_IN_BOUNDS(a.ws, my_s, n, 53)) {
            atomicOr(&bits[my_s >> 5], 1u << (my_s & 31));
          }
        }
      }
    }
  }
  if (redo) {  // (block-uniform) handed to topk_kernel
    if (threadIdx.x == 0) {
      out[0] = kRedoMarker;
      atomicAdd(&a.ws->topk_redo, 1u);
    }
    return;
  }
  __syncthreads();

  // ---- 5. emit: the bitmap holds exactly the kept keys; a scan of the words'
  // populations places each thread's words (a contiguous run) in order
  int32_t* stage = hist;  // the selection, assembled in shared memory
  {
    const int n_words = (n + 31) / 32;
    const int per = (n_words + kFThreads - 1) / kFThreads;
    const int w0 = min(static_cast<int>(threadIdx.x) * per, n_words), w1 = min(w0 + per, n_words);
    int cnt = 0;
    for (int w = w0; w < w1; ++w) cnt += __popc(bits[w]);
    unsigned long long tot;
    int pos = static_cast<int>(block_excl_scan64<kFThreads>(static_cast<unsigned long long>(cnt), &tot, sm));
    if (threadIdx.x == 0 && static_cast<int>(tot) != k) report(a.ws, kDevInternal, static_cast<unsigned>(row));
    for (int w = w0; w < w1; ++w) {
      uint32_t m = bits[w];
      while (m) {
        const int bit = __ffs(m) - 1;
        m &= m - 1u;
        if (pos < k && DSA_IN_BOUNDS(a.ws, pos, kBins, 54)) stage[pos] = 32 * w + bit + key_off;
        ++pos;
      }
    }
  }
  __syncthreads();
  if ((k & 3) == 0) {
    for (int i = threadIdx.x; i < k / 4; i += kFThreads)
      reinterpret_cast<int4*>(out)[i] = reinterpret_cast<const int4*>(stage)[i];
  } else {
    for (int i = threadIdx.x; i < k; i += kFThreads) out[i] = stage[i];
  }
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

namespace {

// Rows up to kOneLevelRow keys are selected in one pass; longer ones in
// segments of at most kMaxSegment keys.
constexpr int kOneLevelRow = 49152;
constexpr int kMaxSegment = 32768;

struct TwoLevel {
  int n_seg = 0, seg_len = 0;
};

TwoLevel two_level(const dsa_dims& d) {
  TwoLevel t;
  const int64_t r = static_cast<int64_t>(d.q_pos0) + d.n_q;  // the longest row
  if (r <= kOneLevelRow) return t;
  t.n_seg = static_cast<int>((r + kMaxSegment - 1) / kMaxSegment);
  t.seg_len = static_cast<int>(((r + t.n_seg - 1) / t.n_seg + 3) & ~int64_t{3});
  return t;
}

template <bool kRefine, int kPass>
cudaError_t launch_instance(const TopkArgs& a, int grid, size_t bytes, cudaStream_t st) {
  const cudaError_t e = cudaFuncSetAttribute(topk_kernel<kRefine, kPass>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             static_cast<int>(bytes));
  if (e != cudaSuccess) return e;
  topk_kernel<kRefine, kPass><<<grid, kThreads, bytes, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_kernel(const TopkArgs& a, int grid, size_t bytes, bool refine, cudaStream_t st) {
  switch (a.pass * 2 + (refine ? 1 : 0)) {
    case 0: return launch_instance<false, 0>(a, grid, bytes, st);
    case 1: return launch_instance<true, 0>(a, grid, bytes, st);
    case 2: return launch_instance<false, 1>(a, grid, bytes, st);
    case 3: return launch_instance<true, 1>(a, grid, bytes, st);
    case 4: return launch_instance<false, 2>(a, grid, bytes, st);
    default: return launch_instance<true, 2>(a, grid, bytes, st);
  }
}

int num_sms_topk() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

// One launch of topk_kernel over `grid` CTAs with rows of up to `row_cap`
// staged scores: picks the shared-memory layout (two CTAs per SM with eight
// re-scoring warps, else one with eight, else one with four) and launches.
cudaError_t launch_pass(TopkArgs a, int row_cap, int grid, bool refine, cudaStream_t st) {
  a.n_cap = (row_cap + 3) & ~3;
  int max_smem = 0, dev = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  // static shared memory of topk_kernel: Scratch and the redo scan's row masks
  const size_t static_bytes = sizeof(Scratch) + sizeof(unsigned int) * kWarps + 64;
  size_t bytes = sizeof(float) * a.n_cap + sizeof(int) * kBins + sizeof(float) * kCandCap;
  a.bcap = 0;
  a.kst_extra = 0;
  a.kst_warps = kRescoreWarps;
  if (refine) {
    // layout after cand: [key staging extra][q row][band cache (>= the slow
    // path's scratch)]
    bytes += kQRowBytes;
    const size_t min_cache = kSlowScratchBytes > 256 * 12 ? kSlowScratchBytes : 256 * 12;
    const size_t full = static_cast<size_t>(max_smem) - static_bytes;
    const size_t half_sm = (228u * 1024u) / 2 - 1024u - static_bytes;
    size_t room;
    if (bytes + kKstExtraBytes + min_cache <= half_sm) {
      a.kst_extra = kKstExtraBytes;
      room = half_sm - bytes - kKstExtraBytes;
    } else if (bytes + kKstExtraBytes + min_cache <= full) {
      a.kst_extra = kKstExtraBytes;
      room = full - bytes - kKstExtraBytes;
    } else if (bytes + min_cache <= full) {
      a.kst_warps = (kBins * 4) / kKstStageBytes;  // the staging fits in hist alone
      room = full - bytes;
    } else {
      return cudaErrorInvalidConfiguration;
    }
    size_t bc = room / (sizeof(unsigned long long) + sizeof(int));
    if (bc > 1024) bc = 1024;
    a.bcap = static_cast<int>(bc);
    bytes += a.kst_extra + a.bcap * (sizeof(unsigned long long) + sizeof(int));
    if (bytes < static_cast<size_t>(a.kst_extra) + kQRowBytes + min_cache) {
      return cudaErrorInvalidConfiguration;  // (unreachable: room >= min_cache)
    }
  } else if (static_cast<size_t>(max_smem) < bytes + static_bytes) {
    return cudaErrorInvalidConfiguration;
  }
  if (a.only_marked) {  // the redo pass scans for handed-back rows with a few CTAs per SM
    const int scan_grid = 2 * num_sms_topk();
    if (grid > scan_grid) grid = scan_grid;
  }
  return launch_kernel(a, grid, bytes, refine, st);
}

// The window select over `grid` rows (or row segments, seg) of at most
// row_cap keys, after clearing the count of handed-back rows.
cudaError_t launch_window(TopkArgs& a, int row_cap, int grid, bool seg, cudaStream_t st) {
  a.fw_words = ((row_cap + 31) / 32 + 3) & ~3;
  const size_t bytes = kFRegionBytes + kQRowBytes +
                       (sizeof(unsigned long long) + sizeof(int)) * kWinCap +
                       sizeof(int) * a.fw_words + (sizeof(int) + sizeof(float)) * kWinCap;
  cudaError_t e = cudaMemsetAsync(&a.ws->topk_redo, 0, sizeof(a.ws->topk_redo), st);
  if (e != cudaSuccess) return e;
  auto go = [&](auto kernel) -> cudaError_t {
    cudaError_t e2 = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          static_cast<int>(bytes));
    if (e2 != cudaSuccess) return e2;
    kernel<<<grid, kFThreads, bytes, st>>>(a);
    return cudaGetLastError();
  };
  if (a.DI == 128) return seg ? go(topk_window_kernel<128, true>) : go(topk_window_kernel<128, false>);
  return seg ? go(topk_window_kernel<32, true>) : go(topk_window_kernel<32, false>);
}

}  // namespace

size_t topk_cand_bytes(const dsa_dims& d) {
  const TwoLevel t = two_level(d);
  return static_cast<size_t>(d.n_q) * t.n_seg * d.top_k * sizeof(int32_t);
}

cudaError_t launch_topk(const dsa_dims& d, const float* scores, int64_t ld, const uint16_t* q_idx,
                        const uint16_t* k_idx, const float* w_idx, int32_t* idx, WsHeader* ws,
                        void* cand, cudaStream_t st) {
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
  a.pass = 0;
  a.seg_len = 0;
  a.n_seg = 0;
  a.cand = nullptr;
  a.fw_words = 0;
  a.only_marked = 0;
  const bool refine = q_idx != nullptr;
  const TwoLevel t = two_level(d);
  const bool window = refine && (d.d_idx == 128 || d.d_idx == 32) && d.n_idx_heads <= 32;
  if (t.n_seg == 0 && window) {
    // the window select, then topk_kernel on the rows it hands back
    const int row_cap = d.q_pos0 + d.n_q;
    cudaError_t e = launch_window(a, row_cap, d.n_q, false, st);
    if (e != cudaSuccess) return e;
    a.only_marked = 1;
    return launch_pass(a, row_cap, d.n_q, refine, st);
  }
  if (t.n_seg == 0) return launch_pass(a, d.q_pos0 + d.n_q, d.n_q, refine, st);
  if (!cand) return cudaErrorInvalidValue;
  a.seg_len = t.seg_len;
  a.n_seg = t.n_seg;
  a.cand = static_cast<int32_t*>(cand);
  a.pass = 1;
  cudaError_t e;
  if (window) {  // the segments through the window select, handed-back ones through topk_kernel
    e = launch_window(a, t.seg_len, d.n_q * t.n_seg, true, st);
    if (e != cudaSuccess) return e;
    a.only_marked = 1;
  }
  e = launch_pass(a, t.seg_len, d.n_q * t.n_seg, refine, st);
  if (e != cudaSuccess) return e;
  a.only_marked = 0;
  a.pass = 2;
  return launch_pass(a, t.n_seg * d.top_k, d.n_q, refine, st);
}

}  // namespace dsa
