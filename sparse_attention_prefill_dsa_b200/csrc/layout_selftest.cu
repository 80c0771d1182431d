// layout_selftest.cu -- a start-up check of the tensor-core operand
// conventions the kernels rely on (the lesson of the "Pre-M5 kernel checks"
// item of the TensorFold issue #743 page: a fragment-layout check that let a
// transposed operand through).
//
// One CTA multiplies matrices of small integers that are not symmetric and
// compares every accumulator element with a CUDA-core sum of the same
// integers; both are exact in float32, so any difference is a layout error
// (a transposed operand, a wrong swizzle, stride or descriptor field, a
// wrong tensor-memory lane or column mapping). Each form writes its operands
// at the byte positions the kernels' own copies produce and builds its
// descriptors with the kernels' helpers:
//   form 0  indexer, bf16: A = key tile [128][128], B = query block [256][128],
//           both K-major in 64-element chunks of 128-byte rows, 128-byte
//           swizzle (as TMA writes them), 8 MMAs of K = 16;
//   form 1  attention QK^T: A = a latent pair read K-major ([128 keys][64 dims]
//           per 16 KB chunk, the gather's swizzle), B = two q chunks
//           ([32 heads][64 dims]), N = 32;
//   form 2  attention PV: A = the same pair read MN-major (M = 128 dims over
//           its two chunks, K = keys), B = P ([128 keys][32 heads] in 64-byte
//           rows, 64-byte swizzle, MN-major), N = 32;
//   form 3  FP8 indexer: e4m3 operands [128][128] and [256][128] in 128-byte
//           rows, kind::f8f6f4, 4 MMAs of K = 32.
// Results read back with tcgen05.ld 32x32b (thread = accumulator row).
// Each form is then timed: its MMAs issued 32 times back to back on the same
// operands, clock64 from the first issue to the completion of the last, which
// gives the form's cycles per MMA on one SM.
#include <cuda_runtime.h>
#include <stdint.h>

#include "dsa_internal.cuh"
#include "sm100_primitives.cuh"

namespace dsa {
namespace {

using namespace sm100;

constexpr int kForms = 4;
constexpr int kThreads = 128;
constexpr int kOperandBytes = 96 * 1024;  // form 0: A 32 KB + B 64 KB
constexpr int kOffB = 32 * 1024;
constexpr int kSmemBytes = kOperandBytes + 64 + 1024;  // + barrier and counters, alignment slack
constexpr unsigned int kSiteMma = 103;     // the wait for a form's MMAs
constexpr int kTimedReps = 32;             // repetitions of a form's MMAs in its timed run

// The test matrices: small integers from a hash of (row, column), exact in
// bf16 and e4m3, with products and 128-term sums exact in float32; no two
// rows or columns of an operand or of a product coincide, so a mixed-up row,
// column, swizzle unit or K chunk changes some accumulator element.
__device__ __forceinline__ uint32_t mix(uint32_t r, uint32_t c, uint32_t seed) {
  uint32_t x = (r * 0x9E3779B1u) ^ (c * 0x85EBCA77u) ^ seed;
  x ^= x >> 15;
  x *= 0x2C1B3C6Du;
  x ^= x >> 12;
  return x;
}
__device__ __forceinline__ int a_val(int m, int k) { return static_cast<int>(mix(m, k, 0x1234u) % 7u) - 3; }
__device__ __forceinline__ int b_val(int n, int k) { return static_cast<int>(mix(n, k, 0x5678u) % 5u) - 2; }

__device__ __forceinline__ uint16_t bf16_of_int(int v) {
  return static_cast<uint16_t>(__float_as_uint(static_cast<float>(v)) >> 16);
}

// e4m3 (sign, 4 exponent bits biased by 7, 3 mantissa bits) of -3 .. 3
__device__ __forceinline__ uint8_t e4m3_of_int(int v) {
  const int a = v < 0 ? -v : v;
  const uint8_t mag = a == 0 ? 0x00 : a == 1 ? 0x38 : a == 2 ? 0x40 : 0x44;
  return static_cast<uint8_t>(mag | (v < 0 && a != 0 ? 0x80 : 0x00));
}

// Byte offset of element e (2-byte elements) of row r in a 128-byte-swizzled
// chunk of 128-byte rows: the 16-byte unit u of row r sits at unit u ^ (r % 8).
__device__ __forceinline__ uint32_t sw128(int r, int e_bytes) {
  return static_cast<uint32_t>(r * 128 + ((((e_bytes >> 4) ^ (r & 7))) << 4) + (e_bytes & 15));
}

// Writes the form's operands; every thread takes a share of the elements.
__device__ void fill_form(int form, unsigned char* s) {
  const int t = threadIdx.x;
  if (form == 0 || form == 1) {
    const int nb = form == 0 ? 256 : 32;     // B rows
    const int b_chunk = nb * 128;            // bytes per 64-element chunk of B
    for (int x = t; x < 128 * 128; x += kThreads) {  // A: key m, dim k
      const int m = x >> 7, k = x & 127;
      *reinterpret_cast<uint16_t*>(s + (k >> 6) * 16384 + sw128(m, (k & 63) * 2)) =
          bf16_of_int(a_val(m, k));
    }
    for (int x = t; x < nb * 128; x += kThreads) {  // B: row n, dim k
      const int n = x >> 7, k = x & 127;
      *reinterpret_cast<uint16_t*>(s + kOffB + (k >> 6) * b_chunk + sw128(n, (k & 63) * 2)) =
          bf16_of_int(b_val(n, k));
    }
  } else if (form == 2) {
    for (int x = t; x < 128 * 128; x += kThreads) {  // A: dim m, key k, stored as row k of chunk m / 64
      const int m = x >> 7, k = x & 127;
      *reinterpret_cast<uint16_t*>(s + (m >> 6) * 16384 + sw128(k, (m & 63) * 2)) =
          bf16_of_int(a_val(m, k));
    }
    for (int x = t; x < 32 * 128; x += kThreads) {  // B = P: head n, key k, stored as row k
      const int n = x >> 7, k = x & 127;
      const int c = (n * 2) >> 4;  // 16-byte unit of eight heads
      *reinterpret_cast<uint16_t*>(s + kOffB + k * 64 + ((c ^ ((k >> 1) & 3)) << 4) + ((n * 2) & 15)) =
          bf16_of_int(b_val(n, k));
    }
  } else {
    for (int x = t; x < 128 * 128; x += kThreads) {
      const int m = x >> 7, k = x & 127;
      s[m * 128 + (((k >> 4) ^ (m & 7)) << 4) + (k & 15)] = e4m3_of_int(a_val(m, k));
    }
    for (int x = t; x < 256 * 128; x += kThreads) {
      const int n = x >> 7, k = x & 127;
      s[kOffB + n * 128 + (((k >> 4) ^ (n & 7)) << 4) + (k & 15)] = e4m3_of_int(b_val(n, k));
    }
  }
}

// Issues the form's MMAs into tensor-memory column 0 (warp-collective), with
// the descriptors as compile-time offsets from two bases, as the kernels do.
template <int form>
__device__ __forceinline__ void issue_form(unsigned char* s, uint32_t tmem) {
  const uint32_t a0 = smem_u32(s), b0 = smem_u32(s + kOffB);
  if constexpr (form == 0) {
    const uint64_t da = smem_desc(a0, 16, 1024, 2), db = smem_desc(b0, 16, 1024, 2);
    constexpr uint32_t idesc = idesc_bf16_f32(128, 256, false, false);
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const uint32_t c = ks / 4, off = (ks % 4) * 32;
      mma_bf16_ss_warp(tmem, da + ((c * 16384 + off) >> 4), db + ((c * 32768 + off) >> 4), idesc,
                       ks > 0 ? 1u : 0u);
    }
  } else if constexpr (form == 1) {
    const uint64_t da = smem_desc(a0, 16, 1024, 2), db = smem_desc(b0, 16, 1024, 2);
    constexpr uint32_t idesc = idesc_bf16_f32(128, 32, false, false);
#pragma unroll
    for (int c = 0; c < 2; ++c)
#pragma unroll
      for (int ks = 0; ks < 4; ++ks)
        mma_bf16_ss_warp(tmem, da + ((c * 16384 + ks * 32) >> 4), db + ((c * 4096 + ks * 32) >> 4),
                         idesc, (c | ks) ? 1u : 0u);
  } else if constexpr (form == 2) {
    const uint64_t da = smem_desc(a0, 16384, 1024, 2), db = smem_desc(b0, 8 * 64, 8 * 64, 4);
    constexpr uint32_t idesc = idesc_bf16_f32(128, 32, true, true);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk)
      mma_bf16_ss_warp(tmem, da + ((kk * 2048) >> 4), db + ((kk * 16 * 64) >> 4), idesc,
                       kk > 0 ? 1u : 0u);
  } else {
    const uint64_t da = smem_desc(a0, 16, 1024, 2), db = smem_desc(b0, 16, 1024, 2);
    constexpr uint32_t idesc = idesc_e4m3_f32(128, 256);
#pragma unroll
    for (int ks = 0; ks < 4; ++ks)
      mma_f8_ss_warp(tmem, da + ((ks * 32) >> 4), db + ((ks * 32) >> 4), idesc, ks > 0 ? 1u : 0u);
  }
}

__device__ __forceinline__ int mmas_of_form(int form) { return form == 3 ? 4 : 8; }

// The form's MMAs once (reps = 1) or kTimedReps times back to back (warp-collective).
template <int form>
__device__ __forceinline__ void issue_reps(unsigned char* s, uint32_t tmem, int reps) {
#pragma unroll 1
  for (int r = 0; r < reps; ++r) issue_form<form>(s, tmem);
}

__device__ __forceinline__ void issue_form_n(int form, unsigned char* s, uint32_t tmem, int reps) {
  switch (form) {
    case 0: issue_reps<0>(s, tmem, reps); break;
    case 1: issue_reps<1>(s, tmem, reps); break;
    case 2: issue_reps<2>(s, tmem, reps); break;
    default: issue_reps<3>(s, tmem, reps); break;
  }
}

__global__ void __launch_bounds__(kThreads, 1) mma_layout_selftest(WsHeader* ws, int* mismatches,
                                                                   float* cycles_per_mma) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* s = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint64_t* bar = reinterpret_cast<uint64_t*>(s + kOperandBytes);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(s + kOperandBytes + 8);
  int* abort_flag = reinterpret_cast<int*>(s + kOperandBytes + 12);
  int* s_mis = reinterpret_cast<int*>(s + kOperandBytes + 16);  // [kForms]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int x = threadIdx.x * 16; x < kOperandBytes; x += kThreads * 16)
    *reinterpret_cast<uint4*>(s + x) = make_uint4(0u, 0u, 0u, 0u);
  if (threadIdx.x == 0) {
    mbar_init(bar, 1);
    *abort_flag = 0;
    for (int f = 0; f < kForms; ++f) s_mis[f] = 0;
    fence_barrier_init();
  }
  if (warp == 0) tmem_alloc(tmem_slot, 256);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int m = 32 * warp + lane;  // this thread's accumulator row (tensor-memory lane)
  bool ok = true;
  uint32_t phase = 0;  // commits made to `bar`
  float s_cyc[kForms] = {0.f, 0.f, 0.f, 0.f};
  for (int form = 0; form < kForms && ok; ++form) {
    fill_form(form, s);
    fence_proxy_async_smem();  // generic-proxy writes, read by the MMAs through the async proxy
    __syncthreads();
    if (warp == 0) {
      tc_fence_after();
      issue_form_n(form, s, tmem, 1);
      mma_commit_warp(bar);
    }
    ok = __all_sync(0xffffffffu, mbar_wait(bar, phase & 1, abort_flag, ws, kSiteMma));
    ++phase;
    if (!ok) break;
    tc_fence_after();
    const int n_cols = (form == 1 || form == 2) ? 32 : 256;
    int bad = 0;
    for (int c0 = 0; c0 < n_cols; c0 += 16) {
      uint32_t r[16];
      tmem_ld_32x32b_x16(tmem + (static_cast<uint32_t>(32 * warp) << 16) + c0, r);
      tmem_ld_wait();
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        int ref = 0;
        for (int k = 0; k < 128; ++k) ref += a_val(m, k) * b_val(c0 + j, k);
        bad += __uint_as_float(r[j]) != static_cast<float>(ref);
      }
    }
    if (bad) atomicAdd(&s_mis[form], bad);
    tc_fence_before();
    __syncthreads();  // every thread has read the accumulator before the timed MMAs
    if (warp == 0) {
      tc_fence_after();
      const long long t0 = clock64();
      issue_form_n(form, s, tmem, kTimedReps);
      mma_commit_warp(bar);
      ok = __all_sync(0xffffffffu, mbar_wait(bar, phase & 1, abort_flag, ws, kSiteMma));
      const long long t1 = clock64();
      s_cyc[form] = static_cast<float>(t1 - t0) / static_cast<float>(kTimedReps * mmas_of_form(form));
    }
    ++phase;
    // every thread reaches this barrier (no short circuit): it also keeps the
    // next form's operand writes behind the timed MMAs
    ok = __syncthreads_and(ok ? 1 : 0) != 0;
    tc_fence_after();
  }
  if (!ok) {
    // a wait gave up: let the MMAs in flight finish (bounded) before TMEM is released
    const long long t0 = clock64();
    while (phase > 0 && !mbar_try_wait(bar, (phase - 1) & 1))
      if (clock64() - t0 > kWaitLimitCycles) break;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int first_bad = -1;
    for (int f = 0; f < kForms; ++f) {
      mismatches[f] = ok ? s_mis[f] : -1;
      cycles_per_mma[f] = ok ? s_cyc[f] : -1.f;
      if (ok && s_mis[f] != 0 && first_bad < 0) first_bad = f;
    }
    if (first_bad >= 0) report(ws, kDevLayout, static_cast<unsigned int>(first_bad));
  }
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace

cudaError_t launch_mma_layout_selftest(WsHeader* ws, int* mismatches, float* cycles_per_mma,
                                      cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(mma_layout_selftest,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
  if (e != cudaSuccess) return e;
  mma_layout_selftest<<<1, kThreads, kSmemBytes, st>>>(ws, mismatches, cycles_per_mma);
  return cudaGetLastError();
}

}  // namespace dsa
