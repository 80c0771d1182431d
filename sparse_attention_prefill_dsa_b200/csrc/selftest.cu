// selftest.cu -- the bounded-wait failure path of the library's kernels, on a
// one-CTA launch that gives up cleanly (no fault, no hang).
//
// Every wait in the indexer, top-k and attention kernels is an mbarrier wait
// with an iteration limit and a per-CTA abort flag (mbar_wait): on a timeout
// the waiting warp records DSA_ERR_TIMEOUT and its site in the workspace
// header and sets the abort flag, and every other wait of the CTA then gives
// up at its next check. Here two warps wait on mbarriers that nothing ever
// arrives at: warp 0 with a short limit, warp 1 with the kernels' own limit
// (about one second), so warp 1 can only finish early through the abort flag.
#include <cuda_runtime.h>
#include <stdint.h>

#include "dsa_internal.cuh"
#include "sm100_primitives.cuh"

namespace dsa {
namespace {

using namespace sm100;

constexpr long long kShortLimitCycles = 1000000;  // about 0.5 ms

__global__ void __launch_bounds__(64, 1) bounded_wait_selftest(WsHeader* ws, long long* cycles) {
  __shared__ __align__(8) uint64_t bar[2];
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar[0], 1);
    mbar_init(&bar[1], 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5;
  const long long t0 = clock64();
  // parity 0: the first phase of a fresh barrier, which completes only when
  // its one expected arrival comes; none does
  bool ok;
  if (warp == 0)
    ok = mbar_wait(&bar[0], 0, &abort_flag, ws, kSelftestSiteShort, kShortLimitCycles);
  else
    ok = mbar_wait(&bar[1], 0, &abort_flag, ws, kSelftestSiteLong);
  const long long t1 = clock64();
  if ((threadIdx.x & 31) == 0 && cycles) cycles[warp] = ok ? -1 : t1 - t0;
  __syncthreads();
}

}  // namespace

cudaError_t launch_bounded_wait_selftest(WsHeader* ws, long long* cycles, cudaStream_t st) {
  bounded_wait_selftest<<<1, 64, 0, st>>>(ws, cycles);
  return cudaGetLastError();
}

}  // namespace dsa
