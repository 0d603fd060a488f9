// selftest.cu -- nvfp4_selftest_wait_timeout: the device-side failure path, run on purpose.
//
// Every wait inside the library's kernels (an mbarrier phase, the bytes of a bulk copy, a
// counter that other CTAs advance) is bounded by wall-clock time; a wait that runs out sets
// bit 1 of the caller's error flag and the kernel leaves its loops and returns, so the CUDA
// context stays usable.  This test hook runs each kind of wait with nothing to complete it
// and a short limit, through the same wait helpers the kernels use.  Nothing here faults:
// no copy is issued, no memory outside the flag is written, and every wait ends.
#include "pipeline.cuh"

namespace nvfp4 {
namespace {

// Never written: a counter that no CTA advances.
__device__ uint32_t g_never_advanced = 0;

__global__ void __launch_bounds__(32) wait_timeout_kernel(int32_t *flag, int kind,
                                                          uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int s_abort;
  if (threadIdx.x != 0) return;
  s_abort = 0;
  mbar_init(&bar, 1);
  mbar_init_fence();
  bool ok = true;
  if (kind == 0) {
    // an mbarrier phase that no thread arrives at
    ok = mbar_wait(&bar, 0, limit_ns);
  } else if (kind == 1) {
    // the arrival is in, but the 16 bytes it announces never land (no copy is issued)
    mbar_arrive_expect_tx(&bar, 16);
    ok = mbar_wait(&bar, 0, limit_ns);
  } else {
    // a grid-wide counter that nobody advances
    ok = wait_geq(&g_never_advanced, 1u, &s_abort, limit_ns);
  }
  if (!ok) report_timeout(flag);
}

}  // namespace
}  // namespace nvfp4

using namespace nvfp4;

extern "C" int nvfp4_selftest_wait_timeout(int32_t *flag, int kind, int64_t limit_ns,
                                           cudaStream_t stream) {
  if (!flag || (reinterpret_cast<uintptr_t>(flag) & 3)) return NVFP4_EINVAL;
  if (kind < 0 || kind > 2) return NVFP4_EINVAL;
  if (limit_ns <= 0 || limit_ns > 1000000000) return NVFP4_EINVAL;
  wait_timeout_kernel<<<1, 32, 0, stream>>>(flag, kind, (uint64_t)limit_ns);
  return check_launch();
}
