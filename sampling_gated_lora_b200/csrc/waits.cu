// Self-test of the library's bounded waits.
//
// Every spin in this library's kernels (a flag another CTA raises, an
// mbarrier that TMA, the tensor core or a peer CTA completes) gives up after
// a time limit, reports UNO_DEV_TIMEOUT in the status words and lets the
// kernel return, so that a lost arrival ends in an error the host can read
// instead of a GPU that stops answering. This kernel runs those same wait
// helpers on conditions that nothing will ever satisfy, with a short limit,
// so the give-up path itself can be tested. It has no copy or MMA in flight:
// giving up leaves nothing behind.
#include "common.cuh"
#include "internal.h"

namespace uno {

namespace {

// Never written by anyone: a flag that stays 0.
__device__ int32_t g_never_raised = 0;

__global__ void wait_selftest_kernel(int which, uint64_t limit_ns, int32_t* result,
                                     int32_t* status) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    fence_mbar_init();
  }
  cta_sync();
  if (threadIdx.x != 0) return;
  bool ok = false;
  switch (which) {
    case 0:   // a flag in global memory that is never raised
      ok = flag_wait(&g_never_raised, 1, limit_ns);
      break;
    case 1:   // an mbarrier phase with no arrival
      ok = mbar_wait(smem_u32(&bar), 0, limit_ns);
      break;
    case 2:   // the same, through the cluster-scope wait used between CTA pairs
      ok = mbar_wait_cluster(smem_u32(&bar), 0, limit_ns);
      break;
    default:  // control: the one expected arrival comes first, the wait succeeds
      mbar_arrive(smem_u32(&bar));
      ok = mbar_wait(smem_u32(&bar), 0, limit_ns);
      break;
  }
  if (!ok) raise_status(status, kDevTimeout);
  *result = ok ? 1 : 0;
}

}  // namespace

uno_status wait_selftest_launch(int32_t which, uint64_t limit_ns, int32_t* result,
                                int32_t* status, cudaStream_t s) {
  const cudaError_t e = launch_kernel(wait_selftest_kernel, dim3(1), dim3(32), 0, s, 1, which,
                                      limit_ns, result, status);
  return e == cudaSuccess ? UNO_OK : cuda_error(e, "wait self-test launch");
}

}  // namespace uno
