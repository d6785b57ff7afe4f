// msa_selftest_wait_timeout: runs the give-up path of the bounded waits that
// every tensor-core kernel of the library uses, on purpose and with nothing in
// flight, so that a test can check it ends and reports.
//
// One CTA of four warps allocates TMEM as the kernels do, then waits on an
// mbarrier that no thread and no copy ever arrives on: warp 1's lane 0 with
// the non-blocking spin of the MMA-issuing threads, warps 2-3 with the
// sleeping wait of the producer and softmax warps.  Each wait gives up after
// `limit` polls; the CTA then raises the abort flag, records status bit 2 in
// the caller's status word, frees its TMEM and returns, exactly the exit the
// kernels take.  No TMA copy, bulk store or MMA is ever issued here, so there
// is nothing to drain.
#include "../../include/msa.h"
#include "common.cuh"
#include "internal.h"
#include "tc_common.cuh"

namespace msa {
namespace {

__global__ void __launch_bounds__(128, 1) wait_timeout_kernel(uint32_t limit, int* status,
                                                              int* gave_up) {
  __shared__ uint64_t bar;
  __shared__ uint32_t tmem_base;
  __shared__ int abort_flag;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    tc::mbar_init(&bar, 1);
    abort_flag = 0;
    tc::fence_mbar_init();
  }
  if (warp == 0) tc::tmem_alloc(&tmem_base, 32);
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  volatile int* abort = &abort_flag;
  bool failed = false;
  if (warp == 1) {
    if (lane == 0) failed = !tc::mbar_spin(&bar, 0, abort, limit);
  } else if (warp >= 2) {
    failed = !__all_sync(MSA_FULL_MASK, tc::mbar_wait(&bar, 0, abort, limit));
  }
  if (failed) {
    abort_flag = 1;
    atomicOr(status, tc::kStatusWaitTimeout);
    if (lane == 0) atomicAdd(gave_up, 1);
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem_base, 32);
  }
}

}  // namespace
}  // namespace msa

extern "C" msa_status_t msa_selftest_wait_timeout(uint32_t limit, int32_t* status,
                                                  int32_t* gave_up, void* stream) {
  if (!status || !gave_up || limit == 0 || limit > msa::tc::kWaitLimit)
    return MSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(status) & 3u) || (reinterpret_cast<uintptr_t>(gave_up) & 3u))
    return MSA_ERR_INVALID_ARG;
  msa::wait_timeout_kernel<<<1, 128, 0, static_cast<cudaStream_t>(stream)>>>(limit, status,
                                                                              gave_up);
  return msa::status_of(cudaGetLastError());
}
