// Check of the bounded waits (failure detection without a GPU fault).
//
// Every kernel of this library waits on mbarriers (TMA tiles landed, a ring
// slot freed, a tensor-core product done) through mbar_wait in common.cuh,
// which gives up after a time limit, ORs PKV_FLAG_TIMEOUT into the caller's
// error word and lets the kernel return, so a lost arrival ends in a status
// the host can read instead of a hung GPU (the murmur post lists fault
// recovery, 故障恢復, among its evaluation criteria).  This file runs that
// same helper on an mbarrier nothing ever arrives on, with no bulk copy,
// TMA load or tensor-core operation in flight, so that giving up is safe.
#include "common.cuh"
#include "kernels.h"

namespace pkv {

__global__ void __launch_bounds__(32) wait_check_kernel(int32_t* flags, uint64_t limit_ns,
                                                        int64_t* waited_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  fence_barrier_init();
  const uint64_t t0 = global_ns();
  // Phase 0 of a fresh barrier completes only after one arrival: none comes.
  const bool arrived = mbar_wait(&bar, 0, flags, 0, limit_ns);
  if (waited_ns) *waited_ns = arrived ? -1 : (int64_t)(global_ns() - t0);
}

}  // namespace pkv

extern "C" int pkv_check_bounded_wait(int32_t* error_flags, int64_t limit_ns,
                                      int64_t* waited_ns, void* stream) {
  if (!error_flags) return PKV_ERR_NULL;
  // at most the library's own limit: the check never waits longer than a kernel would
  if (limit_ns < 0 || (uint64_t)limit_ns > pkv::kWaitLimitNs) return PKV_ERR_SHAPE;
  const uint64_t lim = limit_ns == 0 ? pkv::kWaitLimitNs : (uint64_t)limit_ns;
  pkv::wait_check_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(error_flags, lim,
                                                                          waited_ns);
  return cudaGetLastError() == cudaSuccess ? PKV_OK : PKV_ERR_CUDA;
}
