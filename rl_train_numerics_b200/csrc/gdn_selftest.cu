// gdn_selftest.cu -- gdn_selftest_bounded_wait: runs the boundary walk's
// tensor-memory setup and its bounded completion wait on a barrier that
// nothing arrives at, so that the give-up path (error bit, tensor memory
// released, context still usable) can be tested without faulting or hanging
// the GPU.
#include "../../include/gdn_cpr.h"
#include "gdn_boundary.cuh"

namespace gdn {

__global__ void __launch_bounds__(kTcRows) k_selftest_wait(int polls, int32_t* error) {
  __shared__ uint64_t mbar;
  __shared__ uint32_t tmem;
  TcCtx cx;
  tc_setup(cx, &mbar, &tmem);
  // No product is committed, so the phase never completes: the wait gives up
  // after `polls` polls, as a step whose products never finished would.
  const bool ok = mbar_wait(cx.mbar, cx.phase, polls);
  if (__syncthreads_or(!ok) && threadIdx.x == 0) atomicOr(error, kErrTimeout);
  tc_teardown(cx);
}

}  // namespace gdn

extern "C" int gdn_selftest_bounded_wait(int polls, int32_t* error_word, void* stream) {
  if (polls <= 0 || polls > gdn::kTcWaitPolls || !error_word) return GDN_ERR_INVALID_ARG;
  gdn::k_selftest_wait<<<1, gdn::kTcRows, 0, static_cast<cudaStream_t>(stream)>>>(polls,
                                                                                  error_word);
  return cudaGetLastError() == cudaSuccess ? GDN_OK : GDN_ERR_CUDA;
}
