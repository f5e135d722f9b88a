// k_selftest.cu -- a self-test of the timeout path that every pipelined
// kernel of this library relies on.  One thread initialises an mbarrier and
// waits on its first phase with the same bounded wait the kernels use; unless
// it arrived first, nothing completes the phase, the wait gives up after the
// limit, and the thread sets the device error word to the given code, which
// llsa_device_error reports and clears.  No fault, trap or endless wait is
// involved: the wait ends by the global timer.
#include <stdint.h>

#include "llsa.h"
#include "llsa_internal.cuh"
#include "ptx.cuh"

namespace llsa {

__global__ void selftest_wait_kernel(uint64_t limit_ns, int code, int arrive, int* err) {
  __shared__ __align__(8) uint64_t bar;
  ptx::mbar_init(&bar, 1);
  ptx::fence_mbar_init();
  if (arrive) ptx::mbar_arrive(&bar);
  if (!ptx::mbar_wait_bounded(&bar, 0, limit_ns) && err) atomicExch(err, code);
}

}  // namespace llsa

extern "C" llsa_status llsa_selftest_wait_timeout(unsigned limit_us, int code, int arrive, llsa_stream stream) {
  if (limit_us < 1 || limit_us > 1000000 || code == 0 || (arrive != 0 && arrive != 1)) return LLSA_ERR_ARG;
  int* err = llsa::device_error_word();
  if (!err) return LLSA_ERR_CUDA;
  llsa::selftest_wait_kernel<<<1, 1, 0, (cudaStream_t)stream>>>((uint64_t)limit_us * 1000ull, code, arrive, err);
  llsa::note_launches(1);
  return cudaGetLastError() == cudaSuccess ? LLSA_OK : LLSA_ERR_CUDA;
}
