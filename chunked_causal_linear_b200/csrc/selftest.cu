// A check of the library's failure detection that faults nothing.
//
// Every wait of the library's kernels on an mbarrier (a TMA load landing, an MMA
// completing, another warp's hand-off) is bounded: when it runs out, the kernel records a
// code in the device error word, stops waiting, releases what it holds and returns, and
// kernels launched after it skip their work while the word is set.  The host reads and
// clears the word with lin_attn_device_error.  lin_attn_check_wait_timeout exercises that
// path on purpose: one thread waits, with the given short limit, on an mbarrier that
// nothing ever arrives on; the wait gives up and reports kErrWaitCheck.  No TMA, MMA or
// TMEM is involved, and the context stays usable.

#include <cuda_runtime.h>

#include "../../include/linattn.h"
#include "launch.h"
#include "ptx.cuh"

namespace la {
namespace {

__global__ void wait_timeout_check(int* err, unsigned long long timeout_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);  // one expected arrival, never made
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0 && !mbar_wait(&bar, 0, timeout_ns)) report_error(err, kErrWaitCheck);
}

}  // namespace
}  // namespace la

extern "C" int lin_attn_check_wait_timeout(unsigned int timeout_us, la_stream_t stream) {
  if (timeout_us == 0 || timeout_us > 1000000u) return LA_ERR_INVALID_ARGUMENT;
  int* err = la::device_error_word();
  if (!err) return LA_ERR_CUDA;
  la::wait_timeout_check<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      err, static_cast<unsigned long long>(timeout_us) * 1000ull);
  return cudaGetLastError() == cudaSuccess ? LA_OK : LA_ERR_CUDA;
}
