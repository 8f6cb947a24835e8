// fa_selftest.cu -- a diagnostic for the failure-detection path every kernel relies on.
//
// Each kernel of the library bounds every mbarrier wait: past its time limit the wait
// records FA_ERR_TIMEOUT in the device status word, raises the CTA's abort flag and
// returns, so a stalled pipeline ends the kernel instead of hanging the GPU, and
// fa_check_status reports it.  fa_selftest_wait_timeout runs that same wait helper on a
// barrier that nothing ever completes, with a caller-chosen short limit: the wait must give
// up, the kernel must return, and the status word must read FA_ERR_TIMEOUT afterwards --
// a failure made on purpose without any fault, trap or unbounded loop.
#include <cuda.h>
#include <cuda_runtime.h>

#include "fa.h"
#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {
namespace {

__global__ void __launch_bounds__(32) wait_timeout_probe(DevStatus st, int* waited_ok) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);               // one arrival expected; none will come
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncwarp();
  if (threadIdx.x == 0) {
    const bool ok = mbar_wait(&bar, 0, &abort_flag, st);
    if (waited_ok != nullptr) *waited_ok = ok ? 1 : 0;
  }
}

}  // namespace
}  // namespace fa

extern "C" int fa_selftest_wait_timeout(unsigned int limit_us, int* waited_ok, void* stream) {
  if (limit_us < 1 || limit_us > 1000000u) return FA_ERR_INVALID_ARG;
  int* status = fa::device_status_word();
  if (status == nullptr) return FA_ERR_CUDA;
  fa::DevStatus st{status, (unsigned long long)limit_us * 1000ull};
  fa::wait_timeout_probe<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(st, waited_ok);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}
