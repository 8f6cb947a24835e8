// fa_selftest.cu -- diagnostics: the failure-detection path every kernel relies on, and the
// FMA-pipe exp2 the kernels use for part of their exponentials.
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

// y[i] = 2^x[i] by the FMA-pipe polynomial the kernels use for part of their exponentials,
// evaluated in pairs exactly as in the kernels (an odd tail pairs its last element with 0).
__global__ void __launch_bounds__(256) exp2_poly_probe(const float* x, float* y, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float a = x[i], b = (i + 1 < n) ? x[i + 1] : 0.f;
  const float2 r = exp2_poly2(make_float2(a, b));
  y[i] = r.x;
  if (i + 1 < n) y[i + 1] = r.y;
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

extern "C" int fa_selftest_exp2_poly(const float* x, float* y, int n, void* stream) {
  if (n < 1 || x == nullptr || y == nullptr) return FA_ERR_INVALID_ARG;
  const int pairs = (n + 1) / 2;
  fa::exp2_poly_probe<<<(pairs + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y, n);
  return cudaGetLastError() == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}
