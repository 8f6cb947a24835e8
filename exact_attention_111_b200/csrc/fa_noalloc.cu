// fa_noalloc.cu -- fa_bwd_noalloc: the backward pass for callers that cannot allocate
// device memory at call time.
//
// fa_bwd needs a caller-provided scratch buffer (fp32 dQ accumulator and two per-row
// vectors).  Some callers have no way to provide one when they call: an inference- or
// training-engine plugin whose enqueue step must not allocate, a host program that links
// libfa.so without any device allocator of its own, or code running while the process's
// device memory pool is frozen.  For them this file holds the scratch in a fixed
// file-scope device array instead, and the entry point allocates nothing.
//
// The array (kNoAllocScratchBytes) exists on every GPU that loads the library, until the
// process exits.  The CUDA runtime loads device code lazily, so on each device the array's
// memory is committed when this file's code is first loaded there -- by the first call's
// address lookup -- and that first call must therefore come at start-up, before any stream
// capture or freezing of the device memory pool.  Later calls allocate nothing.  Every call on a device shares that device's array, so calls that overlap
// on the GPU (other streams, other host threads) race on it and must be serialised by the
// caller.  The array keeps the last call's contents; the backward's first kernel rewrites
// every part the later kernels read (it zeroes the dQ accumulator and writes both per-row
// vectors), so nothing has to be cleared between calls.
#include <cuda_runtime.h>

#include <mutex>

#include "fa.h"
#include "fa_internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = (size_t)FA_NOALLOC_SCRATCH_BYTES;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[128] = {nullptr};

// Device address of g_noalloc_scratch on the current device.  In host code the array's name
// is only a host-side stand-in, so the address is asked from the runtime once per device.
int scratch_for_current_device(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return FA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return FA_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return FA_OK;
}

}  // namespace

namespace fa {
int validate_bwd(const fa_bwd_args& x, bool check_workspace);   // fa_host.cu
}

extern "C" int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                              const void* dout, void* dq, void* dk, void* dv, int B, int H, int N, int d,
                              float scale, int causal, const uint8_t* blockmask, void* stream) {
  fa_bwd_args a{};
  a.q = q; a.k = k; a.v = v; a.o = o; a.lse = lse; a.dout = dout;
  a.dq = dq; a.dk = dk; a.dv = dv;
  a.B = B; a.H = H; a.N = N; a.d = d; a.scale = scale; a.causal = causal; a.blockmask = blockmask;
  a.dtype = FA_BF16; a.visit_log = nullptr; a.stream = stream;
  // Argument errors first, exactly as fa_bwd reports them, before any CUDA call.
  int rc = fa::validate_bwd(a, false);
  if (rc != FA_OK) return rc;
  if (fa_bwd_workspace_bytes(B, H, N, d) > kNoAllocScratchBytes) return FA_ERR_WORKSPACE;
  void* scratch = nullptr;
  rc = scratch_for_current_device(&scratch);
  if (rc != FA_OK) return rc;
  a.workspace = scratch;
  a.workspace_bytes = kNoAllocScratchBytes;
  return fa_bwd_ex(&a);
}
