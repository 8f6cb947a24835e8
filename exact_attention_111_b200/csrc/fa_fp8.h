// fa_fp8.h -- argument block and launcher of the FP8 (E4M3) forward, shared by the host
// library (fa_host.cu) and the kernel file (fa_fwd_fp8.cu).  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace fa {

struct F8Args {
  void* o;                  // [BH, N, 128] bf16, or fp32 when o_fp32
  float* lse;               // [BH, N]
  const uint8_t* blockmask; // [T, T] or null
  int* status;
  unsigned long long timeout_ns;
  int N, BH, T, n_units, group_heads;
  int causal, o_fp32;
  float scale_log2;         // scale * dq * dk * log2(e)
  float o_scale;            // dv / 256 (P is stored as E4M3(256 P))
};

// Transposes V into vt ([BH, 128, Np] bytes, Np = T * 128) and runs the forward; tvt is the
// TMA map of vt.  Two launches on `s`.
cudaError_t launch_fwd_fp8(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tvt, const F8Args& a,
                           const uint8_t* v, uint8_t* vt, int Np, cudaStream_t s);

}  // namespace fa
