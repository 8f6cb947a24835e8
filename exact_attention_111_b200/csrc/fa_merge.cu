// fa_merge.cu -- combines attention results computed over disjoint slices of the keys.
//
// Part s holds, for every query row, O_s normalised over its own keys and their log-sum-exp
// LSE_s (fp32).  Over the union of the keys the row's exp-sum is the sum of the parts' sums,
// so with M = max_s LSE_s and w_s = exp(LSE_s - M):
//     LSE = M + ln sum_s w_s,      O = sum_s (w_s / sum_t w_t) O_s,
// the online-softmax rescaling of the running (m, l) statistics (FlashAttention-NeurIPS22
// summary, "核心方法 / Tiling 与 online softmax") applied once per slice.  A row that no part
// saw a key for (every LSE_s = -inf) gets O = 0 and LSE = -inf.
//
// HBM-bound: each row reads n_parts x (4d + 4) bytes and writes 2d + 4 (16-bit O) bytes.
// A row is handled by d/8 consecutive threads, 8 columns (two 16-byte loads per part)
// each, so a warp reads 4 (d = 64) or 2 (d = 128) whole rows of a part per load pair.
// The part pointers may point into another GPU's memory (peer access enabled): the loads are
// plain global loads.
#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {
namespace {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

template <int D>
__global__ void __launch_bounds__(256) merge_kernel(const MergeArgs a) {
  constexpr int kTpr = D / 8;                       // threads per row
  constexpr int kRowsPerBlock = 256 / kTpr;
  const int sub = threadIdx.x % kTpr;
  const int col = sub * 8;
  for (long long row = (long long)blockIdx.x * kRowsPerBlock + threadIdx.x / kTpr; row < a.rows;
       row += (long long)gridDim.x * kRowsPerBlock) {
    float mx = -INFINITY;
    for (int s = 0; s < a.n_parts; ++s) mx = fmaxf(mx, __ldg(a.lse_parts[s] + row));
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    float lse_out = -INFINITY;
    if (mx != -INFINITY) {
      float tot = 0.f;
      for (int s = 0; s < a.n_parts; ++s) {
        const float w = exp2f((__ldg(a.lse_parts[s] + row) - mx) * kLog2e);   // 0 for an empty part
        const float4* src = reinterpret_cast<const float4*>(a.o_parts[s] + row * D + col);
        const float4 x0 = __ldg(src), x1 = __ldg(src + 1);
        if (w > 0.f) {                 // an empty part's O is 0 anyway, but never trust NaN garbage
          acc[0] += w * x0.x; acc[1] += w * x0.y; acc[2] += w * x0.z; acc[3] += w * x0.w;
          acc[4] += w * x1.x; acc[5] += w * x1.y; acc[6] += w * x1.z; acc[7] += w * x1.w;
          tot += w;
        }
      }
      const float inv = 1.f / tot;                  // tot >= 1: the largest part has w = 1
#pragma unroll
      for (int i = 0; i < 8; ++i) acc[i] *= inv;
      lse_out = mx + log2f(tot) * kLn2;
    }
    if (sub == 0) a.lse[row] = lse_out;
    if (a.out_kind == 2) {
      float4* dst = reinterpret_cast<float4*>(static_cast<float*>(a.o) + row * D + col);
      dst[0] = make_float4(acc[0], acc[1], acc[2], acc[3]);
      dst[1] = make_float4(acc[4], acc[5], acc[6], acc[7]);
    } else {
      uint4 w;
      if (a.out_kind == 1) {
        w.x = pack2<true>(acc[0], acc[1]); w.y = pack2<true>(acc[2], acc[3]);
        w.z = pack2<true>(acc[4], acc[5]); w.w = pack2<true>(acc[6], acc[7]);
      } else {
        w.x = pack2<false>(acc[0], acc[1]); w.y = pack2<false>(acc[2], acc[3]);
        w.z = pack2<false>(acc[4], acc[5]); w.w = pack2<false>(acc[6], acc[7]);
      }
      *reinterpret_cast<uint4*>(static_cast<uint16_t*>(a.o) + row * D + col) = w;
    }
  }
}

}  // namespace

cudaError_t launch_merge(const MergeArgs& a, int d, cudaStream_t s) {
  if (a.rows <= 0) return cudaSuccess;
  const long long rows_per_block = 256 / (d / 8);
  long long blocks = (a.rows + rows_per_block - 1) / rows_per_block;
  if (blocks > 148LL * 64) blocks = 148LL * 64;     // grid-stride beyond 64 blocks per SM
  if (d == 64)
    merge_kernel<64><<<(unsigned)blocks, 256, 0, s>>>(a);
  else
    merge_kernel<128><<<(unsigned)blocks, 256, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace fa
