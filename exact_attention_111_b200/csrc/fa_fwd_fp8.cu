// fa_fwd_fp8.cu -- FP8 (E4M3) exact-attention forward for sm_100a, head dimension 128.
//
// The FlashAttention-2 wiki ("FlashAttention-3") lists FP8 low precision among the Hopper
// follow-on's techniques; the pages fix no scaling convention.  This kernel takes Q, K, V
// as E4M3 bytes with one fp32 dequantisation factor per tensor (value = factor * code) and
// computes the exact attention of those values, O = softmax(scale * Q Kᵀ) V, in one fused
// pass with the same online softmax as the 16-bit forward:
//   S  = Q8 K8ᵀ on the tensor cores (kind::f8f6f4, fp32 in TMEM), scaled by
//        scale * dq * dk inside the exp2 argument;
//   P  = 2^(...) in fp32; the row max, exp-sum l and LSE use this P;
//   P8 = E4M3(256 P) (256 P lies in [0, 256], inside E4M3's range, and the factor keeps
//        small probabilities out of the subnormals), written to shared memory;
//   O += P8 V8 (kind::f8f6f4), and the epilogue writes O * dv / (256 l).
// Only the rounding of 256 P to E4M3 (relative 2^-4, absolute 2^-18 on P below the normal
// range) separates the result from the exact attention of the given inputs.
//
// Both products run shared-memory x shared-memory with K-major operands only, the form of
// the 16-bit kernel's S = Q Kᵀ.  At d = 128 every 8-bit row is one 128-byte swizzle panel,
// and each K step covers 32 bytes (32 E4M3 values).  V is first transposed by vt_kernel into
// Vᵀ [BH, 128, Np] (keys contiguous, zero past N), so it too is a K-major operand for
// O += P V.  P goes to shared memory: each softmax thread writes its own 128-byte row in
// the 128-byte-swizzled layout, the pattern the backward kernel uses for dSᵀ.
//
// Warp roles, tile lists, CTA order, causal and block-mask skipping, bounded waits and the
// abort path follow the 16-bit forward (fa_fwd.cu): two query tiles per CTA, softmax groups
// in warps 0-7, the TMA producer in warp 8, the MMA issuer in warp 9.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "fa.h"
#include "fa_fp8.h"
#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {
namespace {

constexpr int kF8D = 128;
constexpr int kF8TileBytes = kTile * 128;      // 128 rows x 128 bytes
constexpr int kF8Stages = 4;                   // K / Vᵀ ring depth
constexpr int kF8SmemTiles = 2 * kF8TileBytes           // Q (two query tiles)
                             + 2 * kF8Stages * kF8TileBytes  // K and Vᵀ rings
                             + 2 * kF8TileBytes;          // P (two query tiles)
constexpr float kF8PScale = 256.0f;
// exp2 pairs per 8 evaluated by the FMA-pipe polynomial instead of the SFU: the SFU is this
// kernel's tightest pipe once the products run at the 8-bit rate (measured at N = 4096 and
// 16384: 2 of 8 is 7 % faster than none; 4 of 8 is slower than none)
constexpr int kF8PolyOf8 = 2;
constexpr float kLn2F8 = 0.693147180559945309f;

struct F8Shared {
  uint64_t q_full;
  uint64_t k_full[kF8Stages], v_full[kF8Stages], k_empty[kF8Stages], v_empty[kF8Stages];
  uint64_t s_full[2], p_full[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort_flag;
  int n_union;
  int n_q[2];
};

// D[tmem] (+)= A[smem desc] * B[smem desc], 8-bit float operands.
__device__ __forceinline__ void mma_ss_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor: D fp32, A and B E4M3 (format code 0), both K-major, M = N = 128.
constexpr uint32_t kIdescF8 = (1u << 4) | (0u << 7) | (0u << 10) | ((128u >> 3) << 17) | ((128u >> 4) << 24);

// Two fp32 -> two E4M3 bytes (lo in the low byte), round to nearest even, saturating.
__device__ __forceinline__ uint32_t pack_e4m3x2(float lo, float hi) {
  unsigned short r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// Vᵀ: v [BH, N, 128] bytes -> vt [BH, 128, Np] bytes, zero for keys >= N.  One block per
// (128-key tile, head): the tile passes through shared memory (rows padded to 144 bytes),
// and a warp then writes 32 consecutive output rows' 16-byte pieces for one key range.
__global__ void __launch_bounds__(256) vt_kernel(const uint8_t* __restrict__ v, uint8_t* __restrict__ vt, int N,
                                                 int Np) {
  __shared__ __align__(16) uint8_t tile[128 * 144];
  const int kt = blockIdx.x, bh = blockIdx.y;
  const uint8_t* src = v + (size_t)bh * N * kF8D;
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int id = threadIdx.x + 256 * r;       // 1024 pieces of 16 bytes
    const int row = id >> 3, c16 = id & 7;
    const int key = kt * kTile + row;
    uint4 x = make_uint4(0u, 0u, 0u, 0u);
    if (key < N) x = *reinterpret_cast<const uint4*>(src + (size_t)key * kF8D + c16 * 16);
    *reinterpret_cast<uint4*>(tile + row * 144 + c16 * 16) = x;
  }
  __syncthreads();
  uint8_t* dst = vt + (size_t)bh * kF8D * Np + (size_t)kt * kTile;
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int id = threadIdx.x + 256 * r;
    const int c = id & 127, k16 = id >> 7;      // output row (head-dim index), 16-key piece
    uint32_t w[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int k0 = k16 * 16 + 4 * u;
      w[u] = (uint32_t)tile[(k0 + 0) * 144 + c] | ((uint32_t)tile[(k0 + 1) * 144 + c] << 8) |
             ((uint32_t)tile[(k0 + 2) * 144 + c] << 16) | ((uint32_t)tile[(k0 + 3) * 144 + c] << 24);
    }
    *reinterpret_cast<uint4*>(dst + (size_t)c * Np + k16 * 16) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

template <bool kOut32>
__global__ void __launch_bounds__(320, 1)
    fwd_fp8_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_vt, const F8Args a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ F8Shared sh;

  const uint32_t pad = (1024u - (smem_addr(smem_raw) & 1023u)) & 1023u;
  uint8_t* sQ = smem_raw + pad;                            // 2 query tiles
  uint8_t* sK = sQ + 2 * kF8TileBytes;                     // kF8Stages key tiles
  uint8_t* sV = sK + kF8Stages * kF8TileBytes;             // kF8Stages Vᵀ tiles
  uint8_t* sP = sV + kF8Stages * kF8TileBytes;             // 2 probability tiles
  int* list = reinterpret_cast<int*>(sP + 2 * kF8TileBytes);

  const int warp = warp_id(), lane = lane_id();
  int bh, ui;
  cta_order(blockIdx.x, a.BH, a.n_units, a.group_heads, bh, ui);
  if (a.causal) ui = a.n_units - 1 - ui;
  const int qt0 = 2 * ui;
  const DevStatus st{a.status, a.timeout_ns};
  volatile int* abort_flag = &sh.abort_flag;

  if (threadIdx.x == 0) {
    mbar_init(&sh.q_full, 1);
    for (int s = 0; s < kF8Stages; ++s) {
      mbar_init(&sh.k_full[s], 1);
      mbar_init(&sh.v_full[s], 1);
      mbar_init(&sh.k_empty[s], 1);
      mbar_init(&sh.v_empty[s], 1);
    }
    for (int q = 0; q < 2; ++q) {
      mbar_init(&sh.s_full[q], 1);
      mbar_init(&sh.p_full[q], 128);
    }
    mbar_init(&sh.mma_done, 1);
    sh.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(&sh.tmem_base, 512);
    tmem_relinquish();
  }
  if (warp == 8) {
    // Union list of key tiles needed by either query tile, with per-tile keep bits.
    int c0, c1;
    const int count = union_tile_list(list, 0, a.T, 0, qt0, true, a.T, a.causal, a.blockmask, c0, c1);
    if (lane == 0) {
      sh.n_union = count;
      sh.n_q[0] = c0;
      sh.n_q[1] = c1;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;
  const int nu = sh.n_union;

  if (warp == 8) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0 && nu > 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_vt);
      const int nq = (qt0 + 1 < a.T) ? 2 : 1;
      mbar_arrive_expect_tx(&sh.q_full, nq * kF8TileBytes);
      for (int q = 0; q < nq; ++q) tma_load_3d(sQ + q * kF8TileBytes, &tm_q, &sh.q_full, 0, (qt0 + q) * kTile, bh);
      // key and value slots are released separately (the key slot a PV product earlier)
      int nk = 0, nv = 0;
      for (int u = 0; u < nu; ++u) {
        const int s = u % kF8Stages;
        const uint32_t ph = ((u / kF8Stages) - 1) & 1;
        const int j = list[u] & 0xFFFF;
        if (u >= kF8Stages && !mbar_wait(&sh.k_empty[s], ph, abort_flag, st)) break;
        mbar_arrive_expect_tx(&sh.k_full[s], kF8TileBytes);
        tma_load_3d(sK + s * kF8TileBytes, &tm_k, &sh.k_full[s], 0, j * kTile, bh);
        ++nk;
        if (u >= kF8Stages && !mbar_wait(&sh.v_empty[s], ph, abort_flag, st)) break;
        mbar_arrive_expect_tx(&sh.v_full[s], kF8TileBytes);
        tma_load_3d(sV + s * kF8TileBytes, &tm_vt, &sh.v_full[s], j * kTile, 0, bh);
        ++nv;
      }
      if (*abort_flag) {
        mbar_wait_drain(&sh.q_full, 0, st);
        for (int uu = (nk > kF8Stages ? nk - kF8Stages : 0); uu < nk; ++uu)
          mbar_wait_drain(&sh.k_full[uu % kF8Stages], (uu / kF8Stages) & 1, st);
        for (int uu = (nv > kF8Stages ? nv - kF8Stages : 0); uu < nv; ++uu)
          mbar_wait_drain(&sh.v_full[uu % kF8Stages], (uu / kF8Stages) & 1, st);
      }
    }
    __syncwarp();
  } else if (warp == 9) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = (nu == 0) || mbar_wait(&sh.q_full, 0, abort_flag, st);
      tc_fence_after();
      const uint32_t aQ = smem_addr(sQ), aK = smem_addr(sK), aV = smem_addr(sV), aP = smem_addr(sP);
      int npv0 = 0, npv1 = 0;
      for (int u = 0; u <= nu && ok; ++u) {
        const int ep = (u > 0) ? list[u - 1] : 0;
        const int ec = (u < nu) ? list[u] : 0;
        const int sp = (u + kF8Stages - 1) % kF8Stages;
        const int sc = u % kF8Stages;
        bool v_ready = false, k_ready = false;
        // Per iteration: O_0 += P_0 V(u-1), S_0 = Q_0 K(u)ᵀ, O_1 += P_1 V(u-1), S_1 = Q_1 K(u)ᵀ, each
        // only where that query tile keeps the tile.
        auto pv = [&](int q, int& npv) -> bool {
          if (u > 0 && ((ep >> (16 + q)) & 1)) {
            if (!v_ready) {
              if (!mbar_wait(&sh.v_full[sp], ((u - 1) / kF8Stages) & 1, abort_flag, st)) return false;
              v_ready = true;
            }
            if (!mbar_wait(&sh.p_full[q], npv & 1, abort_flag, st)) return false;
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {      // 4 x 32 keys
              const uint64_t adesc = smem_desc_sw128(aP + q * kF8TileBytes + kk * 32, 16, 1024);
              const uint64_t bdesc = smem_desc_sw128(aV + sp * kF8TileBytes + kk * 32, 16, 1024);
              mma_ss_f8(tmem + 256 + q * kF8D, adesc, bdesc, kIdescF8, (npv > 0 || kk > 0) ? 1u : 0u);
            }
            ++npv;
          }
          return true;
        };
        auto sq = [&](int q) -> bool {
          if (u < nu && ((ec >> (16 + q)) & 1)) {
            if (!k_ready) {
              if (!mbar_wait(&sh.k_full[sc], (u / kF8Stages) & 1, abort_flag, st)) return false;
              tc_fence_after();
              k_ready = true;
            }
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {      // 4 x 32 head-dim values
              const uint64_t adesc = smem_desc_sw128(aQ + q * kF8TileBytes + kk * 32, 16, 1024);
              const uint64_t bdesc = smem_desc_sw128(aK + sc * kF8TileBytes + kk * 32, 16, 1024);
              mma_ss_f8(tmem + q * 128, adesc, bdesc, kIdescF8, kk > 0 ? 1u : 0u);
            }
            tc_commit(&sh.s_full[q]);
          }
          return true;
        };
        ok = pv(0, npv0) && sq(0) && pv(1, npv1);
        if (u > 0 && ok) tc_commit(&sh.v_empty[sp]);       // V(u-1) free once its PV products are done
        ok = ok && sq(1);
        if (u < nu && ok) tc_commit(&sh.k_empty[sc]);      // K(u) free once its S products are done
      }
      if (ok) {
        tc_commit(&sh.s_full[0]);   // final phase: every MMA into O_0 / O_1 has completed
        tc_commit(&sh.s_full[1]);
      }
      tc_commit(&sh.mma_done);
      mbar_wait_drain(&sh.mma_done, 0, st);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ softmax groups
    const int q = warp >> 2;
    const int wq = warp & 3;
    const int row_local = wq * 32 + lane;
    const int qt = qt0 + q;
    const int row = qt * kTile + row_local;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + q * 128 + lane_off;
    const uint32_t tO = tmem + 256 + q * kF8D + lane_off;
    uint8_t* prow = sP + q * kF8TileBytes + row_local * 128;   // this row of P (128-byte swizzle)
    const float sl2 = a.scale_log2;
    float m = -INFINITY;
    float l = 0.f;
    int c = 0;
    bool ok = true;
    for (int u = 0; u < nu; ++u) {
      const int e = list[u];
      if (!((e >> (16 + q)) & 1)) continue;
      const int key0 = (e & 0xFFFF) * kTile;
      ok = mbar_wait(&sh.s_full[q], c & 1, abort_flag, st);
      if (__any_sync(0xffffffffu, !ok)) { ok = false; break; }
      tc_fence_after();
      uint32_t sr[128];
      tmem_ld32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_ld32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tmem_ld32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[64]));
      tmem_ld32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(&sr[96]));
      tmem_wait_ld();
#pragma unroll
      for (int cq = 0; cq < 4; ++cq) reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&sr[32 * cq]));
      float s[128];
#pragma unroll
      for (int i = 0; i < 128; ++i) s[i] = __uint_as_float(sr[i]);
      if ((a.causal && key0 + kTile - 1 > qt * kTile) || key0 + kTile > a.N) {
        int lim = a.N - key0;
        if (a.causal) lim = min(lim, row - key0 + 1);
#pragma unroll
        for (int i = 0; i < 128; ++i)
          if (i >= lim) s[i] = -INFINITY;
      }
      const float mx = row_max128(s);
      const float mx2 = mx * sl2;
      float alpha = 1.f;
      bool resc = false;
      if (mx2 > m) {
        alpha = ex2(m - mx2);
        resc = (c > 0);
        m = mx2;
      }
      const float mneg = (m == -INFINITY) ? 0.f : -m;
      const float2 sl2v = make_float2(sl2, sl2), mnegv = make_float2(mneg, mneg);
      const float2 p256 = make_float2(kF8PScale, kF8PScale);
      float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        uint32_t pw[8];                            // keys 32h .. 32h+31 as E4M3 bytes
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float2 t = fma2(make_float2(s[32 * h + 2 * i], s[32 * h + 2 * i + 1]), sl2v, mnegv);
          const float2 p = (((16 * h + i) & 7) < kF8PolyOf8) ? exp2_poly2(t) : make_float2(ex2(t.x), ex2(t.y));
          acc[i & 3] = add2(acc[i & 3], p);
          const float2 ps = mul2(p, p256);
          const uint32_t b2 = pack_e4m3x2(ps.x, ps.y);
          if (i & 1) pw[i >> 1] |= b2 << 16;
          else pw[i >> 1] = b2;
        }
        const int sw = row_local & 7;
        *reinterpret_cast<uint4*>(prow + (((2 * h) ^ sw) * 16)) = make_uint4(pw[0], pw[1], pw[2], pw[3]);
        *reinterpret_cast<uint4*>(prow + (((2 * h + 1) ^ sw) * 16)) = make_uint4(pw[4], pw[5], pw[6], pw[7]);
      }
      const float2 a01 = add2(acc[0], acc[1]), a23 = add2(acc[2], acc[3]);
      const float2 a0123 = add2(a01, a23);
      l = l * alpha + (a0123.x + a0123.y);
      if (__any_sync(0xffffffffu, resc)) {
        const float f = resc ? alpha : 1.f;
#pragma unroll
        for (int cc = 0; cc < kF8D; cc += 32) {
          uint32_t o[32];
          tmem_ld32_sync(tO + cc, o);
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            const float2 r = mul2(make_float2(__uint_as_float(o[i]), __uint_as_float(o[i + 1])), make_float2(f, f));
            o[i] = __float_as_uint(r.x);
            o[i + 1] = __float_as_uint(r.y);
          }
          tmem_st32(tO + cc, o);
        }
      }
      fence_async_smem();                          // P rows visible to the tensor cores
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sh.p_full[q]);
      ++c;
    }
    const int nq = sh.n_q[q];
    if (ok) ok = mbar_wait(&sh.s_full[q], nq & 1, abort_flag, st);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
      tc_fence_after();
      const bool valid = row < a.N;
      const float inv = (l > 0.f) ? a.o_scale / l : 0.f;
      if (valid) a.lse[(size_t)bh * a.N + row] = (l > 0.f) ? (m + log2f(l)) * kLn2F8 : -INFINITY;
      const size_t obase = ((size_t)bh * a.N + row) * kF8D;
#pragma unroll
      for (int cc = 0; cc < kF8D; cc += 32) {
        uint32_t o[32];
        if (nq > 0) {
          tmem_ld32_sync(tO + cc, o);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0u;
        }
        if (valid) {
          if constexpr (kOut32) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(a.o) + obase + cc);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              dst[i] = make_float4(__uint_as_float(o[4 * i]) * inv, __uint_as_float(o[4 * i + 1]) * inv,
                                   __uint_as_float(o[4 * i + 2]) * inv, __uint_as_float(o[4 * i + 3]) * inv);
          } else {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(a.o) + obase + cc);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              uint4 w;
              w.x = pack2<false>(__uint_as_float(o[8 * i + 0]) * inv, __uint_as_float(o[8 * i + 1]) * inv);
              w.y = pack2<false>(__uint_as_float(o[8 * i + 2]) * inv, __uint_as_float(o[8 * i + 3]) * inv);
              w.z = pack2<false>(__uint_as_float(o[8 * i + 4]) * inv, __uint_as_float(o[8 * i + 5]) * inv);
              w.w = pack2<false>(__uint_as_float(o[8 * i + 6]) * inv, __uint_as_float(o[8 * i + 7]) * inv);
              dst[i] = w;
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace

cudaError_t launch_fwd_fp8(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tvt, const F8Args& a,
                           const uint8_t* v, uint8_t* vt, int Np, cudaStream_t s) {
  const int T = Np / kTile;
  vt_kernel<<<dim3((unsigned)T, (unsigned)a.BH), 256, 0, s>>>(v, vt, a.N, Np);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t smem = kF8SmemTiles + (size_t)a.T * sizeof(int) + 1024;
  auto kern = a.o_fp32 ? fwd_fp8_kernel<true> : fwd_fp8_kernel<false>;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const unsigned grid = static_cast<unsigned>(a.BH) * static_cast<unsigned>(a.n_units);
  kern<<<grid, 320, smem, s>>>(tq, tk, tvt, a);
  return cudaGetLastError();
}

}  // namespace fa
