// fa_bwd.cu -- fused exact-attention backward pass for sm_100a.
//
// The forward saved only O and the per-row log-sum-exp; the backward recomputes every
// probability tile from Q, K and LSE on chip instead of reading an N x N matrix back
// (FlashAttention-NeurIPS22 summary, "核心方法 / Backward recomputation").  Gradients of
// L = sum(dO o O), from the softmax Jacobian:
//     P = exp(scale*QKᵀ - LSE),  dV = Pᵀ dO,  dP = dO Vᵀ,  D_i = sum_c dO_ic O_ic,
//     dS = P o (dP - D),  dQ = scale * dS K,  dK = scale * dSᵀ Q.
//
// Three kernels on one stream:
//   bwd_pre   -D_i and -LSE_i*log2(e) (padded to whole tiles), and a zeroed fp32 dQ accumulator;
//   bwd_main  one CTA per (b, h, 128-key tile j): K_j, V_j stay in shared memory while the
//             CTA walks the kept 128-row query tiles i (i >= j under causal masking, and
//             blockmask[i][j] != 0); dK_j, dV_j accumulate in tensor memory, the dQ_i
//             partial of each step is added into the fp32 accumulator;
//   bwd_post  dQ = 16-bit(scale * accumulator).
//
// Dropout (kDrop): the mask of the forward pass is regenerated from the same Philox4x32-10
// counters ("核心方法 / Backward recomputation" regenerates it from the generator state):
// dV = (P o M)ᵀ dO, and dS = P o (dP o M - D).  A compute thread owns one key row and 64 query
// columns, while one generator call covers 16 keys of one query row, so each warp draws its
// 128 calls (64 columns x 2 blocks of 16 keys) four per lane and hands each key row its bytes
// with 64 shuffles (see drop_bits).
//
// Deterministic mode (dq_fix set): the dQ partials are added as int64 fixed point (2^-32
// resolution) by 64-bit bulk reduce-adds.  Integer addition is associative, so the sum -- and
// dQ -- is bitwise independent of the order in which CTAs finish; the float path's order-
// dependent fp32 additions are the only non-repeatable step of the backward.
//
// bwd_main roles (320 threads): warps 0-7 two compute groups, one key row per thread (TMEM
// lanes), each group owning half of the query columns and draining half of each dQ partial;
// warp 8 TMA producer; warp 9 MMA issuer.  At d = 64 in the default mode, four groups (warps
// 0-15, a quarter of the query columns each; groups 0 and 1 also drain dQ and write dV / dK),
// producer warp 16, MMA warp 17.
// Tensor memory: Sᵀ/Pᵀ [0,128) (Pᵀ as 16-bit over columns [0,32) and [64,96)), dPᵀ [128,256),
// dV and dK after them; dQ shares the dPᵀ columns when d = 128 and has its own for d = 64.
// Per query tile, the MMAs: Sᵀ = K Q_iᵀ, dPᵀ = V dO_iᵀ, dV += Pᵀ dO_i (Pᵀ from TMEM),
// dK += dSᵀ Q_i, dQ_i = dS K, issued one tile ahead where TMEM allows (see the MMA role)
// where dSᵀ is written once to shared memory (16-bit, 128-byte swizzle) and read both as
// K-major Sᵀ-shaped operand (for dK) and as its transpose, an MN-major operand (for dQ).
#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {
namespace {

constexpr float kLog2e = 1.4426950408889634f;

// ------------------------------------------------------------------------------------
// bwd_pre
// ------------------------------------------------------------------------------------
template <int D, bool kFp16>
__global__ void __launch_bounds__(256) bwd_pre_kernel(const BwdPreArgs a) {
  constexpr int G = D / 8;                 // threads per row, 8 elements (16 B) each
  constexpr int kRowsPerBlock = 256 / G;
  const int g = threadIdx.x % G;
  const long long total = (long long)a.BH * a.Np;
  // Block-uniform trip count: every lane of a warp runs the same iterations (shuffles below).
  for (long long rb = (long long)blockIdx.x * kRowsPerBlock; rb < total; rb += (long long)gridDim.x * kRowsPerBlock) {
    const long long r = rb + threadIdx.x / G;
    const bool active = r < total;
    const int bh = active ? (int)(r / a.Np) : 0;
    const int i = active ? (int)(r % a.Np) : a.N;
    float acc = 0.f;
    if (i < a.N) {
      const size_t off = ((size_t)bh * a.N + i) * D + g * 8;
      const uint4 ov = *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(a.o) + off);
      const uint4 dv = *reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(a.dout) + off);
      const uint32_t ow[4] = {ov.x, ov.y, ov.z, ov.w};
      const uint32_t dw[4] = {dv.x, dv.y, dv.z, dv.w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const float2 of = unpack2<kFp16>(ow[t]);
        const float2 df = unpack2<kFp16>(dw[t]);
        acc = fmaf(of.x, df.x, acc);
        acc = fmaf(of.y, df.y, acc);
      }
      if (a.dq_fix == nullptr) {
        float4* z = reinterpret_cast<float4*>(a.dq_acc + off);
        z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
        z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
      if (a.dk_acc != nullptr) {
        float4* zk = reinterpret_cast<float4*>(a.dk_acc + off);
        float4* zv = reinterpret_cast<float4*>(a.dv_acc + off);
        zk[0] = zk[1] = zv[0] = zv[1] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
    if (a.dq_fix != nullptr && active) {       // every row of the padded accumulator, 4 x 16 bytes
      const long long tile = (long long)bh * (a.Np / 128) + i / 128;
#pragma unroll
      for (int t = 0; t < 4; ++t)
        *reinterpret_cast<longlong2*>(a.dq_fix + fix_index(tile, i & 127, g * 8 + 2 * t, D)) = make_longlong2(0, 0);
    }
#pragma unroll
    for (int s = G / 2; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s, G);
    if (g == 0 && active) {
      a.delta[r] = -acc;                       // stored negated: the main kernel adds it
      float nl2 = -INFINITY;                   // padding rows and rows with no visible key: P = 0
      if (i < a.N) {
        const float lse = a.lse[(size_t)bh * a.N + i];
        if (lse > -INFINITY) nl2 = -lse * kLog2e;
      }
      a.lse2[r] = nl2;                         // -LSE * log2(e)
    }
  }
}

// ------------------------------------------------------------------------------------
// bwd_post
// ------------------------------------------------------------------------------------
template <bool kFp16>
__device__ __forceinline__ void convert8(const float* acc, void* out, long long t, float f) {
  const float4* src = reinterpret_cast<const float4*>(acc) + 2 * t;
  const float4 x = src[0], y = src[1];
  uint4 w;
  w.x = pack2<kFp16>(x.x * f, x.y * f);
  w.y = pack2<kFp16>(x.z * f, x.w * f);
  w.z = pack2<kFp16>(y.x * f, y.y * f);
  w.w = pack2<kFp16>(y.z * f, y.w * f);
  reinterpret_cast<uint4*>(out)[t] = w;
}

template <bool kFp16>
__global__ void __launch_bounds__(256) bwd_post_kernel(const BwdPostArgs a) {
  const long long n8 = a.n_elems / 8;
  for (long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x; t < n8; t += (long long)gridDim.x * blockDim.x) {
    convert8<kFp16>(a.dq_acc, a.dq, t, a.scale);
    if (a.dk_acc != nullptr) {                 // query-range splits: dK and dV from their accumulators
      convert8<kFp16>(a.dk_acc, a.dk, t, a.scale);
      convert8<kFp16>(a.dv_acc, a.dv, t, 1.f);
    }
  }
}

// Deterministic mode: dQ = 16-bit(scale * 2^-32 * int64 accumulator), one thread per row
// and 8 columns (four 16-byte pieces of the tile-blocked layout).
template <int D, bool kFp16>
__global__ void __launch_bounds__(256) bwd_post_fix_kernel(const BwdPostArgs a) {
  constexpr int G = D / 8;
  const long long total = (long long)a.BH * a.N * G;
  const float f = a.scale * (1.0f / kFixOne);
  for (long long t = (long long)blockIdx.x * blockDim.x + threadIdx.x; t < total; t += (long long)gridDim.x * blockDim.x) {
    const long long r = t / G;
    const int g = (int)(t - r * G);
    const int bh = (int)(r / a.N), i = (int)(r % a.N);
    const long long tile = (long long)bh * (a.Np / 128) + i / 128;
    uint32_t w[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const longlong2 x = *reinterpret_cast<const longlong2*>(a.dq_fix + fix_index(tile, i & 127, g * 8 + 2 * u, D));
      w[u] = pack2<kFp16>(__ll2float_rn(x.x) * f, __ll2float_rn(x.y) * f);
    }
    reinterpret_cast<uint4*>(static_cast<uint16_t*>(a.dq) + r * D)[g] = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

// ------------------------------------------------------------------------------------
// bwd_main
// ------------------------------------------------------------------------------------
template <int D>
struct BwdCfg {
  static constexpr int kPanels = D / 64;
  static constexpr int kTileBytes = kTile * D * 2;
  static constexpr int kPanelBytes = kTile * 128;
  static constexpr int kStages = 2;
  // layout (offsets from a 1024-byte aligned base)
  static constexpr int oK = 0;
  static constexpr int oV = oK + kTileBytes;
  static constexpr int oQ = oV + kTileBytes;
  static constexpr int oDO = oQ + kStages * kTileBytes;
  static constexpr int oDS = oDO + kStages * kTileBytes;     // 128 keys x 128 queries, 16-bit
  static constexpr int oLSE = oDS + kTile * kTile * 2;
  static constexpr int oDELTA = oLSE + kStages * kTile * 4;
  static constexpr int oBAR = oDELTA + kStages * kTile * 4;
  // dQ staging for the TMA reduce: its own 32 KB at d = 64 (the reduce's shared-memory read
  // then overlaps the next tile's work); at d = 128 shared memory is full and the dSᵀ panels
  // are reused, so the read must finish before the next dSᵀ tile is stored.
  static constexpr bool kOwnStaging = (D == 64);
  static constexpr int oSTG = ((oBAR + 256 + 1023) / 1024) * 1024;
  static constexpr int kSmem = kOwnStaging ? oSTG + 2 * kPanelBytes : oBAR + 256;
  // exp2 pairs per 8 evaluated by the FMA-pipe polynomial in the P phase (measured: 2 of 8
  // helps slightly at d = 64, any share is slower at d = 128)
  static constexpr int kPolyOf8 = (D == 64) ? 2 : 0;
  static constexpr int tS = 0, tDP = 128, tDV = 256, tDK = 256 + D, tDQ = (D == 128) ? 128 : 384;
  static constexpr bool kDqSharesDp = (D == 128);
};

constexpr int kBwdThreads = 320;   // 2 compute groups (8 warps), producer, MMA issuer
// d = 64, float dQ: four compute groups of 32 query columns (18 warps, 96 registers) instead of
// two.  The twice as many warps hide the phase latencies that bound this kernel at d = 64
// (measured backward main: +5 to +7 % from N = 512 to 16384, causal included; with dropout,
// whose generator work they also share, +7 to +19 %).
constexpr bool kBwdFourGroups = true;

struct BwdBars {
  uint64_t kv_full;
  uint64_t q_full[2], q_empty[2];
  uint64_t s_full, dp_full, p_full, ds_full, dq_full, dq_empty, mma_done;
  uint32_t tmem_base;
  int abort_flag;
};

// Query tiles are visited in the rotated order i = (j + k) mod T, k = 0, 1, ...: every key
// tile starts at its own diagonal, so the CTAs of one head add their dQ partials into
// different accumulator rows at any moment instead of all into the same ones.  Under causal
// masking this is the natural order j, j+1, ..., T-1 (the wrapped part is all masked).
__device__ __forceinline__ int rot_tile(int k, int j, int T) {
  const int i = j + k;
  return i < T ? i : i - T;
}

// Keep bits of the 64 query columns q0 .. q0+63 for this lane's key row (32 * wq + lane of key
// tile j): bit c of the result is the decision for query q0 + c.
// Lane L draws the calls of columns 4 * (L % 16) + k (k = 0..3) for the key block of its
// half-warp, and stores each call's words rotated by L % 4.  Then in round (k, q, s) a lane
// of word group w = (L % 16) / 4 reads slot s from lane 16 * half + 4q + ((w - s) mod 4),
// which holds word w there: 64 shuffles deliver each lane the byte of all 64 columns.
__device__ __forceinline__ uint64_t drop_bits(const Dropout& dr, int j, int wq, int lane, int q0, int bh) {
  const int half = lane >> 4;
  const uint32_t jb = static_cast<uint32_t>((j * kTile + wq * 32) >> 4) + half;
  const int rot = lane & 3;
  uint32_t R[4][4];
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint4 w4 = philox4x32_10(make_uint4(jb, static_cast<uint32_t>(q0 + 4 * (lane & 15) + k),
                                              static_cast<uint32_t>(bh), 0u), dr.seed_lo, dr.seed_hi);
#pragma unroll
    for (int sl = 0; sl < 4; ++sl) {
      const int idx = (sl + rot) & 3;
      R[k][sl] = (idx & 2) ? ((idx & 1) ? w4.w : w4.z) : ((idx & 1) ? w4.y : w4.x);
    }
  }
  const int w = (lane & 15) >> 2;
  const int bsh = 8 * (lane & 3);
  uint32_t lo = 0u, hi = 0u;
#pragma unroll
  for (int k = 0; k < 4; ++k)
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
      for (int sl = 0; sl < 4; ++sl) {
        const int g4 = (w - sl) & 3;
        const uint32_t x = __shfl_sync(0xffffffffu, R[k][sl], (half << 4) | (4 * q + g4));
        const uint32_t bit = ((x >> bsh) & 0xFFu) >= dr.t ? 1u : 0u;
        const int cpos = (16 * q + 4 * g4 + k) & 31;
        if (q < 2) lo |= bit << cpos;
        else hi |= bit << cpos;
      }
  return (static_cast<uint64_t>(hi) << 32) | lo;
}

// The same for the 32 query columns q0 .. q0+31 of a four-group layout: lane L draws the calls
// of columns 2 * (L % 16) + k (k = 0, 1) for the key block of its half-warp, words rotated by
// L % 4; in round (k, q, s) a lane of word group w reads slot s from lane
// 16 * half + 4q + ((w - s) mod 4), whose columns are 2 * (4q + ((w - s) mod 4)) + k: 32 shuffles
// deliver each lane the byte of all 32 columns.  Bit c of the result is query q0 + c.
__device__ __forceinline__ uint32_t drop_bits32(const Dropout& dr, int j, int wq, int lane, int q0, int bh) {
  const int half = lane >> 4;
  const uint32_t jb = static_cast<uint32_t>((j * kTile + wq * 32) >> 4) + half;
  const int rot = lane & 3;
  uint32_t R[2][4];
#pragma unroll
  for (int k = 0; k < 2; ++k) {
    const uint4 w4 = philox4x32_10(make_uint4(jb, static_cast<uint32_t>(q0 + 2 * (lane & 15) + k),
                                              static_cast<uint32_t>(bh), 0u), dr.seed_lo, dr.seed_hi);
#pragma unroll
    for (int sl = 0; sl < 4; ++sl) {
      const int idx = (sl + rot) & 3;
      R[k][sl] = (idx & 2) ? ((idx & 1) ? w4.w : w4.z) : ((idx & 1) ? w4.y : w4.x);
    }
  }
  const int w = (lane & 15) >> 2;
  const int bsh = 8 * (lane & 3);
  uint32_t bits = 0u;
#pragma unroll
  for (int k = 0; k < 2; ++k)
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
      for (int sl = 0; sl < 4; ++sl) {
        const int g4 = (w - sl) & 3;
        const uint32_t x = __shfl_sync(0xffffffffu, R[k][sl], (half << 4) | (4 * q + g4));
        const uint32_t bit = ((x >> bsh) & 0xFFu) >= dr.t ? 1u : 0u;
        bits |= bit << (2 * (4 * q + g4) + k);
      }
  return bits;
}

// Next step k' in [k, k_end) whose query tile the key tile j keeps (k_end when none).
__device__ __forceinline__ int next_kept(int k, int j, int k_end, int T, int causal, const uint8_t* mask) {
  for (; k < k_end; ++k) {
    const int i = rot_tile(k, j, T);
    if (causal && i < j) continue;
    if (mask != nullptr && __ldg(mask + (size_t)i * T + j) == 0) continue;
    break;
  }
  return k;
}

// kG compute groups of 128 threads, each owning 128 / kG query columns of every tile: kG = 2
// (the default) or kG = 4 (d = 64, default mode: twice the warps to hide phase latencies; the
// dQ drain and the dV / dK epilogue stay with groups 0 and 1).
template <int D, bool kFp16, bool kDet, bool kDrop, int kG>
__global__ void __launch_bounds__(128 * kG + 64, 1)
    bwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
               const __grid_constant__ CUtensorMap tm_dq, const BwdArgs a) {
  using C = BwdCfg<D>;
  static_assert(kG == 2 || (kG == 4 && D == 64 && !kDet), "four groups: d = 64, float dQ");
  constexpr int kLoadW = 4 * kG, kMmaW = 4 * kG + 1;
  constexpr int kCols = kTile / kG;                 // query columns per compute group
  extern __shared__ __align__(1024) uint8_t smem[];
  BwdBars& sh = *reinterpret_cast<BwdBars*>(smem + C::oBAR);
  const int warp = warp_id(), lane = lane_id();
  // CTAs resident together share a few heads, so those heads' Q / dO tiles and fp32 dQ
  // accumulator rows stay in L2 (ordering by key tile across all heads thrashed L2); within
  // a group, key tile 0 (the heaviest under causal masking) goes first.
  int bh, j, slot;
  cta_order(blockIdx.x, a.BH, a.T * a.q_splits, a.group_heads, bh, slot);
  j = slot / a.q_splits;
  // query-range split of this CTA: visiting steps k in [k_begin, k_end)
  const int k_begin = (slot - j * a.q_splits) * a.q_chunk;
  const int k_end = min(a.T, k_begin + a.q_chunk);
  const DevStatus st{a.status, a.timeout_ns};
  volatile int* abort_flag = &sh.abort_flag;
  const bool aligned = (smem_addr(smem) & 1023u) == 0;

  if (threadIdx.x == 0) {
    mbar_init(&sh.kv_full, 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&sh.q_full[s], 1);
      mbar_init(&sh.q_empty[s], 1);
    }
    mbar_init(&sh.s_full, 1);
    mbar_init(&sh.dp_full, 1);
    mbar_init(&sh.p_full, 128 * kG);
    mbar_init(&sh.ds_full, 128 * kG);
    mbar_init(&sh.dq_full, 1);
    mbar_init(&sh.dq_empty, 256);
    mbar_init(&sh.mma_done, 1);
    sh.abort_flag = aligned ? 0 : 1;
    if (!aligned) atomicCAS(a.status, 0, kDevBadState);
    fence_barrier_init();
  }
  if (warp == kMmaW) {
    tmem_alloc(&sh.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sh.tmem_base;
  const int k_first = next_kept(k_begin, j, k_end, a.T, a.causal, a.blockmask);
  const bool any = aligned && k_first < k_end;

  if (warp == kLoadW) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0 && any) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      prefetch_tmap(&tm_do);
      mbar_arrive_expect_tx(&sh.kv_full, 2 * C::kTileBytes);
      for (int p = 0; p < C::kPanels; ++p) {
        tma_load_3d(smem + C::oK + p * C::kPanelBytes, &tm_k, &sh.kv_full, p * 64, j * kTile, bh);
        tma_load_3d(smem + C::oV + p * C::kPanelBytes, &tm_v, &sh.kv_full, p * 64, j * kTile, bh);
      }
      int c = 0;
      for (int k = k_first; k < k_end; k = next_kept(k + 1, j, k_end, a.T, a.causal, a.blockmask), ++c) {
        const int i = rot_tile(k, j, a.T);
        const int s = c % C::kStages;
        if (c >= C::kStages && !mbar_wait(&sh.q_empty[s], ((c / C::kStages) - 1) & 1, abort_flag, st)) break;
        mbar_arrive_expect_tx(&sh.q_full[s], 2 * C::kTileBytes + 2 * kTile * 4);
        for (int p = 0; p < C::kPanels; ++p) {
          tma_load_3d(smem + C::oQ + s * C::kTileBytes + p * C::kPanelBytes, &tm_q, &sh.q_full[s], p * 64, i * kTile, bh);
          tma_load_3d(smem + C::oDO + s * C::kTileBytes + p * C::kPanelBytes, &tm_do, &sh.q_full[s], p * 64, i * kTile,
                      bh);
        }
        const size_t roff = (size_t)bh * a.Np + (size_t)i * kTile;
        bulk_load(smem + C::oLSE + s * kTile * 4, a.lse2 + roff, kTile * 4, &sh.q_full[s]);
        bulk_load(smem + C::oDELTA + s * kTile * 4, a.delta + roff, kTile * 4, &sh.q_full[s]);
      }
      if (*abort_flag) {
        mbar_wait_drain(&sh.kv_full, 0, st);
        for (int cc = (c > C::kStages ? c - C::kStages : 0); cc < c; ++cc)
          mbar_wait_drain(&sh.q_full[cc % C::kStages], (cc / C::kStages) & 1, st);
      }
    }
    __syncwarp();
  } else if (warp == kMmaW) {
    // ------------------------------------------------------------------ MMA issuer
    // Issue order per kept query tile c (stage s = c % 2):
    //   [Sᵀ(c), dPᵀ(c) issued one step earlier]  dV += Pᵀ(c) dO(c);  Sᵀ(c+1);
    //   dK += dSᵀ(c) Q(c);  dQ(c) = dS(c) K;  dPᵀ(c+1)
    // so Sᵀ(c+1) runs while the compute groups form dS(c), and dPᵀ(c+1) while they form P(c+1).
    // Sᵀ(c+1) overwrites Pᵀ(c) in TMEM only after dV(c), which reads it, was issued
    // (tcgen05.mma operations from one thread execute in issue order).
    if (lane == 0) {
      const uint32_t id_sq = idesc_f16(128, 128, kFp16, false, false);   // K-major x K-major
      const uint32_t id_kn = idesc_f16(128, D, kFp16, false, true);      // K-major A, MN-major B
      const uint32_t id_mn = idesc_f16(128, D, kFp16, true, true);       // MN-major A and B
      const uint32_t aK = smem_addr(smem + C::oK), aV = smem_addr(smem + C::oV);
      const uint32_t aQ = smem_addr(smem + C::oQ), aDO = smem_addr(smem + C::oDO);
      const uint32_t aDS = smem_addr(smem + C::oDS);
      auto issue_s = [&](int s) {   // Sᵀ = K Q_sᵀ
        const uint32_t qb = aQ + s * C::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = (kk >> 2) * C::kPanelBytes + (kk & 3) * 32;
          mma_ss(tmem + C::tS, smem_desc_sw128(aK + koff, 16, 1024), smem_desc_sw128(qb + koff, 16, 1024), id_sq,
                 kk > 0 ? 1u : 0u);
        }
        tc_commit(&sh.s_full);
      };
      auto issue_dp = [&](int s) {  // dPᵀ = V dO_sᵀ
        const uint32_t dob = aDO + s * C::kTileBytes;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t koff = (kk >> 2) * C::kPanelBytes + (kk & 3) * 32;
          mma_ss(tmem + C::tDP, smem_desc_sw128(aV + koff, 16, 1024), smem_desc_sw128(dob + koff, 16, 1024), id_sq,
                 kk > 0 ? 1u : 0u);
        }
        tc_commit(&sh.dp_full);
      };
      bool ok = any && mbar_wait(&sh.kv_full, 0, abort_flag, st) && mbar_wait(&sh.q_full[0], 0, abort_flag, st);
      int c = 0;
      if (ok) {
        tc_fence_after();
        issue_s(0);
        if (a.visit != nullptr) atomicAdd(&a.visit[((size_t)bh * a.T + rot_tile(k_first, j, a.T)) * a.T + j], 1);
        issue_dp(0);
        for (int k = k_first; k < k_end; ++c) {
          const int s = c % C::kStages;
          const int k_next = next_kept(k + 1, j, k_end, a.T, a.causal, a.blockmask);
          const bool more = k_next < k_end;
          const int i_next = more ? rot_tile(k_next, j, a.T) : 0;
          const uint32_t qb = aQ + s * C::kTileBytes, dob = aDO + s * C::kTileBytes;
          // dV += Pᵀ dO(c)   (Pᵀ read from tensor memory)
          if (!(ok = mbar_wait(&sh.p_full, c & 1, abort_flag, st))) break;
          tc_fence_after();
          // Pᵀ query columns 16kk..16kk+15 sit in TMEM columns kCols*(16kk/kCols) + (16kk mod kCols)/2
          // (each group packs its columns over the first half of its own Sᵀ range)
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk)
            mma_ts(tmem + C::tDV, tmem + C::tS + (16 * kk / kCols) * kCols + ((16 * kk) % kCols) / 2,
                   smem_desc_sw128(dob + kk * 2048, C::kPanelBytes, 1024), id_kn, (c > 0 || kk > 0) ? 1u : 0u);
          // Sᵀ(c+1)
          if (more) {
            const int s1 = (c + 1) % C::kStages;
            if (!(ok = mbar_wait(&sh.q_full[s1], ((c + 1) / C::kStages) & 1, abort_flag, st))) break;
            tc_fence_after();
            issue_s(s1);
            if (a.visit != nullptr) atomicAdd(&a.visit[((size_t)bh * a.T + i_next) * a.T + j], 1);
          }
          // dK += dSᵀ Q(c)
          if (!(ok = mbar_wait(&sh.ds_full, c & 1, abort_flag, st))) break;
          tc_fence_after();
          auto issue_dk = [&]() {
#pragma unroll
            for (int kk = 0; kk < kTile / 16; ++kk) {
              const uint32_t koff = (kk >> 2) * C::kPanelBytes + (kk & 3) * 32;
              mma_ss(tmem + C::tDK, smem_desc_sw128(aDS + koff, 16, 1024),
                     smem_desc_sw128(qb + kk * 2048, C::kPanelBytes, 1024), id_kn, (c > 0 || kk > 0) ? 1u : 0u);
            }
          };
          // d = 128: dK before dQ, so dq_full (the drain may then stage into the dSᵀ panel)
          // also covers dK's reads of that panel; d = 64 stages elsewhere and issues dQ first,
          // so its drain starts while dK runs (measured +0.6 to +1.1 %)
          if constexpr (D == 128) issue_dk();
          // dQ(c) = dS K   (dS = transpose of the stored dSᵀ: an MN-major operand)
          if (!C::kDqSharesDp && c > 0) {
            if (!(ok = mbar_wait(&sh.dq_empty, (c - 1) & 1, abort_flag, st))) break;
            tc_fence_after();
          }
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk)
            mma_ss(tmem + C::tDQ, smem_desc_sw128(aDS + kk * 2048, C::kPanelBytes, 1024),
                   smem_desc_sw128(aK + kk * 2048, C::kPanelBytes, 1024), id_mn, kk > 0 ? 1u : 0u);
          tc_commit(&sh.dq_full);
          if constexpr (D == 64) issue_dk();
          tc_commit(&sh.q_empty[s]);
          // dPᵀ(c+1)   (its columns hold dQ(c) when d = 128: wait for the drain)
          if (more) {
            if (C::kDqSharesDp) {
              if (!(ok = mbar_wait(&sh.dq_empty, c & 1, abort_flag, st))) break;
              tc_fence_after();
            }
            issue_dp((c + 1) % C::kStages);
          }
          k = k_next;
        }
      }
      tc_commit(&sh.mma_done);
      mbar_wait_drain(&sh.mma_done, 0, st);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ key-row compute groups
    // Group g (warps 4g..4g+3) owns query columns [kCols g, kCols (g+1)) of every Sᵀ / dPᵀ
    // tile; each thread owns one key row (TMEM lane).  P stays in registers between the two
    // phases.  Groups 0 and 1 also drain each dQ partial (query rows on TMEM lanes, half the
    // columns each) right after the next P phase: the columns are released as soon as they
    // are read, and the reduction into the accumulator follows from shared memory.
    const int g = warp >> 2;
    const int wq = warp & 3;
    const int r = wq * 32 + lane;                   // key row within the tile == TMEM lane
    const int key = j * kTile + r;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + C::tS + lane_off, tDP = tmem + C::tDP + lane_off;
    constexpr int kHalfD = D / 2;                   // dQ columns drained by each group
    const uint32_t tQ = tmem + C::tDQ + lane_off + kHalfD * g;
    const float sl2 = a.scale_log2;
    const bool key_ok = key < a.N;
    // this group's columns of the key row's dSᵀ: panel (kCols g) / 64, first 16-byte chunk ds_c0
    uint8_t* ds_row = smem + C::oDS + (kCols * g / 64) * C::kPanelBytes + r * 128;
    constexpr int kChunks = kCols / 8;
    const int ds_c0 = ((kCols * g) % 64) / 8;
    int c = 0;
    bool ok = true;
    int i_prev = -1;
    // dQ partial of query tile ip (the cq-th kept one), columns [kHalfD*g, kHalfD*(g+1)),
    // -> fp32 accumulator.  The group's dSᵀ panel (16 KB, free once dq_full says dK / dQ
    // have read it) stages 32 columns at a time in the 128-byte-swizzled layout of the
    // accumulator's TMA map; each warp stages its own 32 rows (4 KB) and its lane 0 issues a
    // TMA tensor reduce-add for them, so the reduction runs on the TMA engine instead of as
    // per-thread atomics, and only warp-level synchronisation is needed.
    uint8_t* stage = smem + (C::kOwnStaging ? C::oSTG : C::oDS) + g * C::kPanelBytes + wq * 32 * 128;
    // After a drain, lane 0 of each warp has reduce operations in flight that still read
    // `stage`; wait_stage_read() must run before `stage` (or, at d = 128, the dSᵀ panel it lives
    // in) is written again.
    auto wait_stage_read = [&]() {
      if (lane == 0) bulk_wait_read_all();
      __syncwarp();
    };
    auto drain = [&](int ip, int cq) -> bool {
      const bool got = mbar_wait(&sh.dq_full, cq & 1, abort_flag, st);
      if (!__all_sync(0xffffffffu, got)) return false;   // warp-uniform before warp-collective loads
      tc_fence_after();
      uint32_t v[kHalfD];
#pragma unroll
      for (int cc = 0; cc < kHalfD; cc += 32) tmem_ld32(tQ + cc, *reinterpret_cast<uint32_t(*)[32]>(&v[cc]));
      tmem_wait_ld();
#pragma unroll
      for (int cc = 0; cc < kHalfD; cc += 32) reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&v[cc]));
      tc_fence_before();
      mbar_arrive(&sh.dq_empty);                    // TMEM columns free for the next MMA
      if constexpr (kDet) {
        // int64 fixed point, 16 columns per bulk add: the warp's 32 rows x 16 columns are one
        // contiguous 4 KB block of the accumulator (fix_index), staged as [pair][lane][2].
        float mx = 0.f;
#pragma unroll
        for (int t = 0; t < kHalfD; ++t) mx = fmaxf(mx, fabsf(__uint_as_float(v[t])));
        if (!(mx < kFixLimit)) atomicCAS(a.status, 0, kDevRange);   // also catches NaN
        const long long tile = (long long)bh * a.T + ip;
#pragma unroll
        for (int ck = 0; ck < kHalfD / 16; ++ck) {
          wait_stage_read();
#pragma unroll
          for (int pr = 0; pr < 8; ++pr) {
            const long long x0 = __float2ll_rn(__uint_as_float(v[16 * ck + 2 * pr]) * kFixOne);
            const long long x1 = __float2ll_rn(__uint_as_float(v[16 * ck + 2 * pr + 1]) * kFixOne);
            *reinterpret_cast<longlong2*>(stage + pr * 512 + lane * 16) = make_longlong2(x0, x1);
          }
          fence_async_smem();
          __syncwarp();
          if (lane == 0) {
            const int col0 = kHalfD * g + 16 * ck;
            bulk_reduce_add_u64(a.dq_fix + fix_index(tile, wq * 32, col0, D), stage, 4096);
            bulk_commit();
          }
        }
      } else {
#pragma unroll
        for (int rd = 0; rd < kHalfD / 32; ++rd) {
          wait_stage_read();                          // previous reduce finished reading `stage`
          uint8_t* row_base = stage + lane * 128;
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            const int phys = ch ^ (lane & 7);
            *reinterpret_cast<uint4*>(row_base + phys * 16) =
                make_uint4(v[32 * rd + 4 * ch], v[32 * rd + 4 * ch + 1], v[32 * rd + 4 * ch + 2], v[32 * rd + 4 * ch + 3]);
          }
          fence_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_reduce_add_3d(&tm_dq, stage, kHalfD * g + 32 * rd, ip * kTile + wq * 32, bh);
            bulk_commit();
          }
        }
      }
      return true;
    };
    if (any) {
      for (int k = k_first; k < k_end; k = next_kept(k + 1, j, k_end, a.T, a.causal, a.blockmask), ++c) {
        const int i = rot_tile(k, j, a.T);
        const int s = c % C::kStages;
        uint32_t keep_lo = 0u, keep_hi = 0u;        // dropout keep bits of this row's kCols columns
        if constexpr (kDrop) {
          if constexpr (kCols == 64) {
            const uint64_t kb = drop_bits(a.drop, j, wq, lane, i * kTile + 64 * g, bh);
            keep_lo = static_cast<uint32_t>(kb);
            keep_hi = static_cast<uint32_t>(kb >> 32);
          } else {
            keep_lo = drop_bits32(a.drop, j, wq, lane, i * kTile + kCols * g, bh);
          }
        }
        ok = mbar_wait(&sh.q_full[s], (c / C::kStages) & 1, abort_flag, st) &&
             mbar_wait(&sh.s_full, c & 1, abort_flag, st);
        if (__any_sync(0xffffffffu, !ok)) { ok = false; break; }
        tc_fence_after();
        // -LSE*log2(e) and -D of this group's 64 query columns (bulk-loaded with the stage)
        const float* nlse2 = reinterpret_cast<const float*>(smem + C::oLSE + s * kTile * 4) + kCols * g;
        const float* ndlt = reinterpret_cast<const float*>(smem + C::oDELTA + s * kTile * 4) + kCols * g;
        const bool diag = a.causal && (i == j);     // key r visible to query column q iff r <= q
        // Phase A: Pᵀ = 2^(scale*log2e*Sᵀ - LSE*log2e), 16-bit, over Sᵀ in TMEM.  Both
        // 32-column chunks are loaded before one wait; -LSE*log2e comes in float4s; the
        // exponent argument is one packed fp32 FMA per pair.
        uint32_t pk[kCols / 2];
        {
          uint32_t sv[kCols];
#pragma unroll
          for (int m = 0; m < kCols / 32; ++m) tmem_ld32(tS + kCols * g + 32 * m, *reinterpret_cast<uint32_t(*)[32]>(&sv[32 * m]));
          tmem_wait_ld();
#pragma unroll
          for (int m = 0; m < kCols / 32; ++m) reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&sv[32 * m]));
          const float4* nl4 = reinterpret_cast<const float4*>(nlse2);
          const float2 sl2v = make_float2(sl2, sl2);
          const bool any_mask = !key_ok || diag;
#pragma unroll
          for (int t4 = 0; t4 < kCols / 4; ++t4) {     // 4 query columns per step
            const float4 nl = nl4[t4];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const int t = 2 * t4 + hh;                // pair index: columns 2t, 2t+1 of the 64
              const float2 x = fma2(make_float2(__uint_as_float(sv[2 * t]), __uint_as_float(sv[2 * t + 1])), sl2v,
                                    hh == 0 ? make_float2(nl.x, nl.y) : make_float2(nl.z, nl.w));
              float2 p = ((t & 7) < C::kPolyOf8) ? exp2_poly2(x) : make_float2(ex2(x.x), ex2(x.y));
              if (any_mask) {
                const int q0 = kCols * g + 2 * t;       // column within the tile
                if (!key_ok || (diag && r > q0)) p.x = 0.f;
                if (!key_ok || (diag && r > q0 + 1)) p.y = 0.f;
              }
              pk[t] = pack2<kFp16>(p.x, p.y);
            }
          }
        }
        // Pᵀ of this group's 64 query columns, packed two per 32-bit column, goes over the
        // first half of the group's own Sᵀ columns [64g, 64g+32): the other group may still be
        // reading its Sᵀ columns, so neither group writes outside its own range.
        if constexpr (kDrop) {
          // dV takes P o M: dropped columns 0, kept ones scaled (pk keeps the undropped P)
#pragma unroll
          for (int h2 = 0; h2 < kCols / 32; ++h2) {
            uint32_t pd[16];
            const uint32_t kw = h2 == 0 ? keep_lo : keep_hi;
#pragma unroll
            for (int t = 0; t < 16; ++t) {
              const float2 p = unpack2<kFp16>(pk[16 * h2 + t]);
              pd[t] = pack2<kFp16>(((kw >> (2 * t)) & 1u) ? p.x * a.drop.scale : 0.f,
                                   ((kw >> (2 * t + 1)) & 1u) ? p.y * a.drop.scale : 0.f);
            }
            tmem_st16(tS + kCols * g + 16 * h2, pd);
          }
        } else {
          if constexpr (kCols == 64) tmem_st32(tS + 64 * g, pk);
          else tmem_st16(tS + kCols * g, pk);
        }
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(&sh.p_full);
        // dQ of the previous query tile (its completion also frees the dSᵀ buffer).  With its
        // own staging (d = 64) the drain waits until this tile's dSᵀ is stored, so dK / dQ of
        // this tile are not held up by it and it fills the wait for the next Sᵀ (measured:
        // +4 % deterministic, +0.5 % default, -3 % with dropout, which keeps the early drain);
        // at d = 128 the staging is the dSᵀ panel, so the drain must come first.
        constexpr bool kLateDrain = C::kOwnStaging && !kDrop;
        if (!kLateDrain && g < 2 && c > 0) {         // groups 0 and 1 drain dQ
          ok = drain(i_prev, c - 1);
          if (__any_sync(0xffffffffu, !ok)) { ok = false; break; }
        }
        // Phase B: dSᵀ = Pᵀ o (dPᵀ - D), 16-bit, into this group's shared-memory panel
        ok = mbar_wait(&sh.dp_full, c & 1, abort_flag, st);
        if (__any_sync(0xffffffffu, !ok)) { ok = false; break; }
        tc_fence_after();
        {
          uint32_t dpv[kCols];
#pragma unroll
          for (int m = 0; m < kCols / 32; ++m) tmem_ld32(tDP + kCols * g + 32 * m, *reinterpret_cast<uint32_t(*)[32]>(&dpv[32 * m]));
          tmem_wait_ld();
#pragma unroll
          for (int m = 0; m < kCols / 32; ++m) reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&dpv[32 * m]));
          const float4* nd4 = reinterpret_cast<const float4*>(ndlt);
          uint32_t w[kCols / 2];
#pragma unroll
          for (int t4 = 0; t4 < kCols / 4; ++t4) {
            const float4 nd = nd4[t4];
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const int t = 2 * t4 + hh;                // pair index within the group's 64 columns
              const float2 p = unpack2<kFp16>(pk[t]);
              float2 dp = make_float2(__uint_as_float(dpv[2 * t]), __uint_as_float(dpv[2 * t + 1]));
              if constexpr (kDrop) {                    // dP o M
                const uint32_t kw = t < 16 ? keep_lo : keep_hi;
                dp.x = ((kw >> ((2 * t) & 31)) & 1u) ? dp.x * a.drop.scale : 0.f;
                dp.y = ((kw >> ((2 * t + 1) & 31)) & 1u) ? dp.y * a.drop.scale : 0.f;
              }
              const float2 ds = mul2(p, add2(dp, hh == 0 ? make_float2(nd.x, nd.y) : make_float2(nd.z, nd.w)));
              w[t] = pack2<kFp16>(ds.x, ds.y);
            }
          }
          // at d = 128 the dQ staging lives in this panel: its reduce must have read it
          if (!C::kOwnStaging) wait_stage_read();
          // 128 bytes = eight 16-byte chunks of this key row (128-byte swizzle)
#pragma unroll
          for (int t = 0; t < kChunks; ++t) {
            const int chunk = (ds_c0 + t) ^ (r & 7);
            *reinterpret_cast<uint4*>(ds_row + chunk * 16) = make_uint4(w[4 * t], w[4 * t + 1], w[4 * t + 2], w[4 * t + 3]);
          }
        }
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(&sh.ds_full);
        if (kLateDrain && g < 2 && c > 0) {
          ok = drain(i_prev, c - 1);
          if (__any_sync(0xffffffffu, !ok)) { ok = false; break; }
        }
        i_prev = i;
      }
      if (g < 2 && ok && c > 0) ok = drain(i_prev, c - 1);
      if (lane == 0) bulk_wait_all();
    }
    // Epilogue: group 0 writes dV, group 1 writes scale * dK, one key row per thread.
    if (ok) ok = mbar_wait(&sh.mma_done, 0, abort_flag, st);
    ok = __all_sync(0xffffffffu, ok);
    if (ok && g < 2 && a.q_splits > 1) {
      // query-range split: add this range's partial (dV, unscaled dK) into the fp32 accumulators
      if (c > 0) {
        tc_fence_after();
        const uint32_t tA = tmem + (g == 0 ? C::tDV : C::tDK) + lane_off;
        float* acc = (g == 0 ? a.dv_acc : a.dk_acc) + ((size_t)bh * a.N + key) * D;
#pragma unroll
        for (int cc = 0; cc < D; cc += 32) {
          uint32_t v[32];
          tmem_ld32_sync(tA + cc, v);
          if (key_ok) {
#pragma unroll
            for (int t = 0; t < 8; ++t)
              red_add_v4(acc + cc + 4 * t, __uint_as_float(v[4 * t]), __uint_as_float(v[4 * t + 1]),
                         __uint_as_float(v[4 * t + 2]), __uint_as_float(v[4 * t + 3]));
          }
        }
      }
    } else if (ok && g < 2) {
      tc_fence_after();
      const size_t base = ((size_t)bh * a.N + key) * D;
      const uint32_t tA = tmem + (g == 0 ? C::tDV : C::tDK) + lane_off;
      const float f = (g == 0) ? 1.f : a.scale;
      uint16_t* dst = static_cast<uint16_t*>(g == 0 ? a.dv : a.dk) + base;
#pragma unroll
      for (int cc = 0; cc < D; cc += 32) {
        uint32_t v[32];
        if (c > 0) {
          tmem_ld32_sync(tA + cc, v);
        } else {
#pragma unroll
          for (int t = 0; t < 32; ++t) v[t] = 0u;
        }
        if (key_ok) {
          uint4* d4 = reinterpret_cast<uint4*>(dst + cc);
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            uint4 wv;
            wv.x = pack2<kFp16>(__uint_as_float(v[8 * t + 0]) * f, __uint_as_float(v[8 * t + 1]) * f);
            wv.y = pack2<kFp16>(__uint_as_float(v[8 * t + 2]) * f, __uint_as_float(v[8 * t + 3]) * f);
            wv.z = pack2<kFp16>(__uint_as_float(v[8 * t + 4]) * f, __uint_as_float(v[8 * t + 5]) * f);
            wv.w = pack2<kFp16>(__uint_as_float(v[8 * t + 6]) * f, __uint_as_float(v[8 * t + 7]) * f);
            d4[t] = wv;
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaW) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int D, bool kFp16>
cudaError_t launch_bwd_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tdo,
                         const CUtensorMap& tdq, const BwdArgs& a, cudaStream_t s) {
  using C = BwdCfg<D>;
  const bool drop = a.drop.t > 0;
  auto kern = a.dq_fix != nullptr ? (drop ? bwd_kernel<D, kFp16, true, true, 2> : bwd_kernel<D, kFp16, true, false, 2>)
                                  : (drop ? bwd_kernel<D, kFp16, false, true, 2> : bwd_kernel<D, kFp16, false, false, 2>);
  int threads = kBwdThreads;
  if constexpr (D == 64) {
    if (kBwdFourGroups && a.dq_fix == nullptr) {
      kern = drop ? bwd_kernel<D, kFp16, false, true, 4> : bwd_kernel<D, kFp16, false, false, 4>;
      threads = 4 * 128 + 64;
    }
  }
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem);
  if (e != cudaSuccess) return e;
  const unsigned grid = static_cast<unsigned>(a.BH) * static_cast<unsigned>(a.T) * static_cast<unsigned>(a.q_splits);
  kern<<<grid, threads, C::kSmem, s>>>(tq, tk, tv, tdo, tdq, a);
  return cudaGetLastError();
}

int grid_for(long long work_items, int per_block) {
  long long g = (work_items + per_block - 1) / per_block;
  const long long cap = 148LL * 16;
  if (g > cap) g = cap;
  if (g < 1) g = 1;
  return (int)g;
}

}  // namespace

cudaError_t launch_bwd_pre(const BwdPreArgs& a, bool fp16, cudaStream_t s) {
  const long long rows = (long long)a.BH * a.Np;
  if (a.d == 64) {
    const int g = grid_for(rows, 256 / 8);
    if (fp16) bwd_pre_kernel<64, true><<<g, 256, 0, s>>>(a);
    else bwd_pre_kernel<64, false><<<g, 256, 0, s>>>(a);
  } else {
    const int g = grid_for(rows, 256 / 16);
    if (fp16) bwd_pre_kernel<128, true><<<g, 256, 0, s>>>(a);
    else bwd_pre_kernel<128, false><<<g, 256, 0, s>>>(a);
  }
  return cudaGetLastError();
}

cudaError_t launch_bwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const CUtensorMap& tdo,
                       const CUtensorMap& tdq, const BwdArgs& a, int d, bool fp16, cudaStream_t s) {
  if (d == 64)
    return fp16 ? launch_bwd_t<64, true>(tq, tk, tv, tdo, tdq, a, s) : launch_bwd_t<64, false>(tq, tk, tv, tdo, tdq, a, s);
  return fp16 ? launch_bwd_t<128, true>(tq, tk, tv, tdo, tdq, a, s) : launch_bwd_t<128, false>(tq, tk, tv, tdo, tdq, a, s);
}

cudaError_t launch_bwd_post(const BwdPostArgs& a, bool fp16, cudaStream_t s) {
  const int g = grid_for(a.n_elems / 8, 256);
  if (a.dq_fix != nullptr) {
    if (a.d == 64) {
      if (fp16) bwd_post_fix_kernel<64, true><<<g, 256, 0, s>>>(a);
      else bwd_post_fix_kernel<64, false><<<g, 256, 0, s>>>(a);
    } else {
      if (fp16) bwd_post_fix_kernel<128, true><<<g, 256, 0, s>>>(a);
      else bwd_post_fix_kernel<128, false><<<g, 256, 0, s>>>(a);
    }
    return cudaGetLastError();
  }
  if (fp16) bwd_post_kernel<true><<<g, 256, 0, s>>>(a);
  else bwd_post_kernel<false><<<g, 256, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace fa
