// fa_fwd.cu -- fused exact-attention forward pass for sm_100a.
//
// Computes O = softmax(scale * Q Kᵀ) V and LSE per row in one pass over the key/value
// tiles, keeping a running row max m and exp-sum l (FlashAttention-NeurIPS22 summary,
// "核心方法 / Tiling 与 online softmax"); the N x N score and probability tiles live only
// in tensor memory and registers ("Kernel fusion").  Only O and LSE are written
// ("Backward recomputation": the forward saves O and the softmax normalisation).
//
// One CTA owns two 128-row query tiles of one (b, h) head (256 rows), so every K/V tile
// it loads feeds two score tiles.  Warp roles (512 threads, four warpgroups):
//   warps 0-3    softmax group 0: query tile 0, one row per thread (TMEM lanes 0..127)
//   warps 4-7    softmax group 1: query tile 1
//   warps 8-11   correction: O_q <- alpha O_q in TMEM for both query tiles, one row per thread
//   warp  12     TMA producer: Q once, then the K/V ring (no multicast)
//   warp  13     MMA issuer (one elected thread) and TMEM allocator
//   warps 14-15  idle (they complete the producer / MMA warpgroup)
// setmaxnreg moves registers from the correction and producer / MMA warpgroups to the
// softmax warpgroups, which hold a whole 128-score row each.
// Tensor memory (512 columns): S0 [0,128), S1 [128,256), O0 [256,256+d), O1 [256+d, 256+2d).
// (The one-query-tile layout of FwdCfg<D, 1>, used for short d = 64 sequences: softmax warps
// 0-3 that also rescale O, producer warp 4, MMA warp 5, 256 columns with S [0,128) and O
// [128,128+d).)
// P (16-bit) is written over the first 64 columns of its S tile and consumed from TMEM by
// the PV MMA.  Per key tile u the MMA thread issues, for each query tile q that keeps u:
//   O_q += P_q(prev) V(prev)   then   S_q = Q_q K(u)ᵀ   (commit -> s_full[q]),
// so completion of S_q(u) also guarantees O_q holds every earlier PV product.  Once the
// softmax group has the row maxima of S_q(u) it publishes the factors alpha = 2^(m_old - m_new);
// the correction warps rescale O_q while the softmax group exponentiates, and the PV product
// of tile u waits for both P_q(u) and the rescaled O_q.  This moves the rescale -- work that is
// not a matrix product (FlashAttention-2 wiki, "最小化非矩阵运算") -- off the softmax's
// critical path.  The row max is refreshed whenever
// it grows, so the largest probability of a row is exactly 1 when it is rounded to 16 bits
// (a stale max would leave it anywhere in [1, 2^k) and add up to 2^-8 relative rounding on the
// dominant term of peaked rows).
// The FA-2 idea of spreading one head over SMs ("改进并行性") is the grid over query tiles;
// its warp repartition to cut shared-memory exchange ("优化块内工作划分") becomes the
// per-row softmax on TMEM lanes, which needs no cross-warp reduction at all.
//
// Key slices.  K/V may hold Nk keys that sit at query-sequence tile kt_off onwards (one GPU's
// shard of a sequence-sharded forward), and the key tiles may be cut into n_splits ranges of
// split_tiles tiles, one CTA per (query pair, range), when there are too few query tiles to
// fill the GPU.  Each range then writes its own normalised O and LSE (fp32) for a separate
// merge kernel to combine; causal and block masks compare query-sequence positions.
//
// Dropout (kDrop, "核心方法 / Kernel fusion"): the softmax thread of row i draws the bytes
// of its scores from Philox4x32-10, one call per 16 keys (counter (key / 16, i, bh, 0)), and
// writes P o M (M = keep * 256/(256 - t)) to TMEM for the PV product, while the row max,
// exp-sum and LSE stay those of the undropped P.
#include "fa_internal.h"
#include "sm100.cuh"

namespace fa {
namespace {

// kQ query tiles per CTA.  kQ = 2 (d = 128, and d = 64 with dropout past 8 key tiles): two
// softmax groups share every K/V tile, one CTA per SM (at d = 128 with a correction warpgroup,
// 512 threads, all 512 TMEM columns).  kQ = 1 (d = 64): one softmax group, 192 threads, 256
// TMEM columns and a 2-stage ring, so two CTAs fit on an SM and one's start-up and epilogue
// overlap the other's tiles.
template <int D, int kQ>
struct FwdCfg {
  static constexpr int kPanels = D / 64;                 // 64-element (128-byte) swizzle panels
  static constexpr int kTileBytes = kTile * D * 2;       // one 128 x D 16-bit tile
  static constexpr int kPanelBytes = kTile * 128;        // 128 rows x 128 bytes
  static constexpr int kStages = (kQ == 1) ? 2 : (D == 64) ? 4 : 2;   // K/V ring depth
  static constexpr int kSmemTiles = kQ * kTileBytes + 2 * kStages * kTileBytes;
  // kQ = 2 at d = 128: a correction warpgroup (warps 8-11) rescales O in TMEM while the
  // softmax warps go on exponentiating; 16 warps, registers rebalanced per warpgroup with
  // setmaxnreg.  At d = 64 the rescale of 64 columns is cheap and the softmax warps keep it
  // (measured: the correction warpgroup costs the d = 64 forward 5-16 %).
  static constexpr bool kCorr = (kQ == 2 && D == 128);
  static constexpr int kThreads = kCorr ? 512 : 128 * kQ + 64;
  static constexpr int kCorrWarp = 8;
  static constexpr int kLoadWarp = kCorr ? 12 : 4 * kQ, kMmaWarp = kCorr ? 13 : 4 * kQ + 1;
  static constexpr int kTmemCols = (kQ == 2) ? 512 : 256;
  static constexpr int kOCol = 128 * kQ;                 // first O column (S tiles before it)
  // One query tile at d = 64 leaves TMEM columns for P of its own (after S and O): S(u+1) is
  // then issued as soon as the softmax has read S(u) instead of after the PV product that
  // reads P(u), which takes that MMA pair off the softmax's chain; the softmax instead waits
  // for PV(u) before it rescales O and stores P(u+1).  Measured forward: +13.5 % at N = 1024,
  // +5 % at N = 512; with two query tiles (which also have the columns) it lost 5-9 %, and
  // the dropout variant (kernel-side switch) spills and lost 27 %.
  static constexpr bool kEarlyS = (D == 64 && kQ == 1);
  static constexpr int kPCol = kQ * (128 + D);           // first P column (kEarlyS)
  static_assert(!kEarlyS || kPCol + 64 * kQ <= kTmemCols, "P columns exceed the allocation");
  // exp2 pairs per 8 evaluated by polynomial on the FMA pipe instead of the SFU
  static constexpr int kPolyOf8 = (D == 64) ? 2 : 0;
  // Registers per thread (kCorr): 128 at launch (65536 / 512), then softmax warpgroups 176,
  // the correction warpgroup 88 and the load / MMA warpgroup 72 (the split with no spills at
  // d = 128).  The shares add up to exactly the launch's 512 x 128, so every setmaxnreg.inc
  // is satisfied.
  static constexpr int kLaunchRegs = 128, kRegSoftmax = 176, kRegCorr = 88, kRegOther = 72;
  static_assert(!kCorr || 8 * 32 * kRegSoftmax + 4 * 32 * kRegCorr + 4 * 32 * kRegOther <= kThreads * kLaunchRegs,
                "register shares exceed the launch allocation");
};

struct FwdShared {
  uint64_t q_full;
  uint64_t k_full[4], v_full[4], k_empty[4], v_empty[4];
  uint64_t s_full[2], p_full[2];
  uint64_t alpha_full[2], o_ready[2];   // softmax -> correction -> MMA (kCorr)
  uint64_t s_free[2], pv_done[2];       // S_q read by the softmax / PV_q product done (kEarlyS)
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort_flag;
  int n_union;
  int n_q[2];
  float alpha[2][kTile];                // per-row O rescale factor of the current tile (kCorr)
};

template <int N>
__device__ __forceinline__ void reg_alloc_inc() { asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N)); }
template <int N>
__device__ __forceinline__ void reg_alloc_dec() { asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N)); }

constexpr float kLn2 = 0.693147180559945309f;

template <int D, bool kFp16, bool kDrop, int kQ>
__global__ void __launch_bounds__(FwdCfg<D, kQ>::kThreads, kQ == 2 ? 1 : 2)
    fwd_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
               const __grid_constant__ CUtensorMap tm_v, const FwdArgs a) {
  using C = FwdCfg<D, kQ>;
  constexpr bool kES = C::kEarlyS && !kDrop;   // P in its own TMEM columns, early S issue
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  __shared__ FwdShared sh;

  const uint32_t pad = (1024u - (smem_addr(smem_raw) & 1023u)) & 1023u;
  uint8_t* sQ = smem_raw + pad;                           // 2 query tiles
  uint8_t* sK = sQ + kQ * C::kTileBytes;                  // kStages key tiles
  uint8_t* sV = sK + C::kStages * C::kTileBytes;          // kStages value tiles
  int* list = reinterpret_cast<int*>(sV + C::kStages * C::kTileBytes);  // T entries

  const int warp = warp_id(), lane = lane_id();
  // CTAs resident together work on a few heads (their K/V tiles then come from L2), and
  // within that group the heaviest query units run first (causal: the last ones).
  int bh, slot;
  cta_order(blockIdx.x, a.BH, a.n_units * a.n_splits, a.group_heads, bh, slot);
  int ui = slot / a.n_splits;
  const int split = slot - ui * a.n_splits;     // key-tile range of this CTA
  if (a.causal) ui = a.n_units - 1 - ui;
  const int qt0 = kQ * ui;
  const DevStatus st{a.status, a.timeout_ns};
  volatile int* abort_flag = &sh.abort_flag;

  if (threadIdx.x == 0) {
    mbar_init(&sh.q_full, 1);
    for (int s = 0; s < C::kStages; ++s) {
      mbar_init(&sh.k_full[s], 1);
      mbar_init(&sh.v_full[s], 1);
      mbar_init(&sh.k_empty[s], 1);
      mbar_init(&sh.v_empty[s], 1);
    }
    for (int q = 0; q < kQ; ++q) {
      mbar_init(&sh.s_full[q], 1);
      mbar_init(&sh.p_full[q], 128);
      mbar_init(&sh.alpha_full[q], 128);
      mbar_init(&sh.o_ready[q], 128);
      mbar_init(&sh.s_free[q], 128);
      mbar_init(&sh.pv_done[q], 1);
    }
    mbar_init(&sh.mma_done, 1);
    sh.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == C::kMmaWarp) {
    tmem_alloc(&sh.tmem_base, C::kTmemCols);
    tmem_relinquish();
  }
  if (warp == C::kLoadWarp) {
    // Union list of this range's key tiles needed by either query tile, with per-tile keep
    // bits; entries hold the K/V tile index, the masks see its query-sequence tile jg.
    int c0, c1;
    const int jb = split * a.split_tiles;
    const int count = union_tile_list(list, jb, min(a.Tk, jb + a.split_tiles), a.kt_off, qt0, kQ == 2, a.T, a.causal,
                                      a.blockmask, c0, c1);
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

  // Each role's register share is set by its whole warpgroup at the top of the role's own
  // branch (kCorr): softmax up to kRegSoftmax, correction and load / MMA down.
  if (warp >= C::kLoadWarp) {
  if constexpr (C::kCorr) reg_alloc_dec<C::kRegOther>();
  if (warp == C::kLoadWarp) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0 && nu > 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      const int nq = (kQ == 2 && qt0 + 1 < a.T) ? 2 : 1;
      mbar_arrive_expect_tx(&sh.q_full, nq * C::kTileBytes);
      for (int q = 0; q < nq; ++q)
        for (int p = 0; p < C::kPanels; ++p)
          tma_load_3d(sQ + q * C::kTileBytes + p * C::kPanelBytes, &tm_q, &sh.q_full, p * 64, (qt0 + q) * kTile, bh);
      // K and V slots are released separately: a key tile's slot frees when the last S product
      // that reads it completes, a full PV product earlier than its value tile's slot, so the
      // next key tile is already resident when the MMA warp reaches it.
      int nk = 0, nv = 0;                         // key / value tiles whose copy was started
      for (int u = 0; u < nu; ++u) {
        const int s = u % C::kStages;
        const uint32_t ph = ((u / C::kStages) - 1) & 1;
        const int j = list[u] & 0xFFFF;
        if (u >= C::kStages && !mbar_wait(&sh.k_empty[s], ph, abort_flag, st)) break;
        mbar_arrive_expect_tx(&sh.k_full[s], C::kTileBytes);
        for (int p = 0; p < C::kPanels; ++p)
          tma_load_3d(sK + s * C::kTileBytes + p * C::kPanelBytes, &tm_k, &sh.k_full[s], p * 64, j * kTile, bh);
        ++nk;
        if (u >= C::kStages && !mbar_wait(&sh.v_empty[s], ph, abort_flag, st)) break;
        mbar_arrive_expect_tx(&sh.v_full[s], C::kTileBytes);
        for (int p = 0; p < C::kPanels; ++p)
          tma_load_3d(sV + s * C::kTileBytes + p * C::kPanelBytes, &tm_v, &sh.v_full[s], p * 64, j * kTile, bh);
        ++nv;
      }
      if (*abort_flag) {
        // Let every copy this thread started land before the CTA's shared memory goes away.
        mbar_wait_drain(&sh.q_full, 0, st);
        for (int uu = (nk > C::kStages ? nk - C::kStages : 0); uu < nk; ++uu)
          mbar_wait_drain(&sh.k_full[uu % C::kStages], (uu / C::kStages) & 1, st);
        for (int uu = (nv > C::kStages ? nv - C::kStages : 0); uu < nv; ++uu)
          mbar_wait_drain(&sh.v_full[uu % C::kStages], (uu / C::kStages) & 1, st);
      }
    }
    __syncwarp();
  } else if (warp == C::kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      bool ok = (nu == 0) || mbar_wait(&sh.q_full, 0, abort_flag, st);
      tc_fence_after();
      const uint32_t idesc_s = idesc_f16(128, 128, kFp16, false, false);
      const uint32_t idesc_pv = idesc_f16(128, D, kFp16, false, true);
      const uint32_t aQ = smem_addr(sQ), aK = smem_addr(sK), aV = smem_addr(sV);
      int npv0 = 0, npv1 = 0;                     // PV products issued per query tile
      int ns[2] = {0, 0};                         // S products issued per query tile
      for (int u = 0; u <= nu && ok; ++u) {
        const int ep = (u > 0) ? list[u - 1] : 0;
        const int ec = (u < nu) ? list[u] : 0;
        const int sp = (u + C::kStages - 1) % C::kStages;
        const int sc = u % C::kStages;
        bool v_ready = false, k_ready = false;
        // Per iteration: O_0 += P_0 V(u-1), S_0 = Q_0 K(u)ᵀ, O_1 += P_1 V(u-1), S_1 = Q_1 K(u)ᵀ, each
        // only where that query tile keeps the tile.
        auto pv = [&](int q, int& npv) -> bool {
          if (u > 0 && ((ep >> (16 + q)) & 1)) {
            if (!v_ready) {
              if (!mbar_wait(&sh.v_full[sp], ((u - 1) / C::kStages) & 1, abort_flag, st)) return false;
              v_ready = true;
            }
            if (!mbar_wait(&sh.p_full[q], npv & 1, abort_flag, st)) return false;
            if constexpr (C::kCorr) {     // O_q rescaled for this tile by the correction warps
              if (!mbar_wait(&sh.o_ready[q], npv & 1, abort_flag, st)) return false;
            }
            tc_fence_after();
            // P_q: its own columns (kEarlyS) or over S_q
            const uint32_t tPq = kES ? tmem + C::kPCol + 64 * q : tmem + q * 128;
#pragma unroll
            for (int kk = 0; kk < kTile / 16; ++kk) {
              const uint64_t bdesc = smem_desc_sw128(aV + sp * C::kTileBytes + kk * 2048, C::kPanelBytes, 1024);
              mma_ts(tmem + C::kOCol + q * D, tPq + kk * 8, bdesc, idesc_pv, (npv > 0 || kk > 0) ? 1u : 0u);
            }
            if constexpr (kES) tc_commit(&sh.pv_done[q]);
            ++npv;
          }
          return true;
        };
        auto sq = [&](int q) -> bool {
          if (u < nu && ((ec >> (16 + q)) & 1)) {
            if (!k_ready) {
              if (!mbar_wait(&sh.k_full[sc], (u / C::kStages) & 1, abort_flag, st)) return false;
              tc_fence_after();
              k_ready = true;
            }
            if constexpr (kES) {            // the softmax has read S_q's previous tile
              if (ns[q] > 0) {
                if (!mbar_wait(&sh.s_free[q], (ns[q] - 1) & 1, abort_flag, st)) return false;
                tc_fence_after();
              }
            }
            ++ns[q];
#pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint32_t koff = (kk >> 2) * C::kPanelBytes + (kk & 3) * 32;
              const uint64_t adesc = smem_desc_sw128(aQ + q * C::kTileBytes + koff, 16, 1024);
              const uint64_t bdesc = smem_desc_sw128(aK + sc * C::kTileBytes + koff, 16, 1024);
              mma_ss(tmem + q * 128, adesc, bdesc, idesc_s, kk > 0 ? 1u : 0u);
            }
            tc_commit(&sh.s_full[q]);
            if (a.visit != nullptr)
              atomicAdd(&a.visit[((size_t)bh * a.T + (qt0 + q)) * a.T + a.kt_off + (ec & 0xFFFF)], 1);
          }
          return true;
        };
        if constexpr (kES) {
          // S_0(u), S_1(u) as soon as the softmax groups have read the previous S, then the PV
          // products of tile u-1 as their P arrive
          ok = sq(0) && (kQ == 1 || sq(1));
          if (u < nu && ok) tc_commit(&sh.k_empty[sc]);
          ok = ok && pv(0, npv0) && (kQ == 1 || pv(1, npv1));
          if (u > 0 && ok) tc_commit(&sh.v_empty[sp]);
        } else {
          ok = pv(0, npv0) && sq(0) && (kQ == 1 || pv(1, npv1));
          if (u > 0 && ok) tc_commit(&sh.v_empty[sp]);     // V(u-1) free once its PV products are done
          ok = ok && (kQ == 1 || sq(1));
          if (u < nu && ok) tc_commit(&sh.k_empty[sc]);    // K(u) free once its S products are done
        }
      }
      if (ok) {
        tc_commit(&sh.s_full[0]);   // final phase: every MMA into O_0 / O_1 has completed
        if (kQ == 2) tc_commit(&sh.s_full[1]);
      }
      tc_commit(&sh.mma_done);
      mbar_wait_drain(&sh.mma_done, 0, st);
    }
    __syncwarp();
  }
  } else if (C::kCorr && warp >= C::kCorrWarp) {
    // ------------------------------------------------------------------ correction warpgroup
    // For every tile a query tile keeps, in list order: wait for its softmax group to publish
    // the per-row factors alpha = 2^(m_old - m_new), rescale that tile's O rows in TMEM (only
    // warps where some row's max grew), and release O to the MMA warp.  The factor is known
    // after the row max, long before P is, so this runs beside the softmax's exponentials.
    // O_q then holds every earlier PV product: completion of S_q(u), which the softmax
    // waited for before publishing, implies completion of PV_q(u-1) issued before it.
    if constexpr (C::kCorr) reg_alloc_dec<C::kRegCorr>();
    const int wq = warp & 3;
    const int r = wq * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    int cq[2] = {0, 0};
    bool ok = true;
    for (int u = 0; u < nu && ok; ++u) {
      const int e = list[u];
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        if (!((e >> (16 + q)) & 1)) continue;
        ok = mbar_wait(&sh.alpha_full[q], cq[q] & 1, abort_flag, st);
        if (__any_sync(0xffffffffu, !ok)) { ok = false; break; }
        const float al = sh.alpha[q][r];
        if (cq[q] > 0 && __any_sync(0xffffffffu, al != 1.f)) {
          tc_fence_after();
          const uint32_t tO = tmem + C::kOCol + q * D + lane_off;
#pragma unroll
          for (int cc = 0; cc < D; cc += 32) {
            uint32_t o[32];
            tmem_ld32_sync(tO + cc, o);
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
              const float2 x = mul2(make_float2(__uint_as_float(o[i]), __uint_as_float(o[i + 1])), make_float2(al, al));
              o[i] = __float_as_uint(x.x);
              o[i + 1] = __float_as_uint(x.y);
            }
            tmem_st32(tO + cc, o);
          }
          tmem_wait_st();
        }
        tc_fence_before();
        mbar_arrive(&sh.o_ready[q]);
        ++cq[q];
      }
    }
  } else {
    // ------------------------------------------------------------------ softmax groups
    if constexpr (C::kCorr) reg_alloc_inc<C::kRegSoftmax>();
    const int q = warp >> 2;
    const int wq = warp & 3;                        // TMEM lane quarter of this warp
    const int row_local = wq * 32 + lane;
    const int qt = qt0 + q;
    const int row = qt * kTile + row_local;
    const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
    const uint32_t tS = tmem + q * 128 + lane_off;
    const uint32_t tO = tmem + C::kOCol + q * D + lane_off;
    const uint32_t tP = kES ? tmem + C::kPCol + 64 * q + lane_off : tS;   // P_q's columns
    const float sl2 = a.scale_log2;
    float m = -INFINITY;   // running max of scale*log2(e)*s over this row
    float l = 0.f;         // running sum of 2^(scale*log2(e)*s - m)
    int c = 0;
    bool ok = true;
    for (int u = 0; u < nu; ++u) {
      const int e = list[u];
      if (!((e >> (16 + q)) & 1)) continue;
      const int key0 = (e & 0xFFFF) * kTile;          // first K/V row of the tile
      const int kpos0 = key0 + a.kt_off * kTile;      // its query-sequence position
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
      if constexpr (kES) {                   // S_q's columns may take the next tile
        tc_fence_before();
        mbar_arrive(&sh.s_free[q]);
      }
      float s[128];
#pragma unroll
      for (int i = 0; i < 128; ++i) s[i] = __uint_as_float(sr[i]);
      if ((a.causal && kpos0 + kTile - 1 > qt * kTile) || key0 + kTile > a.Nk) {
        int lim = a.Nk - key0;                         // K/V rows at or beyond Nk do not exist
        if (a.causal) lim = min(lim, row - kpos0 + 1); // key position <= row
#pragma unroll
        for (int i = 0; i < 128; ++i)
          if (i >= lim) s[i] = -INFINITY;
      }
      const float mx = row_max128(s);
      const float mx2 = mx * sl2;
      float alpha = 1.f;
      bool resc = false;
      if (mx2 > m) {
        alpha = ex2(m - mx2);                       // 0 when m = -inf
        resc = (c > 0);
        m = mx2;
      }
      if constexpr (C::kCorr) {                     // hand the O rescale to the correction warps
        sh.alpha[q][row_local] = alpha;
        mbar_arrive(&sh.alpha_full[q]);
      }
      const float mneg = (m == -INFINITY) ? 0.f : -m;
      const float2 sl2v = make_float2(sl2, sl2), mnegv = make_float2(mneg, mneg);
      if constexpr (kES) {
        // PV_q of the previous kept tile must be done: it reads the P columns about to be
        // rewritten, and O must hold it before the rescale below
        if (c > 0) {
          ok = mbar_wait(&sh.pv_done[q], (c - 1) & 1, abort_flag, st);
          if (__any_sync(0xffffffffu, !ok)) { ok = false; break; }
          tc_fence_after();
        }
      }
      // P = 2^(s*scale*log2e - m) in pairs (packed fp32 FMA), row sum over four packed
      // accumulators; P stored to TMEM in quarters of 32 keys as soon as each is packed.
      float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        uint32_t pk[16];
        uint4 rnd = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          if constexpr (kDrop) {
            // keys kpos0 + 32h + 2i, +1 lie in 16-key block kpos0/16 + 2h + i/8, bytes 2(i%8), +1
            if ((i & 7) == 0)
              rnd = philox4x32_10(make_uint4(static_cast<uint32_t>(kpos0 >> 4) + 2 * h + (i >> 3),
                                             static_cast<uint32_t>(row), static_cast<uint32_t>(bh), 0u),
                                  a.drop.seed_lo, a.drop.seed_hi);
          }
          const float2 t = fma2(make_float2(s[32 * h + 2 * i], s[32 * h + 2 * i + 1]), sl2v, mnegv);
          // kPolyOf8 of every 8 pairs go to the FMA-pipe polynomial, the rest to the SFU
          const float2 p = (((16 * h + i) & 7) < C::kPolyOf8) ? exp2_poly2(t) : make_float2(ex2(t.x), ex2(t.y));
          acc[i & 3] = add2(acc[i & 3], p);
          if constexpr (kDrop) {
            const int wi = (i & 7) >> 1;
            const uint32_t wv = wi == 0 ? rnd.x : wi == 1 ? rnd.y : wi == 2 ? rnd.z : rnd.w;
            const uint32_t b0 = (wv >> (16 * (i & 1))) & 0xFFu, b1 = (wv >> (16 * (i & 1) + 8)) & 0xFFu;
            pk[i] = pack2<kFp16>(b0 >= a.drop.t ? p.x * a.drop.scale : 0.f, b1 >= a.drop.t ? p.y * a.drop.scale : 0.f);
          } else {
            pk[i] = pack2<kFp16>(p.x, p.y);
          }
        }
        tmem_st16(tP + 16 * h, pk);
      }
      const float2 a01 = add2(acc[0], acc[1]), a23 = add2(acc[2], acc[3]);
      const float2 a0123 = add2(a01, a23);
      const float sum0 = a0123.x, sum1 = a0123.y;
      l = l * alpha + (sum0 + sum1);
      // O <- alpha O for the rows whose max grew (O holds every earlier PV product: see above);
      // with a correction warpgroup that work is theirs
      if (!C::kCorr && __any_sync(0xffffffffu, resc)) {
        const float f = resc ? alpha : 1.f;
#pragma unroll
        for (int cc = 0; cc < D; cc += 32) {
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
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sh.p_full[q]);
      ++c;
    }
    // Wait for the final commit: every PV product of this query tile is in O_q.
    const int nq = sh.n_q[q];
    if (ok) ok = mbar_wait(&sh.s_full[q], nq & 1, abort_flag, st);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
      tc_fence_after();
      const bool valid = row < a.N;
      const float inv = (l > 0.f) ? 1.f / l : 0.f;
      if (valid)
        a.lse[split * a.lse_split_stride + (size_t)bh * a.N + row] = (l > 0.f) ? (m + log2f(l)) * kLn2 : -INFINITY;
      const size_t obase = split * a.o_split_stride + ((size_t)bh * a.N + row) * D;
#pragma unroll
      for (int cc = 0; cc < D; cc += 32) {
        uint32_t o[32];
        if (nq > 0) {
          tmem_ld32_sync(tO + cc, o);
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0u;
        }
        if (valid) {
          if (a.o_fp32) {
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
              w.x = pack2<kFp16>(__uint_as_float(o[8 * i + 0]) * inv, __uint_as_float(o[8 * i + 1]) * inv);
              w.y = pack2<kFp16>(__uint_as_float(o[8 * i + 2]) * inv, __uint_as_float(o[8 * i + 3]) * inv);
              w.z = pack2<kFp16>(__uint_as_float(o[8 * i + 4]) * inv, __uint_as_float(o[8 * i + 5]) * inv);
              w.w = pack2<kFp16>(__uint_as_float(o[8 * i + 6]) * inv, __uint_as_float(o[8 * i + 7]) * inv);
              dst[i] = w;
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == C::kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

template <int D, bool kFp16, int kQ>
cudaError_t launch_fwd_q(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const FwdArgs& a0,
                         cudaStream_t s) {
  using C = FwdCfg<D, kQ>;
  FwdArgs a = a0;
  a.n_units = (a.T + kQ - 1) / kQ;
  // CTAs run in groups of heads, heaviest query units first within a group, so a group's K/V
  // tiles are shared through L2.  Non-causal: groups of about two waves.  Causal: a unit's work
  // ranges from 1 to T key tiles, and with two-wave groups the last group's longest CTAs
  // outlast everything else; groups of at least four waves' work, balanced in size, keep those
  // CTAs within half a group's duration (measured on B1 H32 N16384 d128: +6 % forward, DRAM
  // reads 0.59 GB against 0.41 GB; one group of all heads is as fast but reads 2.1 GB).
  {
    const int per_head = a.n_units * a.n_splits;
    if (a.causal) {
      const int gmin = (4 * 148 + per_head - 1) / per_head;
      const int ngroups = (a.BH + gmin - 1) / gmin;
      a.group_heads = (a.BH + ngroups - 1) / ngroups;
    } else {
      a.group_heads = group_heads_for(a.BH, per_head);
    }
  }
  const size_t smem = C::kSmemTiles + (size_t)min(a.Tk, a.split_tiles) * sizeof(int) + 1024;
  auto kern = a.drop.t > 0 ? fwd_kernel<D, kFp16, true, kQ> : fwd_kernel<D, kFp16, false, kQ>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  if constexpr (C::kCorr) {
    // setmaxnreg.inc waits until the block's launch registers cover every warpgroup's share;
    // refuse to launch a build whose register count differs from the one the shares assume.
    static int regs = 0;
    if (regs == 0) {
      cudaFuncAttributes fa_attr;
      e = cudaFuncGetAttributes(&fa_attr, kern);
      if (e != cudaSuccess) return e;
      regs = fa_attr.numRegs;
    }
    if (regs != C::kLaunchRegs) return cudaErrorInvalidConfiguration;
  }
  const unsigned grid = static_cast<unsigned>(a.BH) * static_cast<unsigned>(a.n_units) * static_cast<unsigned>(a.n_splits);
  kern<<<grid, C::kThreads, smem, s>>>(tq, tk, tv, a);
  return cudaGetLastError();
}

// At d = 64 the one-query-tile layout, with its early S issue, is the faster forward at every
// length measured (N = 512 to 16384, causal too: +13 to +19 % over two query tiles from
// N = 2048 on).  With dropout it has no early issue, and pays off only while a CTA's start-up
// and epilogue are large next to its key tiles: up to kSingleMaxTiles key tiles.
constexpr int kSingleMaxTiles = 8;

template <int D, bool kFp16>
cudaError_t launch_fwd_t(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const FwdArgs& a,
                         cudaStream_t s) {
  if constexpr (D == 64) {
    const int tiles = min(a.Tk, a.split_tiles);
    if ((a.drop.t == 0 || tiles <= kSingleMaxTiles) && (long long)a.BH * a.T * a.n_splits <= 0x7fffffffLL)
      return launch_fwd_q<D, kFp16, 1>(tq, tk, tv, a, s);
  }
  return launch_fwd_q<D, kFp16, 2>(tq, tk, tv, a, s);
}

}  // namespace

cudaError_t launch_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const FwdArgs& a,
                       int d, bool fp16, cudaStream_t s) {
  if (d == 64) return fp16 ? launch_fwd_t<64, true>(tq, tk, tv, a, s) : launch_fwd_t<64, false>(tq, tk, tv, a, s);
  return fp16 ? launch_fwd_t<128, true>(tq, tk, tv, a, s) : launch_fwd_t<128, false>(tq, tk, tv, a, s);
}

}  // namespace fa
