// fa_internal.h -- argument blocks passed from the host library to the kernels, and the
// host-side launch functions each kernel file provides.  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace fa {

constexpr int kTile = 128;          // rows per query tile and keys per key/value tile
constexpr int kMaxTiles = 2048;     // tile lists live in shared memory (N <= 2048 * 128)

// Error codes a kernel can record in the device status word.  They live in their own range
// (0x100 and up), disjoint from the public fa_status values, and fa_check_status translates
// each one explicitly (status_from_device_word): a device word is never returned as it is.
enum : int { kDevOk = 0, kDevTimeout = 0x101, kDevBadState = 0x102, kDevRange = 0x103 };

// Deterministic backward: dQ partials are added as int64 fixed point with 32 fraction bits.
// Integer addition is associative, so the sum does not depend on the order in which the
// key-tile CTAs add their partials.  A partial of magnitude >= 2^20 is reported (kDevRange):
// with at most 2^11 key tiles the sum then stays below 2^31, inside the int64 range.
constexpr float kFixOne = 4294967296.0f;      // 2^32
constexpr float kFixLimit = 1048576.0f;       // 2^20

constexpr int kMaxParts = 64;       // most key splits / merged parts per call

// Dropout on the probabilities (off when t == 0).  Score (i, j) of head index bh is dropped
// iff byte j mod 16 of Philox4x32-10(counter (j / 16, i, bh, 0), key (seed_lo, seed_hi)) is
// below t (bytes little-endian within the four output words); kept scores are multiplied
// by scale = 256 / (256 - t).
struct Dropout {
  uint32_t t;
  float scale;
  uint32_t seed_lo, seed_hi;
};

struct FwdArgs {
  void* o;                  // [BH, N, d] 16-bit, or fp32 when o_fp32 (split s at o + s * o_split_stride)
  float* lse;               // [BH, N]                                (split s at lse + s * lse_split_stride)
  const uint8_t* blockmask; // [T, T] or null
  int* visit;               // [BH, T, T] or null
  int* status;              // device status word
  unsigned long long timeout_ns;
  int N, BH, T, n_units;    // queries; n_units = ceil(T / 2): one CTA covers two 128-row query tiles
  int Nk, Tk;               // keys in K/V and their 128-row tiles (N and T for self-attention)
  int kt_off;               // query-sequence tile index of key tile 0 (causal and mask use it)
  int n_splits, split_tiles;// split s takes key tiles [s * split_tiles, (s + 1) * split_tiles)
  long long o_split_stride, lse_split_stride;  // elements between consecutive splits' outputs
  int group_heads;          // CTAs are ordered in groups of this many heads (see cta_order)
  int causal, o_fp32;
  float scale_log2;         // scale * log2(e)
  Dropout drop;
};

struct MergeArgs {
  const float* o_parts[kMaxParts];    // each [rows, d] fp32
  const float* lse_parts[kMaxParts];  // each [rows] fp32
  void* o;                            // [rows, d]: bf16, fp16 or fp32 (out_kind 0, 1, 2)
  float* lse;                         // [rows]
  long long rows;
  int n_parts, out_kind;
};

struct BwdPreArgs {
  const void* o;            // [BH, N, d]
  const void* dout;         // [BH, N, d]
  const float* lse;         // [BH, N]
  float* delta;             // [BH, Np]  -D_i = -sum_c dO_ic O_ic (0 on padding rows)
  float* lse2;              // [BH, Np]  -LSE_i * log2(e) (-inf on padding / empty rows)
  float* dq_acc;            // [BH, N, d] fp32, zeroed here (when dq_fix is null)
  long long* dq_fix;        // deterministic mode: int64 fixed-point accumulator (tile-blocked,
                            // see fix_index), zeroed here; null otherwise
  float* dk_acc;            // query-range splits: fp32 dK / dV accumulators [BH, N, d], zeroed
  float* dv_acc;            // here; null otherwise
  int N, Np, BH, d;
};

struct BwdArgs {
  const float* delta;       // [BH, Np]  -D
  const float* lse2;        // [BH, Np]  -LSE * log2(e)
  float* dq_acc;            // [BH, N, d]
  long long* dq_fix;        // deterministic mode only: [BH, Np, d] int64, tile-blocked
  void* dk;                 // [BH, N, d] 16-bit
  void* dv;                 // [BH, N, d] 16-bit
  const uint8_t* blockmask;
  int* visit;
  int* status;
  unsigned long long timeout_ns;
  int N, Np, BH, T;
  int group_heads;          // CTAs are ordered in groups of this many heads (see cta_order)
  int causal;
  // Query-range splits: key tile j's kept query tiles, in its visiting order k = 0, 1, ..., are
  // cut into q_splits ranges of q_chunk steps, one CTA per (head, key tile, range).  With
  // q_splits > 1 each CTA adds its partial dK (unscaled) and dV into dk_acc / dv_acc (fp32)
  // instead of writing dk / dv, and the post pass converts them.
  int q_splits, q_chunk;
  float* dk_acc;
  float* dv_acc;
  float scale;              // multiplies dK (dQ is scaled in the post pass)
  float scale_log2;
  Dropout drop;
};

struct BwdPostArgs {
  const float* dq_acc;      // [BH, N, d]
  const long long* dq_fix;  // deterministic mode: the int64 accumulator (else null)
  void* dq;                 // [BH, N, d] 16-bit
  const float* dk_acc;      // query-range splits: the fp32 dK / dV accumulators (else null);
  const float* dv_acc;      // dk = 16-bit(scale * dk_acc), dv = 16-bit(dv_acc)
  void* dk;
  void* dv;
  long long n_elems;
  int N, Np, BH, d;
  float scale;
};

// Element (row, col) of query tile `tile` in the int64 accumulator.  Each tile is 128 x d
// values cut into blocks of 32 rows x 16 columns (one compute warp's rows, one 128-byte
// column chunk); a block is 8 column pairs x 32 rows x 2 values, so a warp's block is one
// contiguous 4 KB range that a single bulk reduce adds, and that the warp stages in shared
// memory with conflict-free 16-byte stores (lane = row).
#ifdef __CUDACC__
__host__ __device__
#endif
inline long long fix_index(long long tile, int row, int col, int d) {
  const int blk = (col >> 4) * 4 + (row >> 5);
  return tile * 128LL * d + ((((long long)blk * 8 + ((col & 15) >> 1)) * 32 + (row & 31)) * 2 + (col & 1));
}

// Launchers (defined next to each kernel).  Return a cudaError_t.
cudaError_t launch_fwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv, const FwdArgs& a,
                       int d, bool fp16, cudaStream_t s);
cudaError_t launch_bwd_pre(const BwdPreArgs& a, bool fp16, cudaStream_t s);
cudaError_t launch_bwd(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& tdo, const CUtensorMap& tdq, const BwdArgs& a, int d, bool fp16,
                       cudaStream_t s);   // deterministic when a.dq_fix is set
cudaError_t launch_bwd_post(const BwdPostArgs& a, bool fp16, cudaStream_t s);
cudaError_t launch_merge(const MergeArgs& a, int d, cudaStream_t s);

int* device_status_word();  // address of the per-process device status word
int status_from_device_word(int v);   // fa_status for a device status word

// Heads per CTA-ordering group: about two waves of CTAs (148 SMs, one CTA each) per group, so
// the heads a wave works on keep their tiles in L2 while each group still runs its heaviest
// tiles first.
inline int group_heads_for(int BH, int tiles_per_head) {
  int g = (2 * 148 + tiles_per_head - 1) / tiles_per_head;
  if (g < 1) g = 1;
  if (g > BH) g = BH;
  return g;
}

#ifdef __CUDACC__
// CTA index -> (head, tile slot): heads in groups of G, tile slot outermost inside a group,
// so slot 0 of every head in the group is scheduled before slot 1, and so on.
__device__ __forceinline__ void cta_order(int idx, int BH, int tiles, int G, int& bh, int& slot) {
  const int per = G * tiles;
  const int grp = idx / per;
  const int r = idx - grp * per;
  const int heads_here = min(G, BH - grp * G);
  slot = r / heads_here;
  bh = grp * G + (r - slot * heads_here);
}
#endif

}  // namespace fa
