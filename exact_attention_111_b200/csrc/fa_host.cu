// fa_host.cu -- the C ABI of libfa.so (declared in include/fa.h): argument checks, TMA
// tensor-map encoding, launch sequencing on the caller's stream, status reporting.
// Every argument check happens before the first CUDA call, so invalid calls fail the
// same way with or without a GPU.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "fa.h"
#include "fa_fp8.h"
#include "fa_internal.h"

namespace fa {

__device__ int g_status_word = 0;

namespace {

constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s per barrier wait
thread_local int t_last_launches = 0;

std::mutex g_mu;
int* g_status_ptr[128] = {nullptr};

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

bool get_encode() {
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_encode) return true;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
      q != cudaDriverEntryPointSuccess || fn == nullptr)
    return false;
  g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  return true;
}

// [BH, N, d] 16-bit tensor as a 3-D TMA map with 64 x 128 x 1 boxes, 128-byte swizzle;
// rows past N read as zero.
bool encode_qkv(CUtensorMap* m, const void* base, int BH, int N, int d, bool fp16) {
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)BH};
  const cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)N * d * 2};
  const cuuint32_t box[3] = {64, (cuuint32_t)kTile, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return g_encode(m, fp16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                  const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp32 dQ accumulator [BH, N, d] as a 3-D TMA map with 32 x 32 x 1 boxes (32 columns = 128
// bytes wide, 32 rows: one warp's rows), 128-byte swizzle, for tensor reduce-add from shared
// memory; rows past N are skipped.
bool encode_dqacc(CUtensorMap* m, const void* base, int BH, int N, int d) {
  const cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)N, (cuuint64_t)BH};
  const cuuint64_t strides[2] = {(cuuint64_t)d * 4, (cuuint64_t)N * d * 4};
  const cuuint32_t box[3] = {32, 32, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 8-bit tensor with an innermost extent of 128-byte rows: 3-D map [z, y, x] with a
// 128 x 128 x 1 box, 128-byte swizzle; elements past the extents read as zero.
bool encode_u8(CUtensorMap* m, const void* base, int x, int y, int z) {
  const cuuint64_t dims[3] = {(cuuint64_t)x, (cuuint64_t)y, (cuuint64_t)z};
  const cuuint64_t strides[2] = {(cuuint64_t)x, (cuuint64_t)x * y};
  const cuuint32_t box[3] = {128, (cuuint32_t)kTile, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

int check_shape(int B, int H, int N, int d, float scale, int dtype) {
  if (B < 1 || H < 1 || N < 1) return FA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (dtype != FA_BF16 && dtype != FA_FP16) return FA_ERR_UNSUPPORTED;
  if (N > FA_MAX_SEQLEN) return FA_ERR_UNSUPPORTED;
  if ((long long)B * H > (1LL << 31) - 1) return FA_ERR_UNSUPPORTED;
  if ((long long)B * H * N * d > (1LL << 46)) return FA_ERR_UNSUPPORTED;
  return FA_OK;
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

// Dropout parameters: byte threshold t = floor(256 p + 1/2) (at most 255), scale 256/(256 - t).
bool make_dropout(float p, unsigned long long seed, Dropout* d) {
  if (!(p >= 0.f && p < 1.f)) return false;
  int t = (int)std::floor(256.0 * (double)p + 0.5);
  if (t > 255) t = 255;
  d->t = (uint32_t)t;
  d->scale = (float)(256.0 / (256.0 - t));
  d->seed_lo = (uint32_t)(seed & 0xFFFFFFFFull);
  d->seed_hi = (uint32_t)(seed >> 32);
  return true;
}

// The forward's grid is BH x units x splits CTAs, indexed by an int.
bool fwd_grid_ok(int BH, int units, int splits) {
  return (long long)BH * units * splits <= (long long)0x7fffffff;
}

// Self-attention forward arguments over all T key tiles as one range.
void self_fwd_args(FwdArgs& a, int BH, int N) {
  const int T = (N + kTile - 1) / kTile;
  a.N = N;
  a.BH = BH;
  a.T = T;
  a.n_units = (T + 1) / 2;
  a.Nk = N;
  a.Tk = T;
  a.kt_off = 0;
  a.n_splits = 1;
  a.split_tiles = T;
  a.o_split_stride = 0;
  a.lse_split_stride = 0;
  a.group_heads = group_heads_for(BH, a.n_units);
}

struct SplitLayout {
  size_t o_parts, lse_parts, total;
  long long o_stride, lse_stride;   // elements between consecutive parts
};

SplitLayout split_layout(int B, int H, int N, int d, int S) {
  const size_t rows = (size_t)B * H * N;
  SplitLayout w;
  w.o_parts = 0;
  w.o_stride = (long long)(align256(rows * d * 4) / 4);
  w.lse_parts = align256(rows * d * 4) * S;
  w.lse_stride = (long long)(align256(rows * 4) / 4);
  w.total = w.lse_parts + align256(rows * 4) * S;
  return w;
}

struct WsLayout {
  size_t dq_acc, delta, lse2, dk_acc, dv_acc, total;
};

// The dQ accumulator is fp32 [BH, N, d], or in deterministic mode int64 over whole tiles
// [BH, Np, d] (tile-blocked, fix_index).  With query-range splits (q_splits > 1) fp32 dK and
// dV accumulators [BH, N, d] follow.
WsLayout ws_layout(int B, int H, int N, int d, bool det = false, int q_splits = 1) {
  const size_t BH = (size_t)B * H;
  const size_t Np = (size_t)((N + kTile - 1) / kTile) * kTile;
  WsLayout w;
  w.dq_acc = 0;
  w.delta = det ? align256(BH * Np * d * 8) : align256(BH * N * d * 4);
  w.lse2 = w.delta + align256(BH * Np * 4);
  w.dk_acc = w.lse2 + align256(BH * Np * 4);
  w.dv_acc = w.dk_acc;
  w.total = w.dk_acc;
  if (q_splits > 1) {
    w.dv_acc = w.dk_acc + align256(BH * N * d * 4);
    w.total = w.dv_acc + align256(BH * N * d * 4);
  }
  return w;
}

int status_word(int** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return FA_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_status_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return FA_ERR_CUDA;
    g_status_ptr[dev] = static_cast<int*>(p);
  }
  *out = g_status_ptr[dev];
  return FA_OK;
}

}  // namespace

// Public status for a nonzero device status word: a bounded wait that expired is
// FA_ERR_TIMEOUT, a deterministic-backward partial out of range is FA_ERR_RANGE, and anything
// else (kDevBadState: the kernel found its dynamic shared memory misaligned and did no work)
// is FA_ERR_CUDA.
int status_from_device_word(int v) {
  switch (v) {
    case kDevOk: return FA_OK;
    case kDevTimeout: return FA_ERR_TIMEOUT;
    case kDevRange: return FA_ERR_RANGE;
    default: return FA_ERR_CUDA;
  }
}

// Every check of a backward call that needs no CUDA call: shape, pointers, alignment, the
// dropout probability and (check_workspace) the workspace.  Used by fa_bwd_ex and, before it
// touches the device at all, by fa_bwd_noalloc.
int validate_bwd(const fa_bwd_args& x, bool check_workspace) {
  int rc = check_shape(x.B, x.H, x.N, x.d, x.scale, x.dtype);
  if (rc != FA_OK) return rc;
  if (!x.q || !x.k || !x.v || !x.o || !x.lse || !x.dout || !x.dq || !x.dk || !x.dv) return FA_ERR_INVALID_ARG;
  if (!aligned(x.q, 16) || !aligned(x.k, 16) || !aligned(x.v, 16) || !aligned(x.o, 16) || !aligned(x.dout, 16) ||
      !aligned(x.dq, 16) || !aligned(x.dk, 16) || !aligned(x.dv, 16) || !aligned(x.lse, 4) ||
      !aligned(x.visit_log, 4))
    return FA_ERR_INVALID_ARG;
  Dropout drop{};
  if (!make_dropout(x.dropout_p, x.dropout_seed, &drop)) return FA_ERR_INVALID_ARG;
  if (x.query_splits < 0 || x.query_splits > FA_MAX_PARTS) return FA_ERR_INVALID_ARG;
  // the split ranges add dK / dV partials in fp32 in whatever order they finish
  if (x.query_splits > 1 && x.deterministic) return FA_ERR_UNSUPPORTED;
  const int T = (x.N + kTile - 1) / kTile;
  if ((long long)x.B * x.H * T * (x.query_splits > 1 ? x.query_splits : 1) > 0x7fffffffLL) return FA_ERR_UNSUPPORTED;
  if (check_workspace) {
    const WsLayout w = ws_layout(x.B, x.H, x.N, x.d, x.deterministic != 0, x.query_splits);
    if (!x.workspace || !aligned(x.workspace, 256) || x.workspace_bytes < w.total) return FA_ERR_WORKSPACE;
  }
  return FA_OK;
}

int* device_status_word() {
  int* p = nullptr;
  return status_word(&p) == FA_OK ? p : nullptr;
}

}  // namespace fa

using namespace fa;

extern "C" {

const char* fa_status_string(int s) {
  switch (s) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED";
    case FA_ERR_CUDA: return "FA_ERR_CUDA";
    case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT";
    case FA_ERR_WORKSPACE: return "FA_ERR_WORKSPACE";
    case FA_ERR_RANGE: return "FA_ERR_RANGE";
    default: return "FA_ERR_UNKNOWN";
  }
}

int fa_last_launch_count(void) { return t_last_launches; }

size_t fa_bwd_workspace_bytes(int B, int H, int N, int d) {
  if (check_shape(B, H, N, d, 1.f, FA_BF16) != FA_OK) return 0;
  return ws_layout(B, H, N, d).total;
}

size_t fa_bwd_workspace_bytes_ex(int B, int H, int N, int d, int deterministic) {
  if (check_shape(B, H, N, d, 1.f, FA_BF16) != FA_OK) return 0;
  return ws_layout(B, H, N, d, deterministic != 0).total;
}

size_t fa_bwd_workspace_bytes_split(int B, int H, int N, int d, int query_splits) {
  if (check_shape(B, H, N, d, 1.f, FA_BF16) != FA_OK) return 0;
  if (query_splits < 0 || query_splits > FA_MAX_PARTS) return 0;
  return ws_layout(B, H, N, d, false, query_splits).total;
}

int fa_bwd_splitq_choose(int B, int H, int N, int causal, int num_sms) {
  if (B < 1 || H < 1 || N < 1 || N > FA_MAX_SEQLEN || num_sms < 1) return 0;
  const long long T = (N + kTile - 1) / kTile;
  const long long BH = (long long)B * H;
  const long long total = BH * (causal ? T * (T + 1) / 2 : T * T);   // (key, query) tile pairs
  const long long avg = (total + num_sms - 1) / num_sms;
  int best = 1;
  long long best_cost = -1;
  for (int S = 1; S <= FA_MAX_PARTS; ++S) {
    const long long chunk = (T + S - 1) / S;       // query steps per range
    if (S > 1 && chunk < 4) break;
    const long long s_eff = (T + chunk - 1) / chunk;
    if (s_eff < S) continue;                        // the same cut as a smaller S
    // CTAs with work: under causal masking key tile j keeps T - j steps, so range s is empty
    // for the key tiles past T - s * chunk
    long long ctas = 0;
    for (long long sr = 0; sr < s_eff; ++sr) ctas += causal ? (T - sr * chunk) : T;
    ctas *= BH;
    const long long waves = (ctas + num_sms - 1) / num_sms;
    // Finishing time in tiles: CTAs of equal length (no causal mask) run in whole waves; causal
    // CTAs range from `chunk` tiles down to one, and the heaviest-first order packs them to about
    // the average load per SM, but no faster than the longest.  Plus about two tiles of fixed
    // cost per CTA in each wave.
    const long long span = causal ? (chunk > avg ? chunk : avg) : waves * chunk;
    const long long cost = span + 2 * waves;
    if (best_cost < 0 || 10 * cost < 9 * best_cost) {   // a larger count must win by 10 %
      best_cost = cost;
      best = S;
    }
  }
  return best;
}

int fa_fwd_ex(const fa_fwd_args* p) {
  if (p == nullptr) return FA_ERR_INVALID_ARG;
  const fa_fwd_args& x = *p;
  int rc = check_shape(x.B, x.H, x.N, x.d, x.scale, x.dtype);
  if (rc != FA_OK) return rc;
  if (!x.q || !x.k || !x.v || !x.o || !x.lse) return FA_ERR_INVALID_ARG;
  if (!aligned(x.q, 16) || !aligned(x.k, 16) || !aligned(x.v, 16) || !aligned(x.o, 16) || !aligned(x.lse, 4) ||
      !aligned(x.visit_log, 4))
    return FA_ERR_INVALID_ARG;
  Dropout drop{};
  if (!make_dropout(x.dropout_p, x.dropout_seed, &drop)) return FA_ERR_INVALID_ARG;
  const bool fp16 = x.dtype == FA_FP16;
  const int BH = x.B * x.H;
  const int T = (x.N + kTile - 1) / kTile;
  if (!fwd_grid_ok(BH, (T + 1) / 2, 1)) return FA_ERR_UNSUPPORTED;
  if (!get_encode()) return FA_ERR_CUDA;
  CUtensorMap tq, tk, tv;
  if (!encode_qkv(&tq, x.q, BH, x.N, x.d, fp16) || !encode_qkv(&tk, x.k, BH, x.N, x.d, fp16) ||
      !encode_qkv(&tv, x.v, BH, x.N, x.d, fp16))
    return FA_ERR_CUDA;
  FwdArgs a{};
  a.o = x.o;
  a.lse = x.lse;
  a.blockmask = x.blockmask;
  a.visit = x.visit_log;
  if (status_word(&a.status) != FA_OK) return FA_ERR_CUDA;
  a.timeout_ns = kWaitLimitNs;
  self_fwd_args(a, BH, x.N);
  a.causal = x.causal != 0;
  a.o_fp32 = x.o_fp32 != 0;
  a.drop = drop;
  a.scale_log2 = (float)((double)x.scale * 1.4426950408889634);
  t_last_launches = 0;
  if (launch_fwd(tq, tk, tv, a, x.d, fp16, static_cast<cudaStream_t>(x.stream)) != cudaSuccess) return FA_ERR_CUDA;
  t_last_launches = 1;
  return FA_OK;
}

int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d, float scale,
           int causal, const uint8_t* blockmask, void* stream) {
  fa_fwd_args a{};
  a.q = q; a.k = k; a.v = v; a.o = o; a.lse = lse;
  a.B = B; a.H = H; a.N = N; a.d = d;
  a.scale = scale; a.causal = causal; a.blockmask = blockmask;
  a.dtype = FA_BF16; a.o_fp32 = 0; a.visit_log = nullptr; a.stream = stream;
  return fa_fwd_ex(&a);
}

int fa_bwd_ex(const fa_bwd_args* p) {
  if (p == nullptr) return FA_ERR_INVALID_ARG;
  const fa_bwd_args& x = *p;
  int rc = validate_bwd(x, true);
  if (rc != FA_OK) return rc;
  Dropout drop{};
  make_dropout(x.dropout_p, x.dropout_seed, &drop);
  const bool det = x.deterministic != 0;
  const int qs = x.query_splits > 1 ? x.query_splits : 1;
  const WsLayout w = ws_layout(x.B, x.H, x.N, x.d, det, qs);
  const bool fp16 = x.dtype == FA_FP16;
  const int BH = x.B * x.H;
  const int T = (x.N + kTile - 1) / kTile;
  const int Np = T * kTile;
  if (!get_encode()) return FA_ERR_CUDA;
  CUtensorMap tq, tk, tv, tdo;
  if (!encode_qkv(&tq, x.q, BH, x.N, x.d, fp16) || !encode_qkv(&tk, x.k, BH, x.N, x.d, fp16) ||
      !encode_qkv(&tv, x.v, BH, x.N, x.d, fp16) || !encode_qkv(&tdo, x.dout, BH, x.N, x.d, fp16))
    return FA_ERR_CUDA;
  uint8_t* ws = static_cast<uint8_t*>(x.workspace);
  float* dq_acc = reinterpret_cast<float*>(ws + w.dq_acc);
  long long* dq_fix = det ? reinterpret_cast<long long*>(ws + w.dq_acc) : nullptr;
  CUtensorMap tdq;
  if (!encode_dqacc(&tdq, dq_acc, BH, x.N, x.d)) return FA_ERR_CUDA;
  float* delta = reinterpret_cast<float*>(ws + w.delta);
  float* lse2 = reinterpret_cast<float*>(ws + w.lse2);
  cudaStream_t s = static_cast<cudaStream_t>(x.stream);
  int* status = nullptr;
  if (status_word(&status) != FA_OK) return FA_ERR_CUDA;
  t_last_launches = 0;

  BwdPreArgs pre{};
  pre.o = x.o; pre.dout = x.dout; pre.lse = x.lse;
  pre.delta = delta; pre.lse2 = lse2; pre.dq_acc = dq_acc; pre.dq_fix = dq_fix;
  float* dk_acc = qs > 1 ? reinterpret_cast<float*>(ws + w.dk_acc) : nullptr;
  float* dv_acc = qs > 1 ? reinterpret_cast<float*>(ws + w.dv_acc) : nullptr;
  pre.dk_acc = dk_acc; pre.dv_acc = dv_acc;
  pre.N = x.N; pre.Np = Np; pre.BH = BH; pre.d = x.d;
  if (launch_bwd_pre(pre, fp16, s) != cudaSuccess) return FA_ERR_CUDA;

  BwdArgs b{};
  b.delta = delta; b.lse2 = lse2; b.dq_acc = dq_acc; b.dq_fix = dq_fix; b.dk = x.dk; b.dv = x.dv;
  b.blockmask = x.blockmask; b.visit = x.visit_log; b.status = status; b.timeout_ns = kWaitLimitNs;
  b.N = x.N; b.Np = Np; b.BH = BH; b.T = T; b.causal = x.causal != 0;
  b.q_splits = qs;
  b.q_chunk = (T + qs - 1) / qs;
  b.dk_acc = dk_acc; b.dv_acc = dv_acc;
  b.group_heads = group_heads_for(BH, T * qs);
  b.scale = x.scale;
  b.scale_log2 = (float)((double)x.scale * 1.4426950408889634);
  b.drop = drop;
  if (x.main_start_event && cudaEventRecord(static_cast<cudaEvent_t>(x.main_start_event), s) != cudaSuccess)
    return FA_ERR_CUDA;
  if (launch_bwd(tq, tk, tv, tdo, tdq, b, x.d, fp16, s) != cudaSuccess) return FA_ERR_CUDA;
  if (x.main_stop_event && cudaEventRecord(static_cast<cudaEvent_t>(x.main_stop_event), s) != cudaSuccess)
    return FA_ERR_CUDA;

  BwdPostArgs post{};
  post.dq_acc = dq_acc; post.dq_fix = dq_fix; post.dq = x.dq; post.n_elems = (long long)BH * x.N * x.d;
  post.dk_acc = dk_acc; post.dv_acc = dv_acc; post.dk = x.dk; post.dv = x.dv;
  post.N = x.N; post.Np = Np; post.BH = BH; post.d = x.d; post.scale = x.scale;
  if (launch_bwd_post(post, fp16, s) != cudaSuccess) return FA_ERR_CUDA;
  t_last_launches = 3;
  return FA_OK;
}

int fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dout, void* dq,
           void* dk, void* dv, int B, int H, int N, int d, float scale, int causal, const uint8_t* blockmask,
           void* workspace, size_t workspace_bytes, void* stream) {
  fa_bwd_args a{};
  a.q = q; a.k = k; a.v = v; a.o = o; a.lse = lse; a.dout = dout;
  a.dq = dq; a.dk = dk; a.dv = dv;
  a.B = B; a.H = H; a.N = N; a.d = d; a.scale = scale; a.causal = causal; a.blockmask = blockmask;
  a.dtype = FA_BF16; a.visit_log = nullptr;
  a.workspace = workspace; a.workspace_bytes = workspace_bytes; a.stream = stream;
  return fa_bwd_ex(&a);
}

int fa_fwd_partial(const fa_fwd_partial_args* p) {
  if (p == nullptr) return FA_ERR_INVALID_ARG;
  const fa_fwd_partial_args& x = *p;
  int rc = check_shape(x.B, x.H, x.N, x.d, x.scale, x.dtype);
  if (rc != FA_OK) return rc;
  if (x.Nk < 1 || x.key_offset < 0 || x.key_offset % kTile != 0) return FA_ERR_INVALID_ARG;
  if (x.Nk > FA_MAX_SEQLEN || (long long)x.B * x.H * x.Nk * x.d > (1LL << 46)) return FA_ERR_UNSUPPORTED;
  if ((x.causal || x.blockmask) && (long long)x.key_offset + x.Nk > x.N) return FA_ERR_INVALID_ARG;
  if (!x.q || !x.k || !x.v || !x.o_part || !x.lse_part) return FA_ERR_INVALID_ARG;
  if (!aligned(x.q, 16) || !aligned(x.k, 16) || !aligned(x.v, 16) || !aligned(x.o_part, 16) ||
      !aligned(x.lse_part, 4))
    return FA_ERR_INVALID_ARG;
  const bool fp16 = x.dtype == FA_FP16;
  const int BH = x.B * x.H;
  const int T = (x.N + kTile - 1) / kTile;
  if (!fwd_grid_ok(BH, (T + 1) / 2, 1)) return FA_ERR_UNSUPPORTED;
  if (!get_encode()) return FA_ERR_CUDA;
  CUtensorMap tq, tk, tv;
  if (!encode_qkv(&tq, x.q, BH, x.N, x.d, fp16) || !encode_qkv(&tk, x.k, BH, x.Nk, x.d, fp16) ||
      !encode_qkv(&tv, x.v, BH, x.Nk, x.d, fp16))
    return FA_ERR_CUDA;
  FwdArgs a{};
  a.o = x.o_part;
  a.lse = x.lse_part;
  a.blockmask = x.blockmask;
  a.visit = nullptr;
  if (status_word(&a.status) != FA_OK) return FA_ERR_CUDA;
  a.timeout_ns = kWaitLimitNs;
  self_fwd_args(a, BH, x.N);
  a.Nk = x.Nk;
  a.Tk = (x.Nk + kTile - 1) / kTile;
  a.kt_off = x.key_offset / kTile;
  a.split_tiles = a.Tk;
  a.causal = x.causal != 0;
  a.o_fp32 = 1;
  a.scale_log2 = (float)((double)x.scale * 1.4426950408889634);
  t_last_launches = 0;
  if (launch_fwd(tq, tk, tv, a, x.d, fp16, static_cast<cudaStream_t>(x.stream)) != cudaSuccess) return FA_ERR_CUDA;
  t_last_launches = 1;
  return FA_OK;
}

int fa_lse_merge(const float* const* o_parts, const float* const* lse_parts, int n_parts, void* o, float* lse,
                 int B, int H, int N, int d, int out_dtype, void* stream) {
  if (B < 1 || H < 1 || N < 1) return FA_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
  if (out_dtype != FA_BF16 && out_dtype != FA_FP16 && out_dtype != FA_FP32) return FA_ERR_UNSUPPORTED;
  if ((long long)B * H * N * d > (1LL << 46)) return FA_ERR_UNSUPPORTED;
  if (n_parts < 1 || n_parts > FA_MAX_PARTS) return FA_ERR_INVALID_ARG;
  if (!o_parts || !lse_parts || !o || !lse || !aligned(o, 16) || !aligned(lse, 4)) return FA_ERR_INVALID_ARG;
  MergeArgs m{};
  for (int i = 0; i < n_parts; ++i) {
    if (!o_parts[i] || !lse_parts[i] || !aligned(o_parts[i], 16) || !aligned(lse_parts[i], 4))
      return FA_ERR_INVALID_ARG;
    m.o_parts[i] = o_parts[i];
    m.lse_parts[i] = lse_parts[i];
  }
  m.o = o;
  m.lse = lse;
  m.rows = (long long)B * H * N;
  m.n_parts = n_parts;
  m.out_kind = out_dtype;
  t_last_launches = 0;
  if (launch_merge(m, d, static_cast<cudaStream_t>(stream)) != cudaSuccess) return FA_ERR_CUDA;
  t_last_launches = 1;
  return FA_OK;
}

size_t fa_fwd_splitkv_workspace_bytes(int B, int H, int N, int d, int num_splits) {
  if (check_shape(B, H, N, d, 1.f, FA_BF16) != FA_OK) return 0;
  if (num_splits < 1 || num_splits > FA_MAX_PARTS) return 0;
  return split_layout(B, H, N, d, num_splits).total;
}

int fa_splitkv_choose(int B, int H, int N, int causal, int num_sms) {
  if (B < 1 || H < 1 || N < 1 || N > FA_MAX_SEQLEN || num_sms < 1) return 0;
  const int T = (N + kTile - 1) / kTile;
  const long long units = (long long)B * H * ((T + 1) / 2);
  int best = 1;
  long long best_cost = -1;
  for (int S = 1; S <= FA_MAX_PARTS; ++S) {
    const int sp = (T + S - 1) / S;                 // key tiles per range
    if (S > 1 && sp < 4) break;
    const int s_eff = (T + sp - 1) / sp;            // ranges that hold any tile
    if (s_eff < S) continue;                        // same cut as a smaller S
    // causal CTAs average half the tiles: the light ones free their SMs early
    const long long load = units * s_eff / (causal ? 2 : 1);
    const long long waves = (load + num_sms - 1) / num_sms;
    const long long cost = (waves < 1 ? 1 : waves) * (sp + 2);
    if (best_cost < 0 || 10 * cost < 9 * best_cost) {   // a new cut must win by 10 % (merge cost)
      best_cost = cost;
      best = S;
    }
  }
  return best;
}

int fa_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
                   float scale, int causal, const uint8_t* blockmask, int num_splits, void* workspace,
                   size_t workspace_bytes, void* stream) {
  int rc = check_shape(B, H, N, d, scale, FA_BF16);
  if (rc != FA_OK) return rc;
  if (num_splits < 1 || num_splits > FA_MAX_PARTS) return FA_ERR_INVALID_ARG;
  if (num_splits == 1) return fa_fwd(q, k, v, o, lse, B, H, N, d, scale, causal, blockmask, stream);
  if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4))
    return FA_ERR_INVALID_ARG;
  const SplitLayout w = split_layout(B, H, N, d, num_splits);
  if (!workspace || !aligned(workspace, 256) || workspace_bytes < w.total) return FA_ERR_WORKSPACE;
  const int BH = B * H;
  const int T = (N + kTile - 1) / kTile;
  const int sp = (T + num_splits - 1) / num_splits;
  const int s_eff = (T + sp - 1) / sp;              // ranges past the last tile are dropped
  if (!fwd_grid_ok(BH, (T + 1) / 2, s_eff)) return FA_ERR_UNSUPPORTED;
  if (!get_encode()) return FA_ERR_CUDA;
  CUtensorMap tq, tk, tv;
  if (!encode_qkv(&tq, q, BH, N, d, false) || !encode_qkv(&tk, k, BH, N, d, false) ||
      !encode_qkv(&tv, v, BH, N, d, false))
    return FA_ERR_CUDA;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* o_parts = reinterpret_cast<float*>(ws + w.o_parts);
  float* lse_parts = reinterpret_cast<float*>(ws + w.lse_parts);
  FwdArgs a{};
  a.o = o_parts;
  a.lse = lse_parts;
  a.blockmask = blockmask;
  a.visit = nullptr;
  if (status_word(&a.status) != FA_OK) return FA_ERR_CUDA;
  a.timeout_ns = kWaitLimitNs;
  self_fwd_args(a, BH, N);
  a.n_splits = s_eff;
  a.split_tiles = sp;
  a.o_split_stride = w.o_stride;
  a.lse_split_stride = w.lse_stride;
  a.group_heads = group_heads_for(BH, a.n_units * s_eff);
  a.causal = causal != 0;
  a.o_fp32 = 1;
  a.scale_log2 = (float)((double)scale * 1.4426950408889634);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  t_last_launches = 0;
  if (launch_fwd(tq, tk, tv, a, d, false, s) != cudaSuccess) return FA_ERR_CUDA;
  MergeArgs m{};
  for (int i = 0; i < s_eff; ++i) {
    m.o_parts[i] = o_parts + i * w.o_stride;
    m.lse_parts[i] = lse_parts + i * w.lse_stride;
  }
  m.o = o;
  m.lse = lse;
  m.rows = (long long)BH * N;
  m.n_parts = s_eff;
  m.out_kind = FA_BF16;
  if (launch_merge(m, d, s) != cudaSuccess) return FA_ERR_CUDA;
  t_last_launches = 2;
  return FA_OK;
}

size_t fa_fwd_fp8_workspace_bytes(int B, int H, int N, int d) {
  if (check_shape(B, H, N, d, 1.f, FA_BF16) != FA_OK || d != 128) return 0;
  const size_t Np = (size_t)((N + kTile - 1) / kTile) * kTile;
  return align256((size_t)B * H * 128 * Np);
}

int fa_fwd_fp8(const fa_fwd_fp8_args* p) {
  if (p == nullptr) return FA_ERR_INVALID_ARG;
  const fa_fwd_fp8_args& x = *p;
  int rc = check_shape(x.B, x.H, x.N, x.d, x.scale, FA_BF16);
  if (rc != FA_OK) return rc;
  if (x.d != 128) return FA_ERR_UNSUPPORTED;
  for (float f : {x.descale_q, x.descale_k, x.descale_v})
    if (!(f > 0.f) || !std::isfinite(f)) return FA_ERR_INVALID_ARG;
  if (!x.q || !x.k || !x.v || !x.o || !x.lse) return FA_ERR_INVALID_ARG;
  if (!aligned(x.q, 16) || !aligned(x.k, 16) || !aligned(x.v, 16) || !aligned(x.o, 16) || !aligned(x.lse, 4))
    return FA_ERR_INVALID_ARG;
  const size_t need = fa_fwd_fp8_workspace_bytes(x.B, x.H, x.N, x.d);
  if (!x.workspace || !aligned(x.workspace, 256) || x.workspace_bytes < need) return FA_ERR_WORKSPACE;
  const int BH = x.B * x.H;
  const int T = (x.N + kTile - 1) / kTile;
  const int Np = T * kTile;
  if (!fwd_grid_ok(BH, (T + 1) / 2, 1)) return FA_ERR_UNSUPPORTED;
  if (!get_encode()) return FA_ERR_CUDA;
  CUtensorMap tq, tk, tvt;
  if (!encode_u8(&tq, x.q, 128, x.N, BH) || !encode_u8(&tk, x.k, 128, x.N, BH) ||
      !encode_u8(&tvt, x.workspace, Np, 128, BH))
    return FA_ERR_CUDA;
  F8Args a{};
  a.o = x.o;
  a.lse = x.lse;
  a.blockmask = x.blockmask;
  if (status_word(&a.status) != FA_OK) return FA_ERR_CUDA;
  a.timeout_ns = kWaitLimitNs;
  a.N = x.N;
  a.BH = BH;
  a.T = T;
  a.n_units = (T + 1) / 2;
  a.group_heads = group_heads_for(BH, a.n_units);
  a.causal = x.causal != 0;
  a.o_fp32 = x.o_fp32 != 0;
  a.scale_log2 = (float)((double)x.scale * x.descale_q * x.descale_k * 1.4426950408889634);
  a.o_scale = x.descale_v / 256.0f;
  t_last_launches = 0;
  if (launch_fwd_fp8(tq, tk, tvt, a, static_cast<const uint8_t*>(x.v), static_cast<uint8_t*>(x.workspace), Np,
                     static_cast<cudaStream_t>(x.stream)) != cudaSuccess)
    return FA_ERR_CUDA;
  t_last_launches = 2;
  return FA_OK;
}

int fa_check_status(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return FA_ERR_CUDA;
  int* p = nullptr;
  if (status_word(&p) != FA_OK) return FA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return FA_ERR_CUDA;
  if (v != 0) {
    const int zero = 0;
    if (cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return FA_ERR_CUDA;
    return status_from_device_word(v);
  }
  return FA_OK;
}

}  // extern "C"
