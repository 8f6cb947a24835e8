/*
 * fa.h -- C ABI of the B200 (sm_100a) fused exact-attention library (libfa.so).
 *
 * The operation (FlashAttention-NeurIPS22 summary, "问题与动机" and "核心方法"):
 *     O = softmax(scale * Q Kᵀ) V            per (b, h) head, over [B, H, N, d] tensors,
 * computed in one fused tiled pass that never writes the N x N score or probability
 * matrices to memory ("核心方法 / Tiling 与 online softmax", "Kernel fusion"); the forward
 * saves only O and the row log-sum-exp LSE, and the backward recomputes each probability
 * tile from Q, K and LSE ("核心方法 / Backward recomputation").
 *
 * Conventions shared by every entry point
 *   - Q, K, V, O, dO, dQ, dK, dV: device pointers, dense row-major [B, H, N, d] of 16-bit
 *     elements (bf16 unless a *_ex call says fp16), 16-byte aligned; d is 64 or 128.
 *   - LSE: device fp32 [B, H, N], natural log of the row sum of exp(scale * q_i . k_j)
 *     over the visible keys; -inf for a row that sees no key (whose O row is then 0).
 *   - causal != 0: key j is visible to query i iff j <= i (equal query/key length N).
 *   - blockmask: NULL (dense) or a DEVICE pointer to uint8 [T, T], T = ceil(N / 128),
 *     row-major, shared by all (b, h); tile (i, j) of 128 x 128 scores is computed iff
 *     blockmask[i * T + j] != 0 ("核心方法 / Block-sparse 扩展": zero blocks are skipped
 *     and never read).  causal and blockmask compose by intersection.
 *   - stream: a cudaStream_t passed as void* (NULL = legacy default stream).  Calls are
 *     stream-ordered and asynchronous; they allocate no memory and keep no state across
 *     calls except a per-process device status word (see fa_check_status).
 *   - The caller allocates and owns every buffer.  Inputs are read only.
 *   - Return value: FA_OK, or an fa_status error.  Argument errors return before anything
 *     is launched.  FA_ERR_CUDA means a CUDA runtime call failed at launch time.
 *   - The library caches, per device ordinal, the device addresses of its own device
 *     variables (the status word, fa_bwd_noalloc's array) for the life of the process, so it
 *     must not be used across cudaDeviceReset (or any other teardown of a device's primary
 *     context): after one, the cached addresses are stale.
 */
#ifndef FA_B200_H_
#define FA_B200_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  FA_OK = 0,
  FA_ERR_INVALID_ARG = 1,   /* NULL pointer, N < 1, B/H < 1, misaligned pointer, bad sizes */
  FA_ERR_UNSUPPORTED = 2,   /* d not in {64, 128}, dtype not bf16/fp16, N too large        */
  FA_ERR_CUDA = 3,          /* a CUDA runtime/driver call failed (no device, launch error)  */
  FA_ERR_TIMEOUT = 4,       /* a kernel's bounded wait expired (reported by fa_check_status) */
  FA_ERR_WORKSPACE = 5,     /* workspace pointer NULL/misaligned or smaller than required   */
  FA_ERR_RANGE = 6          /* deterministic backward: a dQ partial was non-finite or too
                               large for the fixed-point accumulator (fa_check_status)       */
} fa_status;

typedef enum {
  FA_BF16 = 0,
  FA_FP16 = 1,
  FA_FP32 = 2              /* output type of fa_lse_merge only */
} fa_dtype;

/* Largest sequence length accepted (tile lists live in shared memory: T <= 2048). */
#define FA_MAX_SEQLEN (2048 * 128)

/*
 * Forward pass (FlashAttention-NeurIPS22, "核心方法": tiling + online softmax + fusion).
 *   q, k, v : in,  [B, H, N, d] bf16
 *   o       : out, [B, H, N, d] bf16
 *   lse     : out, [B, H, N] fp32 (natural log, see above)
 *   scale   : multiplies Q Kᵀ before the softmax (typically 1/sqrt(d))
 */
int fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
           int B, int H, int N, int d, float scale, int causal,
           const uint8_t* blockmask, void* stream);

/*
 * Bytes of device workspace fa_bwd needs for this shape (fp32 dQ accumulator plus two
 * fp32 per-row vectors padded to whole 128-row tiles, each part 256-byte aligned).
 * Pure host arithmetic; returns 0 for invalid sizes.
 * (NeurIPS22 summary, "核心方法 / Backward recomputation": the backward keeps O(N d) state
 * besides its inputs -- the per-row statistics and one dQ accumulator -- never an N x N
 * matrix; this is that state's size: B*H*N*(4*d) + 2 * B*H*ceil(N/128)*128*4 bytes, rounded
 * up per part to 256 bytes.)
 */
size_t fa_bwd_workspace_bytes(int B, int H, int N, int d);

/*
 * Backward pass ("核心方法 / Backward recomputation"): recomputes P tile by tile from
 * q, k and the forward's lse, and writes the gradients of sum(dout o O).
 *   q, k, v, o, lse : in, exactly as given to / produced by fa_fwd
 *   dout            : in,  [B, H, N, d] bf16 upstream gradient
 *   dq, dk, dv      : out, [B, H, N, d] bf16
 *   workspace       : device scratch of at least fa_bwd_workspace_bytes(B, H, N, d) bytes,
 *                     256-byte aligned; overwritten, needs no initialisation
 * Three launches on `stream`: row preprocess (D = rowsum(dO o O), dQ accumulator = 0),
 * the fused main kernel (one CTA per 128-key tile), and the dQ conversion.
 */
int fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
           const void* dout, void* dq, void* dk, void* dv,
           int B, int H, int N, int d, float scale, int causal, const uint8_t* blockmask,
           void* workspace, size_t workspace_bytes, void* stream);

/*
 * General forms of fa_fwd / fa_bwd (the same operation, "核心方法"; the pages fix no calling
 * convention): element type bf16 or fp16, optional fp32 O output, optional tile visit log
 * (the evidence that block-sparse skipping, "核心方法 / Block-sparse 扩展", computed exactly
 * the kept tiles), per-kernel timing events, and the modes below (dropout, deterministic
 * backward).  Errors as fa_fwd / fa_bwd.
 */
typedef struct {
  const void* q; const void* k; const void* v;
  void* o;                 /* bf16/fp16 like q, or fp32 when o_fp32 != 0            */
  float* lse;
  int B, H, N, d;
  float scale;
  int causal;
  const uint8_t* blockmask;
  int dtype;               /* fa_dtype of q, k, v (and of o unless o_fp32)           */
  int o_fp32;              /* nonzero: o is fp32 [B, H, N, d]                        */
  int* visit_log;          /* NULL, or device int32 [B, H, T, T] that the kernel
                              increments once per (query tile, key tile) it computes */
  void* stream;
  float dropout_p;         /* 0 (off) or a dropout probability in [0, 1), see below  */
  unsigned long long dropout_seed;
} fa_fwd_args;

typedef struct {
  const void* q; const void* k; const void* v; const void* o; const float* lse;
  const void* dout; void* dq; void* dk; void* dv;
  int B, H, N, d;
  float scale;
  int causal;
  const uint8_t* blockmask;
  int dtype;               /* fa_dtype of every 16-bit tensor                        */
  int* visit_log;          /* as in fa_fwd_args, for the main backward kernel        */
  void* workspace; size_t workspace_bytes;
  void* stream;
  void* main_start_event;  /* NULL, or a cudaEvent_t recorded on `stream` right before the
                              fused main backward kernel (for per-kernel timing)       */
  void* main_stop_event;   /* NULL, or a cudaEvent_t recorded right after it           */
  int deterministic;       /* nonzero: bitwise repeatable dQ (see below); the workspace
                              must then hold fa_bwd_workspace_bytes_ex(..., 1) bytes    */
  float dropout_p;         /* exactly the forward's dropout_p and dropout_seed        */
  unsigned long long dropout_seed;
  int query_splits;        /* 0 or 1: off; S >= 2: split each key tile's query range, see
                              below (the workspace must then hold
                              fa_bwd_workspace_bytes_split(..., S) bytes)               */
} fa_bwd_args;

int fa_fwd_ex(const fa_fwd_args* args);
int fa_bwd_ex(const fa_bwd_args* args);

/*
 * Dropout on the attention probabilities, fused into both passes (FlashAttention-NeurIPS22
 * summary, "核心方法 / Kernel fusion"; the backward regenerates the mask from the generator
 * state instead of storing it, "Backward recomputation").  With dropout_p > 0:
 *   - score (i, j) of head (b, h) draws byte (j mod 16) of Philox4x32-10 (Salmon et al.,
 *     SC'11) at counter (j / 16, i, b * H + h, 0) with key (seed mod 2^32, seed / 2^32),
 *     bytes little-endian within the four 32-bit output words;
 *   - it is dropped iff that byte < t = floor(256 * dropout_p + 1/2) (at most 255), so the
 *     probability is applied in steps of 1/256; kept probabilities are scaled by
 *     256 / (256 - t), so the mask has mean exactly 1;
 *   - O = (P o M) V, while LSE stays the log-sum-exp of the undropped scores;
 *   - the backward must get the same dropout_p and dropout_seed as the forward.
 * dropout_p outside [0, 1) (or NaN) returns FA_ERR_INVALID_ARG.  A value small enough that
 * t = 0 means no dropout.  The split-KV and key-slice entry points take no dropout.
 */

/*
 * Deterministic backward (fa_bwd_args.deterministic != 0).  "Exact and deterministic" is a
 * property the FlashAttention-2 wiki claims ("性能与效率"); the forward has it as built, but
 * the default backward adds each key tile's fp32 dQ partial into the accumulator in whatever
 * order the CTAs finish, and fp32 addition is not associative.  This mode adds the partials
 * as int64 fixed point with 32 fraction bits instead: integer addition is associative, so
 * dQ (and dK, dV, which never depended on order) are bitwise identical from run to run.
 *   - cost: an int64 accumulator (twice the bytes of the fp32 one) over whole 128-row tiles;
 *   - precision: each partial is rounded to a multiple of 2^-32 before the (exact) sum, an
 *     absolute error of at most T * 2^-33 on scale^-1 * dQ;
 *   - range: a partial with magnitude >= 2^20 (or non-finite) makes the call report
 *     FA_ERR_RANGE through fa_check_status; the sum of up to 2048 tiles then stays inside
 *     the int64 range, so no result is silently wrapped.
 * Workspace bytes for either mode; fa_bwd_workspace_bytes(...) == ..._ex(..., 0).
 */
size_t fa_bwd_workspace_bytes_ex(int B, int H, int N, int d, int deterministic);

/*
 * Query-range splits of the backward (fa_bwd_args.query_splits = S >= 2), its counterpart of the
 * split-KV forward.  The FlashAttention-2 wiki ("改进并行性") spreads one head's work over the
 * SMs because a small batch of long sequences otherwise leaves SMs idle.  The backward runs one
 * CTA per (head, 128-key tile), and that CTA walks the key tile's query tiles; with few heads
 * there are too few CTAs, and under causal masking key tile 0 walks all T query tiles while
 * the last walks one.  With S splits each key tile's visited query tiles are cut into S ranges
 * of ceil(T / S) steps, one CTA per (head, key tile, range).  Each range's dK and dV partials
 * are added in fp32 into workspace accumulators and a final pass converts them, so:
 *   - the result equals the unsplit one up to fp32 summation order (not bitwise);
 *   - it does not combine with deterministic != 0 (FA_ERR_UNSUPPORTED);
 *   - the workspace grows by two fp32 [B, H, N, d] accumulators:
 *     fa_bwd_workspace_bytes_split(B, H, N, d, S) (== fa_bwd_workspace_bytes for S <= 1).
 * 0 <= query_splits <= FA_MAX_PARTS, else FA_ERR_INVALID_ARG.
 * fa_bwd_splitq_choose: host arithmetic, the S to use on a GPU with num_sms SMs: minimises the
 * finishing time in tiles -- whole waves of equal ranges without causal masking, else
 * max(longest range, average (key, query) tile pairs per SM) -- plus 2 per wave of CTAs, over
 * 1 .. FA_MAX_PARTS with at least 4 steps per range; a larger S must win by 10 %.  Returns 1
 * when the key tiles alone fill the GPU, 0 for invalid sizes.
 */
size_t fa_bwd_workspace_bytes_split(int B, int H, int N, int d, int query_splits);
int fa_bwd_splitq_choose(int B, int H, int N, int causal, int num_sms);

/*
 * Synchronises `stream`, then reads and clears the device status word that kernels set
 * when a bounded wait expires (FA_ERR_TIMEOUT) or a deterministic backward meets a partial
 * outside its range (FA_ERR_RANGE).  Returns FA_OK, FA_ERR_TIMEOUT, FA_ERR_RANGE or
 * FA_ERR_CUDA.  FA_ERR_CUDA also stands for a kernel that found its own launch state
 * unusable (its dynamic shared memory not 1024-byte aligned) and did no work; the device
 * records such states under codes of its own, which are never returned as they are.
 * (No counterpart in the pages: failure reporting of this library.)
 */
int fa_check_status(void* stream);

/* Size of the fixed device scratch array that fa_bwd_noalloc uses: 64 MiB. */
#define FA_NOALLOC_SCRATCH_BYTES (64u << 20)

/*
 * fa_bwd_noalloc -- fa_bwd for callers that cannot allocate device memory when they call.
 * (No counterpart in the paper: this is a deployment variant of the backward entry point.)
 *
 * Who needs it: callers with no device allocator at call time, such as an engine plugin
 * whose enqueue step must not allocate, a host program linking libfa.so without any device
 * allocator of its own, or code running while the device memory pool is frozen.  fa_bwd
 * asks them for a workspace they cannot provide; this entry point instead uses one fixed
 * file-scope device array of FA_NOALLOC_SCRATCH_BYTES that lives on every GPU that loads
 * the library until the process exits.
 *
 * Arguments and results are exactly those of fa_bwd without the workspace pair.
 * Limits and behaviour:
 *   - returns FA_ERR_WORKSPACE, launching nothing, when fa_bwd_workspace_bytes(B, H, N, d)
 *     exceeds FA_NOALLOC_SCRATCH_BYTES (roughly B*H*N*(4*d + 8) bytes must fit in 64 MiB);
 *   - allocates nothing: no cudaMalloc / cudaFree and no allocating library routine;
 *   - the first call on a device does a one-time set-up there: the CUDA runtime loads the
 *     library's device code lazily, so that call loads the code that holds the array, which
 *     commits its FA_NOALLOC_SCRATCH_BYTES of device memory, and looks up the array's device
 *     address (cudaGetSymbolAddress).  Make that first call at start-up, before any stream
 *     capture and before device memory is frozen or exhausted; every later call allocates
 *     nothing at all;
 *   - argument errors are those of fa_bwd and come back before any CUDA call;
 *   - every call on a device shares the one array, which keeps the last call's contents
 *     (the backward rewrites all of it that it reads, so nothing needs clearing); calls that
 *     overlap on the GPU -- other streams or host threads -- race on it, so the caller
 *     must serialise them.
 */
int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                   const void* dout, void* dq, void* dk, void* dv,
                   int B, int H, int N, int d, float scale, int causal, const uint8_t* blockmask,
                   void* stream);

/*
 * ---------------------------------------------------------------------------------------
 * Attention over a slice of the keys, and the merge of slices (split-KV forward).
 *
 * The FlashAttention-2 wiki ("改进并行性") spreads one head's work over the GPU's SMs because
 * long sequences with small batches otherwise leave SMs idle; the NeurIPS22 summary leaves
 * decode-style small-batch long-context use and multi-GPU sequence parallelism to follow-on
 * work ("边界条件", "局限与 Future Work").  Cutting the KEYS of a head into slices serves both:
 * each slice's attention is independent, and the results combine exactly through their
 * log-sum-exps (the online-softmax rescaling of "核心方法 / Tiling 与 online softmax"):
 *     LSE = ln sum_s exp(LSE_s),    O = sum_s exp(LSE_s - LSE) O_s.
 * ---------------------------------------------------------------------------------------
 */

/* Most key splits of fa_fwd_splitkv and most parts of fa_lse_merge. */
#define FA_MAX_PARTS 64

/*
 * Forward over a slice of the keys: every query row of q attends only to the Nk keys of k/v.
 *   q          : in,  [B, H, N, d] (dtype), all query rows of the sequence
 *   k, v       : in,  [B, H, Nk, d] (dtype), key rows that sit at query-sequence positions
 *                key_offset .. key_offset + Nk - 1
 *   o_part     : out, [B, H, N, d] fp32, normalised over this slice's keys (0 where a row
 *                sees none of them)
 *   lse_part   : out, [B, H, N] fp32, natural log-sum-exp over this slice (-inf if none)
 *   key_offset : a multiple of 128, >= 0.  causal keeps key position <= query row; the
 *                blockmask ([T, T], T = ceil(N / 128), as for fa_fwd) is indexed by the
 *                query-sequence tiles of the keys.  With causal or a blockmask,
 *                key_offset + Nk must not exceed N; without either, Nk and key_offset are
 *                free (cross-attention over any key set).
 * One launch.  Errors: FA_ERR_INVALID_ARG for NULL or misaligned pointers, Nk < 1, a bad
 * key_offset; otherwise as fa_fwd.
 */
typedef struct {
  const void* q; const void* k; const void* v;
  float* o_part;
  float* lse_part;
  int B, H, N, Nk, d;
  int key_offset;
  float scale;
  int causal;
  const uint8_t* blockmask;
  int dtype;               /* fa_dtype of q, k, v: FA_BF16 or FA_FP16 */
  void* stream;
} fa_fwd_partial_args;

int fa_fwd_partial(const fa_fwd_partial_args* args);

/*
 * Combine n_parts results over disjoint key slices of the same rows.
 *   o_parts, lse_parts : HOST arrays of n_parts DEVICE pointers; part s is fp32
 *                        [B, H, N, d] and fp32 [B, H, N], 16- and 4-byte aligned.  The
 *                        pointers may address another GPU's memory where peer access is
 *                        enabled (the kernel reads them with plain loads).
 *   o                  : out, [B, H, N, d] of out_dtype (FA_BF16, FA_FP16 or FA_FP32)
 *   lse                : out, [B, H, N] fp32
 * 1 <= n_parts <= FA_MAX_PARTS.  A row no part saw a key for gets O = 0 and LSE = -inf.
 * One launch; nothing is allocated.
 */
int fa_lse_merge(const float* const* o_parts, const float* const* lse_parts, int n_parts,
                 void* o, float* lse, int B, int H, int N, int d, int out_dtype, void* stream);

/*
 * Split-KV forward: the same result as fa_fwd (bf16), computed with the key tiles of every
 * head cut into num_splits ranges of ceil(T / num_splits) tiles, one CTA per (pair of query
 * tiles, range), and merged.  For heads too few to fill the GPU (small batch, long N).
 *   num_splits : 1 .. FA_MAX_PARTS (1 = fa_fwd itself: one launch, no workspace used);
 *                fa_splitkv_choose gives a good value
 *   workspace  : device scratch of fa_fwd_splitkv_workspace_bytes(B, H, N, d, num_splits)
 *                bytes, 256-byte aligned (the fp32 partial O and LSE of every range)
 * Two launches (the split forward, then the merge) when num_splits > 1.  LSE and O equal
 * fa_fwd's up to fp32 rounding of the merge; ranges past the last key tile are empty and
 * cost one short CTA each.
 */
size_t fa_fwd_splitkv_workspace_bytes(int B, int H, int N, int d, int num_splits);
int fa_fwd_splitkv(const void* q, const void* k, const void* v, void* o, float* lse,
                   int B, int H, int N, int d, float scale, int causal, const uint8_t* blockmask,
                   int num_splits, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Host arithmetic: the split count fa_fwd_splitkv should use on a GPU with num_sms SMs (one
 * forward CTA per SM).  Minimises (waves of CTAs) x (key tiles per CTA + 2), the 2 standing
 * for a CTA's fixed cost in tiles and causal CTAs counting half, over 1 .. FA_MAX_PARTS
 * with at least 4 key tiles per range; a larger count must win by 10 % (the merge's cost).  Returns 1 when the query tiles alone fill the GPU, and 0
 * for invalid sizes.
 */
int fa_splitkv_choose(int B, int H, int N, int causal, int num_sms);

/*
 * ---------------------------------------------------------------------------------------
 * FP8 (E4M3) forward, head dimension 128.  The FlashAttention-2 wiki ("FlashAttention-3")
 * names FP8 low precision for the Hopper follow-on without a scaling convention; here each
 * of Q, K, V is given as E4M3 codes (OCP FP8 E4M3, the "fn" variant: finite, max 448) with
 * one fp32 dequantisation factor per tensor, value = descale * code.
 *
 * The result is the exact attention of those values, O = softmax(scale * Q Kᵀ) V, up to one
 * rounding: the probabilities enter the P V product as E4M3(256 P) / 256, i.e. with relative
 * error <= 2^-4 (absolute <= 2^-18 below E4M3's normal range), so elementwise
 *     |O - O_exact| <= 2^-4 * sum_j P_ij |V_jc| + 2^-18 * sum_j |V_jc|  (+ fp32 / output rounding).
 * LSE is computed from the unrounded P in fp32, as in fa_fwd.
 *   q, k, v   : in,  E4M3 bytes [B, H, N, 128], 16-byte aligned
 *   o         : out, [B, H, N, 128] bf16, or fp32 when o_fp32 != 0
 *   lse       : out, [B, H, N] fp32
 *   workspace : device scratch of fa_fwd_fp8_workspace_bytes(B, H, N, 128) bytes, 256-byte
 *               aligned: V transposed to [B, H, 128, ceil(N/128)*128] (keys contiguous)
 * causal and blockmask as for fa_fwd.  Two launches (the V transpose, then the fused
 * forward).  d != 128 returns FA_ERR_UNSUPPORTED; a descale that is not finite and > 0
 * returns FA_ERR_INVALID_ARG.  There is no FP8 backward.
 */
typedef struct {
  const void* q; const void* k; const void* v;
  float descale_q, descale_k, descale_v;
  void* o;
  float* lse;
  int B, H, N, d;
  float scale;
  int causal;
  const uint8_t* blockmask;
  int o_fp32;
  void* workspace; size_t workspace_bytes;
  void* stream;
} fa_fwd_fp8_args;

size_t fa_fwd_fp8_workspace_bytes(int B, int H, int N, int d);
int fa_fwd_fp8(const fa_fwd_fp8_args* args);

/*
 * Diagnostic of failure detection (no counterpart in the pages).  Launches one small kernel
 * that runs the library's bounded mbarrier wait on a barrier nothing ever completes, with
 * a limit of limit_us microseconds (1 .. 1000000).  The wait must give up at the limit and
 * the kernel return; the next fa_check_status on `stream` then returns FA_ERR_TIMEOUT (and
 * clears the word).  waited_ok: NULL, or a device int that receives 0 when the wait gave up
 * (1 would mean the barrier completed, which cannot happen).  Nothing faults, traps or
 * loops without bound.  Returns FA_OK once launched, FA_ERR_INVALID_ARG for a limit out of
 * range, FA_ERR_CUDA on a launch error.
 */
int fa_selftest_wait_timeout(unsigned int limit_us, int* waited_ok, void* stream);

/*
 * Diagnostic (no counterpart in the pages): y[i] = 2^x[i] for i < n, evaluated by the
 * polynomial the kernels use for part of their exponentials to take load off the
 * special-function unit (the FlashAttention-2 wiki, "最小化非矩阵运算", counts these
 * non-matmul operations as the cost to cut).  x and y are device fp32 arrays of n elements.
 * Claimed accuracy: relative error <= 1.1e-4 for x in [-126, 0]; exactly 1 at x = 0;
 * exactly +0 for x <= -127 and for x = -inf; below 2^-126 in absolute value for x in
 * (-127, -126).  One launch on `stream`; FA_ERR_INVALID_ARG for n < 1 or a NULL pointer.
 */
int fa_selftest_exp2_poly(const float* x, float* y, int n, void* stream);

/* Static human-readable name of a status code (no counterpart in the pages). */
const char* fa_status_string(int status);

/* Number of kernel launches made by the last successful fa_fwd / fa_bwd call (any form) on this
   host thread. */
int fa_last_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif  /* FA_B200_H_ */
