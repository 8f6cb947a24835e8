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
  FA_ERR_WORKSPACE = 5      /* workspace pointer NULL/misaligned or smaller than required   */
} fa_status;

typedef enum { FA_BF16 = 0, FA_FP16 = 1 } fa_dtype;

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

/* General forms: element type, optional fp32 O output, optional tile visit log. */
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
} fa_bwd_args;

int fa_fwd_ex(const fa_fwd_args* args);
int fa_bwd_ex(const fa_bwd_args* args);

/*
 * Synchronises `stream`, then reads and clears the device status word that kernels set
 * when a bounded wait expires.  Returns FA_OK, FA_ERR_TIMEOUT, or FA_ERR_CUDA.
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
 *   - the first call on a device looks up the array's device address for that device
 *     (cudaGetSymbolAddress); make that first call before any stream capture;
 *   - every call on a device shares the one array, which keeps the last call's contents
 *     (the backward rewrites all of it that it reads, so nothing needs clearing); calls that
 *     overlap on the GPU -- other streams or host threads -- race on it, so the caller
 *     must serialise them.
 */
int fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse,
                   const void* dout, void* dq, void* dk, void* dv,
                   int B, int H, int N, int d, float scale, int causal, const uint8_t* blockmask,
                   void* stream);

/* Static human-readable name of a status code. */
const char* fa_status_string(int status);

/* Number of kernel launches made by the last successful fa_fwd / fa_bwd call (any form) on this
   host thread. */
int fa_last_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif  /* FA_B200_H_ */
