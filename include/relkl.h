/*
 * relkl.h -- C ABI of librelkl.so: the linear-memory relation-distillation KL
 * loss of LinearARD and its gradient, on NVIDIA B200 (sm_100a).
 *
 * What is computed.  LinearARD (arXiv 2604.00004; pith.science verdict page,
 * field pith_extraction.key_machinery, repeated in core_discovery; the
 * abstract on the mlsanity.com index page) distils, for every head and for
 * X in {Q, K, V}, the row-wise distributions of the masked self-relation
 *
 *     Z_m = X_m X_m^T * scale + M,   R_m = softmax_rows(Z_m),  m in {t, s},
 *
 * of a frozen teacher (t) into a RoPE-scaled student (s) by the forward KL
 *
 *     kl_i = KL(R_t(i,:) || R_s(i,:)),   L = (1/n) sum_i kl_i,
 *
 * and backpropagates through the identity dL/dZ_s(i,j) = (R_s - R_t)(i,j)/n.
 * With an upstream gradient dkl_i per row, G(i,j) = dkl_i (R_s - R_t)(i,j) on
 * allowed entries and, because X_s appears on both sides of Z_s,
 *
 *     dX_s = scale * (G + G^T) X_s.
 *
 * M is the causal mask (column j allowed for row i iff j <= i) when
 * `causal` is set, and no mask otherwise; the pages name M without defining
 * it.  No N x N matrix is ever stored: the forward keeps O(N) row statistics
 * and the backward recomputes the logit tiles (the pages' two-phase scheme).
 *
 * A "unit" is one (batch b, head h) slice of one relation: an [N, d] teacher
 * matrix and the matching student matrix.  Units are independent.
 *
 * Conventions for every entry point below:
 *  - All tensor pointers are DEVICE pointers, owned by the caller, and must
 *    stay valid until the work queued on `stream` has finished.  The library
 *    allocates no device or host memory and keeps no pointer after a call.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls
 *    only enqueue work on it and return; nothing synchronises except
 *    relkl_get_device_error().
 *  - The current CUDA device (cudaSetDevice) must be the one that owns the
 *    tensors and `stream`: the library reads its properties and launches on
 *    it.
 *  - Arguments are validated before anything is enqueued; on any error code
 *    other than RELKL_OK nothing was enqueued, except RELKL_ERR_CUDA, which
 *    reports a failed launch (see relkl_last_cuda_error()).
 *  - Row statistics and gradients are float32.  Teacher and student inputs
 *    are bf16 (tensor-core path, d in {64, 128}) or float32 (CUDA-core path,
 *    1 <= d <= 128).
 */
#ifndef RELKL_H
#define RELKL_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  RELKL_OK = 0,
  RELKL_ERR_INVALID = 1,      /* null pointer, bad shape, stride or alignment      */
  RELKL_ERR_UNSUPPORTED = 2,  /* well-formed but not provided (e.g. bf16 with d=96) */
  RELKL_ERR_CUDA = 3,         /* a CUDA runtime or driver call failed               */
  RELKL_ERR_WORKSPACE = 4,    /* workspace missing, misaligned or too small          */
  RELKL_ERR_TIMEOUT = 5       /* a bounded device-side wait ran out (device record)  */
} relkl_status;

typedef enum { RELKL_BF16 = 0, RELKL_FP32 = 1 } relkl_dtype;

/* Shape of one relation's teacher AND student tensors (both use it).
 * Logical shape [B, H, N, d]; element (b,h,n,k) lives at
 *   base + b*stride[0] + h*stride[1] + n*stride[2] + k      (elements).
 * stride[3] must be 1.  For the bf16 path the base address and stride[0..2]
 * (in bytes) must be multiples of 16 (a TMA requirement).                    */
typedef struct {
  int32_t B, H, N, d;
  int64_t stride[4];
  int32_t dtype;     /* relkl_dtype                                         */
  int32_t causal;    /* 1: row i sees columns j <= i; 0: every column       */
  float scale;       /* logit scale; 0 means 1/sqrt(d)                      */
  int32_t reserved;  /* must be 0                                           */
  /* Optional right padding: DEVICE pointer to B int32 valid lengths (NULL: all
   * N rows valid).  For batch b, rows and columns >= L_b = clamp(lengths[b],
   * 0, N) are padding: no row distribution includes them, their kl rows and
   * stats are 0, their dX_s rows are 0, and the default upstream gradient of
   * a valid row is 1/L_b.  Read on the device; must stay valid until the
   * queued work has finished; 4-byte aligned.                               */
  const int32_t* lengths;
  /* Optional packed variable-length sequences (cu_seqlens NULL: none).  The
   * tensors are [1, H, N, d] (B must be 1, lengths NULL) and hold n_seq
   * sequences back to back on the token axis: sequence k owns tokens
   * [cu_seqlens[k], cu_seqlens[k+1]) (DEVICE int32 [n_seq + 1],
   * non-decreasing, cu_seqlens[0] = 0, cu_seqlens[n_seq] <= N; read on the
   * device, 4-byte aligned).  Each (sequence, head) is a unit of its own: its
   * rows see only its own tokens (causal or full inside it), its default
   * upstream gradient is 1/L_k, and kl, stats and dX_s use the [1, H, N]
   * layout of the tokens.  Tokens past cu_seqlens[n_seq] belong to no
   * sequence: the forward leaves their kl and stats rows untouched and their
   * dX_s rows are 0.  max_seqlen must be >= every sequence's length (it sizes
   * the work; rows of a longer sequence past max_seqlen are not computed).  */
  const int32_t* cu_seqlens;
  int32_t n_seq;
  int32_t max_seqlen;
} relkl_desc;

/* Bytes of device workspace a call needs (for every entry point, any desc):
 * a 256-byte, 256-byte-aligned record that the kernels use to report a
 * bounded wait that ran out.  Zero it once after allocation
 * (relkl_workspace_init); calls never clear it, so a reported error sticks
 * until the caller clears it again.                                          */
size_t relkl_workspace_bytes(void);
relkl_status relkl_workspace_init(void* ws, size_t ws_bytes, void* stream);

/* Forward (Phase 1 on the pages: per-row statistics, O(N) memory).
 *   x_t, x_s : teacher / student, layout `desc`.
 *   kl       : float [B, H, N] contiguous, out: kl_i per row.
 *   stats    : float [B, H, N, 4] contiguous, out, per row
 *              (m, lse_t, lse_s, w): m = max_j max(Z_t, Z_s)(i,j) over allowed
 *              j, lse_m = log sum_j exp Z_m(i,j), w = sum_j R_t (Z_t - Z_s)(i,j).
 *              kl_i = w_i + lse_s(i) - lse_t(i).  Needed by relkl_bwd.      */
relkl_status relkl_fwd(const relkl_desc* desc, const void* x_t, const void* x_s,
                       float* kl, float* stats, void* ws, size_t ws_bytes,
                       void* stream);

/* Backward (Phase 2 on the pages: recompute the logit tiles, rebuild R_t and
 * R_s from the stored LSEs, form G and stream it into dX_s).
 *   stats    : the forward's statistics for the same inputs.
 *   dkl      : float [B, H, N] contiguous upstream gradient of kl, or NULL for
 *              1/N on every row (the gradient of L = (1/N) sum_i kl_i).
 *   dx_s     : float [B, H, N, d] contiguous, out: overwritten with dL/dX_s.
 * The teacher is frozen and gets no gradient.  dx_s is zeroed on `stream`
 * and then accumulated by float32 reduce-adds performed in L2 (TMA bulk-tensor
 * reductions on the tensor-core path, atomics on the CUDA-core path); the
 * order of those additions depends on scheduling, so the last bits of dx_s
 * may differ between runs.                                                  */
relkl_status relkl_bwd(const relkl_desc* desc, const void* x_t, const void* x_s,
                       const float* stats, const float* dkl, float* dx_s,
                       void* ws, size_t ws_bytes, void* stream);

/* Several relations (Q, K, V of one layer; GQA gives K and V fewer heads)
 * in ONE persistent launch.  n_rel in 1..3; descs[r] describes relation r.
 * All descs must share N, d, dtype, causal and scale; B and H may differ.
 * Arrays are indexed by relation, with the meaning of relkl_fwd / relkl_bwd.
 * dkl may be NULL (all relations use 1/N) or an array whose entries may be NULL. */
relkl_status relkl_fwd_qkv(int32_t n_rel, const relkl_desc* descs,
                           const void* const* x_t, const void* const* x_s,
                           float* const* kl, float* const* stats,
                           void* ws, size_t ws_bytes, void* stream);
relkl_status relkl_bwd_qkv(int32_t n_rel, const relkl_desc* descs,
                           const void* const* x_t, const void* const* x_s,
                           const float* const* stats, const float* const* dkl,
                           float* const* dx_s, void* ws, size_t ws_bytes,
                           void* stream);

/* One part of the fused calls above, for splitting one problem's rows over
 * several GPUs (row-sharded context parallelism: the pages give the method
 * for one device; this split follows from rows of the relation being
 * independent in the forward and additive in the backward).
 *
 * Every unit's rows are grouped into work items (pairs of 128-row blocks on
 * the tensor-core path, 32-row blocks on the CUDA-core path); part `part` of
 * `n_parts` (0 <= part < n_parts) takes items part, part + n_parts, ...
 * of every unit, so the parts hold nearly equal causal work.
 *   relkl_fwd_qkv_part writes kl and stats for the rows of its items only and
 *     leaves every other row untouched: zero the outputs, run every part and
 *     add (or all-reduce) them to obtain relkl_fwd_qkv's result.
 *   relkl_bwd_qkv_part needs stats for every row its items read (in general
 *     all rows: combine the parts' forward statistics first).  dx_s is
 *     overwritten with the contributions of this part's rows of G to both
 *     sides of dX_s = scale (G + G^T) X_s; the sum of dx_s over all parts is
 *     relkl_bwd_qkv's result.
 * Teacher and student must hold every row of every unit (gather them first).
 * n_parts = 1 is relkl_fwd_qkv / relkl_bwd_qkv.  RELKL_ERR_INVALID for a bad
 * part index.                                                               */
relkl_status relkl_fwd_qkv_part(int32_t n_rel, const relkl_desc* descs,
                                const void* const* x_t, const void* const* x_s,
                                float* const* kl, float* const* stats, int32_t part,
                                int32_t n_parts, void* ws, size_t ws_bytes, void* stream);
relkl_status relkl_bwd_qkv_part(int32_t n_rel, const relkl_desc* descs,
                                const void* const* x_t, const void* const* x_s,
                                const float* const* stats, const float* const* dkl,
                                float* const* dx_s, int32_t part, int32_t n_parts, void* ws,
                                size_t ws_bytes, void* stream);

/* Debug aid, host only (no GPU needed): replays the work decomposition of the
 * tensor-core kernels that a call with these descs would launch (the forward
 * when is_bwd is 0, else the backward the library picks; where that choice
 * depends on the SM count, see relkl_bwd_kernel_for, both candidates), for every part of
 * n_parts (n_parts = 1: the whole call), and checks that every (unit, row
 * block, column tile) the mask requires is visited exactly once over the
 * parts, that no other tile is, and that every visited tile's TMA row
 * coordinates lie inside the tensors.  The descs' device pointers are not
 * read: a desc with lengths or packed sequences needs HOST copies of them in
 * host_lengths[r] / host_cu_seqlens[r] (arrays indexed by relation; may be
 * NULL when no desc uses them).  RELKL_OK when the schedule is sound,
 * RELKL_ERR_INVALID with a one-line reason in why (if not NULL) otherwise,
 * RELKL_ERR_UNSUPPORTED for descs the tensor-core path does not take.        */
relkl_status relkl_check_schedule(int32_t n_rel, const relkl_desc* descs, int32_t is_bwd,
                                  int32_t n_parts, const int32_t* const* host_lengths,
                                  const int32_t* const* host_cu_seqlens, char* why,
                                  size_t why_len);

/* Synchronises `stream`, then reads the workspace record.  Returns RELKL_OK
 * or RELKL_ERR_TIMEOUT; *where (if not NULL) receives the code of the wait
 * that ran out (0 when none).                                                */
relkl_status relkl_get_device_error(const void* ws, void* stream, uint32_t* where);

/* Test hook: bound every device-side wait of later launches from this
 * process by `ns` nanoseconds (default 2e9).  0 makes any wait that is not
 * satisfied at once run out, which exercises the timeout path without a
 * hang.  Returns the previous value.                                         */
uint64_t relkl_set_wait_timeout_ns(uint64_t ns);

/* Human-readable name of a status code (static string).                     */
const char* relkl_status_string(relkl_status s);

/* The cudaError_t of the last failing CUDA call in this thread (0 if none). */
int32_t relkl_last_cuda_error(void);

/* Which kernel family a desc would run: 1 = tcgen05 tensor-core path,
 * 2 = CUDA-core float32 path, 0 = unsupported.  Validation-free.            */
int32_t relkl_path_for(const relkl_desc* desc);

/* Which backward kernel relkl_bwd_qkv would launch for these relations on a
 * GPU with n_sms SMs: 1 = CUDA-core float32 kernel, 2 = one 128-row block per
 * pass (tensor cores), 3 = adjacent row-block pairs (tensor cores, d = 128),
 * 4 = adjacent row-block pairs at d = 64; 0 for invalid descs or n_sms < 1.
 * A causal mask of 16 to 32 row blocks takes 2 or 3 by an estimate of their
 * times on n_sms SMs; fewer row blocks take 2, more take 3, a full mask 3.
 * Host only (no device access); validation as in relkl_check_schedule.     */
int32_t relkl_bwd_kernel_for(int32_t n_rel, const relkl_desc* descs, int32_t n_sms);

/* Forward that needs no workspace from the caller and allocates nothing.
 * The paper has no counterpart: this entry point exists for callers that
 * cannot obtain device memory for a workspace, such as a host framework that
 * plans every device buffer itself and hands a custom operation only its
 * inputs and outputs.
 *
 * Same arguments and results as relkl_fwd, without ws / ws_bytes; tensor-core
 * path only (bf16, d in {64, 128}; anything else returns
 * RELKL_ERR_UNSUPPORTED).  The kernel's scratch -- the record a device-side
 * wait writes when it runs out -- lives in a static device array of
 * RELKL_NOALLOC_SCRATCH_BYTES bytes inside the library, which every GPU that
 * loads the library keeps until the process exits.  A call whose scratch need
 * (relkl_workspace_bytes()) exceeded that size would be refused with
 * RELKL_ERR_WORKSPACE; the need does not grow with B, H or N.
 *  - The first call on a device looks up the array's device address (with
 *    that device current) and keeps it together with the device's current
 *    context; make that first call before any stream capture.  A later call
 *    that finds another context current on the device (after cudaDeviceReset,
 *    for example) looks the address up again.
 *  - The current device must be the one that owns the tensors and `stream`.
 *  - All calls share the one array, which keeps what the last call wrote;
 *    each call clears the record on its stream before its kernel starts.
 *    Calls that overlap on the GPU (other streams, other threads) race on the
 *    record.
 *  - A wait that ran out is recorded but cannot be read back through this
 *    entry point; use relkl_fwd with a workspace when that report matters.  */
#define RELKL_NOALLOC_SCRATCH_BYTES 256
relkl_status relkl_fwd_noalloc(const relkl_desc* desc, const void* x_t, const void* x_s,
                               float* kl, float* stats, void* stream);

/* ---------------------------------------------------------------------------
 * Chain rule from dX_s to the student's projection weights.
 *
 * LinearARD trains only the student's Q/K/V projections (pith.science
 * verdict page, pith_extraction.minor_comments); the student's relation
 * inputs are X_s = RoPE_s(H_s W_x) for x in {q, k} and X_s = H_s W_v for V,
 * with H_s [B, N, D] the student's hidden states and the heads of X laid side
 * by side per token.  The pages stop at the logit gradient; the two steps
 * below are the plain chain rule applied to relkl_bwd's dX_s.
 */

/* Rotate-half RoPE (RoFormer's rotary embedding in LLaMA's pairing): pair
 * (i, i + d/2) of token n rotates by pos(n) * base^(-2i/d), with
 * pos(n) = pos_offset + n * pos_scale (pos_scale = 1/s for positional
 * interpolation by s).                                                       */
typedef struct {
  double base;        /* > 1, e.g. 10000 */
  double pos_scale;   /* finite */
  double pos_offset;  /* finite */
  int32_t apply;      /* 1: the input carried RoPE (Q, K); 0: it did not (V) */
  int32_t reserved;   /* must be 0 */
} relkl_rope;

/* RoPE backward with the head/token transpose the weight gradient needs.
 *
 *   dx_pre[b, n, h, :] = R(pos(n))^T dx_post[b, h, n, :]
 *
 * where R is the rotation above (the identity when rope->apply == 0): for
 * each pair, (g_a, g_b) -> (g_a cos + g_b sin, g_b cos - g_a sin).  Angles are
 * formed in double precision, the rotation in float32.
 *   dx_post  : float [B, H, N, d] contiguous (relkl_bwd's dx_s), in.
 *   dx_pre   : [B, N, H, d] contiguous, out, overwritten; element type
 *              out_dtype (RELKL_BF16 to feed relkl_weight_grad, or RELKL_FP32).
 * d must be even and 2 <= d <= 512; B, H, N >= 0 (zero work is a no-op).
 * RELKL_ERR_INVALID for bad shapes, null pointers with work to do, a
 * non-finite or non-positive base, non-finite positions or reserved != 0.    */
relkl_status relkl_rope_bwd(int32_t B, int32_t H, int32_t N, int32_t d, const float* dx_post,
                            const relkl_rope* rope, int32_t out_dtype, void* dx_pre,
                            void* stream);

/* bfloat16 copy of a float32 array, for a caller that keeps dX_s in bf16:
 *
 *   dst[i] = src[i] rounded to the nearest bf16, ties to even
 *
 * (overflow rounds to infinity, NaN stays NaN).  The pages fix only that dX_s
 * is accumulated in float32 (the verdict page's Phase 2 streams it to the
 * student's Q/K/V); the copy is a storage convenience and runs as its own
 * HBM-bound pass, since a row of dX_s is complete only after every CTA that
 * adds into it has done so.  Issue it on the stream of the relkl_bwd call.
 *   src : float [n] (relkl_bwd's dx_s), in, 4-byte aligned.
 *   dst : bf16 [n], out, 2-byte aligned; must not overlap src.
 * n == 0 is a no-op (pointers unused).  RELKL_ERR_INVALID for n < 0, null or
 * misaligned pointers, or overlapping ranges.  Asynchronous on `stream`.     */
relkl_status relkl_cast_bf16(const float* src, void* dst, int64_t n, void* stream);

/* Weight gradient over the token rows:
 *
 *   dw[D, cols] = h[rows, D]^T dx_pre[rows, cols]
 *
 * (rows = B*N tokens, cols = heads * d), overwriting dw: one dense GEMM on
 * the tensor cores (the library's own tcgen05 kernel), bf16 operands, float32
 * accumulation and result.
 *   h      : bf16 [rows, D] row-major (the student's hidden states), in.
 *   dx_pre : bf16 [rows, cols] row-major (relkl_rope_bwd's output), in.
 *   dw     : float [D, cols] row-major, out.
 *   ws     : the workspace record of the other calls (bounded waits).
 * 1 <= rows <= 2^31 - 1, D >= 1, cols >= 1; pointers 16-byte aligned and
 * D, cols multiples of 8.  RELKL_ERR_INVALID otherwise.                      */
relkl_status relkl_weight_grad(int64_t rows, int32_t D, int32_t cols, const void* h,
                               const void* dx_pre, float* dw, void* ws, size_t ws_bytes,
                               void* stream);

#ifdef __cplusplus
}
#endif
#endif /* RELKL_H */
