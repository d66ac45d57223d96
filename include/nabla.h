/*
 * nabla.h -- C ABI of the NABLA (Neighborhood Adaptive Block-Level Attention) hot path
 * for NVIDIA B200 (sm_100a).
 *
 * The method (arXiv 2507.13546) as described by:
 *   [ZH-TS]  "NABLA: Neighborhood Adaptive Block-Level Attention", gist.science (Chinese
 *            edition), technical summary, section "Methodology".
 *   [LSD-2]  lsdiaocha.cn article on NABLA, section 2 ("core innovation": pooled
 *            scouting, CDF filtering, exact mapping back to N x N tiles, OR with STA).
 *   [LSD-4]  same article, section 4 ("technical principles").
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Tensors are dense, contiguous, row-major [B, H, S, D] with S = T * Hg * W tokens.
 *    Every call except nabla_reorder's source works in the reordered ("fractal") token
 *    order: block i = tokens [i*N, (i+1)*N), N = P*P, nb = S / N blocks.
 *  - bf16 tensors are IEEE bfloat16 stored as uint16.  All pointers are DEVICE pointers
 *    of the current CUDA device unless stated otherwise.
 *  - Ownership: the caller allocates and frees every buffer, workspaces included.  The
 *    library allocates no device memory and keeps no state between calls.
 *  - Asynchrony: every call only enqueues work on `stream` (a cudaStream_t; NULL = the
 *    legacy default stream) and returns.  All arguments are validated on the host
 *    first; when a call returns anything but NABLA_OK nothing has been enqueued.
 *  - Supported: P = 8 (N = 64), D in {64, 128}, Hg and W multiples of P, B*H >= 1,
 *    nb <= 16384.  Pointers to bf16/f32 tensors must be 16-byte aligned.
 *  - Device-side status: kernels that wait on hardware barriers bound every wait; on
 *    a timeout they record a code in the first 16 bytes of the call's workspace and
 *    return early.  nabla_read_device_status() reads it.
 */
#ifndef NABLA_H_
#define NABLA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *nabla_stream_t; /* identical to cudaStream_t */

typedef enum {
  NABLA_OK = 0,
  NABLA_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad shape, thr out of range */
  NABLA_ERR_UNSUPPORTED = 2,  /* valid request outside the supported set (D, P, nb) */
  NABLA_ERR_WORKSPACE = 3,    /* workspace pointer null or smaller than required */
  NABLA_ERR_CUDA = 4,         /* a CUDA runtime/driver call failed (launch, encode) */
  NABLA_ERR_DEVICE_CHECK = 5  /* a kernel recorded a device-side failure (bounded wait) */
} nabla_status;

typedef enum { NABLA_BF16 = 0, NABLA_F32 = 1, NABLA_F16 = 2 } nabla_dtype;

/* Token order of the attention tensors: the reordered order of nabla_reorder (blocks of
 * N = P*P consecutive tokens), or the natural order (t, h, w) of the latent, in which a
 * block is an 8 x 8 spatial patch of one frame, gathered by the kernel as it loads. */
typedef enum { NABLA_LAYOUT_REORDERED = 0, NABLA_LAYOUT_NATURAL = 1 } nabla_layout;

/* Problem shape.  S = T*Hg*W, N = P*P, nb = S/N.  Hg is the (padded) latent height. */
typedef struct {
  int32_t B, H, T, Hg, W, D, P;
} nabla_shape;

/* Static STA window in blocks on the (T, Hg/P, W/P) block grid; odd sizes, centred on
 * the query block and truncated at the grid edges.  {0,0,0} = no STA part. */
typedef struct {
  int32_t t, h, w;
} nabla_window;

/* Human-readable name of a status code (static string, never NULL). */
const char *nabla_status_string(nabla_status s);

/* ---------------------------------------------------------------------------------
 * Token reordering ("fractal flatten")                                       [ZH-TS]
 * [ZH-TS] Methodology, "token reordering": the tokens of each P x P spatial patch are
 * grouped into one contiguous run; frames stay in order.  Natural index
 * n = (t*Hg + h)*W + w maps to r = ((t*Hb + h/P)*Wb + w/P)*N + (h%P)*P + (w%P) with
 * Hb = Hg/P, Wb = W/P (row-major patches, row-major inside a patch).
 *
 * inverse == 0: dst[b,h,r,:] = src[b,h,n(r),:] (natural -> reordered).  src_dtype must be
 *   NABLA_BF16; dst_dtype NABLA_BF16 (copy) or NABLA_F16 (converted on the way, for the
 *   V operand of the attention kernels; exact for 2^-14 <= |x| <= 65504, larger
 *   magnitudes become +-inf).
 * inverse == 1: dst[b,h,n(r),:] = src[b,h,r,:] (reordered -> natural), src_dtype ==
 *   dst_dtype in {NABLA_BF16, NABLA_F16, NABLA_F32} (e.g. to restore an output O).
 * inverse == 2: dst[b,h,n,:] = src[b,h,n,:] converted (natural order kept), src_dtype
 *   NABLA_BF16, dst_dtype NABLA_BF16 or NABLA_F16: the fp16 V of the natural-layout
 *   training path (see nabla_attn_bwd), in one pass, optionally with pool_out.
 * Any other value of inverse: INVALID_ARG.
 * src, dst: [B,H,S,D] of those dtypes; must not overlap.  With inverse == 0 and pool_out
 *   given, dst may be NULL: only the block means are computed, src is read once and
 *   nothing is reordered (the natural-layout forward then reads src directly).
 * pool_out (nullable, with inverse == 0 or 2): fp64 [B,H,nb,D], the mean of each
 *   block's N reordered token vectors (sum in token order in fp64, then / N), i.e.
 *   the pooled Q or K of [ZH-TS] "downsampling", ready for nabla_build_mask.
 * Errors: INVALID_ARG (nulls, overlap, shape), UNSUPPORTED (D, P), CUDA (launch).
 * --------------------------------------------------------------------------------- */
nabla_status nabla_reorder(const void *src, nabla_dtype src_dtype, void *dst,
                           nabla_dtype dst_dtype, double *pool_out, nabla_shape s,
                           int32_t inverse, nabla_stream_t stream);

/* ---------------------------------------------------------------------------------
 * Adaptive mask construction                                         [ZH-TS, LSD-2]
 * [ZH-TS] Methodology, "adaptive mask construction": Q and K are average-pooled per
 * block of N tokens; full attention is computed on the pooled map (logits scaled by
 * `scale`); each row is softmax-normalised; per row the CDF is taken and the blocks
 * whose cumulative probability exceeds 1 - thr are kept; the binary mask defines which
 * N x N tiles are computed.  "Hybrid integration": M = M_nabla OR M_STA.
 * Ranking inside a row: probability descending, ties by lower block index.  Block j is
 * kept iff the probability mass ranked strictly before it is < thr (equivalently the
 * ascending CDF at j is > 1 - thr).  thr >= 1 keeps every block; thr == 0 keeps none,
 * so the result is the pure STA mask.  The decision is taken in fp64.
 *
 * q, k       : bf16 [B,H,S,D] in the token order given by layout (read only when the
 *              matching pool is NULL; given both without pools, the call pools them in
 *              the same pass that prepares its tensor-core operands).
 * q_pool,
 * k_pool     : nullable fp64 [B,H,nb,D] block means from nabla_reorder; when given, the
 *              call reads them instead of q / k (q / k may then be NULL).
 * thr        : in [0, 1]; scale > 0 (usually 1/sqrt(D)).  thr >= 1 keeps every block
 *              and thr <= 0 keeps none but the static window (pure STA); neither depends
 *              on the data, and q, k, q_pool and k_pool may then all be NULL.
 * sta        : window, {0,0,0} = off; each size must be 0 (all off) or odd >= 1.
 * mask_bits  : out uint32 [B,H,nb,ceil(nb/32)]; bit (j%32) of word j/32 of row i is 1
 *              iff query block i attends to key block j.  Padding bits are 0.
 * row_idx    : out, nullable, int32 [B,H,nb,nb]: kept key blocks of row i ascending in
 *              row_idx[..,i,0:row_cnt[..,i]]; the rest is not written.
 * row_cnt    : out, nullable, int32 [B,H,nb]: kept blocks per row (required when row_idx
 *              is given; may be given alone for the counts only).
 * col_idx,
 * col_cnt    : out, nullable: the transpose (query blocks that keep key block j,
 *              ascending), same shapes and the same rule; used by the backward pass.
 * layout     : token order of q and k: NABLA_LAYOUT_REORDERED or NABLA_LAYOUT_NATURAL
 *              (each 8 x 8 patch of a frame gathered as it is read); ignored for pools.
 * workspace  : >= nabla_mask_workspace_bytes(s) bytes, 256-byte aligned.
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA.
 * --------------------------------------------------------------------------------- */
size_t nabla_mask_workspace_bytes(nabla_shape s);
nabla_status nabla_build_mask(const void *q, const void *k, const double *q_pool,
                              const double *k_pool, nabla_shape s, double thr,
                              nabla_window sta, double scale, uint32_t *mask_bits,
                              int32_t *row_idx, int32_t *row_cnt, int32_t *col_idx,
                              int32_t *col_cnt, nabla_layout layout, void *workspace,
                              size_t workspace_bytes, nabla_stream_t stream);

/* ---------------------------------------------------------------------------------
 * Several thresholds on one pooled map ("mask reuse").
 * The pages tune thr per model (lsdiaocha.cn article, section 3: thr 0.2-0.9 swept
 * against quality and speed; gist.science, Chinese edition, "Experimental results":
 * sparsity and quality per thr); this call builds the masks of n_thr thresholds from one
 * computation of the pooled means and the pooled logits, the per-row cut (and its fp64
 * check) running once per threshold.  Each mask is identical, bit for bit, to the one
 * nabla_build_mask returns for that thr with the same inputs.
 *
 * q, k, q_pool,
 * k_pool, sta,
 * scale      : as nabla_build_mask (q, k and the pools may all be NULL when every thr is
 *              <= 0 or >= 1).
 * thrs       : host array of n_thr values in [0, 1]; 1 <= n_thr <= 64.
 * mask_bits  : out uint32 [n_thr][B,H,nb,ceil(nb/32)]: mask t at offset
 *              t * B*H*nb*ceil(nb/32) words.
 * row_cnt    : out, nullable, int32 [n_thr][B,H,nb]: kept blocks per row of each mask
 *              (row lists: nabla_mask_lists on a mask).
 * workspace  : >= nabla_mask_workspace_bytes(s) bytes, 256-byte aligned (reused by the
 *              thresholds one after another).
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA.
 * --------------------------------------------------------------------------------- */
nabla_status nabla_build_mask_sweep(const void *q, const void *k, const double *q_pool,
                                    const double *k_pool, nabla_shape s, const double *thrs,
                                    int n_thr, nabla_window sta, double scale,
                                    uint32_t *mask_bits, int32_t *row_cnt, void *workspace,
                                    size_t workspace_bytes, nabla_stream_t stream);

/* Row and column lists of an arbitrary block mask (e.g. a dense all-ones mask for the
 * dense comparator, or a caller-made mask).  Same layouts as nabla_build_mask; any of
 * the two list pairs may be NULL.  Padding bits of mask_bits are ignored. */
nabla_status nabla_mask_lists(const uint32_t *mask_bits, nabla_shape s, int32_t *row_idx,
                              int32_t *row_cnt, int32_t *col_idx, int32_t *col_cnt,
                              nabla_stream_t stream);

/* ---------------------------------------------------------------------------------
 * Block-sparse attention forward                                    [ZH-TS, LSD-2]
 * [ZH-TS] Methodology, "expansion" + FlexAttention: exact softmax attention restricted
 * to the kept N x N tiles.  For token row r of query block i:
 *   O_r = sum_c softmax_c(scale * Q_r . K_c) V_c over tokens c of the kept key blocks
 *   of row i;  LSE_r = ln sum_c exp(scale * Q_r . K_c).
 * A row with no kept block gives O = 0 and LSE = -inf.
 *
 * q, k       : bf16 [B,H,S,D] in the token order given by layout.
 * v, v_dtype : [B,H,S,D] in that order, NABLA_BF16 or NABLA_F16.  With fp16 V the
 *              probabilities P enter the PV product as fp16 (11-bit significand)
 *              instead of bf16 (8-bit): about 8x smaller output error.
 * mask_bits  : the block mask as from nabla_build_mask (padding bits are ignored).
 * o          : out [B,H,S,D], bf16 or f32 per o_dtype.   lse: out f32 [B,H,S] (natural
 *              log; nullable when not needed).  Both in the token order given by layout.
 * layout     : NABLA_LAYOUT_REORDERED, or NABLA_LAYOUT_NATURAL: q, k, v, o and lse in
 *              the natural order of the latent, nothing reordered beforehand (the
 *              fractal flatten of [ZH-TS] "token reordering" is done by the loads; the
 *              mask and block indices are unchanged).
 * workspace  : >= nabla_fwd_workspace_bytes(s) bytes (tile schedule + status word).
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA.
 * --------------------------------------------------------------------------------- */
size_t nabla_fwd_workspace_bytes(nabla_shape s);
nabla_status nabla_attn_fwd(const void *q, const void *k, const void *v, nabla_dtype v_dtype,
                            const uint32_t *mask_bits, nabla_shape s, float scale, void *o,
                            nabla_dtype o_dtype, float *lse, nabla_layout layout,
                            void *workspace, size_t workspace_bytes, nabla_stream_t stream);

/* ---------------------------------------------------------------------------------
 * Block-sparse attention backward (mask constant)                   [ZH-TS, LSD-2]
 * The pages credit NABLA with faster training as well as inference; the binary mask
 * has no gradient, so gradients flow through attention on the kept tiles only:
 *   P = exp(scale*Q K^T - LSE), Dr = rowsum(dO * O), dS = P * (dO V^T - Dr),
 *   dV = P^T dO, dK = scale * dS^T Q, dQ = scale * dS K   (kept tiles only).
 * q, k, dout: bf16 [B,H,S,D]; v: bf16 or fp16 (v_dtype); o: forward output (o_dtype);
 * lse: forward LSE.  The MMAs run on fp16 copies of Q, K, V and dO made in the
 * workspace (P and dS rounded to fp16): inputs must satisfy |x| <= 65504, otherwise the
 * device status word reports it (0x201); an fp16 V is checked for infinite or NaN
 * values when it is gathered (natural layout) and used as given in the reordered layout.
 * row_* and col_* lists from nabla_build_mask / nabla_mask_lists.
 * dq, dk, dv : out f32 [B,H,S,D] (fully overwritten; deterministic, no atomics).
 * layout     : token order of q, k, v, o, dout, lse, dq, dk and dv: NABLA_LAYOUT_REORDERED,
 *              or NABLA_LAYOUT_NATURAL (the latent's natural order, as the natural-layout
 *              forward reads and writes them; the fractal flatten of [ZH-TS] "token
 *              reordering" is done by the backward's own gather into its fp16 copies, and
 *              the gradients are written at the tokens' natural indices).
 * workspace  : >= nabla_bwd_workspace_bytes(s) bytes.
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, CUDA.
 * --------------------------------------------------------------------------------- */
size_t nabla_bwd_workspace_bytes(nabla_shape s);
nabla_status nabla_attn_bwd(const void *q, const void *k, const void *v, nabla_dtype v_dtype,
                            const void *o,
                            nabla_dtype o_dtype, const void *dout, const float *lse,
                            const int32_t *row_idx, const int32_t *row_cnt,
                            const int32_t *col_idx, const int32_t *col_cnt, nabla_shape s,
                            float scale, float *dq, float *dk, float *dv, nabla_layout layout,
                            void *workspace, size_t workspace_bytes, nabla_stream_t stream);

/* ---------------------------------------------------------------------------------
 * Allocation-free forward (no counterpart in the NABLA pages; a library convenience).
 * For callers that cannot call cudaMalloc where they run attention -- e.g. a host
 * framework that owns all device memory through its own pool and forbids driver
 * allocations on its hot path, or a latency-critical loop that must not pay for an
 * allocation -- and so cannot provide nabla_attn_fwd's workspace.  Same arguments and
 * results as nabla_attn_fwd without the workspace: the workspace is a fixed 1 MiB
 * array in the library's own device memory (every GPU that loads the library holds it
 * until the process exits).  Problems whose workspace (nabla_fwd_workspace_bytes)
 * exceeds 1 MiB are rejected with NABLA_ERR_UNSUPPORTED before anything is enqueued
 * (the 720p-like 40-head problem needs about 200 KB).  The first call on a device looks
 * up that array's device address (cudaGetSymbolAddress, with the device current); make
 * that first call before any stream capture.  A re-created context (cudaDeviceReset)
 * is detected by its context id and the lookup is repeated on the next call.  The call
 * allocates nothing.  All calls share the one array, which keeps the last call's
 * contents (each call clears what must start at zero): calls that can overlap on the
 * GPU (different streams, or several host threads on one device) race on it and must
 * be serialised by the caller.  The device status word of the last call on the current
 * device (a bounded wait that gave up leaves O incomplete) is read, and cleared, with
 * nabla_attn_fwd_noalloc_status().
 * --------------------------------------------------------------------------------- */
nabla_status nabla_attn_fwd_noalloc(const void *q, const void *k, const void *v,
                                    nabla_dtype v_dtype, const uint32_t *mask_bits, nabla_shape s,
                                    float scale, void *o, nabla_dtype o_dtype, float *lse,
                                    nabla_layout layout, nabla_stream_t stream);

/* Status of the last nabla_attn_fwd_noalloc call on the current device: waits for
 * `stream`, then behaves as nabla_read_device_status on the fixed array (NABLA_OK, or
 * NABLA_ERR_DEVICE_CHECK with the code in `code`, nullable; the word is then cleared).
 * Allocates nothing.  Errors: CUDA. */
nabla_status nabla_attn_fwd_noalloc_status(uint32_t *code, nabla_stream_t stream);

/* Failure-path self-test (no counterpart in the pages).  Enqueues one warp that waits,
 * through the same bounded barrier wait as every kernel of the library, for a barrier
 * phase that nothing completes.  The wait gives up after its limit (about 2 s), records
 * the code 0x10A in the status word of `workspace` (>= 256 bytes, 256-byte aligned) and
 * the kernel returns: nabla_read_device_status() then reports NABLA_ERR_DEVICE_CHECK
 * with code 0x10A, and the stream and context stay usable.  No trap, fault or hang.
 * Errors: WORKSPACE, CUDA. */
nabla_status nabla_selftest_bounded_wait(void *workspace, size_t workspace_bytes,
                                         nabla_stream_t stream);

/* Reads (synchronously on `stream`) the device status word that the kernels of the
 * last call on `workspace` recorded: 0 = fine, otherwise a code naming the barrier
 * wait that gave up.  Returns NABLA_ERR_DEVICE_CHECK when the word is non-zero, and
 * clears it.  `code` (nullable) receives the raw word. */
nabla_status nabla_read_device_status(void *workspace, uint32_t *code,
                                      nabla_stream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* NABLA_H_ */
