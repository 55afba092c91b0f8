/*
 * fp8mlp -- fused FP8 ReLU^2 MLP block for NVIDIA B200 (sm_100a).
 *
 * C ABI.  Plain pointers and sizes; no C++ or framework types.
 *
 * The block (one transformer MLP, d -> h -> d):
 *     pre  = x . W1^T                       (never stored)
 *     post = relu(pre)^2                    BF16, kept for the backward
 *     q    = e4m3(post * s_t)               FP8 copy under the delayed scale s_t
 *     out  = (q . W2q_t^T) * s_t^-1 * s_w^-1   FP8 down-projection
 * and its BF16 backward, which rebuilds relu(pre) as sqrt(post).
 *
 * Sources (page title, section):
 *   "NanoGPT Speedrun (Track 1)", section "Changes vs Record #83", item 4:
 *       the MLP kernel stores only post = relu(pre)^2; the backward rebuilds
 *       relu(pre) = sqrt(post) in-kernel.
 *   same page, "From Unoptimized / Approach", item 5: FP8 e4m3 MLP GEMMs in
 *       the training forward, BF16 backward, BF16 at evaluation.
 *   "A Retrospective on Our World Records", Modded-NanoGPT Main Track: the
 *       fused up-projection writes BF16 post, an FP8 copy and a tiny
 *       partial-amax tensor while post sits in registers; the scale of step t
 *       comes from amax(t-1) times a safety margin; a transposed FP8 cache of
 *       W2 is refreshed after optimizer updates; the BF16 backward is left
 *       unchanged.  Same page, "A few implementation notes": an exact,
 *       non-delayed W2 refresh is viable.
 *
 * Layouts (all row-major, element strides implied by the sizes):
 *   x [M,d] bf16      W1 [h,d] bf16 (nn.Linear(d,h).weight)   W2 [h,d] bf16
 *   post [M,h] bf16   post_fp8 [M,h] e4m3   W2q_t [d,h] e4m3 (W2 transposed)
 *   out [M,d] bf16    dOut [M,d] bf16   dPre [M,h] bf16   dX [M,d] bf16
 *   dW1 [h,d] fp32    dW2 [h,d] fp32
 * BF16 and e4m3 tensors are passed as raw bit patterns (uint16 / uint8).
 *
 * Conventions shared by every entry point:
 *   - Ownership: the caller owns and allocates every buffer; the library
 *     allocates no device memory and keeps no pointer after the call.
 *   - Device pointers must be 16-byte aligned (TMA).  Tensors are dense.
 *   - Shapes: M >= 0 is arbitrary; d and h must be multiples of 16 and at
 *     least 16.  M = 0 returns FP8MLP_OK and writes nothing, except the
 *     results an empty batch defines: zero weight gradients (fp8mlp_bwd_dw,
 *     fp8mlp_mlp_bwd, fp8mlp_linear_bwd) and zero cross-entropy totals
 *     (fp8mlp_ce_fwd, fp8mlp_ce_fwd_fp8).
 *   - Asynchrony: every call enqueues work on `stream` (NULL = the legacy
 *     default stream) of the current device and returns without waiting.
 *     No call reads device data back to the host, except
 *     fp8mlp_get_device_status.
 *   - Errors: argument checks run on the host before any CUDA call and
 *     return FP8MLP_ERR_INVALID_ARG / FP8MLP_ERR_UNSUPPORTED_SHAPE with
 *     nothing enqueued.  FP8MLP_ERR_NO_DEVICE: the current device is not a
 *     compute-capability 10.0 GPU (or there is none).  FP8MLP_ERR_CUDA: a
 *     CUDA call failed (fp8mlp_last_error_detail() says which).  Faults
 *     found on the device (a bounded wait that gave up) are reported through
 *     the device status word, read with fp8mlp_get_device_status.
 *     There is no CPU fallback.
 */
#ifndef FP8MLP_H
#define FP8MLP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* fp8mlp_stream_t; /* same type as cudaStream_t */

/* return codes */
#define FP8MLP_OK 0
#define FP8MLP_ERR_INVALID_ARG 1
#define FP8MLP_ERR_UNSUPPORTED_SHAPE 2
#define FP8MLP_ERR_CUDA 3
#define FP8MLP_ERR_TIMEOUT 4
#define FP8MLP_ERR_NO_DEVICE 5

/* device status word bits (fp8mlp_get_device_status) */
#define FP8MLP_STATUS_TIMEOUT 1u          /* a kernel's bounded wait gave up */
#define FP8MLP_STATUS_NONFINITE_AMAX 2u   /* amax was NaN/inf: scale kept */
#define FP8MLP_STATUS_W2_DEGENERATE 4u    /* max|W2| was 0 or not finite: s_w = 1 */

/* Largest finite e4m3 value; the delayed scale maps margin * amax onto it. */
#define FP8MLP_E4M3_MAX 448.0f

/*
 * Delayed-scaling state, device-resident, caller-allocated (32 bytes,
 * 16-byte aligned).  "A Retrospective on Our World Records", Main Track: the
 * FP8 activation scale of step t is derived from the amax measured at step
 * t-1 multiplied by a safety margin; no rolling window.
 * The caller may copy it out and back in to checkpoint / resume.
 */
typedef struct fp8mlp_scale_state {
  float amax_prev; /* A_{t-1}: amax of post reduced at the last update       */
  float scale;     /* s_t = 448 / (margin * A_{t-1}), used to quantise post  */
  float scale_inv; /* 1 / s_t (fp32, round-to-nearest)                       */
  float margin;    /* safety margin (> 0)                                     */
  int32_t step;    /* number of updates applied                              */
  int32_t flags;   /* FP8MLP_STATE_KEPT_SCALE: last update kept the scale    */
  int32_t pad[2];
} fp8mlp_scale_state;

#define FP8MLP_STATE_KEPT_SCALE 1

/* mlp_fwd / up_proj_fused flags */
#define FP8MLP_FWD_EVAL_BF16 1 /* evaluation: BF16 down-projection from post and W2; no FP8 copy */
#define FP8MLP_FWD_CALIBRATE 2 /* write post and partial amax only (step 0: no amax(t-1) yet)   */

/* ------------------------------------------------------------------------
 * Forward
 * ------------------------------------------------------------------------ */

/*
 * Fused up-projection ("A Retrospective on Our World Records", Main Track:
 * while the up-projection has the post-activation values in registers it
 * writes the BF16 tensor for the backward, emits the FP8 version and
 * accumulates a tiny partial-amax tensor; "NanoGPT Speedrun (Track 1)",
 * Changes vs Record #83, item 4: only post = relu(pre)^2 is stored).
 *
 *   post[m,i]     = bf16( fp32(r*r) ),  r = max(fp32(x[m,:] . W1[i,:]), 0)
 *   post_fp8[m,i] = e4m3_satfinite( fp32(post[m,i] * st->scale) )
 *   partial_amax  = max of post over blocks of block_rows x block_cols
 *                   (32 x 64), fp32, row-major [row_blocks][col_blocks]
 *                   with the sizes of fp8mlp_partial_amax_shape
 *                   (8*ceil(M/256) x 4*ceil(h/256)); blocks that lie
 *                   wholly past row M or column h hold 0
 *   pre_debug     = optional fp32 pre [M,h] (NULL to skip; slow, for tests)
 *
 * st->scale is read on the device; the host never waits for it.
 * flags: FP8MLP_FWD_CALIBRATE or FP8MLP_FWD_EVAL_BF16 skip post_fp8 (may be
 * NULL then).  post and partial_amax are always written.
 */
int fp8mlp_up_proj_fused(int M, int d, int h, const uint16_t* x, const uint16_t* W1,
                         const fp8mlp_scale_state* st, uint16_t* post, uint8_t* post_fp8,
                         float* partial_amax, float* pre_debug, int flags, fp8mlp_stream_t stream);

/*
 * FP8 scaled down-projection ("A Retrospective on Our World Records", Main
 * Track: the down-projection runs as an FP8 scaled matmul on both operands,
 * against the transposed FP8 cache of W2):
 *   out[m,j] = bf16( fp32( sum_i q[m,i] * W2q_t[j,i] ) * fp32(st->scale_inv * w2_scale_inv[0]) )
 * with fp32 accumulation.  post_fp8 [M,h], W2q_t [d,h].
 */
int fp8mlp_down_proj_fp8(int M, int d, int h, const uint8_t* post_fp8, const uint8_t* W2q_t,
                         const float* w2_scale_inv, const fp8mlp_scale_state* st, uint16_t* out,
                         fp8mlp_stream_t stream);

/*
 * BF16 down-projection for evaluation ("NanoGPT Speedrun (Track 1)", From
 * Unoptimized, item 5: BF16 at eval):  out = bf16(post . W2), W2 [h,d].
 */
int fp8mlp_down_proj_bf16(int M, int d, int h, const uint16_t* post, const uint16_t* W2, uint16_t* out,
                          fp8mlp_stream_t stream);

/*
 * Whole forward: fp8mlp_up_proj_fused, then
 *   default flags:          fp8mlp_down_proj_fp8 (W2q_t, w2_scale_inv used; W2 may be NULL)
 *   FP8MLP_FWD_EVAL_BF16:   fp8mlp_down_proj_bf16 (W2 used; W2q_t, w2_scale_inv, post_fp8 may be NULL)
 *   FP8MLP_FWD_CALIBRATE:   no down-projection (out, W2*, post_fp8 may be NULL)
 */
int fp8mlp_mlp_fwd(int M, int d, int h, const uint16_t* x, const uint16_t* W1, const uint8_t* W2q_t,
                   const float* w2_scale_inv, const uint16_t* W2, const fp8mlp_scale_state* st, uint16_t* post,
                   uint8_t* post_fp8, float* partial_amax, uint16_t* out, float* pre_debug, int flags,
                   fp8mlp_stream_t stream);

/* ------------------------------------------------------------------------
 * FP8 up-projection ("NanoGPT Speedrun (Track 1)", From Unoptimized, item 5:
 * the MLP GEMMs in e4m3 in the training forward, BF16 backward).  x and W1
 * enter the up-projection as e4m3 copies: x under its own delayed scale s_x
 * (the same recurrence as post's, from max |x| of the previous step), W1
 * under an exact cache scale.  The backward keeps the BF16 x and W1.
 * ------------------------------------------------------------------------ */

/* x_fp8 = e4m3_satfinite(fp32(x * st_x->scale)), x [M,d] bf16 -> x_fp8 [M,d];
 * partial_amax_x[b] = max |x| over elements [8192 b, 8192 b + 8192) of the
 * flat x (fp8mlp_x_partial_amax_count entries; reduce them with
 * fp8mlp_amax_reduce_update_scale into st_x for the next step). */
int fp8mlp_quantize_x(int M, int d, const uint16_t* x, const fp8mlp_scale_state* st_x, uint8_t* x_fp8,
                      float* partial_amax_x, fp8mlp_stream_t stream);
/* Entries of fp8mlp_quantize_x's partial_amax_x: ceil(M*d / 8192). */
int fp8mlp_x_partial_amax_count(int M, int d);

/* Exact FP8 copy of W1 (not transposed; W1 [h,d] is K-major for the
 * up-projection): s_w1 = fp32(448 / max|W1|) (1 if 0 or not finite),
 * W1q[i,k] = e4m3_satfinite(fp32(W1[i,k] * s_w1)), w1_scale_inv[0] = 1/s_w1.
 * workspace: fp8mlp_workspace_size(0,d,h) bytes, as for the W2 cache. */
int fp8mlp_w1_fp8_cache_refresh(int h, int d, const uint16_t* W1, uint8_t* W1q, float* w1_scale_inv,
                                void* workspace, fp8mlp_stream_t stream);

/* fp8mlp_up_proj_fused on e4m3 inputs: the accumulator is dequantised in the
 * epilogue, pre = fp32(acc * fp32(st_x->scale_inv * w1_scale_inv[0])), then
 * post, the FP8 copy of post and the partial amax exactly as in
 * fp8mlp_up_proj_fused.  x_fp8 [M,d], W1q [h,d] e4m3. */
int fp8mlp_up_proj_fused_fp8(int M, int d, int h, const uint8_t* x_fp8, const uint8_t* W1q,
                             const float* w1_scale_inv, const fp8mlp_scale_state* st_x, const fp8mlp_scale_state* st,
                             uint16_t* post, uint8_t* post_fp8, float* partial_amax, float* pre_debug, int flags,
                             fp8mlp_stream_t stream);

/* ------------------------------------------------------------------------
 * Generic FP8 linear layer y = x . W^T (nn.Linear(K, N).weight = W [N,K]) on
 * the same kernels: the attention QKV / output projections that "NanoGPT
 * Speedrun (Track 1)", Changes vs Record #83, item 1 runs in e4m3 in the
 * forward (BF16 backward, BF16 at eval).  x_fp8 from fp8mlp_quantize_x (its
 * own delayed scale st_x), Wq from fp8mlp_weight_fp8_cache_refresh.
 * ------------------------------------------------------------------------ */

/* y[m,n] = bf16( fp32( sum_k x_fp8[m,k] Wq[n,k] ) * fp32(st_x->scale_inv * w_scale_inv[0]) ),
 * x_fp8 [M,K] e4m3, Wq [N,K] e4m3, y [M,N] bf16.  K and N multiples of 16. */
int fp8mlp_linear_fwd_fp8(int M, int K, int N, const uint8_t* x_fp8, const uint8_t* Wq, const float* w_scale_inv,
                          const fp8mlp_scale_state* st_x, uint16_t* y, fp8mlp_stream_t stream);

/* Exact FP8 copy of a weight W [N,K] (= fp8mlp_w1_fp8_cache_refresh with
 * N, K for h, d). */
int fp8mlp_weight_fp8_cache_refresh(int N, int K, const uint16_t* W, uint8_t* Wq, float* w_scale_inv,
                                    void* workspace, fp8mlp_stream_t stream);

/* BF16 backward of the linear layer: dX = bf16(dY . W) [M,K] (skipped when
 * dX is NULL) and dW = fp32(dY^T . x) [N,K].  x [M,K], W [N,K], dY [M,N].
 * The dW GEMM, which does not depend on dX, starts while the dX GEMM
 * finishes.  flags: 0, or FP8MLP_LAUNCH_OVERLAP_PREVIOUS for the first GEMM
 * launched (dX, or dW when dX is NULL), with the meaning given at
 * fp8mlp_bwd_dpre.
 * workspace: NULL, or fp8mlp_linear_bwd_workspace_size(M, K, N) bytes
 * (16-byte aligned, no initial contents needed; calls that may overlap on
 * the GPU need workspaces of their own).  When dW has so few
 * 256x256 output tiles that they would keep at most half of the CTA pairs
 * busy (768 -> 2304: 27 tiles for 74 pairs), the tokens are split in two at
 * a multiple of 64 rows: the first part accumulates into dW, the second
 * into the workspace in the same launch, and a last kernel adds the
 * workspace to dW (dW = fp32(first part) + fp32(second part), a fixed
 * order).  With NULL, or when the split does not apply, the workspace is
 * not touched. */
int fp8mlp_linear_bwd(int M, int K, int N, const uint16_t* x, const uint16_t* W, const uint16_t* dY, uint16_t* dX,
                      float* dW, void* workspace, int flags, fp8mlp_stream_t stream);

/* Bytes of the optional workspace of fp8mlp_linear_bwd: 4*N*K when M >= 128,
 * else 0. */
size_t fp8mlp_linear_bwd_workspace_size(int M, int K, int N);

/* ------------------------------------------------------------------------
 * Softcapped cross-entropy over a language-model head, without [M,V] logits.
 * "NanoGPT Speedrun (Track 1)", From Unoptimized / Approach, item 5: a fused
 * softcapped cross-entropy that never materialises the [M,V] logits in fp32;
 * "A Retrospective on Our World Records", SlowRun section: one LM head scored
 * against several successive targets at each position through an FP8
 * soft-capped cross-entropy kernel; Changes vs Record #83, item 1: FP8 in the
 * LM head.
 *
 *   y = x . W^T          x [M,d] bf16, W [V,d] bf16  (or their e4m3 copies:
 *                        y = fp32(acc) * fp32(st_x->scale_inv * w_scale_inv[0]))
 *   z = c tanh(y / c)    the softcap, 0 < c <= 40
 *   lse[m] = logsumexp_v z[m,v]
 *   loss_m = sum over t < T with 0 <= targets[m,t] < V of w_t (lse[m] - z[m, targets[m,t]])
 *   loss[0] = sum_m loss_m, loss[1] = sum of the valid weights,
 *   loss[2] = loss[0] / loss[1] (0 when no target is valid)
 *
 * targets [M,T] int32 row-major, 1 <= T <= 4; a target outside [0,V) is
 * ignored.  target_weights: HOST array of T floats, or NULL for all 1.
 * V and d multiples of 16 (pad the vocabulary; padded columns take part in
 * the softmax).  The cap bounds |z| by c, so exp(z - c) never overflows and
 * never falls below e^-80: no running maximum is kept.  lse [M] and loss[3]
 * fp32 (caller-owned, 4-byte aligned); row_loss [M] fp32 or NULL.  The
 * reductions run in double in a fixed order (deterministic).
 * ------------------------------------------------------------------------ */
#define FP8MLP_CE_SUM 0  /* the backward differentiates loss[0] */
#define FP8MLP_CE_MEAN 1 /* the backward differentiates loss[2]  */

/* Bytes of workspace (16-byte aligned, caller-owned, no initial contents)
 * that fp8mlp_ce_fwd / fp8mlp_ce_fwd_fp8 need for M rows, V columns and T
 * targets: per-row partial sums over 128-column groups, z at the targets and
 * per-block sums.  0 for M = 0. */
size_t fp8mlp_ce_workspace_size(int M, int V, int T);

/* Forward on BF16 x and W: one GEMM whose epilogue softcaps and sums the
 * logits tile by tile (nothing [M,V] is written), then two small passes. */
int fp8mlp_ce_fwd(int M, int d, int V, int T, const uint16_t* x, const uint16_t* W, const int32_t* targets,
                  const float* target_weights, float softcap, float* lse, float* row_loss, float* loss,
                  void* workspace, fp8mlp_stream_t stream);

/* Forward on the e4m3 copies: x_fp8 [M,d] from fp8mlp_quantize_x under st_x,
 * Wq [V,d] from fp8mlp_weight_fp8_cache_refresh (scale 1 / w_scale_inv[0]). */
int fp8mlp_ce_fwd_fp8(int M, int d, int V, int T, const uint8_t* x_fp8, const fp8mlp_scale_state* st_x,
                      const uint8_t* Wq, const float* w_scale_inv, const int32_t* targets,
                      const float* target_weights, float softcap, float* lse, float* row_loss, float* loss,
                      void* workspace, fp8mlp_stream_t stream);

/* Gradient of the loss with respect to the logits, recomputing y exactly as
 * the forward did (same kernel, same precision):
 *   dlogits[m,v] = bf16( g (W_m softmax(z_m)_v - sum_t w_t [v == targets[m,t]]) (1 - (z/c)^2) )
 * W_m = sum of row m's valid weights; g = dloss[0] (NULL: 1), divided by
 * loss[1] when reduction is FP8MLP_CE_MEAN (0 when loss[1] is 0).  lse and
 * loss from the forward; dlogits [M,V] bf16.  The BF16 backward through the
 * head is then fp8mlp_linear_bwd(M, d, V, x, W, dlogits, dX, dW, 0, stream). */
int fp8mlp_ce_bwd_dlogits(int M, int d, int V, int T, const uint16_t* x, const uint16_t* W, const int32_t* targets,
                          const float* target_weights, float softcap, const float* lse, const float* loss,
                          const float* dloss, int reduction, uint16_t* dlogits, fp8mlp_stream_t stream);

/* fp8mlp_ce_bwd_dlogits for a forward run on the e4m3 copies. */
int fp8mlp_ce_bwd_dlogits_fp8(int M, int d, int V, int T, const uint8_t* x_fp8, const fp8mlp_scale_state* st_x,
                              const uint8_t* Wq, const float* w_scale_inv, const int32_t* targets,
                              const float* target_weights, float softcap, const float* lse, const float* loss,
                              const float* dloss, int reduction, uint16_t* dlogits, fp8mlp_stream_t stream);

/* Number of row blocks and column blocks of the partial-amax tensor for an
 * [M,h] post, and the block size in rows / columns.  Returns FP8MLP_OK. */
int fp8mlp_partial_amax_shape(int M, int h, int* row_blocks, int* col_blocks, int* block_rows,
                              int* block_cols);
/* Number of fp32 entries of that tensor, row_blocks * col_blocks: the n to
 * pass to fp8mlp_amax_reduce_update_scale and the length of the buffer to
 * allocate for partial_amax (0 for negative sizes). */
int fp8mlp_partial_amax_count(int M, int h);

/* ------------------------------------------------------------------------
 * Delayed scaling and the W2 cache
 * ------------------------------------------------------------------------ */

/* Initialise a state on the device: amax_prev 0, scale = initial_scale,
 * scale_inv = 1/initial_scale, margin, step 0, flags 0.  margin > 0 and
 * initial_scale > 0 (finite), else FP8MLP_ERR_INVALID_ARG. */
int fp8mlp_scale_state_init(fp8mlp_scale_state* st, float margin, float initial_scale,
                            fp8mlp_stream_t stream);

/*
 * Reduce the partial amax of this step and derive the next step's scale
 * ("A Retrospective on Our World Records", Main Track: "we only reduce those
 * partial amax values later"; scale of step t from amax(t-1) times a margin):
 *   A = max(partial_amax[0..n)),   st->amax_prev = A,   st->step += 1
 *   if A finite and > 0:  st->scale = fp32(448 / fp32(margin * A)),
 *                         st->scale_inv = fp32(1 / st->scale), flag cleared
 *   else (0, NaN, inf):   scale kept, FP8MLP_STATE_KEPT_SCALE set
 *                         (NaN/inf also set FP8MLP_STATUS_NONFINITE_AMAX)
 * n >= 0 (n = 0 gives A = 0).  One CTA; no host synchronisation.
 */
int fp8mlp_amax_reduce_update_scale(const float* partial_amax, int n, fp8mlp_scale_state* st,
                                    fp8mlp_stream_t stream);

/*
 * Refresh the transposed FP8 cache of W2 ("A Retrospective on Our World
 * Records", Main Track: transposed FP8 cache of W2 refreshed after optimizer
 * updates; implementation notes: exact, non-delayed refresh is viable):
 *   s_w = fp32(448 / max|W2|)   (1 if max|W2| is 0 or not finite)
 *   W2q_t[j,i] = e4m3_satfinite( fp32(W2[i,j] * s_w) ),  w2_scale_inv[0] = fp32(1/s_w)
 * W2 [h,d] bf16, W2q_t [d,h] e4m3.  workspace: at least
 * fp8mlp_workspace_size(0,d,h) bytes of caller-owned device memory (one
 * partial maximum per 8192 elements of W2; no initial contents needed).
 */
int fp8mlp_w2_fp8_cache_refresh(int h, int d, const uint16_t* W2, uint8_t* W2q_t, float* w2_scale_inv,
                                void* workspace, fp8mlp_stream_t stream);

/*
 * The same refresh for callers that cannot allocate device memory.  The
 * pages describe no such call: this entry point exists for integration only.  Some
 * callers cannot provide a workspace: code inside another framework's
 * operator hook that owns every device allocation through its own pool and
 * exposes none to the op, or a runtime that forbids cudaMalloc/cudaFree on its
 * hot path because they can synchronise the whole device.  It launches the
 * same two kernels as fp8mlp_w2_fp8_cache_refresh, so the results are the
 * same bits.
 *   - Scratch: a fixed 8 KiB device array owned by the library (2048 partial
 *     maxima, one per 8192 elements of W2); every GPU that loads the library
 *     holds it until the process exits.  h*d above 16,777,216 elements is
 *     rejected with FP8MLP_ERR_UNSUPPORTED_SHAPE (use the workspace version).
 *   - The first call on a device looks up the array's device address with
 *     that device current; make that first call before any stream capture.
 *   - All calls share the array and it keeps the last call's contents; no
 *     entry needs to start at zero (each call writes every entry it reads).
 *     Calls that overlap on the GPU (other streams, other host threads) race.
 *   - No cudaMalloc, cudaFree or other allocating call is made.
 */
int fp8mlp_w2_fp8_cache_refresh_noalloc(int h, int d, const uint16_t* W2, uint8_t* W2q_t, float* w2_scale_inv,
                                        fp8mlp_stream_t stream);

/* Device workspace in bytes needed by the calls that take one. */
size_t fp8mlp_workspace_size(int M, int d, int h);

/* ------------------------------------------------------------------------
 * Backward ("NanoGPT Speedrun (Track 1)", Changes vs Record #83, item 4;
 * "A Retrospective on Our World Records": BF16 backward from the BF16 post)
 * ------------------------------------------------------------------------ */

/* Launch flag of fp8mlp_bwd_dpre and fp8mlp_bwd_dw (no counterpart on the
 * pages; a scheduling hint).  The caller asserts that the kernel enqueued
 * immediately before this call on the same stream was launched by this
 * library, and that this call reads nothing that kernel writes and writes
 * nothing it reads or writes (e.g. dPre right after the FP8 down-projection,
 * dW right after dX).  The GEMM then starts while that kernel finishes its
 * last wave of tiles and waits for it only before completing, so work
 * enqueued later still sees both complete.  (Every kernel of the library
 * waits for its own predecessor before it lets the next kernel start -- a
 * kernel launched with this flag lets it start only after that final wait --
 * so the inputs produced two launches back are complete.)  With
 * programmatic launch switched off, or when the previous kernel is not the
 * library's, the flag changes nothing.  A false assertion is a data race. */
#define FP8MLP_LAUNCH_OVERLAP_PREVIOUS 1

/*
 * dPost = dOut . W2^T (fp32 accumulate);  relu(pre) rebuilt as sqrt(post):
 *   dPre[m,i] = bf16( fp32(2 * sqrt(post[m,i])) * dPost[m,i] )
 * sqrt is the hardware approximation (sqrt.approx.f32, about one fp32 ulp),
 * far below the BF16 rounding of dPre that follows.
 * dOut [M,d], W2 [h,d], post [M,h] -> dPre [M,h].
 * flags: 0 or FP8MLP_LAUNCH_OVERLAP_PREVIOUS (see above).
 */
int fp8mlp_bwd_dpre(int M, int d, int h, const uint16_t* dOut, const uint16_t* W2, const uint16_t* post,
                    uint16_t* dPre, int flags, fp8mlp_stream_t stream);

/* dX = bf16(dPre . W1):  dPre [M,h], W1 [h,d] -> dX [M,d]. */
int fp8mlp_bwd_dx(int M, int d, int h, const uint16_t* dPre, const uint16_t* W1, uint16_t* dX,
                  fp8mlp_stream_t stream);

/* dW1 = dPre^T . x and dW2 = post^T . dOut, fp32 [h,d] each, in one launch.
 * flags: 0 or FP8MLP_LAUNCH_OVERLAP_PREVIOUS (see above). */
int fp8mlp_bwd_dw(int M, int d, int h, const uint16_t* x, const uint16_t* dPre, const uint16_t* post,
                  const uint16_t* dOut, float* dW1, float* dW2, int flags, fp8mlp_stream_t stream);

/* Whole backward: fp8mlp_bwd_dpre, fp8mlp_bwd_dx, fp8mlp_bwd_dw. */
int fp8mlp_mlp_bwd(int M, int d, int h, const uint16_t* x, const uint16_t* W1, const uint16_t* W2,
                   const uint16_t* post, const uint16_t* dOut, uint16_t* dPre, uint16_t* dX, float* dW1,
                   float* dW2, fp8mlp_stream_t stream);

/*
 * One whole training step of the block, scheduled for the GPU ("A
 * Retrospective on Our World Records", Main Track: the transposed FP8 W2
 * cache refreshed after the optimizer update, the fused up-projection, the
 * FP8 down-projection, the BF16 backward, the partial amax reduced into the
 * next step's scale).  Results, bit for bit, are those of
 *   fp8mlp_w2_fp8_cache_refresh (from the current W2, into W2q_t),
 *   fp8mlp_mlp_fwd (default flags), fp8mlp_mlp_bwd,
 *   fp8mlp_amax_reduce_update_scale (fp8mlp_partial_amax_count(M, h) entries),
 * called in that order on `stream`.  The schedule: the cache refresh runs on
 * a second stream beside the up-projection (which does not read the cache)
 * and is joined before the down-projection; dPre and dW start while the
 * GEMM before each finishes its last wave (FP8MLP_LAUNCH_OVERLAP_PREVIOUS);
 * the scale update runs on the second stream beside dX and dW and is joined
 * at the end, so work enqueued later on `stream` sees every result.
 * Buffers and layouts as in those calls; workspace: fp8mlp_workspace_size
 * (M, d, h) bytes for the cache refresh.  The second stream and its four
 * events are the library's own, one set per device, created by the first
 * call on that device: make that call before any stream capture.  A call
 * enqueues its whole sequence under that device's lock, so calls from
 * several host threads are safe, but their second-stream work runs one
 * call after another.  M = 0: the cache is refreshed, dW1 and dW2 are
 * zeroed and the scale update keeps the scale (amax 0).
 */
int fp8mlp_mlp_train_step(int M, int d, int h, const uint16_t* x, const uint16_t* W1, const uint16_t* W2,
                          const uint16_t* dOut, uint8_t* W2q_t, float* w2_scale_inv, fp8mlp_scale_state* st,
                          uint16_t* post, uint8_t* post_fp8, float* partial_amax, uint16_t* out, uint16_t* dPre,
                          uint16_t* dX, float* dW1, float* dW2, void* workspace, fp8mlp_stream_t stream);

/* ------------------------------------------------------------------------
 * Layer stack helpers (RMSNorm without gain, eps = 1e-6; residual add).
 * The pages train 9-layer, 768-dim models with ReLU^2 MLPs ("nanochat
 * autoresearch result", Method); they do not describe the norm, so this is
 * the plain RMSNorm reading.
 * ------------------------------------------------------------------------ */

/* x = bf16(r * rstd), rstd[m] = 1/sqrt(mean(r[m,:]^2) + 1e-6) (fp32). */
int fp8mlp_rmsnorm_fwd(int M, int d, const uint16_t* r, uint16_t* x, float* rstd, fp8mlp_stream_t stream);

/* RMSNorm forward fused with the x quantiser of the FP8 up-projection
 * ("NanoGPT Speedrun (Track 1)", From Unoptimized, item 5: e4m3 MLP GEMMs in
 * the training forward), so that x is read once: x and rstd as
 * fp8mlp_rmsnorm_fwd, and
 *   x_fp8[m,k] = e4m3_satfinite( fp32(x[m,k] * st_x->scale) )   (the BF16 x)
 *   row_amax[m] = max_k |x[m,k]|                                (fp32, [M])
 * -- the codes of fp8mlp_quantize_x on this x.  The next step's x-scale is
 * fp8mlp_amax_reduce_update_scale(row_amax, M, st_x). */
int fp8mlp_rmsnorm_fwd_quant(int M, int d, const uint16_t* r, uint16_t* x, float* rstd,
                             const fp8mlp_scale_state* st_x, uint8_t* x_fp8, float* row_amax,
                             fp8mlp_stream_t stream);

/* dr_out = bf16( dr_in + rstd * (dx - xhat * mean(dx * xhat)) ), xhat = r * rstd.
 * dr_in may equal dr_out (in place). */
int fp8mlp_rmsnorm_bwd(int M, int d, const uint16_t* r, const float* rstd, const uint16_t* dx,
                       const uint16_t* dr_in, uint16_t* dr_out, fp8mlp_stream_t stream);

/* r_next = bf16(r + out), [M,d]. */
int fp8mlp_residual_add(int M, int d, const uint16_t* r, const uint16_t* out, uint16_t* r_next,
                        fp8mlp_stream_t stream);

/* ------------------------------------------------------------------------
 * Status and diagnostics
 * ------------------------------------------------------------------------ */

/* Synchronise `stream`, then copy the device status word of the current
 * device into *status (FP8MLP_STATUS_* bits; 0 = clean). */
int fp8mlp_get_device_status(unsigned int* status, fp8mlp_stream_t stream);
/* Clear the device status word (enqueued on `stream`). */
int fp8mlp_clear_device_status(fp8mlp_stream_t stream);
/* Programmatic dependent launch (default on): every kernel of the library is
 * launched so that it may start while the previous kernel on the stream is
 * finishing (its set-up overlaps that kernel's tail); each kernel waits for
 * the previous one to complete before it touches global memory, so results
 * do not depend on this setting.  0 turns it off for later launches. */
int fp8mlp_set_programmatic_launch(int enable);
/* Per-wait limit of the kernels' bounded waits, in ns (default 2e9). */
int fp8mlp_set_wait_timeout_ns(unsigned long long ns);
/* Test hooks for the bounded waits.  FP8MLP_DEBUG_STALL_PRODUCER makes the
 * next GEMM launches' load warp issue nothing, so the MMA warp's bounded wait
 * runs out.  FP8MLP_DEBUG_STALL_AUX makes the epilogue of the next
 * fp8mlp_bwd_dpre launches issue none of its loads of post, so the
 * epilogue's own waits for them run out (and then the MMA warp's wait for a
 * free accumulator).  Either way the kernel returns with
 * FP8MLP_STATUS_TIMEOUT set and the context stays usable.  0 restores normal
 * runs. */
#define FP8MLP_DEBUG_STALL_PRODUCER 1
#define FP8MLP_DEBUG_STALL_AUX 2
int fp8mlp_set_debug_flags(int flags);

/* Static text of a return code. */
const char* fp8mlp_error_string(int code);
/* Text of the last error on this thread (empty if none). */
const char* fp8mlp_last_error_detail(void);
/* Library version string. */
const char* fp8mlp_version(void);
/* Number of CUDA kernels the library has launched in this process. */
unsigned long long fp8mlp_kernel_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* FP8MLP_H */
