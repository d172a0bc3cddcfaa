/*
 * dig.h -- C ABI of the B200 (sm_100a) DiG token mixer: chunkwise Gated Linear
 * Attention forward and backward, and the SREM reorient + 3x3 depthwise conv.
 *
 * Source of the operations ("DiG: Scalable and Efficient Diffusion Models with
 * Gated Linear Attention"; docswell study-group slides, page 2 of the reference
 * set, and the volcengine translation of the paper, page 3):
 *   GLA        slide "Gated Linear Attention Transformer (GLA) の導入", eq. (5)-(8):
 *              alpha_t = sigmoid(z_t)^(1/tau)        (gate, per key channel)
 *              S_t = diag(alpha_t) S_{t-1} + k_t^T v_t   (S_0 = 0, d_k x d_v)
 *              o_t = q_t S_t
 *   epilogue   same slide, eq. (9)-(10): y_t = Swish(r_t) * RMSNorm(o_t) * gamma
 *              (the projections X W_r and W_O are outside this library)
 *   chunking   slide "計算効率の分析" / paper "Efficiency Analysis": the sequence is
 *              split into chunks that fit on-chip memory
 *   SREM       slide "SREM (Spatial Reorient & Enhancement Module) の導入" and the
 *              paper's "DiG Block" section: 3x3 depthwise conv on the 2-D token grid
 *              and one of four scan orders (transpose / flip)
 *   backward   gradients of the three operations by the chain rule, for training
 *              (the paper trains DiG end to end)
 *
 * Conventions shared by every entry point
 *   - All tensor pointers are DEVICE pointers owned by the caller.  The library
 *     never allocates, frees or keeps device memory, and never synchronises
 *     (except dig_read_status).  Work is enqueued on `stream` (a cudaStream_t;
 *     NULL = legacy default stream) and the call returns without waiting.
 *     Stream order holds as for plain launches: the kernels are launched with
 *     programmatic stream serialization, so one may be scheduled while the
 *     previous kernel of the stream finishes, but each reads or writes global
 *     memory written by that kernel only after waiting for its completion, and
 *     writes nothing before then (any caller-side kernel that precedes a call
 *     has completed before the call's first kernel touches memory).
 *   - Tensors are dense, row-major, tokens in GRID row-major order
 *     (token g = row * grid_w + col, L = grid_h * grid_w).  Pointers must be
 *     16-byte aligned.
 *   - Element types: `dtype` is the storage type of q, k, v, dO, r and of the
 *     conv input x (DIG_F32 or DIG_BF16); `out_dtype` is the storage type of o,
 *     y, dq, dk, dv and the conv output.  z, dlog_alpha, gamma, the conv weights
 *     and bias are always fp32.  Arithmetic is fp32: tensor-core products take
 *     each operand as a sum of bf16 terms (two for bf16 inputs, three for fp32
 *     inputs) and accumulate in fp32.
 *   - Errors in the arguments are reported synchronously and nothing is
 *     launched.  A failed launch returns DIG_ERR_CUDA.  Conditions found on the
 *     device (a bounded wait that ran out, a gate outside the supported range)
 *     are recorded in a status word inside the workspace; read it with
 *     dig_read_status.  dig_last_error() gives a message for the last failure
 *     of the calling thread.
 */
#ifndef DIG_H_
#define DIG_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int dig_status;
enum {
  DIG_OK = 0,
  DIG_ERR_INVALID_ARGUMENT = 1,   /* bad shape, pointer, mode or dtype             */
  DIG_ERR_UNSUPPORTED = 2,        /* valid but not built (head dims, see below)      */
  DIG_ERR_MISALIGNED = 3,         /* a pointer is not 16-byte aligned                */
  DIG_ERR_WORKSPACE_TOO_SMALL = 4,
  DIG_ERR_CUDA = 5,               /* a CUDA call failed (launch, attribute query)    */
  DIG_ERR_DEVICE_TIMEOUT = 6,     /* device status: a bounded inter-CTA wait ran out  */
  DIG_ERR_GATE_RANGE = 7          /* device status: a chunk's gate decay left the
                                     exponent range of the chunked factorisation
                                     (dig_gla_fwd_ext / dig_gla_bwd_ext only; the
                                     plain entry points compute such chunks)          */
};

/* Scan orders (DiG scanning directions; layer l of the model uses mode l % 4).
 * Scan position t visits grid token g = pi(t):
 *   ROW_FWD  pi(t) = t                    ROW_REV  pi(t) = L-1-t
 *   COL_FWD  pi(t) = (t % grid_h) * grid_w + t / grid_h
 *   COL_REV  pi(t) = COL_FWD(L-1-t)                                          */
enum { DIG_SCAN_ROW_FWD = 0, DIG_SCAN_ROW_REV = 1, DIG_SCAN_COL_FWD = 2, DIG_SCAN_COL_REV = 3 };

enum { DIG_F32 = 0, DIG_BF16 = 1 };

/* Head dimensions built into this library: (d_k, d_v) in
 * {(32,64), (36,72), (64,64)}; any other pair returns DIG_ERR_UNSUPPORTED. */
int dig_gla_supported(int d_k, int d_v);

/* Bytes of device workspace dig_gla_fwd (pass = 0) or dig_gla_bwd (pass = 1)
 * needs for this shape (gate_heads: 1 or H, as passed to those calls) on the
 * current device.  The workspace must be
 * zero-filled before its first use; every call that ends with status DIG_OK
 * leaves it ready for the next call (no re-zeroing needed).  After a device
 * status other than DIG_OK, zero it again.  Calls that may run concurrently
 * need separate workspaces.  Returns 0 for invalid shapes. */
size_t dig_gla_workspace_bytes(int B, int H, int gate_heads, int L, int d_k, int d_v, int pass);

/* GLA forward (slide eq. (5)-(8), chunkwise).
 *   q, k   [B, L, H, d_k]   dtype        queries / keys (no extra 1/sqrt(d) scale)
 *   v      [B, L, H, d_v]   dtype
 *   z      [B, L, gate_heads, d_k] fp32  gate logits; alpha = exp(inv_tau*logsigmoid(z));
 *                                        gate_heads is 1 (one gate shared by all heads)
 *                                        or H
 *   o      [B, L, H, d_v]   out_dtype    o_t = q_t S_t, written at the token's grid slot
 *   r      [B, L, H, d_v]   dtype        optional (NULL): output-gate input
 *   gamma  [d_v] fp32                    optional (NULL = ones): RMSNorm weight
 *   y      [B, L, H, d_v]   out_dtype    optional: Swish(r) * o / sqrt(mean(o^2)+eps) * gamma;
 *                                        written only when both r and y are non-NULL
 * The recurrence runs in the scan order `scan_mode` over the grid_h x grid_w
 * grid; no reordered copy of any tensor is written.
 * Any finite z is computed: a chunk whose decay over half a chunk exceeds 2^115
 * in some key channel (the range of the chunk factorisation in fp32) is
 * recomputed exactly in fp32 token by token, inside the same kernels, and the
 * backward does the same (strong gates; the device status stays DIG_OK). */
dig_status dig_gla_fwd(const void *q, const void *k, const void *v, const float *z,
                       int gate_heads, float inv_tau, void *o,
                       const void *r, const float *gamma, float eps, void *y,
                       int B, int H, int L, int d_k, int d_v, int grid_h, int grid_w,
                       int scan_mode, int dtype, int out_dtype,
                       void *workspace, size_t workspace_bytes, void *stream);

/* Forward without a caller-allocated workspace, for callers that cannot call
 * cudaMalloc (plug-ins hosted by a runtime that owns all device memory and
 * forbids its extensions to allocate; host programs that link only this library
 * and have no device allocator).  The paper has no counterpart: this is an
 * interface convenience.  Same arguments and results as dig_gla_fwd, but the
 * workspace is a 16 MiB scratch array built into the library (one per GPU that
 * loads it, held until the process exits); nothing is allocated or freed.
 *   - Shapes whose dig_gla_workspace_bytes(B, H, gate_heads, L, d_k, d_v, 0)
 *     exceeds 16 MiB
 *     are rejected with DIG_ERR_WORKSPACE_TOO_SMALL (see dig_last_error).
 *   - The first call on a device looks up the scratch array's device address
 *     (with that device current); make that first call before any stream capture.
 *     The address is kept for the life of the process: after a cudaDeviceReset
 *     in the host process it is stale, so do not use this entry point after one.
 *   - Every argument check of dig_gla_fwd runs first; an invalid call returns
 *     before anything is enqueued on `stream`.
 *   - Every call clears the scratch's status word (a small memset on `stream`)
 *     and shares the one array: calls that overlap on the GPU (other
 *     streams, other threads) race on it and must not be issued.
 *   - device_status (optional, device pointer): receives the call's device
 *     status word (DIG_OK, DIG_ERR_DEVICE_TIMEOUT, DIG_ERR_GATE_RANGE) in
 *     stream order. */
dig_status dig_gla_fwd_noalloc(const void *q, const void *k, const void *v, const float *z,
                               int gate_heads, float inv_tau, void *o,
                               const void *r, const float *gamma, float eps, void *y,
                               int B, int H, int L, int d_k, int d_v, int grid_h, int grid_w,
                               int scan_mode, int dtype, int out_dtype,
                               unsigned int *device_status, void *stream);

/* GLA forward with a value gate and state input / output (slide "Gated Linear
 * Attention Transformer (GLA) の導入", eq. (5): G_t = alpha_t^T beta_t (outer
 * product), S_t = G_t (*) S_{t-1} + k_t^T v_t, o_t = q_t S_t, the recurrence
 * started from S_0 instead of zero).  Arguments as dig_gla_fwd, plus:
 *   zb       [B, L, gate_heads, d_v] fp32  value-gate logits, beta = exp(inv_tau *
 *                                          logsigmoid(zb)); NULL: beta = 1
 *   S0       [B, H, d_k, d_v] fp32         initial state (S0[b][h][c][j] = S_0[c][j]);
 *                                          NULL: zero
 *   S_final  [B, H, d_k, d_v] fp32         written: the state after the last scan
 *                                          position (the S0 of a following segment);
 *                                          may be NULL
 * A sequence cut into segments and run segment by segment, each from the last
 * one's S_final, gives the same o as one call over the whole sequence (in the
 * scan order of each call).  d_v must be 64 or 72.  The call runs the fp32
 * kernels (64-token chunks); bf16 inputs are widened into the workspace, whose
 * size dig_gla_ext_workspace_bytes(..., dtype, 0) gives (zero-filled before the
 * first use).  Errors as dig_gla_fwd, except that a chunk whose key or value
 * gate decays beyond 2^115 over half a 64-token chunk is not recomputed: it
 * sets DIG_ERR_GATE_RANGE in the device status word (dig_read_status). */
dig_status dig_gla_fwd_ext(const void *q, const void *k, const void *v, const float *z, const float *zb,
                           int gate_heads, float inv_tau, const float *S0, void *o,
                           const void *r, const float *gamma, float eps, void *y, float *S_final,
                           int B, int H, int L, int d_k, int d_v, int grid_h, int grid_w,
                           int scan_mode, int dtype, int out_dtype,
                           void *workspace, size_t workspace_bytes, void *stream);

/* Gradients for dig_gla_fwd_ext of sum(o * dO) + sum(S_final * dS_final).
 *   o          [B, L, H, d_v] out_dtype  the forward's output (read only for
 *                                        dlog_beta; may be NULL without it)
 *   dS_final   [B, H, d_k, d_v] fp32     gradient of S_final; NULL: zero
 *   dlog_beta  [B, L, gate_heads, d_v] fp32  dLoss/dlog(beta), summed over heads
 *                                        when gate_heads == 1; NULL: not formed
 *                                        (then zb may be NULL)
 *   dS0        [B, H, d_k, d_v] fp32     written: gradient of S0; may be NULL
 * Other arguments and results as dig_gla_bwd; the workspace size is
 * dig_gla_ext_workspace_bytes(..., dtype, 1). */
dig_status dig_gla_bwd_ext(const void *q, const void *k, const void *v, const float *z, const float *zb,
                           int gate_heads, float inv_tau, const float *S0, const void *o, const void *dO,
                           const float *dS_final, void *dq, void *dk, void *dv, float *dlog_alpha,
                           float *dlog_beta, float *dS0,
                           int B, int H, int L, int d_k, int d_v, int grid_h, int grid_w,
                           int scan_mode, int dtype, int out_dtype,
                           void *workspace, size_t workspace_bytes, void *stream);

/* Bytes of workspace dig_gla_fwd_ext (pass = 0) or dig_gla_bwd_ext (pass = 1)
 * needs; 0 for invalid or unsupported shapes. */
size_t dig_gla_ext_workspace_bytes(int B, int H, int gate_heads, int L, int d_k, int d_v, int dtype, int pass);

/* GLA backward: gradients of sum(o * dO) for the forward above.
 *   dO          [B, L, H, d_v]  dtype
 *   dq, dk      [B, L, H, d_k]  out_dtype
 *   dv          [B, L, H, d_v]  out_dtype
 *   dlog_alpha  [B, L, gate_heads, d_k] fp32: dLoss/dlog(alpha), summed over heads
 *               when gate_heads == 1.  The gradient of the logits is
 *               dz = dlog_alpha * inv_tau * sigmoid(-z) (left to the caller).
 * When gate_heads == 1 the heads' contributions to dlog_alpha are added with
 * floating-point atomics, so its last bits may differ between runs. */
dig_status dig_gla_bwd(const void *q, const void *k, const void *v, const float *z,
                       int gate_heads, float inv_tau, const void *dO,
                       void *dq, void *dk, void *dv, float *dlog_alpha,
                       int B, int H, int L, int d_k, int d_v, int grid_h, int grid_w,
                       int scan_mode, int dtype, int out_dtype,
                       void *workspace, size_t workspace_bytes, void *stream);

/* GLA backward that reuses the records of the forward call on the same inputs
 * (training steps run the forward first): the gate factors and the state
 * entering every chunk are read from `fwd_workspace` instead of being
 * recomputed, so this pass reads neither z nor the forward's k^T v per chunk.
 *   fwd_workspace   the workspace of the last dig_gla_fwd call with the same
 *                   q, k, v, z, gate_heads, inv_tau, shapes, scan_mode and dtype,
 *                   unchanged since (device pointer; only read)
 *   workspace       this pass's own workspace, as for dig_gla_bwd
 * Results equal dig_gla_bwd's up to rounding.  Where the two passes cut the
 * sequence into different chunks (the head dims or dtype give the backward a
 * shorter chunk), the forward's records do not apply and the call runs
 * dig_gla_bwd.  There is no check that fwd_workspace matches the inputs: a
 * stale or foreign workspace gives wrong gradients, not an error. */
dig_status dig_gla_bwd_saved(const void *q, const void *k, const void *v, const float *z,
                             int gate_heads, float inv_tau, const void *dO,
                             void *dq, void *dk, void *dv, float *dlog_alpha,
                             int B, int H, int L, int d_k, int d_v, int grid_h, int grid_w,
                             int scan_mode, int dtype, int out_dtype,
                             const void *fwd_workspace, size_t fwd_workspace_bytes,
                             void *workspace, size_t workspace_bytes, void *stream);

/* SREM reorient + 3x3 depthwise conv (zero "same" padding, cross-correlation as
 * in a depthwise nn.Conv2d):
 *   x     [B, grid_h, grid_w, C] dtype, grid order
 *   w     [C, 3, 3] fp32;  bias [C] fp32 or NULL
 *   y     [B, L, C] out_dtype, in SCAN order: y[b, t] = conv(x)[b, pi(t)]
 * With the identity kernel (centre tap 1) this is exactly the reorient
 * permutation. */
dig_status dig_srem_reorient_dwconv(const void *x, const float *w, const float *bias, void *y,
                                    int B, int grid_h, int grid_w, int C, int scan_mode,
                                    int dtype, int out_dtype, void *stream);

/* Backward of dig_srem_reorient_dwconv: gradients of sum(dY * y).
 *   x      [B, grid_h, grid_w, C] dtype, grid order: the forward's input (only read
 *          for dw; may be NULL when dw and dbias are both NULL)
 *   w      [C, 3, 3] fp32: the forward's weights
 *   dY     [B, L, C] dtype, SCAN order (the layout of the forward's y)
 *   dx     [B, grid_h, grid_w, C] out_dtype, grid order:
 *          dx[g] = sum_{di,dj} w[di+1, dj+1] * dY at the scan position of g - (di, dj)
 *   dw     [C, 3, 3] fp32 or NULL; dbias [C] fp32 or NULL: sums over B and the
 *          grid.  Overwritten: the call zeroes them on `stream` first.  With an
 *          even C the partial sums of the thread blocks are added with
 *          floating-point atomics, so their last bits may differ between runs.
 * Same element types, alignment and stream rules as the forward. */
dig_status dig_srem_reorient_dwconv_bwd(const void *x, const float *w, const void *dY, void *dx,
                                        float *dw, float *dbias,
                                        int B, int grid_h, int grid_w, int C, int scan_mode,
                                        int dtype, int out_dtype, void *stream);

/* Backward of the epilogue (slide eq. (9)-(10)): gradients of sum(dY * y) for
 * y = Swish(r) * o / sqrt(mean(o^2) + eps) * gamma, taken row by row over d_v as
 * dig_gla_fwd computes it (rows = B * L * H for its [B, L, H, d_v] tensors; any
 * row order, as long as o, r, dY, d_o and d_r share it).
 *   o, r, dY   [rows, d_v] dtype       the forward's o and r, and dLoss/dy
 *   gamma      [d_v] fp32 or NULL (ones)
 *   eps        the forward's eps (>= 0)
 *   d_o        [rows, d_v] out_dtype   dLoss/do: the dO to pass to dig_gla_bwd
 *   d_r        [rows, d_v] out_dtype   dLoss/dr
 *   d_gamma    [d_v] fp32 or NULL: dLoss/dgamma summed over the rows.  Overwritten:
 *              the call zeroes it on `stream` first, then adds the thread blocks'
 *              partial sums with floating-point atomics (last bits may differ
 *              between runs).
 * d_v up to 8192 (DIG_ERR_UNSUPPORTED above).  Same element types, alignment and
 * stream rules as the forward. */
dig_status dig_epilogue_bwd(const void *o, const void *r, const float *gamma, float eps,
                            const void *dY, void *d_o, void *d_r, float *d_gamma,
                            long long rows, int d_v, int dtype, int out_dtype, void *stream);

/* Gate projection (slide eq. (5): the gate logits are a projection of the block
 * input, low-rank in DiG: D -> R -> d_k):
 *   u = x W1,   z = u W2 + b
 *   x    [rows, D] dtype          rows = B * L tokens (grid order), D % 8 == 0
 *   W1   [D, R] fp32;  W2 [R, d_k] fp32;  b [d_k] fp32 or NULL (zero)
 *   z    [rows, d_k] fp32         the z of dig_gla_fwd with gate_heads = 1
 *   u    [rows, R] fp32 or NULL   x W1, kept for dig_gate_proj_bwd
 * Built for R <= 32 and d_k <= 128 with the weights in shared memory (D * R
 * floats, plus D * R more for the backward, up to 227 KB): DIG_ERR_UNSUPPORTED
 * otherwise.  Same alignment and stream rules as the other calls. */
dig_status dig_gate_proj_fwd(const void *x, const float *W1, const float *W2, const float *b,
                             float *z, float *u, long long rows, int D, int R, int d_k,
                             int dtype, void *stream);

/* Backward of the gate projection from the GLA backward's dlog_alpha (the gate
 * is log(alpha) = inv_tau * logsigmoid(z), so dz = dlog_alpha * inv_tau * sigmoid(-z)):
 *   x, W1, W2   as passed to dig_gate_proj_fwd;  u, z its outputs
 *   dlog_alpha  [rows, d_k] fp32 (dig_gla_bwd with gate_heads = 1)
 *   dx          [rows, D] out_dtype:  dz W2^T W1^T
 *   dW1 [D, R], dW2 [R, d_k], db [d_k] (db may be NULL) fp32: sums over the rows.
 *               Overwritten (zeroed on `stream` first); the thread blocks' partial
 *               sums are added with floating-point atomics, so their last bits may
 *               differ between runs. */
dig_status dig_gate_proj_bwd(const void *x, const float *W1, const float *W2, const float *u,
                             const float *z, const float *dlog_alpha, float inv_tau,
                             void *dx, float *dW1, float *dW2, float *db,
                             long long rows, int D, int R, int d_k, int dtype, int out_dtype,
                             void *stream);

/* Element-wise steps of a DiG block around its token mixer (slide "DiG" Fig. 4,
 * the DiG block: adaLN scale / shift / gate regressed from the conditioning,
 * RMS normalisation, gated residuals, SiLU in the conditioning MLP, GELU in the
 * feed-forward network).  The paper gives the block's structure, not these
 * interfaces; they serve the library's synthetic block.  Tensors are bf16 rows
 * of D values, B batches of rows_per_batch rows each; the modulation vectors are
 * fp32, D values per batch at stride mod_stride (so that slices of one [B, 6 D]
 * projection can be passed; mod_stride a multiple of 4).  Pointers, including the
 * modulation slices, 16-byte aligned; D a multiple of 8.
 *   rmsnorm_modulate:  y = x / sqrt(mean(x^2) + eps) * (1 + scale[b]) + shift[b]
 *                      (D up to 2048)
 *   gated_add:         x += gate[b] * y
 *   activation:        x in place, n values: kind 0 SiLU a sigmoid(a), kind 1 GELU
 *                      (tanh form) */
dig_status dig_block_rmsnorm_modulate(const void *x, const float *shift, const float *scale,
                                      long long mod_stride, float eps, void *y, int B,
                                      long long rows_per_batch, int D, void *stream);
dig_status dig_block_gated_add(void *x, const float *gate, long long mod_stride, const void *y, int B,
                               long long rows_per_batch, int D, void *stream);
dig_status dig_block_activation(void *x, long long n, int kind, void *stream);

/* Synchronises `stream`, returns the device status word kept in `workspace`
 * (DIG_OK, DIG_ERR_DEVICE_TIMEOUT or DIG_ERR_GATE_RANGE) and clears it. */
dig_status dig_read_status(void *workspace, void *stream);

const char *dig_status_string(dig_status s);
const char *dig_last_error(void);

#ifdef __cplusplus
}
#endif
#endif /* DIG_H_ */
