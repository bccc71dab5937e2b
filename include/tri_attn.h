/*
 * tri_attn.h — C ABI of the B200 (sm_100a) triangle attention library.
 *
 * One call computes the pair-biased triangle attention block over a protein
 * pair representation Z of shape [N][N][c_z] (channels last), in either the
 * starting-node or the ending-node orientation:
 *
 *   x      = LayerNorm(z)                      per pair, over c_z channels
 *   q,k,v  = Wq x, Wk x, Wv x                  H heads of width d
 *   g      = sigmoid(Wg x + bg)
 *   beta_h = Wb x                              one logit bias per head
 *   starting node: o_ij = sum_k softmax_k(q_ij.k_ik/sqrt(d) + beta_h(j,k)) v_ik
 *   ending node:   o_ij = sum_k softmax_k(q_ij.k_kj/sqrt(d) + beta_h(k,i)) v_kj
 *   out_ij = z_ij + Wo (g_ij * o_ij) + bo
 *
 * Sources.  The pair representation (Ns, Ns, Hz), Hz typically 128, as the
 * bottleneck of protein structure models: LightNobel article
 * ("蛋白质结构预测模型的量化优化与硬件加速"), §1.1; LayerNorm ahead of the
 * linear layers and the residual path: same article §2.2.3 (groups A and B)
 * and §3.1, which also names triangular attention.  Attention scores are
 * computed tile by tile with an online softmax and never stored as an N x N
 * matrix: Design-CP technical summary, §Metodología 1 (2D grid sharding,
 * ring attention).  Kernel fusion of attention to cut memory traffic:
 * OpenFold-TRT summary, §2 Metodología.  The pages give no equations for
 * triangular attention; the formulas above are the standard definition of
 * the block and are what this library computes.
 *
 * Masking: mask[k] == 0 removes residue k as a key (probability exactly 0);
 * rows and columns of masked residues are still computed.  If every key is
 * masked the attention output is 0 and out = z + bo.
 *
 * Threading and streams: calls are asynchronous on the given stream unless
 * stated otherwise.  A handle is not thread-safe; use one handle per host
 * thread.  Results are deterministic (no floating-point atomics).
 * There is no CPU fallback: without a usable sm_100 device every call that
 * needs one returns TRI_ATTN_ERR_NO_DEVICE.
 *
 * Diagnostics: with the environment variable TRIATTN_LOG=1 the library prints
 * to stderr why a call failed (the CUDA call and its error, a rejected size)
 * and, per forward, the row chunking and workspace size it chose.
 */
#ifndef TRI_ATTN_H
#define TRI_ATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------ */
#define TRI_ATTN_OK                 0
#define TRI_ATTN_ERR_INVALID_ARG   -1  /* NULL/misaligned pointer, N < 1, bad enum */
#define TRI_ATTN_ERR_UNSUPPORTED   -2  /* shape or dtype the kernels do not cover */
#define TRI_ATTN_ERR_ALIAS         -3  /* out overlaps Z without being equal to it */
#define TRI_ATTN_ERR_OOM           -4  /* device or host allocation failed */
#define TRI_ATTN_ERR_CUDA          -5  /* a CUDA runtime call or launch failed */
#define TRI_ATTN_ERR_TIMEOUT       -6  /* a kernel's bounded wait expired (device status) */
#define TRI_ATTN_ERR_NO_DEVICE     -7  /* no sm_100 device is available */

/* ---- flags for tri_attn_forward --------------------------------------- */
#define TRI_ATTN_FLAG_SYNC          1u  /* synchronise the stream and return the device status */
#define TRI_ATTN_FLAG_TIME_KERNELS  2u  /* record CUDA events around each kernel (see tri_attn_kernel_times) */
/* Fault injection, for tests of the error paths.  None of them faults, traps or
 * hangs the GPU: a withheld copy makes the waiting threads' bounded waits
 * (2 s) expire, those threads free what they hold and leave, and the call
 * reports TRI_ATTN_ERR_TIMEOUT through the device status; the handle and the
 * CUDA context stay usable. */
#define TRI_ATTN_FLAG_DEBUG_STALL   4u  /* tri_attn_fwd: one CTA's producer withholds its first stage
                                       (also through tri_attn_attention_forward_bf16); in
                                       tri_attn_attention_backward_bf16 the same in each of its
                                       three tensor-core kernels */
#define TRI_ATTN_FLAG_DEBUG_STALL_PROJ 8u   /* pair_ln_proj: one group of one CTA never gets its first
                                               tile of Z (every launch of the call) */
#define TRI_ATTN_FLAG_DEBUG_STALL_GATE 16u  /* gate_out: one CTA's producer withholds its first stage
                                               (every launch of the call) */
#define TRI_ATTN_FLAG_DEBUG_FAIL_ALLOC 32u  /* if the call has to grow the handle's workspace, that
                                               allocation fails as if cudaMalloc had run out of memory:
                                               the call returns TRI_ATTN_ERR_OOM before any launch and
                                               the handle holds no workspace afterwards (the old one is
                                               released first); the next call allocates again */

typedef enum { TRI_ATTN_F32 = 0, TRI_ATTN_BF16 = 1 } tri_attn_dtype;
typedef enum { TRI_ATTN_STARTING = 0, TRI_ATTN_ENDING = 1 } tri_attn_orientation;

typedef struct tri_attn_handle tri_attn_handle;  /* opaque */

/* Weights of one block.  All pointers are DEVICE memory holding `dtype`
 * elements, row-major, contiguous.  Shapes (out x in):
 *   ln_gamma, ln_beta [c_z];  w_q, w_k, w_v, w_g [H*d][c_z];  b_g [H*d] or NULL (= 0);
 *   w_b [H][c_z];  w_o [c_z][H*d];  b_o [c_z] or NULL (= 0).
 * The kernels are specialised to c_z = 128, H = 4, d = 32; other shapes give
 * TRI_ATTN_ERR_UNSUPPORTED. */
typedef struct {
  int c_z, n_heads, head_dim;
  tri_attn_dtype dtype;
  float ln_eps;                 /* LayerNorm epsilon, e.g. 1e-5 */
  const void *ln_gamma, *ln_beta;
  const void *w_q, *w_k, *w_v, *w_g;
  const void *b_g;
  const void *w_b;
  const void *w_o;
  const void *b_o;
} tri_attn_params;

/* Create a handle on the current CUDA device.  Copies and repacks the weights
 * into the handle's own device buffers (synchronously), so the caller may
 * free its copies on return.  *out is set only on TRI_ATTN_OK. */
int tri_attn_create(const tri_attn_params *params, tri_attn_handle **out);

/* Run the block once on `stream` (a cudaStream_t; NULL = legacy default).
 *   Z    [N][N][c_z] device, dtype of the handle, 16-byte aligned.
 *   mask [N] device uint8 (1 = valid key) or NULL (all valid).
 *   out  [N][N][c_z] device, same dtype; out == Z (in place) is allowed,
 *        any other overlap returns TRI_ATTN_ERR_ALIAS.
 * Argument checks happen before any launch; on error nothing is launched.
 * The handle grows its workspace on demand (cudaMalloc); see
 * tri_attn_set_workspace_limit.  Returns TRI_ATTN_OK once the kernels are
 * enqueued, or, with TRI_ATTN_FLAG_SYNC, after the stream has drained, with
 * the device status of the call. */
int tri_attn_forward(tri_attn_handle *h, const void *Z, int N, const uint8_t *mask,
                     tri_attn_orientation orientation, void *out, void *stream,
                     unsigned flags);

/* End-to-end call on HOST buffers: copies Z (and mask) to the device, applies
 * the blocks orientations[0], orientations[1], ... in sequence, each on the
 * output of the previous one (in place in a device staging buffer owned by
 * the handle), and copies the final result back to out_host.  Synchronous:
 * returns after out_host is written.  Z_host and out_host may be the same
 * buffer; pinned host memory gives full PCIe bandwidth.  Z is copied in
 * pieces that the first block's projection consumes as they arrive, and the
 * last block runs in row chunks whose results are copied back while later
 * chunks compute, so the copies overlap the computation where the block's
 * data dependencies allow. */
int tri_attn_forward_host(tri_attn_handle *h, const void *Z_host, int N,
                          const uint8_t *mask_host, const int *orientations,
                          int n_orientations, void *out_host, void *stream,
                          unsigned flags);

/* Asynchronous form of tri_attn_forward_host, for a stream of independent
 * problems: same arguments and result, but the call returns once the copies
 * and the blocks are enqueued.  The uploads run on a copy stream of the
 * handle, the blocks on `stream`, the downloads on a second copy stream of the
 * handle, ordered by events; the handle keeps three device staging buffers
 * (allocated on first use, each N x N x c_z elements), so consecutive calls
 * overlap one call's upload, another's computation and a third's download
 * (PCIe carries both directions at once).
 * Rules: every asynchronous call on a handle uses the same `stream`; Z_host,
 * mask_host and out_host must stay valid and unmodified until
 * tri_attn_host_wait returns; one in-flight call's out_host must not be
 * another in-flight call's Z_host (a call's own Z_host may be its out_host;
 * in-flight calls may share one out_host: the downloads run in call order).
 * A call with a larger N than before waits for the calls in flight first.
 * Errors are those of tri_attn_forward_host, returned by the call that
 * detects them; device errors (a timed-out wait) by tri_attn_host_wait. */
int tri_attn_forward_host_async(tri_attn_handle *h, const void *Z_host, int N,
                                const uint8_t *mask_host, const int *orientations,
                                int n_orientations, void *out_host, void *stream,
                                unsigned flags);

/* Wait until every tri_attn_forward_host_async call on the handle has
 * completed (its results are in out_host) and return the sticky device status
 * (TRI_ATTN_OK or TRI_ATTN_ERR_TIMEOUT), then clear it. */
int tri_attn_host_wait(tri_attn_handle *h);

/* Synchronise `stream` and return the sticky device status of the handle
 * (TRI_ATTN_OK or TRI_ATTN_ERR_TIMEOUT), then clear it. */
int tri_attn_get_status(tri_attn_handle *h, void *stream);

/* Device milliseconds spent in each kernel, summed over every launch made
 * with TRI_ATTN_FLAG_TIME_KERNELS since the previous call of this function
 * (which resets the record): ms[0] = pair_ln_proj, ms[1] = tri_attn_fwd,
 * ms[2] = gate_out; launches[k] (may be NULL) = number of launches timed.
 * Each launch is bracketed by CUDA events on the stream it runs on.
 * Synchronises on the events. */
int tri_attn_kernel_times(tri_attn_handle *h, float ms[3], int launches[3]);

/* Upper bound on the workspace (bytes) the handle may allocate; above it the
 * rows are processed in chunks.  0 restores the default (48 GiB). */
int tri_attn_set_workspace_limit(tri_attn_handle *h, size_t bytes);

/* Device workspace in bytes that a forward of size N needs without chunking. */
size_t tri_attn_workspace_bytes(tri_attn_dtype dtype, int N);

/* Device pointers of the intermediate tensors of the last forward call (for
 * inspection by tests).  Layouts, for rows r of the last chunk and head h:
 *   q, k, v, g, o: [rows][H][N][d];  bias: [H][N][ld_bias]
 * (bias already scaled by log2(e); at masked keys and at columns >= N it is
 * -inf for F32 handles and the finite -3e38 for BF16 handles, which keeps the
 * sums it enters finite and still gives those keys probability exactly 0;
 * q already scaled by log2(e)/sqrt(d)).  Element type: bf16 for a BF16
 * handle, fp32 for F32.  A BF16 handle keeps no gate tensor (gate_out
 * recomputes the gate from LayerNorm(z)), so *g is set to NULL for it.  Any
 * output pointer may be NULL. */
int tri_attn_debug_workspace(tri_attn_handle *h, void **q, void **k, void **v, void **g,
                             void **bias, void **o, int *ld_bias, int *rows);

/* ---- row-sharded execution (bf16) -----------------------------------------
 *
 * A starting-node block splits over devices by problem rows i: row i needs
 * only its own K and V (pairs (i, k)) plus the logit bias of every pair, so a
 * device that holds the row slab Z[row0 .. row0+nrows-1][0..N-1][c_z] can
 * compute those output rows once the whole bias is known (the 1D row sharding
 * of the Design-CP technical summary, §Metodología 1, with the bias as the one
 * exchanged quantity).  The caller runs the exchange between the two calls:
 *
 *   1. tri_attn_rows_bias: the slab's bias rows, bias_rows[h][r][k] for the
 *      problem rows row0+r, heads h, keys k < ld (ld = tri_attn_bias_ld(N));
 *   2. gather every device's rows into bias_all[h][i][k] ([H][N][ld]);
 *   3. tri_attn_rows_forward: the block on the slab, reading bias_all.
 *
 * An ending-node block is the starting-node block of the transposed pair
 * tensor (pair (i, j) -> (j, i)): shard its rows, i.e. the columns of Z.
 * Bias values: bf16, already scaled by log2(e), -3e38 at masked keys and at
 * k >= N.  Results are bitwise identical to tri_attn_forward on the whole
 * tensor.  These calls are asynchronous on `stream` like tri_attn_forward
 * (TRI_ATTN_FLAG_SYNC and TRI_ATTN_FLAG_TIME_KERNELS apply), need a BF16
 * handle (else TRI_ATTN_ERR_UNSUPPORTED) and device pointers aligned to 16
 * bytes; mask is the whole [N] key mask.  Z_rows and out_rows are
 * [nrows][N][c_z]; out_rows may equal Z_rows, any other overlap returns
 * TRI_ATTN_ERR_ALIAS.  Invalid row ranges return TRI_ATTN_ERR_INVALID_ARG. */

/* Row length (elements) of the logit-bias buffers for a problem of size N:
 * N rounded up to a multiple of 64; 0 for N < 1. */
int tri_attn_bias_ld(int N);

/* Phase 1: bias_rows ([H][nrows][ld] bf16, device) for the slab's rows. */
int tri_attn_rows_bias(tri_attn_handle *h, const void *Z_rows, int N, int row0, int nrows,
                       const uint8_t *mask, void *bias_rows, void *stream, unsigned flags);

/* Phase 3: out_rows = the starting-node block on the slab, with bias_all
 * ([H][N][ld] bf16, device) the whole problem's logit bias. */
int tri_attn_rows_forward(tri_attn_handle *h, const void *Z_rows, int N, int row0, int nrows,
                          const uint8_t *mask, const void *bias_all, void *out_rows,
                          void *stream, unsigned flags);

/* One forward of the bf16 block that allocates no device memory at all.
 *
 * For callers that are not allowed to call cudaMalloc: code embedded in a host
 * application that owns every byte of device memory through its own pool or
 * budget, and latency-critical paths where the implicit synchronisation and
 * unpredictable cost of a device allocation is not acceptable.  Such callers
 * cannot create a handle (tri_attn_create allocates), so this entry point takes
 * the weights directly (`params`, device pointers, bf16 only) together with the
 * usual Z, mask, out, N, orientation and stream; the arguments mean what they
 * mean for tri_attn_forward.  There is no counterpart of this call on the pages
 * this library follows.
 *
 * Scratch: everything besides the caller's buffers (the repacked weights, the
 * status word and the workspace) lives in one statically allocated device array
 * of 32 MiB inside this library; every GPU that loads the library holds it
 * until the process exits.  Rows are processed in chunks that fit the array.
 * Sizes it cannot hold (the whole logit bias plus one three-row chunk must fit,
 * which allows N up to 1856) return TRI_ATTN_ERR_UNSUPPORTED before anything
 * is launched.  The first call on a device also looks up the array's
 * device address (cudaGetSymbolAddress); make that first call before any stream
 * capture.  All calls share the one array, which keeps the last call's contents
 * (the status word is cleared at the start of each call): calls that overlap on
 * the GPU, e.g. on two streams of the same device, race and corrupt each other;
 * serialise them.  Flags: TRI_ATTN_FLAG_SYNC synchronises the stream and returns
 * the device status; the timing and fault-injection flags are ignored. */
int tri_attn_forward_noalloc(const tri_attn_params *params, const void *Z, int N,
                             const uint8_t *mask, tri_attn_orientation orientation, void *out,
                             void *stream, unsigned flags);

/* ---- backward pass of the attention core (fp32) ---------------------------
 *
 * Gradients of the starting-node attention core for training (the training
 * setting of the BioNeMo context-parallelism page).  For R problem rows r,
 * head h, query j and key k:
 *   s_jk = q_j . k_k / sqrt(d) + bias[h][j][k]  over keys with mask[k] != 0,
 *   p = softmax over k,  o_j = sum_k p_jk v_k.
 * Given dO = d loss / d o, this writes
 *   dQ_j = sum_k ds_jk k_k / sqrt(d),  dK_k = sum_j ds_jk q_j / sqrt(d),
 *   dV_k = sum_j p_jk dO_j,  dbias[h][j][k] = sum_r ds_jk,
 * with ds_jk = p_jk (dO_j . v_k - dO_j . o_j) (the softmax Jacobian applied to
 * d loss / d p).  Masked keys, and queries whose every key is masked, get zero
 * gradients.  The ending-node core is this computation on the transposed
 * problem (its rows are the columns of Z).  Note the natural-unit logits:
 * q is not pre-scaled and the bias is not multiplied by log2(e), unlike the
 * forward's workspace.
 *
 * Layouts (device memory, fp32, contiguous): Q, K, V, dO, dQ, dK, dV
 * [rows][H][N][d] with H = 4, d = 32 (the head-major layout of the forward's
 * workspace); bias, dbias [H][N][N]; mask [N] (1 = valid key) or NULL.
 * Q, K, V, dO, dQ, dK, dV and workspace must be 16-byte aligned.  The caller
 * owns every buffer; the call allocates nothing.  `workspace` holds the row
 * statistics and must have at least
 * tri_attn_attention_backward_workspace_bytes(rows, N) bytes.
 * Asynchronous on `stream` (four kernel launches, SIMT fp32 arithmetic: each
 * gradient agrees with an fp64 evaluation to ~1e-6 relative); dbias is written
 * once per element (no atomics), so the result is deterministic.
 * Errors: TRI_ATTN_ERR_INVALID_ARG (NULL or misaligned pointer, rows or N < 1,
 * workspace too small), TRI_ATTN_ERR_UNSUPPORTED (rows > 65535 or N > 46340),
 * TRI_ATTN_ERR_NO_DEVICE, TRI_ATTN_ERR_CUDA (launch failure).
 * Flags: TRI_ATTN_FLAG_SYNC synchronises the stream before returning. */
size_t tri_attn_attention_backward_workspace_bytes(int rows, int N);

/* The forward of the same attention core (fp32), for training loops that pair
 * it with tri_attn_attention_backward: writes o [rows][H][N][d] (16-byte
 * aligned) and the natural-log log-sum-exp lse [rows][H][N] of each query's
 * scores (+inf for a query whose every key is masked; its o is 0).  Same
 * inputs, layouts and errors as the backward; one kernel launch (the backward's
 * row-statistics kernel with o written out).  Flags: TRI_ATTN_FLAG_SYNC. */
int tri_attn_attention_forward(const float *Q, const float *K, const float *V,
                               const float *bias, const uint8_t *mask, int rows, int N,
                               float *O, float *lse, void *stream, unsigned flags);
int tri_attn_attention_backward(const float *Q, const float *K, const float *V,
                                const float *bias, const uint8_t *mask, const float *dO,
                                int rows, int N, float *dQ, float *dK, float *dV,
                                float *dbias, void *workspace, size_t workspace_bytes,
                                void *stream, unsigned flags);

/* ---- the same attention core on the tensor cores (bf16 operands) ---------
 *
 * The mathematics, layouts and natural units of the two fp32 calls above, with
 * bf16 operands: Q, K, V, O, dO bf16 [rows][H][N][d] (H = 4, d = 32), bias
 * bf16 [H][N][N], mask uint8 [N] (1 = valid key) or NULL.  Products run on
 * tcgen05 tensor cores in bf16 with fp32 accumulation: q * log2(e)/sqrt(d),
 * the bias in base 2, and the probabilities and ds_jk fed to the gradient
 * products are rounded to bf16 (relative 2^-9 each); lse, the row statistics
 * and every sum are fp32.
 *
 * `workspace` (16-byte aligned, at least
 * tri_attn_attention_bf16_workspace_bytes(rows, N) bytes, caller-owned, the
 * same size for both calls) holds the device status word, the scaled q, the
 * padded base-2 bias (and its transpose) and the per-query statistics.  Both
 * calls are asynchronous on `stream`; with TRI_ATTN_FLAG_SYNC they wait and
 * return the device status (TRI_ATTN_ERR_TIMEOUT if a kernel's bounded wait
 * expired; TRI_ATTN_FLAG_DEBUG_STALL injects that).  The calls allocate nothing.
 * Errors: TRI_ATTN_ERR_INVALID_ARG (NULL or misaligned pointer: Q, K, V, O,
 * dO, dQ, dK, dV, dbias and workspace must be 16-byte aligned, lse 4-byte;
 * rows or N < 1; workspace too small), TRI_ATTN_ERR_UNSUPPORTED (rows > 65535
 * or N > 46340), TRI_ATTN_ERR_NO_DEVICE, TRI_ATTN_ERR_CUDA (launch failure). */
size_t tri_attn_attention_bf16_workspace_bytes(int rows, int N);

/* o (bf16) and lse (fp32 [rows][H][N], natural log, +inf for a query whose
 * every key is masked; its o is 0) — the flash-style forward kernel of the
 * block (tri_attn_fwd, scores never in memory) run on the caller's Q, K, V
 * and bias, after two preparation kernels (q scaled; the bias in base 2 with
 * the mask folded in).  lse may be NULL. */
int tri_attn_attention_forward_bf16(const void *Q, const void *K, const void *V,
                                    const void *bias, const uint8_t *mask, int rows, int N,
                                    void *O, float *lse, void *workspace,
                                    size_t workspace_bytes, void *stream, unsigned flags);

/* Gradients dQ, dK, dV (fp32 [rows][H][N][d]) and dbias (fp32 [H][N][N],
 * summed over the rows) from the operands, the forward's o and lse (those of
 * tri_attn_attention_forward_bf16 on the same operands) and dO.  Five kernel
 * launches after the preparation: dQ (a CTA per 3 rows x 128 queries x head,
 * walking the keys), dK and dV (per 2 rows x 128 keys x head, walking the
 * queries), dbias (per 128 queries x 64 keys x head, walking every row, so it
 * is written once per element: no atomics, deterministic). */
int tri_attn_attention_backward_bf16(const void *Q, const void *K, const void *V,
                                     const void *bias, const uint8_t *mask, const void *O,
                                     const float *lse, const void *dO, int rows, int N,
                                     float *dQ, float *dK, float *dV, float *dbias,
                                     void *workspace, size_t workspace_bytes, void *stream,
                                     unsigned flags);

/* ---- block-level calls (BF16 handle): the 2D grid of devices -------------
 *
 * The Design-CP technical summary (§Metodología 1, 2D grid sharding) splits
 * the pair tensor over a sqrt(P) x sqrt(P) grid of devices and passes K/V
 * column blocks round a ring with an online softmax.  For a starting-node
 * block on such a grid, device (a, b) holds the pairs of rows A_a and columns
 * B_b; its outputs need the K/V of rows A_a over every column block (held
 * along its grid row) and the logit bias of the pairs (B_b, B_c) for every c.
 * These calls are the block's three kernels on caller-owned tensors, plus the
 * merge of partial attention outputs, so that a driver can move K/V, bias and
 * partial outputs between devices itself.  All device pointers, bf16 unless
 * stated, 16-byte aligned (lse: 4-byte); asynchronous on `stream`
 * (TRI_ATTN_FLAG_SYNC waits and returns the device status).  A block of pairs
 * is Z[rows][cols][c_z], taken as a starting-node problem whose rows are its
 * rows and whose keys are its columns.  Errors: TRI_ATTN_ERR_INVALID_ARG,
 * TRI_ATTN_ERR_UNSUPPORTED (F32 handle, rows > 65535, cols > 46340),
 * TRI_ATTN_ERR_ALIAS (block_gate: out overlaps Z without equalling it),
 * TRI_ATTN_ERR_NO_DEVICE, TRI_ATTN_ERR_CUDA. */

/* LayerNorm and the projections of every pair of the block: Q, K, V
 * [rows][H][cols][d] (q scaled by log2(e)/sqrt(d)) and the logit bias
 * [H][rows][tri_attn_bias_ld(cols)] (times log2(e); -3e38 at keys with
 * mask[col] == 0 and at columns >= cols).  mask: [cols] or NULL. */
int tri_attn_block_project(tri_attn_handle *h, const void *Z, int rows, int cols,
                           const uint8_t *mask, void *Q, void *K, void *V, void *bias,
                           void *stream, unsigned flags);

/* Flash attention of `rows` problem rows over one key block: o[r][h][j] =
 * softmax_k(q[r][h][j] . k[r][h][k] + bias[h][j][k]) v[r][h][k] for n queries
 * and n keys (the tensors of tri_attn_block_project: Q, K, V [rows][H][n][d],
 * bias [H][n][ld_bias], ld_bias >= tri_attn_bias_ld(n), a multiple of 8, with
 * its columns n..ld_bias-1 masked), O [rows][H][n][d] normalised within the
 * block, and lse [rows][H][n] (fp32, natural log of the block's sum; +inf when
 * the block has no unmasked key) or NULL. */
int tri_attn_block_attend(tri_attn_handle *h, const void *Q, const void *K, const void *V,
                          const void *bias, int ld_bias, int rows, int n, void *O, float *lse,
                          void *stream, unsigned flags);

/* The gate, the output projection and the residual of the block: out =
 * z + Wo (g * o) + bo with g recomputed from LayerNorm(z); O [rows][H][cols][d],
 * out [rows][cols][c_z] (out == Z allowed). */
int tri_attn_block_gate(tri_attn_handle *h, const void *Z, int rows, int cols, const void *O,
                        void *out, void *stream, unsigned flags);

/* Merge a block's partial output into a running one, for `count` queries:
 * lse = log(exp(lse_acc) + exp(lse_part)), O_acc = the weighted mean of O_acc
 * and O_part (weights exp(lse_x - lse)); a part with lse = +inf (no unmasked
 * key) has weight 0.  With `first` the accumulator is taken as empty (its
 * contents are not read).  O_acc [count][d] fp32 and lse_acc [count] fp32 are
 * updated in place; O_part [count][d] bf16, lse_part [count] fp32; O_out
 * [count][d] bf16 receives the merged output, or NULL.  No handle. */
int tri_attn_merge_partial(float *O_acc, float *lse_acc, const void *O_part,
                           const float *lse_part, long long count, int first, void *O_out,
                           void *stream, unsigned flags);

/* Release everything the handle owns.  NULL-safe.  Not stream-ordered:
 * call it after the work that uses the handle has completed. */
int tri_attn_destroy(tri_attn_handle *h);

/* Static string for a status code. */
const char *tri_attn_status_string(int code);

#ifdef __cplusplus
}
#endif

#endif /* TRI_ATTN_H */
