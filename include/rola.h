/*
 * rola.h -- C ABI of librola.so: RoLA hybrid block-sparse + rotary low-rank
 * linear attention for video diffusion transformers, and the W8A8 FP8 E4M3
 * projections around it, for NVIDIA B200 (sm_100a).
 *
 * The method: SparkDiffusion write-up (「首次定义“高稀疏陷阱”」, 0539edu.com
 * news page), section 05 "RoLA": a block-sparse branch keeps the high-energy
 * query-key block interactions, and a rotary-positioned low-rank linear branch
 * restores the global context that sparsification dropped; section 07: the
 * attention and FFN projections run as W8A8 FP8 E4M3 with activation scaling
 * and type conversion fused.  The arXiv listing of the SparkDiffusion paper
 * (montaan.com, "Sources") names the sibling idea "3D RoPE-driven
 * Sparse-LowRank Attention", hence the 3-D rotary embedding.  The pages print
 * no formula; the concrete form fixed here is stated at each entry point.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every tensor pointer is a DEVICE pointer owned by the caller (except in
 *    rola_layer_fwd_host, which takes host buffers); the library never
 *    allocates device memory.  Scratch space, where needed, is a
 *    caller-provided workspace whose size a *_workspace_bytes() call reports.
 *  - "bf16" buffers hold bfloat16 bit patterns (uint16_t).
 *  - Calls are asynchronous on the given stream (a cudaStream_t; NULL is the
 *    legacy default stream) and stateless, apart from the two copy streams and
 *    seven events rola_layer_fwd_host creates once per device; concurrent
 *    calls on different streams are safe as long as their buffers do not
 *    overlap.
 *  - Shape, pointer and alignment problems are reported synchronously as a
 *    status code and nothing is launched.  A failed launch returns
 *    ROLA_ERR_CUDA.  No C++ exception crosses this boundary.
 *  - Device-side checks (a block index out of range or not strictly
 *    ascending, a bounded wait that ran out) never trap: the kernel skips the
 *    offending work, ORs a ROLA_DEVERR_* bit into *dev_err (one int32 the
 *    caller zeroes), and returns.
 *  - q, k, v and out are [B, N, H, d] row-major (token-major, heads
 *    interleaved as in a DiT's [tokens, H*d] activations).  Tokens sit on a
 *    (T, Hg, W) latent grid in frame-major raster order:
 *    token n -> t = n / (Hg*W), y = (n / W) % Hg, x = n % W.
 *  - Blocks are `block` consecutive tokens; n_blocks = ceil(N / block); the
 *    last block may be partly padding, and padding never takes part in any
 *    sum, mean or softmax.
 */
#ifndef ROLA_H
#define ROLA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ROLA_OK = 0,
  ROLA_ERR_INVALID_ARG = 1,   /* null pointer, inconsistent or out-of-range shape */
  ROLA_ERR_UNSUPPORTED = 2,   /* valid shape this build has no kernel for        */
  ROLA_ERR_WORKSPACE = 3,     /* workspace missing, too small or misaligned      */
  ROLA_ERR_CUDA = 4,          /* a CUDA runtime call or launch failed            */
  ROLA_ERR_ALIGNMENT = 5      /* a pointer misses the documented alignment       */
} rola_status_t;

/* Bits a kernel ORs into *dev_err. */
#define ROLA_DEVERR_BAD_INDEX 0x1   /* idx entry out of [0, n_blocks) or not ascending */
#define ROLA_DEVERR_TIMEOUT 0x2     /* a bounded pipeline wait ran out                  */

/* Every size is at least 1: an empty batch, head set or grid is rejected with
 * ROLA_ERR_INVALID_ARG (there is nothing to launch). */
typedef struct {
  int32_t B, H, d;       /* batch, heads, head dim (64 or 128)                    */
  int32_t N;             /* valid tokens; must equal T * Hg * W                   */
  int32_t T, Hg, W;      /* latent grid (frames, height, width)                   */
  int32_t block;         /* tokens per block: 64 or 128                            */
  int32_t k_b;           /* kept key blocks per query block, 1..n_blocks          */
  int32_t r;             /* rank of the linear branch: 16 or 32 (even, <= d)      */
  float rope_base;       /* rotary base, e.g. 10000                                */
} rola_shape_t;

/* Human-readable name of a status code (static string, never NULL). */
const char* rola_status_string(rola_status_t s);

/* ceil(N / block), or -1 for an invalid shape pointer. */
int32_t rola_num_blocks(const rola_shape_t* shape);

/* Kept blocks for a sparsity given in permille:
 * ceil((1000 - sparsity_permille) * n_blocks / 1000), computed in integers so
 * that 97 % of 100 blocks keeps exactly 3.  SparkDiffusion write-up, section
 * 01: 90 % -> 97 % sparsity keeps 3 % instead of 10 % of the blocks.
 * Returns -1 for n_blocks < 1 or a sparsity outside [0, 1000). */
int32_t rola_kb_from_sparsity(int32_t n_blocks, int32_t sparsity_permille);

/* ---------------------------------------------------------------- selector */

/* Workspace rola_select_blocks needs: 256-byte aligned, contents scratch.
 * 0 for an invalid shape. */
size_t rola_select_workspace_bytes(const rola_shape_t* shape);

/* The same number under the generic name: rola_select_blocks is the only one
 * of the three hot-path steps (select, states, attention) that takes a
 * workspace. */
size_t rola_workspace_bytes(const rola_shape_t* shape);

/* Block selector (write-up section 05: keep the high-energy query-key block
 * interactions).  For every (b, h): mean-pool q and k over each block's valid
 * tokens, score sigma[a][j] = qbar_a . kbar_j / sqrt(d), and keep, per query
 * block a, the k_b key blocks that come first in the order (-sigma, j) --
 * larger score first, ties to the lower index; no block is forced in.
 * Pooling and scores are computed in float64 (the bf16 block sums are exact),
 * so the selection is decided in float64.
 *   q, k        bf16 [B, N, H, d], 16-byte aligned
 *   idx         out, int32 [B, H, n_blocks, k_b], each row strictly ascending
 *   scores_opt  out, optional (NULL to skip), float64 [B, H, n_blocks, n_blocks]
 *   ws          workspace of rola_select_workspace_bytes(shape) bytes */
rola_status_t rola_select_blocks(const rola_shape_t* shape, const uint16_t* q, const uint16_t* k,
                                 int32_t* idx, double* scores_opt, void* ws, size_t ws_bytes,
                                 void* stream);

/* The selector above without a caller workspace: its scratch is a fixed
 * 16 MiB device array inside this library (the pages describe no such call;
 * it exists for callers that cannot provide device memory at the call site).
 * Same inputs, output and results as rola_select_blocks (no scores output).
 * ROLA_ERR_WORKSPACE when rola_select_workspace_bytes(shape) exceeds 16 MiB.
 * Every call looks up the array's device address on the current device, so
 * the entry point stays valid across a device reset; the first call on a
 * device also loads the library's device code there (set-up work: make it
 * before any stream capture).  Nothing is allocated and nothing needs
 * clearing; calls that overlap in time on one device share the array and
 * race, so callers serialise them. */
rola_status_t rola_select_blocks_noalloc(const rola_shape_t* shape, const uint16_t* q,
                                         const uint16_t* k, int32_t* idx, void* stream);

/* ---------------------------------------------------------------- states */

/* Linear-branch key/value states (write-up section 05: the low-rank linear
 * branch restores the context of the dropped blocks).  Per (b, h) with the
 * head's projection P_h [d, r]:
 *   psi_j = phi(k_j P_h), phi(u) = elu(u) + 1 (u + 1 for u > 0, else e^u);
 *   rho_j = R(t_j, y_j, x_j) psi_j, the 3-D rotary rotation of interleaved
 *           pairs (2p, 2p+1): the first r_t = r - 4 floor(r/6) dims turn with
 *           t, the next r_h = 2 floor(r/6) with y, the last r_w = r_h with x;
 *           pair m of an axis with r_a dims turns by pos * base^(-2m / r_a);
 *   S_blk[b,h,j] = sum over the block's valid keys of rho v^T   (r x d)
 *   z_blk[b,h,j] = sum over the block's valid keys of psi       (r)
 *   S_glb[b,h]   = sum_j S_blk[b,h,j],   z_glb[b,h] = sum_j z_blk[b,h,j]
 *     (the totals are summed in float64 and stored as float32).
 *   k, v   bf16 [B, N, H, d], 16-byte aligned;  P  bf16 [H, d, r]
 *   S_blk  out, fp32 [B, H, n_blocks, r, d];  z_blk  out, fp32 [B, H, n_blocks, r]
 *   S_glb  out, fp32 [B, H, r, d];            z_glb  out, fp32 [B, H, r] */
rola_status_t rola_block_states(const rola_shape_t* shape, const uint16_t* k, const uint16_t* v,
                                const uint16_t* P, float* S_blk, float* z_blk, float* S_glb,
                                float* z_glb, void* stream);

/* ---------------------------------------------------------------- attention */

/* RoLA attention forward for a given block mask.  For query token n in
 * query block a with kept set K_a = idx[b,h,a,:] and complement U_a:
 *   o_sp  = softmax over the valid tokens of the blocks in K_a of
 *           q_n . k_j / sqrt(d), applied to v;
 *   S_U   = S_glb - sum_{j in K_a} S_blk[j],  z_U likewise;
 *   o_lin = rho_n^T S_U / (psi_n^T z_U)   (rotation in the numerator only),
 *           and 0 when U_a is empty;
 *   out   = o_sp + gate[h] * o_lin, rounded to bf16.
 * The softmax runs with fp32 accumulation and bf16 probabilities for P.V, on
 * the tensor cores (tcgen05, accumulators in tensor memory).  Rows of padding
 * are not written.
 *   q, k, v  bf16 [B, N, H, d], 16-byte aligned
 *   idx      int32 [B, H, n_blocks, k_b], rows strictly ascending; a bad entry
 *            is skipped and sets ROLA_DEVERR_BAD_INDEX
 *   P        bf16 [H, d, r];  S_blk, z_blk, S_glb, z_glb as produced by
 *            rola_block_states (S_blk, S_glb 16-byte aligned);  gate  fp32 [H]
 *   out      out, bf16 [B, N, H, d], 16-byte aligned
 *   dev_err  one int32 the caller zeroed; may be NULL (then device-side
 *            problems are still skipped but not reported)
 * For d = 128, 128-token blocks and k_b <= 256 a persistent kernel walks pairs
 * of adjacent query blocks over the union of their kept lists; it reads the
 * states 32 bytes and P 16 bytes at a time, so it is chosen when S_blk and
 * S_glb are 32-byte and P 16-byte aligned (otherwise, and for the other
 * shapes, a one-tile kernel runs; both give the results stated above). */
rola_status_t rola_attention_fwd(const rola_shape_t* shape, const uint16_t* q, const uint16_t* k,
                                 const uint16_t* v, const int32_t* idx, const uint16_t* P,
                                 const float* S_blk, const float* z_blk, const float* S_glb,
                                 const float* z_glb, const float* gate, uint16_t* out,
                                 int32_t* dev_err, void* stream);

/* rola_attention_fwd with the bound on each of the kernel's pipeline waits
 * given in nanoseconds (rola_attention_fwd uses 1 s).  The pages describe no
 * such call: it is this library's failure detection.  A wait that runs out
 * makes its CTA stop, wait (at most 1 s each) for the copies and MMAs it has
 * in flight, free its tensor memory and return; the launch's later CTAs skip
 * their work, ROLA_DEVERR_TIMEOUT is ORed into *dev_err and `out` is
 * incomplete.  The device stays usable: later calls run normally.
 * wait_limit_ns = 0 makes a wait give up as soon as it finds its stage not
 * ready yet, so a test can run the timeout path without any fault.  Other
 * arguments, results and errors as rola_attention_fwd. */
rola_status_t rola_attention_fwd_bounded(const rola_shape_t* shape, const uint16_t* q,
                                         const uint16_t* k, const uint16_t* v, const int32_t* idx,
                                         const uint16_t* P, const float* S_blk, const float* z_blk,
                                         const float* S_glb, const float* z_glb, const float* gate,
                                         uint16_t* out, int32_t* dev_err, uint64_t wait_limit_ns,
                                         void* stream);

/* ---------------------------------------------------------------- backward */

/* rola_attention_fwd (d = 128, 128-token blocks, k_b <= 256, n_blocks <= 1024)
 * that also saves what rola_attention_bwd reads:
 *   out_lo  bf16 [B, N, H, d]: the output's rounding residual, bf16(o - out)
 *        with o the float32 result (out + out_lo carries ~16 mantissa bits,
 *        which the backward's D = dout . o_sp needs);
 *   lse  float [B, H, N]: natural log of sum over the kept valid keys of
 *        exp(q . k / sqrt(d)) (-inf for a row without kept blocks);
 *   den  float [B, H, N]: the linear branch's denominator psi_q . z_U (NaN
 *        when the complement is empty).
 * Other arguments, results and errors as rola_attention_fwd; other shapes:
 * ROLA_ERR_UNSUPPORTED.  S_blk and S_glb 32-byte aligned, P 16-byte. */
rola_status_t rola_attention_fwd_train(const rola_shape_t* shape, const uint16_t* q, const uint16_t* k,
                                       const uint16_t* v, const int32_t* idx, const uint16_t* P,
                                       const float* S_blk, const float* z_blk, const float* S_glb,
                                       const float* z_glb, const float* gate, uint16_t* out,
                                       uint16_t* out_lo, float* lse, float* den, int32_t* dev_err,
                                       void* stream);

/* Workspace of rola_attention_bwd (256-byte aligned), 0 for an invalid or
 * unsupported shape. */
size_t rola_attention_bwd_workspace_bytes(const rola_shape_t* shape);

/* Gradients of sum(dout * out) for the forward above, the block mask held
 * fixed (selection passes no gradient).  The SparkDiffusion write-up (section
 * 05) and project blog ("A simple staging principle", item 1) adapt the dense
 * model to 97 % sparsity by a short sparse warm-up that trains through RoLA;
 * the pages print no backward, so the gradient is the chain rule through the
 * forward's steps in reverse: the sparse branch from the saved log-sum-exp
 * (P = exp(S / sqrt(d) - lse), D = dout . o_sp), the linear branch through
 * o_lin = rho_q^T S_U / (psi_q . z_U), the complement S_U = S - sum_kept S_b,
 * the block states S_b = sum rho_k v^T, z_b = sum psi_k, the rotary
 * rotation, the feature map elu + 1 and the projection P_h.
 *   q, k, v, idx, P, S_blk, z_blk, S_glb, z_glb, gate: the forward's inputs
 *   out, out_lo, lse, den: its output and saved quantities (rola_attention_fwd_train)
 *   dout   bf16 [B, N, H, d], the gradient reaching out
 *   dq, dk, dv  out, bf16 [B, N, H, d] (padding rows not written)
 *   dP     out, float [H, d, r];   dgate  out, float [H]
 * Two passes, no atomics (deterministic): a query-major pass (dq, the query
 * side of the linear branch, D) and a key-major pass over the query blocks
 * that keep each key block (dk, dv, the key side); contractions on the
 * tensor cores (tcgen05).  Supported: d = 128, 128-token blocks, r 16 or 32,
 * k_b <= 256, n_blocks <= 1024 (else ROLA_ERR_UNSUPPORTED).  16-byte aligned
 * activations and gradients; dev_err as in rola_attention_fwd. */
rola_status_t rola_attention_bwd(const rola_shape_t* shape, const uint16_t* q, const uint16_t* k,
                                 const uint16_t* v, const int32_t* idx, const uint16_t* P,
                                 const float* S_blk, const float* z_blk, const float* S_glb,
                                 const float* z_glb, const float* gate, const uint16_t* out,
                                 const uint16_t* out_lo, const float* lse, const float* den,
                                 const uint16_t* dout, uint16_t* dq,
                                 uint16_t* dk, uint16_t* dv, float* dP, float* dgate, void* ws,
                                 size_t ws_bytes, int32_t* dev_err, void* stream);

/* ---------------------------------------------------------------- whole layer */

/* Workspace of rola_layer_fwd: selector scratch, idx and the states. */
size_t rola_layer_workspace_bytes(const rola_shape_t* shape);

/* One RoLA attention layer: the selection, block states and attention of
 * rola_select_blocks, rola_block_states and rola_attention_fwd back to back on
 * `stream`, intermediates in `ws` (256-byte aligned, rola_layer_workspace_bytes
 * bytes).  For d = 128 and 128-token blocks one pass over q, k and v computes
 * both the block means and the block states (same results as the separate
 * calls; q, k, v and P 16-byte aligned).  idx_out (optional, NULL to skip)
 * receives a copy of the kept-block index. */
rola_status_t rola_layer_fwd(const rola_shape_t* shape, const uint16_t* q, const uint16_t* k,
                             const uint16_t* v, const uint16_t* P, const float* gate, uint16_t* out,
                             int32_t* idx_out, void* ws, size_t ws_bytes, int32_t* dev_err,
                             void* stream);

/* rola_layer_fwd with CUDA events recorded on `stream` at its stage
 * boundaries, for profiling.  `events` points to n_events cudaEvent_t the
 * caller created (or is NULL, which makes the call identical to
 * rola_layer_fwd; n_events is then ignored):
 *   n_events = 3: before the first kernel, once the selection and the block
 *                 states are done, after the attention kernel;
 *   n_events = 5: before the first kernel, after the pass over q, k, v
 *                 (block means and states), after the scores and top-k,
 *                 after the state totals, after the attention kernel.
 * (For shapes without the fused pass, the second event follows the
 * selector and the fourth the block states.)  Other counts:
 * ROLA_ERR_INVALID_ARG. */
rola_status_t rola_layer_fwd_timed(const rola_shape_t* shape, const uint16_t* q, const uint16_t* k,
                                   const uint16_t* v, const uint16_t* P, const float* gate,
                                   uint16_t* out, int32_t* idx_out, void* ws, size_t ws_bytes,
                                   int32_t* dev_err, void* stream, void* const* events,
                                   int32_t n_events);

/* Options of rola_layer_fwd_ex. */
typedef struct {
  /* Per-head kept counts, device int32 [H] (each in 1..shape->k_b), or NULL
   * for shape->k_b in every head.  The Video-Generation-101 chapter page on
   * sparse attention lists head-adaptive block sparsity (AdaSpa) among the
   * sparse-attention methods: heads differ in how concentrated their
   * attention is, so each head may keep its own number of blocks.  idx rows
   * keep the stride shape->k_b; a head keeping kb_h blocks fills the first
   * kb_h entries of its rows (ascending) and the selector writes -1 into the
   * rest.  A count outside 1..k_b is clamped into it and reported through
   * ROLA_DEVERR_BAD_INDEX. */
  const int32_t* kb_per_head;
  /* 0: select the mask and (when idx_io is not NULL) write it to idx_io.
   * Nonzero: idx_io holds the mask to use (for example the one selected at an
   * earlier diffusion step: the same chapter page lists cross-step reuse of
   * the sparsity pattern, RAPID); no selection kernel runs, the block states
   * and the attention run as usual. */
  int32_t reuse_mask;
} rola_layer_opts_t;

/* rola_layer_fwd_timed with options (opts may be NULL: then the call equals
 * rola_layer_fwd_timed with idx_out = idx_io).  idx_io: int32 [B, H,
 * n_blocks, k_b], an output unless opts->reuse_mask, then an input (required,
 * rows validated by the attention kernel as in rola_attention_fwd).
 * events / n_events as in rola_layer_fwd_timed (NULL / 0 for none); with a
 * reused mask the scores-and-top-k interval is empty. */
rola_status_t rola_layer_fwd_ex(const rola_shape_t* shape, const rola_layer_opts_t* opts,
                                const uint16_t* q, const uint16_t* k, const uint16_t* v,
                                const uint16_t* P, const float* gate, uint16_t* out,
                                int32_t* idx_io, void* ws, size_t ws_bytes, int32_t* dev_err,
                                void* stream, void* const* events, int32_t n_events);

/* Number of kernels one rola_layer_fwd call launches for `shape` (0 for an
 * invalid or unsupported shape); memory copies are not counted. */
int rola_layer_kernel_launches(const rola_shape_t* shape);

/* Device staging the host-buffer variant needs: P and gate of all heads, two
 * slots of q, k, v and out for one head group, and the layer workspace of one
 * head group. */
size_t rola_layer_host_workspace_bytes(const rola_shape_t* shape);

/* The same layer with q, k, v, P, gate and out in HOST memory (pinned for
 * asynchronous copies).  Every (b, h) is independent, so the heads are taken
 * in groups whose slice of a token row is at least 2 KB (8 heads of d = 128):
 * a group's q, k, v are copied (strided rows) into one of two device slots
 * while the previous group computes, and each group's output is copied back
 * into its columns of out while the next one computes.  The copies run on two
 * streams the library creates once per device; events order them after the
 * work already on `stream`, the compute runs on `stream`, and `stream` waits
 * for the last copy back before anything enqueued after this call.  The call
 * returns once the work is enqueued; the caller synchronises `stream` before
 * reading `out`.  Calls on one device are enqueued under a lock.  The result
 * is bit-identical to rola_layer_fwd.  ws: device workspace of
 * rola_layer_host_workspace_bytes(shape) bytes, 256-byte aligned; dev_err:
 * device pointer or NULL. */
rola_status_t rola_layer_fwd_host(const rola_shape_t* shape, const uint16_t* q_host,
                                  const uint16_t* k_host, const uint16_t* v_host,
                                  const uint16_t* P_host, const float* gate_host,
                                  uint16_t* out_host, void* ws, size_t ws_bytes, int32_t* dev_err,
                                  void* stream);

/* ---------------------------------------------------------------- FP8 W8A8 */

/* Per-row E4M3 quantisation (write-up section 07: W8A8 FP8 E4M3 with fused
 * activation scaling and cast).  For each row m of x [M, K]:
 *   amax = max_k |x[m,k]|;  scale[m] = amax / 448 (1 if amax == 0);
 *   q[m,k] = E4M3(x[m,k] * (448 / amax)), round to nearest even, saturating,
 *   with the reciprocal and the product each rounded to float32.
 * fp8_quantize_rows_bf16 takes bf16 activations (per-token scales);
 * fp8_quantize_weight takes fp32 weights [N, K] (per-output-channel scales).
 * K must be a multiple of 16. */
rola_status_t fp8_quantize_rows_bf16(int32_t M, int32_t K, const uint16_t* x, uint8_t* x_q,
                                     float* scale, void* stream);
rola_status_t fp8_quantize_weight(int32_t N, int32_t K, const float* w, uint8_t* w_q,
                                  float* w_scale, void* stream);

/* y[m,n] = bf16( (sum_k dec(x_q[m,k]) dec(w_q[n,k])) * x_scale[m] * w_scale[n] )
 * on the tensor cores (tcgen05 kind::f8f6f4, fp32 accumulation in tensor
 * memory); write-up section 07 (W8A8 FP8 E4M3 projections).
 * x_q [M, K], w_q [N, K] row-major E4M3 bytes (both K-major), x_scale [M],
 * w_scale [N] float32, y [M, N] row-major bf16; all device pointers, owned by
 * the caller.  N a multiple of 32, K a multiple of 16 (a K tail inside the
 * last 128-wide slice is zero-padded by the copy engine).  x_q, w_q, y and
 * w_scale 16-byte aligned, x_scale 4-byte aligned.  Asynchronous on `stream`.
 * dev_err: optional device int32 that receives ROLA_DEVERR_TIMEOUT if a
 * pipeline wait ran out (y is then incomplete). */
rola_status_t fp8_gemm_w8a8(int32_t M, int32_t N, int32_t K, const uint8_t* x_q,
                            const float* x_scale, const uint8_t* w_q, const float* w_scale,
                            uint16_t* y, int32_t* dev_err, void* stream);

/* Activation applied in the GEMM epilogue (fp8_gemm_w8a8_act). */
#define ROLA_ACT_NONE 0
#define ROLA_ACT_GELU_TANH 1 /* 0.5 u (1 + tanh(sqrt(2/pi) (u + 0.044715 u^3))) */

/* fp8_gemm_w8a8 with an activation applied to the scaled fp32 product
 * before the bf16 rounding: y = bf16(act(product * x_scale * w_scale)).
 * GELU in its tanh form serves the FFN's up projection (write-up section 07:
 * the FFN projections run in W8A8 FP8 too; the pages name no activation, so
 * this library takes the tanh form).  act must be ROLA_ACT_NONE or
 * ROLA_ACT_GELU_TANH, else ROLA_ERR_INVALID_ARG; other arguments as
 * fp8_gemm_w8a8. */
rola_status_t fp8_gemm_w8a8_act(int32_t M, int32_t N, int32_t K, const uint8_t* x_q,
                                const float* x_scale, const uint8_t* w_q, const float* w_scale,
                                int32_t act, uint16_t* y, int32_t* dev_err, void* stream);

/* Workspace of fp8_linear_w8a8: the quantised activations and their scales. */
size_t fp8_linear_workspace_bytes(int32_t M, int32_t K);

/* x (bf16 [M, K]) -> per-token quantisation into ws -> fp8_gemm_w8a8.
 * Same constraints as the two calls; dev_err as in fp8_gemm_w8a8. */
rola_status_t fp8_linear_w8a8(int32_t M, int32_t N, int32_t K, const uint16_t* x,
                              const uint8_t* w_q, const float* w_scale, uint16_t* y, void* ws,
                              size_t ws_bytes, int32_t* dev_err, void* stream);

/* Workspace of fp8_ffn_w8a8 (256-byte aligned): codes and scales of x, the
 * bf16 hidden activation [M, F], and its codes and scales. */
size_t fp8_ffn_workspace_bytes(int32_t M, int32_t D, int32_t F);

/* The transformer block's FFN with both projections in W8A8 FP8 E4M3
 * (write-up section 07: the FFN projections are quantised like the attention
 * ones):  y = W2 gelu_tanh(W1 x)  for x bf16 [M, D], w1_q [F, D], w2_q [D, F]
 * (E4M3 bytes, K-major) with per-output-channel scales w1_scale [F],
 * w2_scale [D], and y bf16 [M, D].  Steps, in order: per-token quantisation of
 * x; the up projection with GELU in its epilogue, written as bf16 [M, F] into
 * the workspace; per-token quantisation of that hidden activation; the down
 * projection.  D and F multiples of 32 (and of 16 for the quantisation), at
 * most 16384.  Device pointers owned by the caller; ws of
 * fp8_ffn_workspace_bytes(M, D, F) bytes; dev_err as in fp8_gemm_w8a8. */
rola_status_t fp8_ffn_w8a8(int32_t M, int32_t D, int32_t F, const uint16_t* x,
                           const uint8_t* w1_q, const float* w1_scale, const uint8_t* w2_q,
                           const float* w2_scale, uint16_t* y, void* ws, size_t ws_bytes,
                           int32_t* dev_err, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* ROLA_H */
