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
 * The first call on a device looks up the array's address (set-up work: make
 * it before any stream capture).  Nothing is allocated and nothing needs
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

/* Workspace of fp8_linear_w8a8: the quantised activations and their scales. */
size_t fp8_linear_workspace_bytes(int32_t M, int32_t K);

/* x (bf16 [M, K]) -> per-token quantisation into ws -> fp8_gemm_w8a8.
 * Same constraints as the two calls; dev_err as in fp8_gemm_w8a8. */
rola_status_t fp8_linear_w8a8(int32_t M, int32_t N, int32_t K, const uint16_t* x,
                              const uint8_t* w_q, const float* w_scale, uint16_t* y, void* ws,
                              size_t ws_bytes, int32_t* dev_err, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* ROLA_H */
