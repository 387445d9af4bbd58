/*
 * oft.h -- C ABI of the B200 (sm_100a) OFT hot path: an orthogonal (OFT)
 * adapter in front of a frozen low-precision linear layer, its backward, and
 * the active-expert-chunked MoE variant.
 *
 * Method (the pages describe it in words only; the formulas are the standard
 * OFT definition):
 *   - The frozen base stays in deployment precision (INT4 / FP4 / FP8) and a
 *     BF16 OFT adapter carries all gradients ("Orbit", chooseai.io news 4086,
 *     section "技术原理：低精度基座 + BF16 适配器 + OFT"; m.xxlwj.com 771001,
 *     sections on the Kimi-K2.6 and DeepSeek V4 Flash runs).
 *   - Per b x b block, Q is skew-symmetric and R = (I + Q)(I - Q)^-1 (Cayley).
 *   - Each sub-projection p of a fused QKV or gate/up weight has its own
 *     block-diagonal rotation R_p ("split-projection", chooseai.io news 4086,
 *     item "自定义适配器核函数" and item "分投影适配器支持").
 *   - Forward, row-major: X'_p = X R_p, Y_p = X'_p deq(W_p), Y = [Y_0 | Y_1 ...]
 *     (for a column token x this is y_p = W_p^T (R_p^T x)).
 *   - Backward skips the frozen weight's gradient (m.xxlwj.com 771001, section
 *     "技术细节", DeepSeek V4 paragraph): dX'_p = dY_p W_p^T, dX = sum_p dX'_p R_p^T,
 *     G_p = blockdiag(X^T dX'_p), dQ = skew part of 1/2 (I+R)^T G (I+R)^T.
 *   - MoE: router-selected experts are grouped into fixed-size chunks, each
 *     chunk is dequantised into a transient bf16 buffer and fed to a grouped
 *     GEMM (m.xxlwj.com 771001, section "技术细节", paragraph
 *     "Active-expert-chunked dequantization"; chooseai.io news 4086, section
 *     "对低精度 MoE 模型的专门优化").
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller.  The library
 *     allocates no device memory; scratch comes from a caller buffer `ws` of at
 *     least the size the matching *_workspace() call returns (16-byte aligned).
 *   - bf16 tensors are passed as uint16_t bit patterns.  Row-major, densely packed.
 *   - Every pointer must be 16-byte aligned.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls are
 *     asynchronous on that stream: they return after enqueueing work.
 *   - Return value: OFT_OK, or an error code.  On error nothing, or a prefix of
 *     the work, has been enqueued; oft_last_error() gives a message (per host
 *     thread).  No C++ exception crosses this ABI.
 *   - Device-side waits are bounded.  A wait that runs out sets a device error
 *     word and the kernel returns; oft_check_device() reports it as
 *     OFT_ERR_TIMEOUT.
 *   - Some calls (the MoE entry points, and oft_linear_fwd from 2048 tokens) run
 *     part of their work on a library-owned side stream of the device, forked from
 *     and joined back to `stream` with events, so they stay ordered with everything
 *     else on `stream`.  The side stream is created on the first such call on a
 *     device; make that call before capturing `stream` into a CUDA graph.  Calls
 *     from several host threads share it, which orders their side work but never
 *     breaks the ordering on each caller's stream.
 *
 * Weight storage (stored transposed, one row per output channel: W^T [N][K]):
 *   OFT_W_INT4   codes uint8 [N][K/2]  (element k in byte k/2, low nibble for
 *                even k, two's complement in [-8,7]); scales bf16 [K/G][N].
 *                dequant: w = bf16_rne(q * s).
 *   OFT_W_FP8    codes uint8 [N][K] (OCP e4m3fn); scales fp32 [N] (per output
 *                channel).  dequant: w = bf16_rne(f32_rne(v * s_n)).
 *   OFT_W_MXFP4  codes uint8 [N][K/2] (OCP e2m1, low nibble for even k);
 *                scales uint8 e8m0 [K/32][N].  dequant: w = v * 2^(e-127).
 *   An expert bank (n_experts > 1) stacks these arrays expert-major:
 *   codes [E][N][...], scales [E][...].
 *
 * Adapter storage: Q is bf16, the strict upper triangle of each skew block,
 * row-major ((0,1),(0,2),...,(0,b-1),(1,2),...), laid out [P][K/b][b(b-1)/2].
 * R is fp32 [P][K/b][b][b] row-major.  dQ is fp32 in Q's packed layout.
 */
#ifndef OFT_H_
#define OFT_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum {
  OFT_OK = 0,
  OFT_ERR_INVALID_ARG = 1, /* null or misaligned pointer, bad size or layout   */
  OFT_ERR_UNSUPPORTED = 2, /* b not in {16,32,64}, K % b, K % G, > 4 splits ... */
  OFT_ERR_CUDA = 3,        /* a CUDA runtime/driver call or launch failed       */
  OFT_ERR_TIMEOUT = 4,     /* a bounded device-side wait ran out               */
  OFT_ERR_WORKSPACE = 5    /* ws too small                                     */
};

enum { OFT_W_INT4 = 1, OFT_W_FP8 = 2, OFT_W_MXFP4 = 3 };

/* A frozen low-precision weight (or expert bank), see "Weight storage" above. */
typedef struct {
  int fmt;            /* OFT_W_INT4 | OFT_W_FP8 | OFT_W_MXFP4                  */
  const void* codes;  /* device                                                 */
  const void* scales; /* device                                                 */
  int d_in;           /* K                                                      */
  int d_out;          /* N (per expert for a bank)                              */
  int group;          /* INT4: 32, 64 or 128 along d_in; MXFP4: 32; FP8: 0      */
  int n_experts;      /* 0 or 1: a single weight; > 1: an expert bank           */
} oft_weight;

/* Sub-projections of a fused weight: d_out = sum(sizes[0..n-1]); each size is a
 * multiple of 8.  Sub-projection p owns output columns [off_p, off_p + sizes[p]). */
typedef struct {
  int n;
  int sizes[4];
} oft_split;

/* Library version string. */
const char* oft_version(void);

/* Message for the last error returned on this host thread ("" if none). */
const char* oft_last_error(void);

/* Synchronises `stream`, then reads and clears the device error word.
 * Returns OFT_OK, OFT_ERR_TIMEOUT if a bounded wait ran out since the last
 * check, or OFT_ERR_CUDA if the stream reports an error. */
int oft_check_device(void* stream);

/* Cayley build (the standard OFT parameterisation; the pages only name OFT).
 * Q: bf16 [n_blocks][b(b-1)/2] packed skew entries.  R: fp32 [n_blocks][b][b],
 * R = (I + Q)(I - Q)^-1, computed in fp32 by Gauss-Jordan elimination without
 * pivoting (I - Q has symmetric part I, so every pivot is >= 1 in exact
 * arithmetic).  b in {16, 32, 64}. */
int oft_build_rotation(const uint16_t* Q, int n_blocks, int b, float* R, void* stream);

/* Bytes of scratch oft_linear_fwd needs for this shape. */
size_t oft_linear_fwd_workspace(int M, const oft_weight* W, const oft_split* S, int b);

/* Split-projection OFT linear forward (chooseai.io news 4086, item "分投影适配器支持";
 * the frozen base dequantised on the fly, section "技术原理：低精度基座 + BF16 适配器 + OFT"):
 *   Y[:, cols of p] = (X R_p) deq(W_p).
 * X bf16 [M][K]; R fp32 [P][K/b][b][b] (from oft_build_rotation); Y bf16 [M][N].
 * fp32 accumulation, bf16 output (round to nearest even).  K % 32 == 0. */
int oft_linear_fwd(const uint16_t* X, int M, const oft_weight* W, const oft_split* S, int b, const float* R,
                   uint16_t* Y, void* ws, size_t ws_bytes, void* stream);

/* Bytes of scratch oft_linear_fwd_weight_side needs: two bf16 copies of the weight. */
size_t oft_linear_fwd_weight_side_workspace(const oft_weight* W);

/* Weight-side variant of oft_linear_fwd: the same product, with the rotation moved
 * onto the weight, Y_p = X (R_p deq(W_p)).  deq(W) is written to bf16, the rows of
 * each sub-projection are rotated (V_p^T = deq(W_p)^T R_p^T, bf16, on the tensor
 * cores), and one plain bf16 GEMM gives Y = X V over all N columns.  It does
 * 2 N K b rotation FLOP instead of 2 M K b P, so it is the cheaper rotation when
 * N < M P, and it keeps no X' copy.  Same arguments and limits as oft_linear_fwd;
 * here V is rounded to bf16 instead of X'. */
int oft_linear_fwd_weight_side(const uint16_t* X, int M, const oft_weight* W, const oft_split* S, int b,
                               const float* R, uint16_t* Y, void* ws, size_t ws_bytes, void* stream);

/* Bytes of scratch oft_linear_bwd needs for this shape. */
size_t oft_linear_bwd_workspace(int M, const oft_weight* W, const oft_split* S, int b);

/* Adapter backward (no gradient for the frozen weight: m.xxlwj.com 771001, section
 * "技术细节", DeepSeek V4 paragraph; the adapter alone carries the gradient,
 * chooseai.io news 4086, section "技术原理：低精度基座 + BF16 适配器 + OFT").
 * dY bf16 [M][N], X bf16 [M][K], R as in the forward.
 * Outputs: dX bf16 [M][K] = sum_p (dY_p W_p^T) R_p^T;
 *          dQ fp32 [P][K/b][b(b-1)/2], fully overwritten (not accumulated):
 *          dq_ij = D_ij - D_ji with D = 1/2 (I+R)^T G (I+R)^T, G = X_blk^T dX'_p,blk. */
int oft_linear_bwd(const uint16_t* dY, const uint16_t* X, int M, const oft_weight* W, const oft_split* S, int b,
                   const float* R, uint16_t* dX, float* dQ, void* ws, size_t ws_bytes, void* stream);

/* Bytes of scratch moe_chunked_oft_fwd needs (includes the transient bf16
 * chunk buffer of `chunk` experts). */
size_t moe_chunked_oft_workspace(int T, int E, int top_k, int chunk, const oft_weight* W_experts, int b);

/* Active-expert-chunked MoE OFT forward.
 * X bf16 [T][K]; logits fp32 [T][E]; W_experts: an INT4 expert bank with
 * d_out = 2 * n_proj per expert (gate rows, then up rows); Q_experts bf16
 * [E][2][K/b][b(b-1)/2] (gate, up).
 * Routing: top_k experts per token by logit (ties: lower expert id first),
 * weights = softmax over the selected logits.  Entries (t, k) are bucketed by
 * expert, stable in (t, k); active experts (count > 0) ascending are cut into
 * chunks of `chunk`; each chunk is dequantised to a bf16 buffer and run as one
 * grouped GEMM.  Y bf16 [T][2*n_proj] = sum_k w_tk [X_t R_e,g W_e,g | X_t R_e,u W_e,u].
 * Routing outputs (device, written every call):
 *   topk_idx int32 [T][top_k], topk_w fp32 [T][top_k], offsets int32 [E+1],
 *   bucket int32 [T*top_k] (entries t*top_k + k), chunk_table int32
 *   [ceil(E/chunk)][chunk] (-1 padded), n_active int32 [1].
 * Limits: E <= 512, top_k <= 8, chunk <= 32, 16 <= b <= 64. */
int moe_chunked_oft_fwd(const uint16_t* X, int T, const float* logits, int E, int top_k, int chunk,
                        const oft_weight* W_experts, int b, const uint16_t* Q_experts, uint16_t* Y,
                        int32_t* topk_idx, float* topk_w, int32_t* offsets, int32_t* bucket, int32_t* chunk_table,
                        int32_t* n_active, void* ws, size_t ws_bytes, void* stream);

/* Bytes of scratch moe_fused_oft_fwd needs (no chunk buffers). */
size_t moe_fused_oft_workspace(int T, int E, int top_k, int chunk, const oft_weight* W_experts, int b);

/* MoE OFT forward with the dequant fused into the grouped GEMM: the next step after
 * the chunked variant above (the chunk dequantisation is the pages' design: "技术细节"
 * of m.xxlwj.com 771001).  Same arguments, same routing outputs (chunk_table still
 * lists the active experts in chunks of `chunk`) and the same result Y.  There is no
 * bf16 chunk buffer: one launch covers every (active expert, projection) group and
 * decodes the INT4 codes straight into the tensor-core operand, so each active
 * expert's weight crosses HBM once, as 4-bit codes.  Same limits. */
int moe_fused_oft_fwd(const uint16_t* X, int T, const float* logits, int E, int top_k, int chunk,
                      const oft_weight* W_experts, int b, const uint16_t* Q_experts, uint16_t* Y,
                      int32_t* topk_idx, float* topk_w, int32_t* offsets, int32_t* bucket, int32_t* chunk_table,
                      int32_t* n_active, void* ws, size_t ws_bytes, void* stream);

/* Bytes of scratch moe_chunked_oft_layer_fwd needs: that of moe_chunked_oft_fwd plus
 * the routing tables, the down adapters' rotations, the gated activations (bf16
 * [T*top_k][n_proj]) and the per-slot down outputs (fp32 [T*top_k][d_in]). */
size_t moe_chunked_oft_layer_workspace(int T, int E, int top_k, int chunk, const oft_weight* W_experts,
                                       const oft_weight* W_down, int b);

/* Full MoE expert layer, forward: the chunked gate/up projections above, SwiGLU, and
 * a down projection with its own OFT adapter, every expert weight INT4 and
 * dequantised chunk by chunk ("技术细节" of m.xxlwj.com 771001).  For every (t, k)
 * routed to e, with [g | u] = [X_t R_e,g W_e,g | X_t R_e,u W_e,u]:
 *   h = silu(g) * u (fp32),  Z_tk = (h R_e,down) W_e,down,  Y_t = sum_k w_tk Z_tk.
 * W_down: INT4 bank with d_in = n_proj, d_out = d_in of W_experts (one row per output
 * channel, n_experts = E); Q_down bf16 [E][n_proj/b][b(b-1)/2].  Y bf16 [T][K].
 * h R_e,down is rounded to bf16 as the GEMM operand; everything else accumulates in
 * fp32.  Same limits as moe_chunked_oft_fwd, and n_proj % b == 0. */
int moe_chunked_oft_layer_fwd(const uint16_t* X, int T, const float* logits, int E, int top_k, int chunk,
                              const oft_weight* W_experts, const oft_weight* W_down, int b, const uint16_t* Q_experts,
                              const uint16_t* Q_down, uint16_t* Y, void* ws, size_t ws_bytes, void* stream);

/* Bytes of scratch moe_chunked_oft_bwd needs: routing tables, the active experts'
 * rotations, dY gathered in bucket order, two transposed bf16 chunk buffers,
 * and fp32 per-slot gradients (2 x T*top_k x K for dY W^T, T*top_k x K for the
 * rotated-back rows). */
size_t moe_chunked_oft_bwd_workspace(int T, int E, int top_k, int chunk, const oft_weight* W_experts, int b);

/* Adapter backward of the chunked MoE layer above (the frozen experts get no
 * gradient; the pages train the adapters only: "技术细节" of m.xxlwj.com 771001).
 * Inputs as for moe_chunked_oft_fwd, plus dY bf16 [T][2*n_proj] (gate | up), the
 * gradient of Y.  The routing is recomputed from `logits` (it is deterministic).
 * With D_p = dY_p[t] W_e,p^T for every (t, k) routed to e:
 *   dX bf16 [T][K]          = sum_k w_tk sum_p D_p R_e,p^T;
 *   dQ fp32 [E][2][K/b][b(b-1)/2], fully overwritten: the Cayley backward of
 *       G_e,p = sum over e's entries of blockdiag(X_t^T w_tk D_p); zero for experts
 *       that no token selected;
 *   dlogits fp32 [T][E], fully overwritten (NULL: not computed): through the
 *       softmax over the selected logits, w_tk (dw_tk - sum_j w_tj dw_tj) with
 *       dw_tk = <dY[t], Y_tk>; zero for logits that were not selected.
 * Each expert's weight is dequantised transposed, chunk by chunk, into a bf16
 * buffer ([chunk][gate/up][K][n_proj]) and contracted by one grouped GEMM per chunk.
 * Same limits as the forward; the result does not depend on scheduling. */
int moe_chunked_oft_bwd(const uint16_t* dY, const uint16_t* X, int T, const float* logits, int E, int top_k,
                        int chunk, const oft_weight* W_experts, int b, const uint16_t* Q_experts, uint16_t* dX,
                        float* dQ, float* dlogits, void* ws, size_t ws_bytes, void* stream);

/* ---- test hooks: single steps of the path, same kernels ---- */

/* Dequantise a single weight to bf16: out [N][K] (transpose = 0) or [K][N]. */
int oft_dequant_weight(const oft_weight* W, uint16_t* out, int transpose, void* stream);

/* Block-diagonal rotation: Xr[p] = X R_p for p < P.  Xr bf16 [P][M][K]. */
int oft_rotate(const uint16_t* X, int M, int K, int P, int b, const float* R, uint16_t* Xr, void* stream);

/* Cayley backward: dQ[blk] = pack(D - D^T), D = 1/2 (I+R)^T G (I+R)^T.
 * R, G fp32 [n_blocks][b][b]; dQ fp32 [n_blocks][b(b-1)/2]. */
int oft_cayley_backward(const float* R, const float* G, int n_blocks, int b, float* dQ, void* stream);

/* One chunk of the MoE transient dequant (the pages' "Active-expert-chunked
 * dequantization", section "技术细节" of m.xxlwj.com 771001), with the kernels and
 * launch shapes the MoE calls use.  bank: an INT4 expert bank (n_experts = E,
 * d_out = N per expert); chunk_table: device int32, slot s of chunk c is entry
 * c * chunk + s, an expert id or -1 (empty).  For every non-empty slot s of chunk
 * chunk_idx, with e its expert:
 *   transpose = 0: out[s][r][k]    = deq(W_e)[r][k],       out bf16 [chunk][N][K]
 *                  (the forward's chunk buffer; the full layer's down projections
 *                  use it with the down bank);
 *   transpose = 1: out[s][p][k][j] = deq(W_e)[p*N/2 + j][k], out bf16 [chunk][2][K][N/2]
 *                  (the backward's transposed buffer; N % 16 == 0).
 * Slots of -1 are left untouched.  Bit-exact: w = bf16_rne(q * s). */
int oft_moe_chunk_dequant(const oft_weight* bank, const int32_t* chunk_table, int chunk_idx, int chunk, int transpose,
                          uint16_t* out, void* stream);

/* Selects the GEMM inside oft_linear_fwd / oft_linear_bwd and
 * oft_linear_fwd_weight_side (test and benchmarking hook; process-wide, not
 * thread-safe against concurrent calls): 0 = by problem size (default: from 2048
 * tokens, deq(W) to a bf16 workspace and the plain tcgen05 GEMM on 2-SM pairs; below
 * that the fused-decode kernels, the 2-SM pair kernel for launches of at least two
 * waves of one-CTA tiles, and for forwards of 1 to 128 tokens the small-M split-K
 * kernel), 1 = always the one-CTA fused kernel, 2 = always the 2-SM pair fused
 * kernel, 3 = always the bf16 copy and the plain pair GEMM, 4 = always the bf16 copy
 * and the plain one-CTA GEMM.  The weight-side forward always takes the
 * plain GEMM: the pair kernel unless the mode is 4.  All compute the same product.  Query the *_workspace
 * sizes after setting the mode.  Returns OFT_ERR_INVALID_ARG for any other value. */
int oft_set_gemm_mode(int mode);

/* The static tile schedule of the plain GEMM (host only, launches nothing).  Groups
 * g < n_groups are m[g] x n[g] outputs contracted over k[g], cut into tile_rows x 256
 * tiles numbered group by group, row band by row band, as the kernel numbers them.
 * A worker is a CTA of the one-CTA kernel (tile_rows = 128) or a CTA pair of the 2-SM
 * kernel (tile_rows = 256).  When the groups differ in depth (the dX' product of
 * sub-projections of different widths), tiles in decreasing depth go to the worker
 * with the least work so far (ties to the lowest index).  For `grid` workers, sets
 * *used = 1 and writes off[0..grid] and tiles[0..off[grid]): worker c runs
 * tiles[off[c] .. off[c+1]) in that order.  Sets
 * *used = 0 and writes nothing else when the kernel runs round-robin instead: equal
 * depths, more than 2048 tiles or more than 160 workers.  `tiles` holds at least the
 * total tile count.  OFT_ERR_INVALID_ARG: a NULL pointer, n_groups outside 1..32,
 * tile_rows not 128 or 256, grid < 1. */
int oft_gemm_schedule(int n_groups, const int* m, const int* n, const int* k, int tile_rows, int grid, int* used,
                      int* off, int* tiles);

/* Launches a kernel that waits on a barrier nothing will complete, bounded by
 * timeout_us microseconds; it must return on its own and set the device error
 * word.  Exercises the timeout path without faulting or hanging the GPU. */
int oft_debug_bounded_wait(int timeout_us, void* stream);

/* ---- forward without a caller workspace ----
 * The pages have no counterpart to this entry point; it exists for callers that
 * cannot allocate device memory or pass a workspace: for example a runtime
 * whose memory pool already owns all free HBM (a serving engine that reserves
 * the card for its KV cache, where cudaMalloc would fail), or a plugin
 * interface whose signature carries only inputs and outputs.
 *
 * Same result as oft_linear_fwd given a workspace of OFT_NOALLOC_SCRATCH_BYTES
 * (same kernels, same launch sequence), but the scratch (rotated activations and,
 * from 2048 tokens when it fits too, the bf16 copy of the weight) lives in a
 * fixed file-scope device array of OFT_NOALLOC_SCRATCH_BYTES (32 MiB) that every
 * GPU loading this library holds until the process exits.  Allocates nothing:
 * no cudaMalloc/cudaFree and no allocating library call.
 *   - From 2048 tokens the bf16-weight path runs when X' (2 P M K bytes) and the
 *     weight copy (2 N K bytes) both fit in the array, else the fused-decode path,
 *     which needs X' only.
 *   - Shapes whose X' alone exceeds OFT_NOALLOC_SCRATCH_BYTES are rejected with
 *     OFT_ERR_WORKSPACE and a message giving both sizes.
 *   - The first call on a device (with that device current) looks up the
 *     array's device address; make that first call before any stream capture.
 *   - All calls share the one array and it keeps the last call's contents.
 *     Every scratch byte a call reads is written earlier in the same call, so
 *     nothing needs clearing, but calls whose kernels overlap on the GPU (two
 *     streams, or two host threads) race on the array: serialise them. */
#define OFT_NOALLOC_SCRATCH_BYTES (32u << 20)

int oft_linear_fwd_noalloc(const uint16_t* X, int M, const oft_weight* W, const oft_split* S, int b,
                           const float* R, uint16_t* Y, void* stream);

/* ---- profiling hooks (measurement plumbing, not part of the method) ---- */

/* Kernel classes reported by oft_profile_end(). */
enum {
  OFT_K_GEMM = 0,     /* tcgen05 GEMM (forward, dX', MoE grouped)          */
  OFT_K_ROTATE = 1,   /* block rotations (X R, dX' R^T, MoE gather-rotate) */
  OFT_K_DEQUANT = 2,  /* standalone dequantisation (incl. MoE chunks)      */
  OFT_K_CAYLEY = 3,   /* Cayley forward / backward                          */
  OFT_K_GRAD = 4,     /* dR = X^T dX' partial reductions                    */
  OFT_K_ROUTE = 5,    /* MoE top-k, bucketing, combine                      */
  OFT_K_NUM = 6
};

/* Starts recording a CUDA event pair around every kernel this library launches
 * (on the launch stream), for up to max_launches launches.  Host-side only:
 * creates events, allocates no device memory. */
int oft_profile_begin(int max_launches);

/* Synchronises the recorded events, stops recording and writes, per kernel
 * class (n_kinds <= OFT_K_NUM entries), the summed device time in ms and the
 * number of launches.  Launches beyond max_launches are counted but not timed;
 * *dropped (optional) receives how many. */
int oft_profile_end(double* ms_by_kind, int* launches_by_kind, int n_kinds, int* dropped);

#ifdef __cplusplus
}
#endif

#endif /* OFT_H_ */
