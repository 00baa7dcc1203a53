/*
 * moe_b200.h -- C ABI of the DeepSeekMoE layer forward for one NVIDIA B200
 * (sm_100a).
 *
 * The layer (per token t, N routed experts, one shared expert):
 *   s_i   = sigmoid(x_t . e_i)                       affinity
 *   s'_i  = s_i + b_i                                biased score, selection only
 *   keep the topG of G contiguous expert groups by group score (sum of the two
 *   largest s' in the group), then idx = the K largest s' inside kept groups
 *   gate_k = s_{idx_k} / sum_j s_{idx_j}             un-biased, renormalised
 *   y_t = E_shared(x_t) + sum_k gate_k * E_{idx_k}(x_t)
 *   E(a) = (silu(a W1^T) * (a W3^T)) W2^T            SwiGLU expert
 *   after the step: b_i -= gamma if expert i took more than T*K/N rows,
 *                   b_i += gamma if it took fewer.
 *
 * Sources (web pages on DeepSeek-V3):
 *   [P1] "DeepSeek-V3 高效训练关键技术分析" (mhpq.cn): §1.1 DeepSeekMoE (1 shared +
 *        256 routed experts, 8 active), §1.2 auxiliary-loss-free balancing (bias
 *        adjusted every step from the measured load), §2.2 forward order
 *        DISPATCH -> MLP -> COMBINE, §3.1 each token reaches at most 4 nodes,
 *        §4.1 FP8 GEMMs with 1x128 activation / 128x128 weight scaling and
 *        online max-abs scales, FP32 accumulation.
 *   [P2] "解读 DeepSeek-V3" reading notes (gkm0120.cn), Q3: the bias enters
 *        routing only, never the gate value.
 *   [P4] DeepSeek-V3 walk-through (kaiyunto.com), DeepSeekMoE paragraphs:
 *        sigmoid affinity, gate = normalisation over the selected affinities,
 *        bias -gamma when overloaded, +gamma when under-loaded.
 *   [P5] "DeepSeek-V3核心技术解析" (wenxiaobai), §二(一)4: top-K by affinity,
 *        the shared expert always participates.
 * Readings where the pages are silent: top-2-sum group score, contiguous groups,
 * SwiGLU without biases, no routed scaling factor, lower index wins exact ties,
 * FP8 scale = amax/448 in fp32.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers owned by the caller, row-major and
 *     16-byte aligned; the library allocates and frees nothing.
 *   - `stream` is a cudaStream_t (passed as void*); every call only enqueues
 *     work on it and returns without synchronising.
 *   - Return value: MOE_OK or a negative MOE_ERR_* status; nothing is enqueued
 *     when an argument check fails.  No exception or exit crosses the ABI.
 *   - Device-side failures (a pipeline wait that gave up, an expert index out
 *     of range, inconsistent counts) are OR-ed into the status word at the
 *     start of the workspace; read it with moe_read_device_status().
 */
#ifndef MOE_B200_H_
#define MOE_B200_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Layer shape.  dtype selects the expert-GEMM arithmetic:
 *   MOE_DTYPE_FP32: x, weights, y fp32; SIMT fp32 experts.
 *   MOE_DTYPE_BF16: x, weights, y bf16; tcgen05 bf16 MMAs, fp32 accumulate.
 *   MOE_DTYPE_E4M3: x, y bf16; expert GEMMs in E4M3 with fp32 block scales
 *                   (1x128 activations, 128x128 weights), fp32 accumulate.
 * The router is fp32 in every mode. */
typedef struct moe_shape {
  int32_t T;     /* tokens */
  int32_t d;     /* model width */
  int32_t N;     /* routed experts (the shared expert is index N) */
  int32_t K;     /* routed experts per token */
  int32_t G;     /* expert groups (contiguous, N/G experts each) */
  int32_t topG;  /* groups a token may reach */
  int32_t f;     /* expert inner width */
  int32_t dtype; /* MOE_DTYPE_* */
} moe_shape;

enum {
  MOE_DTYPE_FP32 = 0,
  MOE_DTYPE_BF16 = 1,
  MOE_DTYPE_E4M3 = 2
};

enum {
  MOE_OK = 0,
  MOE_ERR_ARG = -1,         /* null pointer, non-positive size, misaligned pointer */
  MOE_ERR_UNSUPPORTED = -2, /* shape or dtype outside what the kernels handle */
  MOE_ERR_WORKSPACE = -3,   /* workspace smaller than moe_workspace_size() */
  MOE_ERR_CUDA = -4,        /* a CUDA launch or API call failed */
  MOE_ERR_DEVICE = -5       /* the device status word is non-zero */
};

/* Device status bits (moe_read_device_status). */
enum {
  MOE_DEV_WAIT_TIMEOUT = 1,   /* a tensor-core pipeline wait gave up after ~2 s */
  MOE_DEV_COUNT_MISMATCH = 2, /* counts[] disagree with the expert indices */
  MOE_DEV_BAD_INDEX = 4       /* an expert index outside [0, N) */
};

/* Human-readable text for a MOE_* status.  Never NULL; static storage. */
const char* moe_status_string(int status);

/* Text of the last CUDA failure recorded on this thread (the failing call and
 * CUDA's message), "" if none; explains a MOE_ERR_CUDA status.  Static,
 * thread-local storage, overwritten by the next failure. */
const char* moe_last_error(void);

/* Check a shape: MOE_OK, MOE_ERR_ARG or MOE_ERR_UNSUPPORTED.
 * Supported: T >= 1; 1 <= K <= min(32, topG*N/G); N <= 256; G divides N;
 * 1 <= topG <= G; for BF16 and E4M3 also d % 256 == 0 and f % 128 == 0;
 * for FP32 also d % 4 == 0. */
int moe_check_shape(const moe_shape* shape);

/* Bytes of scratch every entry point of this shape may use (one buffer serves
 * all of them; calls on the same stream may share it).  The first 256 bytes
 * hold the device status word and the expert GEMMs' work counters (each
 * launch leaves them at zero): zero them once after allocating
 * (moe_workspace_init) and read the status with moe_read_device_status.
 * Returns 0 for an invalid shape. */
size_t moe_workspace_size(const moe_shape* shape);

/* Zero the device status word of `ws` (enqueued on `stream`). */
int moe_workspace_init(void* ws, void* stream);

/* Synchronise `stream`, then copy the device status word of `ws` into
 * *status_out (0 = no device-side failure).  When `clear` is non-zero the word
 * is reset to 0 afterwards.  Returns MOE_OK, or MOE_ERR_DEVICE when the word
 * was non-zero. */
int moe_read_device_status(void* ws, void* stream, uint32_t* status_out, int clear);

/* Measurement aid, not a step of the method: the expert GEMM kernels add,
 * on every launch, the SM cycles and wall-clock nanoseconds of their first
 * CTA (start to end) to counters in the workspace head (bytes 128..159).
 * This synchronises `stream` and copies them into counters_out[4] =
 * {bf16 cycles, bf16 ns, FP8 cycles, FP8 ns}; cycles / ns is the average SM
 * clock, in GHz, over the launches since the last clear.  `clear` non-zero
 * zeroes them afterwards.  MOE_ERR_ARG for a NULL pointer. */
int moe_read_gemm_clock(void* ws, void* stream, uint64_t* counters_out, int clear);

/* Routing: affinity, biased group-limited top-K, gates and per-expert counts.
 * [P4] sigmoid affinity and gate normalisation; [P2] Q3 / [P1] §1.2 bias for
 * selection only; [P1] §3.1 group limit; [P5] top-K by affinity.
 *   x          [T, d]  fp32 (FP32 mode) or bf16 (BF16/E4M3 modes)
 *   router_w   [N, d]  fp32, row i = e_i
 *   bias       [N]     fp32
 *   topk_idx   [T, K]  int32 out, ascending expert id per token
 *   topk_gate  [T, K]  fp32 out, gate of topk_idx[t, k]; each row sums to 1
 *   counts     [N]     int32 out, tokens routed to each expert (sum = T*K)
 *   ws         workspace of moe_workspace_size(shape) bytes
 * Scores are fp32 (dot products accumulated in fp32); an exact tie between
 * two scores goes to the lower expert (or group) index. */
int moe_route(const moe_shape* shape, const void* x, const float* router_w, const float* bias,
              int32_t* topk_idx, float* topk_gate, int32_t* counts, void* ws, void* stream);

/* moe_route_softmax: the conventional softmax gate that the bias method
 * replaces, kept as a baseline to contrast with it ([P4] gating paragraph: a
 * softmax on top of a classifier, balanced by an auxiliary penalty; [P2] Q3).
 * Per token: p = softmax(x . e_i) over all N experts; the K largest p (no
 * groups, no bias; shape->G and topG are ignored), ascending expert id;
 * gate_k = p_k / sum of the selected p.  BF16 and E4M3 shapes (x bf16).
 *   topk_idx, topk_gate, counts   as at moe_route
 *   prob_sum   [N] fp32 out or NULL: sum over the T tokens of p[t, i], added
 *              in a fixed order (deterministic).  With counts it gives the
 *              conventional balance statistic N * sum_i (counts_i / (K T)) *
 *              (prob_sum_i / T), 1 for uniform routing.
 * Returns MOE_ERR_UNSUPPORTED for FP32 shapes. */
int moe_route_softmax(const moe_shape* shape, const void* x, const float* router_w,
                      int32_t* topk_idx, float* topk_gate, int32_t* counts, float* prob_sum,
                      void* ws, void* stream);

/* Dispatch ([P1] §2.2 DISPATCH, single-GPU permutation): group the T*K
 * (token, expert) pairs by expert.  Row order is experts ascending, tokens
 * ascending within an expert, so the result is deterministic.
 *   topk_idx   [T, K]  int32 (from moe_route)
 *   counts     [N]     int32 (from moe_route)
 *   offsets    [N+1]   int32 out, first row of each expert; offsets[N] = T*K
 *   perm_tok   [T*K]   int32 out, token of each row
 *   slot       [T, K]  int32 out, row holding (t, topk_idx[t, k])
 *   x_perm     [T*K, d] out: bf16 copy of x rows (BF16), fp32 (FP32), or E4M3
 *                      codes (E4M3 mode, one byte per element).  May be NULL
 *                      in BF16 and FP32 modes: then only offsets, perm_tok and
 *                      slot are written (for moe_expert_ffn_gathered)
 *   x_perm_scales [d/128, L] fp32 out, E4M3 mode only (NULL otherwise), with
 *                      L = T*K rounded up to a multiple of 4: the scale
 *                      amax/448 of row r's 1x128 tile j is at [j, r] ([P1]
 *                      §4.1).  Block-major, so a tile of rows at one K block
 *                      is contiguous; columns r >= T*K are not written.
 * Sets MOE_DEV_COUNT_MISMATCH if counts disagree with topk_idx. */
int moe_dispatch(const moe_shape* shape, const void* x, const int32_t* topk_idx,
                 const int32_t* counts, int32_t* offsets, int32_t* perm_tok, int32_t* slot,
                 void* x_perm, float* x_perm_scales, void* ws, void* stream);

/* Experts: the N routed SwiGLU experts on their dispatched rows and the shared
 * expert (index N) on all T rows of x, in one pass per GEMM
 * ([P1] §1.1, [P5]; SwiGLU is this library's reading of "FFN").
 *   x_perm, x_perm_scales, offsets   from moe_dispatch
 *   x          [T, d]  layer input (fp32 or bf16), input of the shared expert
 *   w13        [N+1, 2f, d] packed W1/W3 (moe_pack_w13): for each 128-row block
 *              j of W1 and W3, rows 256j..256j+127 are W1 rows 128j.. and rows
 *              256j+128..256j+255 are W3 rows 128j..  (bf16 / fp32 / E4M3 codes)
 *   w2         [N+1, d, f]  (bf16 / fp32 / E4M3 codes)
 *   w13_scales [N+1, 2f/128, d/128], w2_scales [N+1, d/128, f/128] fp32,
 *              E4M3 mode only (from moe_quantize_weights), else NULL
 *   y_perm     [T*K, d] out (fp32 in FP32 mode, else bf16): E_{expert}(row)
 *   y_shared   [T, d]   out: E_shared(x)
 * The hidden activation h is held in the workspace as bf16 (BF16), fp32 (FP32)
 * or E4M3 with 1x128 scales (E4M3). */
int moe_expert_ffn(const moe_shape* shape, const void* x_perm, const float* x_perm_scales,
                   const int32_t* offsets, const void* x, const void* w13, const void* w2,
                   const float* w13_scales, const float* w2_scales, void* y_perm,
                   void* y_shared, void* ws, void* stream);

/* moe_expert_ffn_gathered (BF16 mode only): moe_expert_ffn without the
 * permuted copy of x.  GEMM1 reads each routed row straight from x, row
 * perm_tok[r] for row r of the expert-major order (the producer warp's
 * 16-byte cp.async copies, written in the 128-byte-swizzled operand layout),
 * so moe_dispatch may be called with x_perm = NULL.
 *   x          [T, d] bf16 layer input
 *   perm_tok   [T*K] int32, offsets [N+1] int32   from moe_dispatch
 *   w13, w2, y_perm, y_shared, ws   as at moe_expert_ffn
 * Same results as moe_expert_ffn on the same inputs (bit-identical rows).
 * Returns MOE_ERR_UNSUPPORTED for other dtypes. */
int moe_expert_ffn_gathered(const moe_shape* shape, const void* x, const int32_t* perm_tok,
                            const int32_t* offsets, const void* w13, const void* w2,
                            void* y_perm, void* y_shared, void* ws, void* stream);

/* moe_expert_ffn_combine (BF16 mode only): moe_expert_ffn followed by
 * moe_combine, with the COMBINE step inside GEMM2's epilogue ([P1] §2.2 runs
 * DISPATCH -> MLP -> COMBINE within one chunk).  After storing a row of
 * y_perm or y_shared, the epilogue counts one arrival for (token, 256-column
 * tile) in the workspace; the token's K+1-th arrival (its K routed rows and
 * its shared-expert row) forms that tile of
 *   y[t] = y_shared[t] + sum_k topk_gate[t,k] * y_perm[slot[t,k]]
 * with fp32 fused multiply-adds in k order and one bf16 rounding: the same
 * operations in the same order as moe_combine, so y is bit-identical to
 * moe_expert_ffn + moe_combine.  The shared expert's tiles run first.
 *   x_perm, offsets, perm_tok, slot   from moe_dispatch
 *   topk_gate  [T, K] fp32 from moe_route
 *   x, w13, w2, y_perm, y_shared, ws  as at moe_expert_ffn
 *   y          [T, d] bf16 out
 * The arrival counters ([T, d/256] int32 in the workspace) are cleared at the
 * start of every call.  Returns MOE_ERR_UNSUPPORTED for other dtypes. */
int moe_expert_ffn_combine(const moe_shape* shape, const void* x_perm, const int32_t* offsets,
                           const int32_t* perm_tok, const int32_t* slot, const float* topk_gate,
                           const void* x, const void* w13, const void* w2, void* y_perm,
                           void* y_shared, void* y, void* ws, void* stream);

/* Backward of the expert FFNs, input gradients ([P1] §2.2: the backward
 * pass runs COMBINE -> MLP_B -> MLP_W -> DISPATCH; this is MLP_B), BF16 mode.
 * With g = a W1^T, u = a W3^T (a = a dispatched row, or an x row for the
 * shared expert) and dy the gradient of that expert's output row:
 *   dh = dy W2;  dg = dh * u * silu'(g);  du = dh * silu(g);  da = dg W1 + du W3
 * g and u are recomputed (GEMM1) and stored bf16; dh accumulates in fp32;
 * dg, du are rounded to bf16 (operands of the last GEMM); da is bf16.
 *   x_perm, offsets, x, w13   as at moe_expert_ffn
 *   w13t [N+1, d, 2f], w2t [N+1, f, d]  bf16, from moe_transpose_weights
 *   dy_perm [T*K, d], dy_shared [T, d]  bf16 output gradients (y_perm order)
 *   dx_perm [T*K, d], dx_shared [T, d]  bf16 out: input gradients per
 *              dispatched row and for the shared expert's rows
 *   ws_bwd     moe_backward_workspace_size(shape) bytes; its first 256 bytes
 *              are a status word like the forward workspace's (zero them once)
 * MOE_ERR_UNSUPPORTED for other dtypes.  moe_transpose_weights takes the
 * bf16 weights of a BF16 or E4M3 shape (MOE_ERR_UNSUPPORTED for FP32);
 * moe_backward_workspace_size is 0 for an FP32 shape. */
size_t moe_backward_workspace_size(const moe_shape* shape);
int moe_transpose_weights(const moe_shape* shape, const void* w13, const void* w2, void* w13t,
                          void* w2t, void* stream);
int moe_expert_ffn_backward_dx(const moe_shape* shape, const void* x_perm,
                               const int32_t* offsets, const void* x, const void* w13,
                               const void* w13t, const void* w2t, const void* dy_perm,
                               const void* dy_shared, void* dx_perm, void* dx_shared,
                               void* ws_bwd, void* stream);

/* FP8 input gradients of the experts, E4M3 mode with f % 256 == 0: E4M3
 * operands in the forward and E5M2 gradients in the backward ([P3]), each
 * scaled per 1x128 tile or 128x128 block from its online max-abs ([P1] §4.1):
 *   1. g, u recomputed from the forward's E4M3 operands, stored bf16;
 *   2. dy quantised to E5M2 per 1x128 along d;
 *   3. dh = dy W2 against W2^T's E4M3 blocks, fp32 with per-slice promotion;
 *      dg = dh * u * silu'(g), du = dh * silu(g), stored bf16;
 *   4. [dg du] quantised to E5M2 per 1x128 along 2f;
 *   5. da = [dg du] W13 against W13^T's E4M3 blocks -> bf16.
 *   x_perm, x_perm_scales, offsets   E4M3 dispatch outputs (moe_dispatch)
 *   x          [T, d] bf16 layer input (the shared expert's rows)
 *   w13, w13_scales   the forward's E4M3 weights (moe_quantize_weights)
 *   w13t, w13t_scales, w2t, w2t_scales   E4M3 codes [N+1, d, 2f], [N+1, f, d]
 *              and block scales [N+1, d/128, 2f/128], [N+1, f/128, d/128]
 *              from moe_quantize_weights_transposed
 *   dy_perm, dy_shared, dx_perm, dx_shared   bf16, as at moe_expert_ffn_backward_dx
 *   ws_bwd     moe_backward_workspace_size(shape) bytes (status word first)
 * moe_quantize_weights_transposed quantises the bf16 transposes (from
 * moe_transpose_weights) per 128x128 block: the blocks are the forward's
 * blocks transposed, so codes and scales are the forward's, transposed. */
int moe_quantize_weights_transposed(const moe_shape* shape, const void* w13t, const void* w2t,
                                    void* w13t_q, float* w13t_scales, void* w2t_q,
                                    float* w2t_scales, void* stream);
int moe_expert_ffn_backward_dx_fp8(const moe_shape* shape, const void* x_perm,
                                   const float* x_perm_scales, const int32_t* offsets,
                                   const void* x, const void* w13, const float* w13_scales,
                                   const void* w13t, const float* w13t_scales, const void* w2t,
                                   const float* w2t_scales, const void* dy_perm,
                                   const void* dy_shared, void* dx_perm, void* dx_shared,
                                   void* ws_bwd, void* stream);

/* moe_expert_ffn_backward_dw_fp8: FP8 weight gradients, E4M3 mode with
 * f % 256 == 0, to be called after moe_expert_ffn_backward_dx_fp8 with the
 * same ws_bwd (it reads the g, u and dg, du left there):
 *   dW2_e = dY_e^T H_e,  dW13_e = [dg du]_e^T A_e  (packed like W13)
 * with the gradient operand in E5M2 and the activation in E4M3, each column
 * of each scaled per 128-row tile of the expert's rows ([P3]; [P1] §4.1),
 * fp32 per-slice promotion, bf16 results.  A is the layer input x gathered
 * through perm_tok (E4M3 mode keeps no bf16 copy of the dispatched rows).
 *   perm_tok [T*K], offsets [N+1]   from moe_dispatch
 *   x        [T, d] bf16;  dy_perm, dy_shared as at the _dx_fp8 call
 *   dw13 [N+1, 2f, d], dw2 [N+1, d, f] bf16 out; an expert without rows gets zeros */
int moe_expert_ffn_backward_dw_fp8(const moe_shape* shape, const int32_t* perm_tok,
                                   const int32_t* offsets, const void* x, const void* dy_perm,
                                   const void* dy_shared, void* dw13, void* dw2, void* ws_bwd,
                                   void* stream);

/* moe_expert_ffn_backward_dw: the weight gradients ([P1] §2.2 MLP_W), BF16
 * mode with f % 256 == 0, to be called after moe_expert_ffn_backward_dx with
 * the same ws_bwd (it reads the g, u and dg, du that call leaves there):
 *   dW2_e = dY_e^T H_e,  H = silu(g) * u          -> dw2  [N+1, d, f]
 *   dW13_e = [dg du]_e^T A_e (packed like W13)     -> dw13 [N+1, 2f, d]
 * for every routed expert e on its dispatched rows and the shared expert on
 * x.  Each product contracts over the expert's rows in fp32 (tensor cores,
 * the rows transposed into zero-padded per-expert column blocks first); the
 * gradients are bf16.  An expert without rows gets zeros.
 *   x_perm, offsets, x, dy_perm, dy_shared   as at the _dx call */
int moe_expert_ffn_backward_dw(const moe_shape* shape, const void* x_perm,
                               const int32_t* offsets, const void* x, const void* dy_perm,
                               const void* dy_shared, void* dw13, void* dw2, void* ws_bwd,
                               void* stream);

/* Combine ([P1] §2.2 COMBINE): y[t] = y_shared[t] + sum_k gate[t,k] *
 * y_perm[slot[t,k]], accumulated in fp32 in k order, rounded once to the
 * output dtype (fp32 in FP32 mode, else bf16).  No atomics: deterministic. */
int moe_combine(const moe_shape* shape, const void* y_perm, const void* y_shared,
                const int32_t* slot, const float* topk_gate, void* y, void* stream);

/* ---- backward of COMBINE, of the gates and of DISPATCH --------------------
 * [P1] §2.2 orders the backward pass COMBINE -> MLP_B -> MLP_W -> DISPATCH.
 * These three calls are the steps around the expert backward
 * (moe_expert_ffn_backward_dx/_dw).  The routing of the forward is held
 * fixed; the bias receives no gradient ([P2] Q3: it only selects).
 * Activations are fp32 in FP32 mode and bf16 otherwise (E4M3 mode keeps its
 * layer input and outputs in bf16); gradients of the gates and of the router
 * are fp32.  Every sum runs in fp32 in a fixed order: deterministic, no
 * atomics.  All pointers are device pointers owned by the caller, 16-byte
 * aligned; a NULL or misaligned pointer gives MOE_ERR_ARG.
 *
 * moe_combine_backward: for y[t] = y_shared[t] + sum_k gate[t,k] y_perm[slot[t,k]]
 * and dy = dL/dy [T, d]:
 *   dy_perm[slot[t,k]] = gate[t,k] * dy[t]          [T*K, d], one rounding
 *   dgate[t,k]         = dy[t] . y_perm[slot[t,k]]   [T, K] fp32
 * The shared expert's output gradient is dy itself.  Rows that no slot names
 * are not written; a slot outside [0, T*K) gives dgate 0. */
int moe_combine_backward(const moe_shape* shape, const void* dy, const void* y_perm,
                         const int32_t* slot, const float* topk_gate, void* dy_perm,
                         float* dgate, void* stream);

/* moe_route_backward: the gates gate_k = s_k / S (S = sum over the K selected
 * experts, s = sigmoid(x . e_i), [P4]) given dgate [T, K]:
 *   dlogit[t,k] = s_k (1 - s_k) (dgate_k - sum_j gate_j dgate_j) / S   [T, K] fp32
 *   dx_route[t] = sum_k dlogit[t,k] e_{idx[t,k]}                      [T, d] fp32
 *   drouter[i]  = sum over expert i's dispatched rows r (in row order)
 *                 of dlogit * x[perm_tok[r]]                          [N, d] fp32
 * The logits are recomputed in fp32 from x and router_w [N, d] fp32.
 *   topk_idx [T, K] int32 from moe_route; offsets, perm_tok, slot from
 *   moe_dispatch.  An expert with no rows gets a zero row of drouter. */
int moe_route_backward(const moe_shape* shape, const void* x, const float* router_w,
                       const int32_t* topk_idx, const float* dgate, const int32_t* offsets,
                       const int32_t* perm_tok, const int32_t* slot, float* dlogit,
                       float* dx_route, float* drouter, void* stream);

/* moe_dispatch_backward: each copy that DISPATCH made returns its gradient,
 *   dx[t] = dx_shared[t] + sum_k dx_perm[slot[t,k]] (+ dx_route[t])
 * accumulated in fp32 in that order and rounded once to the activation type.
 *   dx_perm [T*K, d], dx_shared [T, d]   from moe_expert_ffn_backward_dx
 *   dx_route [T, d] fp32 from moe_route_backward, or NULL to leave it out */
int moe_dispatch_backward(const moe_shape* shape, const void* dx_perm, const void* dx_shared,
                          const int32_t* slot, const float* dx_route, void* dx, void* stream);

/* moe_quantize_rows_e5m2: fine-grained quantisation of gradient rows to
 * FP8-E5M2, the backward pass's format ([P3]: E4M3 forward, E5M2 backward;
 * the 1x128 online scaling of [P1] §4.1).  Per 1x128 tile of each row:
 *   scale = amax / 57344 and inverse = 57344 / amax (fp32, IEEE division),
 *   code  = E5M2 round-to-nearest-even with saturation of v * inverse;
 * an all-zero tile gets scale 1 and zero codes.
 *   g       [rows, cols] bf16 row-major, cols % 128 == 0
 *   codes   [rows, cols] uint8 E5M2 bit patterns
 *   scales  block-major [cols/128, sc_ld] fp32, sc_ld >= rows (scales of one
 *           128-column block contiguous over rows, like x_perm_scales)
 * MOE_ERR_ARG for a bad size or a NULL / misaligned pointer. */
int moe_quantize_rows_e5m2(const void* g, int64_t rows, int cols, uint8_t* codes,
                           float* scales, int64_t sc_ld, void* stream);

/* Auxiliary-loss-free bias update ([P4]; [P1] §1.2): for every expert,
 * bias[i] -= gamma if counts[i] * N > T * K, += gamma if counts[i] * N < T * K,
 * unchanged otherwise; fp32, in place. */
int moe_bias_update(const moe_shape* shape, const int32_t* counts, float* bias, float gamma,
                    void* stream);

/* moe_gather_rows: dst[i] = src[idx[i]] for i < n, whole rows of row_bytes
 * bytes (any element type).  Expert parallelism ([P1] §2.1: each GPU holds a
 * contiguous share of the routed experts; §3.1: tokens reach them by
 * all-to-all) receives rows grouped by source GPU, then by expert; this
 * regroups them by expert for the grouped expert GEMM, and puts the results
 * back in arrival order.
 *   src  [src_rows, row_bytes] device, 16-byte aligned
 *   idx  [n] int32 device; an index outside [0, src_rows) writes a zero row
 *   dst  [n, row_bytes] device, 16-byte aligned, must not overlap src
 * row_bytes % 16 == 0.  MOE_ERR_ARG for a bad size or pointer; n = 0 is a
 * no-op. */
int moe_gather_rows(const void* src, int64_t src_rows, const int32_t* idx, int64_t n,
                    int row_bytes, void* dst, void* stream);

/* Weight preparation (not part of the timed forward).
 * moe_pack_w13: w1, w3 [N+1, f, d] -> w13 [N+1, 2f, d] in the 128-row block
 * interleave described at moe_expert_ffn (element type per shape->dtype; for
 * E4M3 pass the bf16 weights here, then moe_quantize_weights). */
int moe_pack_w13(const moe_shape* shape, const void* w1, const void* w3, void* w13, void* stream);

/* moe_quantize_weights (E4M3 mode): per 128x128 block of each expert matrix,
 * scale = amax/448 (fp32), codes = E4M3_RNE_satfinite(w * (448/amax)).
 *   w13_bf16 [N+1, 2f, d] (packed), w2_bf16 [N+1, d, f]
 *   w13_q / w2_q: E4M3 codes of the same shapes; scales as at moe_expert_ffn. */
int moe_quantize_weights(const moe_shape* shape, const void* w13_bf16, const void* w2_bf16,
                         void* w13_q, float* w13_scales, void* w2_q, float* w2_scales,
                         void* stream);

/* moe_dispatch_noalloc: moe_dispatch for callers that cannot allocate device
 * memory when they call in -- for example code that runs while a framework
 * forbids new allocations, or a host application that hands the library only
 * its input and output buffers -- and so cannot provide a workspace.  The
 * pages describe no such entry point; it has no counterpart there.
 * Arguments, layouts and results are those of moe_dispatch, without `ws`;
 * as there, x_perm may be NULL (offsets, perm_tok and slot only).
 * Scratch: a fixed static device array of 1 MiB + 256 bytes inside the
 * library (held on every GPU that loads the library until the process
 * exits).  The dispatch needs a 256-byte status word plus two tables of
 * ceil(T/32) * N * 4 bytes each (each rounded up to 256 bytes); a shape that
 * needs more than the array (at N = 256: T > 16384) returns
 * MOE_ERR_WORKSPACE before anything is enqueued.  E4M3 mode returns
 * MOE_ERR_UNSUPPORTED.
 * The first call on a device looks up the array's device address (with
 * that device current) and caches it; make that first call before any
 * stream capture.  All calls share the one array, so calls whose work
 * overlaps on the GPU (different streams without ordering) race; calls on
 * one stream are safe.  The device status word lives in the array and is
 * cleared at the start of every call; it cannot be read back, but all
 * writes stay in bounds as in moe_dispatch. */
int moe_dispatch_noalloc(const moe_shape* shape, const void* x, const int32_t* topk_idx,
                         const int32_t* counts, int32_t* offsets, int32_t* perm_tok,
                         int32_t* slot, void* x_perm, float* x_perm_scales, void* stream);

/* The whole forward in order: route, dispatch, experts, combine, then the bias
 * update; intermediate buffers are caller-provided as in the calls above. */
int moe_forward(const moe_shape* shape, const void* x, const float* router_w, float* bias,
                float gamma, const void* w13, const void* w2, const float* w13_scales,
                const float* w2_scales, int32_t* topk_idx, float* topk_gate, int32_t* counts,
                int32_t* offsets, int32_t* perm_tok, int32_t* slot, void* x_perm,
                float* x_perm_scales, void* y_perm, void* y_shared, void* y, void* ws,
                void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H_ */
