// Internal declarations shared by the kernel files and the C-ABI layer.
#pragma once
#include <cuda_bf16.h>
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/moe_b200.h"

namespace moe {

constexpr int kRouteTokens = 32;   // tokens per routing CTA (4 per warp)
constexpr int kRouteMaxN = 256;    // experts a routing warp holds (8 per lane)
constexpr int kChunkTokens = 32;   // tokens per dispatch chunk
constexpr int kMaxK = 32;

inline int chunks_of(int T) { return (T + kChunkTokens - 1) / kChunkTokens; }

// Byte offsets of the workspace regions (each 256-byte aligned).
struct WsLayout {
  size_t status = 0;      // uint32 device status word (+ padding to 256)
  size_t chunk_hist = 0;  // int32 [chunks, N]
  size_t chunk_base = 0;  // int32 [chunks, N]
  size_t router_split = 0;  // bf16 [N, 3d] exact three-part split of the router (bf16 x)
  size_t scores = 0;        // fp32 [splits <= 8, T, N] partial router logits (bf16 x)
  size_t prob_part = 0;     // fp32 [ceil(T/8), N] softmax-probability sums per selection CTA
  size_t h = 0;           // hidden activation [T*K + T, f] (bf16 / fp32 / e4m3)
  size_t h_scales = 0;    // fp32 block-major [f/128, scale_ld(T*K + T)] (E4M3)
  size_t xq = 0;          // E4M3 codes of x for the shared expert [T, d]
  size_t xq_scales = 0;   // fp32 block-major [d/128, scale_ld(T)]
  size_t arrive = 0;      // int32 [T, d/256] arrival counters of the fused combine (BF16)
  size_t sc_rows = 0;     // fp32 [T*K, round8(d/128)] dispatch scales by row (E4M3)
  size_t total = 0;
};
WsLayout ws_layout(const moe_shape& s);

inline size_t dtype_bytes(int dtype) {
  return dtype == MOE_DTYPE_FP32 ? 4 : (dtype == MOE_DTYPE_BF16 ? 2 : 1);
}
// Bytes per element of the layer input x and output y.
inline size_t io_bytes(int dtype) { return dtype == MOE_DTYPE_FP32 ? 4 : 2; }
// Rows of a W1/W3 block in the packed w13 layout.
inline int pack_block(int f) { return f < 128 ? f : 128; }

// ---- error text (errors.cu) ------------------------------------------------------
// Record `e` (if not cudaSuccess) with the failing call's name; returns e.
cudaError_t note_cuda(cudaError_t e, const char* where);
void note_text(const char* what);

// FP8 activation scales are stored block-major, [K/128][ld] with ld = the row
// count rounded up to 4, so the 128 scales of a token tile at one K block are
// contiguous and one TMA copy (16-byte aligned row pitch) brings them in.
inline long long scale_ld(long long rows) { return (rows + 3) & ~3LL; }

// Clock record in a workspace head (after the status word, inside its 256
// bytes, clear of the status word and the schedule counters at bytes 64-75):
// u64 pairs {SM cycles, ns} summed over launches by the first CTA of
// the bf16 expert GEMMs (pair 0) and of the FP8 expert GEMMs (pair 1).
constexpr size_t kClockRecordOffset = 128;

// ---- host helpers (tma_host.cu) ------------------------------------------------
// 2-D row-major tensor [rows, inner] with a (box_inner x box_rows) box and the
// 128-byte swizzle; out-of-range rows read as zero.
bool make_map(CUtensorMap* map, const void* ptr, CUtensorMapDataType dt, size_t elem_bytes,
              uint64_t inner, uint64_t rows, uint32_t box_inner, uint32_t box_rows);
// The same with a chosen swizzle and no L2 promotion (used for TMA stores).
bool make_map_swizzled(CUtensorMap* map, const void* ptr, CUtensorMapDataType dt,
                       size_t elem_bytes, uint64_t inner, uint64_t rows, uint32_t box_inner,
                       uint32_t box_rows, CUtensorMapSwizzle swizzle);
// `rank`-D tensor (2..5) given by its dims (innermost first), the byte strides of
// dims 1..rank-1 and the box; 128-byte swizzle, out-of-range elements read as zero.
bool make_map_nd(CUtensorMap* map, const void* ptr, CUtensorMapDataType dt, int rank,
                 const uint64_t* dims, const uint64_t* strides_bytes, const uint32_t* box);
// fp32 matrix [rows, inner] (inner a multiple of 4) read one row segment at a
// time: box {box_inner, 1}, no swizzle, out-of-range elements read as zero.
bool make_map_f32_rows(CUtensorMap* map, const float* ptr, uint64_t inner, uint64_t rows,
                       uint32_t box_inner);
int num_sms();

// ---- launchers (return cudaError_t of the launch) -----------------------------
// Softmax top-K baseline routing (bf16 / E4M3 shapes): idx, gate, counts and,
// when prob_sum is set, the per-expert sums of the softmax probabilities.
int launch_route_softmax(const moe_shape& s, const void* x, const float* router, int32_t* idx,
                         float* gate, int32_t* counts, float* prob_sum, void* ws,
                         cudaStream_t st);
int launch_route(const moe_shape& s, const void* x, const float* router, const float* bias,
                 int32_t* idx, float* gate, int32_t* counts, void* ws, cudaStream_t st);
cudaError_t launch_dispatch(const moe_shape& s, const void* x, const int32_t* idx,
                            const int32_t* counts, int32_t* offsets, int32_t* perm_tok,
                            int32_t* slot, void* x_perm, float* x_perm_scales, void* ws,
                            cudaStream_t st);
cudaError_t launch_combine(const moe_shape& s, const void* y_perm, const void* y_shared,
                           const int32_t* slot, const float* gate, void* y, cudaStream_t st);
cudaError_t launch_bias_update(const moe_shape& s, const int32_t* counts, float* bias,
                               float gamma, cudaStream_t st);
cudaError_t launch_pack_w13(const moe_shape& s, const void* w1, const void* w3, void* w13,
                            cudaStream_t st);
cudaError_t launch_ffn_simt(const moe_shape& s, const float* x_perm, const int32_t* offsets,
                            const float* x, const float* w13, const float* w2, float* y_perm,
                            float* y_shared, void* ws, cudaStream_t st);
// Router logits on the tensor cores (bf16 x): Z[split, t, i] = partial sums
// of x_t . e_i over K split `split`; sum the splits in order for z.
int router_k_splits(const moe_shape& s);
int launch_router_scores_tc(const moe_shape& s, const void* x, const float* router, float* Z,
                            int k_splits, void* ws, cudaStream_t st);
// Returns MOE_OK or a MOE_ERR_* status (tensor maps can fail to encode).
// Expert backward workspace: status word, the recomputed gate/up GU and the
// input pass's dGU [T*K+T, 2f] bf16, then the weight-gradient pass's column
// blocks and transposed operands (gemm_wgrad.cu).
struct BwdLayout {
  size_t gu = 0, dgu = 0, colbase = 0, at = 0, dyt = 0, ht = 0, dgut = 0;
  size_t total = 0;
};
// Backward workspace of the FP8 (E4M3) mode: status word, then the stored g, u
// and dg, du (bf16 [T*K + T, 2f], packed like W13), x in E4M3 for the shared
// expert, and the E5M2 gradients dY [T*K + T, d] and dGU [T*K + T, 2f] with
// their block-major 1x128 scales.
struct BwdLayoutFp8 {
  size_t gu = 0, dgu = 0, xq = 0, xs = 0, dyq = 0, dys = 0, dguq = 0, dgus = 0;
  // weight-gradient pass: column blocks, the transposed operands (bf16), their
  // codes (per 1x128 tile of each row) and block-major scales [R/128][C]
  size_t colbase = 0, at = 0, dyt = 0, ht = 0, dgut = 0;
  size_t atq = 0, dytq = 0, htq = 0, dgutq = 0, ats = 0, dyts = 0, hts = 0, dguts = 0;
  size_t total = 0;
};
long long wgrad_cols_fp8(const moe_shape& s);
int launch_ffn_bwd_dw_e4m3(const moe_shape& s, const int32_t* perm_tok, const int32_t* offsets,
                           const void* x, const void* dy_perm, const void* dy_shared, void* dw13,
                           void* dw2, void* ws_bwd, cudaStream_t st);
BwdLayoutFp8 bwd_layout_fp8(const moe_shape& s);
int launch_ffn_bwd_dx_e4m3(const moe_shape& s, const void* x_perm, const float* x_perm_scales,
                           const int32_t* offsets, const void* x, const void* w13q,
                           const float* w13_scales, const void* w13tq, const float* w13t_scales,
                           const void* w2tq, const float* w2t_scales, const void* dy_perm,
                           const void* dy_shared, void* dx_perm, void* dx_shared, void* ws_bwd,
                           cudaStream_t st);
cudaError_t launch_quantize_weights_transposed(const moe_shape& s, const void* w13t,
                                               const void* w2t, void* w13t_q, float* w13t_scales,
                                               void* w2t_q, float* w2t_scales, cudaStream_t st);
cudaError_t launch_group_transposes(const moe_shape& s, int pad, const void* a_routed,
                                    const int32_t* a_perm, const void* x, const void* dy_perm,
                                    const void* dy_shared, const __nv_bfloat16* GU,
                                    const __nv_bfloat16* dGU, const int32_t* offsets,
                                    int32_t* colbase, long long R, __nv_bfloat16* AT,
                                    __nv_bfloat16* dYT, __nv_bfloat16* HT, __nv_bfloat16* dGUT,
                                    cudaStream_t st);
long long wgrad_cols(const moe_shape& s);
BwdLayout bwd_layout(const moe_shape& s);
size_t backward_ws_bytes(const moe_shape& s);
int launch_ffn_bwd_dw_bf16(const moe_shape& s, const void* x_perm, const int32_t* offsets,
                           const void* x, const void* dy_perm, const void* dy_shared,
                           void* dw13, void* dw2, void* ws_bwd, cudaStream_t st);
int launch_ffn_bwd_dx_bf16(const moe_shape& s, const void* x_perm, const int32_t* offsets,
                           const void* x, const void* w13, const void* w13t, const void* w2t,
                           const void* dy_perm, const void* dy_shared, void* dx_perm,
                           void* dx_shared, void* ws_bwd, cudaStream_t st);
cudaError_t launch_combine_backward(const moe_shape& s, const void* dy, const void* y_perm,
                                    const int32_t* slot, const float* gate, void* dy_perm,
                                    float* dgate, cudaStream_t st);
cudaError_t launch_route_backward(const moe_shape& s, const void* x, const float* router_w,
                                  const int32_t* idx, const float* dgate, const int32_t* offsets,
                                  const int32_t* perm_tok, const int32_t* slot, float* dlogit,
                                  float* dx_route, float* drouter, cudaStream_t st);
cudaError_t launch_dispatch_backward(const moe_shape& s, const void* dx_perm,
                                     const void* dx_shared, const int32_t* slot,
                                     const float* dx_route, void* dx, cudaStream_t st);
cudaError_t launch_transpose_weights(const moe_shape& s, const void* w13, const void* w2,
                                     void* w13t, void* w2t, cudaStream_t st);
// bf16 expert GEMMs; with perm_tok set, GEMM1 gathers the routed rows from x
// (x_perm unused), else it reads x_perm.
int launch_ffn_tc_bf16(const moe_shape& s, const void* x_perm, const int32_t* perm_tok,
                       const int32_t* offsets, const void* x, const void* w13, const void* w2,
                       void* y_perm, void* y_shared, void* ws, cudaStream_t st);
// The same two GEMMs on CTA pairs (tcgen05 cta_group::2), gemm2sm.cu.
// The same GEMMs with the COMBINE step fused into GEMM2's epilogue: y is
// written directly (bit-identical to the standalone combine).
int launch_ffn_combine_bf16(const moe_shape& s, const void* x_perm, const int32_t* offsets,
                            const int32_t* perm_tok, const int32_t* slot, const float* gate,
                            const void* x, const void* w13, const void* w2, void* y_perm,
                            void* y_shared, void* y, void* ws, cudaStream_t st);
int launch_ffn_tc_bf16_dual(const moe_shape& s, const void* x_perm, const int32_t* offsets,
                            const void* x, const void* w13, const void* w2, void* y_perm,
                            void* y_shared, void* ws, cudaStream_t st);
int launch_ffn_tc_bf16_pair(const moe_shape& s, const void* x_perm, const int32_t* offsets,
                            const void* x, const void* w13, const void* w2, void* y_perm,
                            void* y_shared, void* ws, cudaStream_t st);
int launch_ffn_tc_e4m3(const moe_shape& s, const void* x_perm, const float* x_perm_scales,
                       const int32_t* offsets, const void* x, const void* w13, const void* w2,
                       const float* w13_scales, const float* w2_scales, void* y_perm,
                       void* y_shared, void* ws, cudaStream_t st);
// x [rows, d] bf16 -> E4M3 codes [rows, d] and fp32 scales [rows, d/128].
cudaError_t launch_quant_rows_e5m2(const void* g, long long rows, int d, uint8_t* q, float* sc,
                                   long long sc_ld, cudaStream_t st);
cudaError_t launch_quant_rows(const void* x, long long rows, int d, uint8_t* q, float* sc,
                              long long sc_ld,
                              cudaStream_t st);
cudaError_t launch_quantize_weights(const moe_shape& s, const void* w13, const void* w2,
                                    void* w13_q, float* w13_scales, void* w2_q,
                                    float* w2_scales, cudaStream_t st);

}  // namespace moe
