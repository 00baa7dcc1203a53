// C-ABI entry points: argument checks, workspace layout, and the launches.
// Every entry point validates before enqueuing anything; nothing here
// synchronises except moe_read_device_status.
#include <cstring>

#include "internal.h"

namespace moe {

static size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

WsLayout ws_layout(const moe_shape& s) {
  WsLayout L;
  size_t off = 256;
  const size_t nch = (size_t)chunks_of(s.T);
  L.chunk_hist = off;
  off = align256(off + nch * s.N * 4);
  L.chunk_base = off;
  off = align256(off + nch * s.N * 4);
  if (s.dtype != MOE_DTYPE_FP32) {
    L.router_split = off;
    off = align256(off + (size_t)s.N * 3 * s.d * 2);
    L.scores = off;
    off = align256(off + (size_t)8 * s.T * s.N * 4);
    L.prob_part = off;
    off = align256(off + (size_t)((s.T + 7) / 8) * s.N * 4);
  }
  const size_t rows = (size_t)s.T * s.K + s.T;
  L.h = off;
  off = align256(off + rows * s.f * dtype_bytes(s.dtype));
  if (s.dtype == MOE_DTYPE_E4M3) {
    L.h_scales = off;
    off = align256(off + (size_t)scale_ld((long long)rows) * (s.f / 128) * 4);
    L.xq = off;
    off = align256(off + (size_t)s.T * s.d);
    L.xq_scales = off;
    off = align256(off + (size_t)scale_ld(s.T) * (s.d / 128) * 4);
    L.sc_rows = off;
    off = align256(off + (size_t)s.T * s.K * ((s.d / 128 + 7) / 8 * 8) * 4);
  }
  if (s.dtype == MOE_DTYPE_BF16) {
    L.arrive = off;
    off = align256(off + (size_t)s.T * (s.d / 256) * 4);
  }
  L.total = off;
  return L;
}

}  // namespace moe

using namespace moe;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool ptr_ok(const void* p) { return p != nullptr && aligned16(p); }

int check(const moe_shape* s) {
  if (!s) return MOE_ERR_ARG;
  if (s->T <= 0 || s->d <= 0 || s->N <= 0 || s->K <= 0 || s->G <= 0 || s->topG <= 0 ||
      s->f <= 0)
    return MOE_ERR_ARG;
  if (s->dtype < MOE_DTYPE_FP32 || s->dtype > MOE_DTYPE_E4M3) return MOE_ERR_UNSUPPORTED;
  if (s->N > kRouteMaxN || s->N % s->G != 0 || s->G > 32 || s->topG > s->G)
    return MOE_ERR_UNSUPPORTED;
  if (s->K > kMaxK || s->K > s->topG * (s->N / s->G)) return MOE_ERR_UNSUPPORTED;
  if (s->d % 32 != 0) return MOE_ERR_UNSUPPORTED;
  if (s->dtype == MOE_DTYPE_FP32) {
    if (s->f >= 128 ? (s->f % 128 != 0) : false) return MOE_ERR_UNSUPPORTED;
  } else {
    if (s->d % 256 != 0 || s->f % 128 != 0) return MOE_ERR_UNSUPPORTED;
  }
  if ((long long)s->T * s->K + s->T >= (1ll << 31)) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

int ws_check(const moe_shape* s, void* ws) {
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & 255u)) return MOE_ERR_ARG;
  (void)s;
  return MOE_OK;
}

int cuda_status(cudaError_t e) {
  note_cuda(e, "kernel launch");
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}


}  // namespace

extern "C" {

const char* moe_status_string(int status) {
  switch (status) {
    case MOE_OK: return "ok";
    case MOE_ERR_ARG: return "bad argument (null or misaligned pointer, non-positive size)";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case MOE_ERR_WORKSPACE: return "workspace too small";
    case MOE_ERR_CUDA: return "CUDA launch or API error";
    case MOE_ERR_DEVICE: return "device-side failure recorded in the workspace status word";
    default: return "unknown status";
  }
}

int moe_check_shape(const moe_shape* shape) { return check(shape); }

size_t moe_workspace_size(const moe_shape* shape) {
  if (check(shape) != MOE_OK) return 0;
  return ws_layout(*shape).total;
}

int moe_workspace_init(void* ws, void* stream) {
  if (!ws) return MOE_ERR_ARG;
  return cuda_status(cudaMemsetAsync(ws, 0, 256, static_cast<cudaStream_t>(stream)));
}

int moe_read_device_status(void* ws, void* stream, uint32_t* status_out, int clear) {
  if (!ws || !status_out) return MOE_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint32_t v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, ws, sizeof(v), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  *status_out = v;
  if (clear && v) {
    e = cudaMemsetAsync(ws, 0, sizeof(uint32_t), st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return MOE_ERR_CUDA;
  }
  return v ? MOE_ERR_DEVICE : MOE_OK;
}

int moe_read_gemm_clock(void* ws, void* stream, uint64_t* counters_out, int clear) {
  if (!ws || !counters_out) return MOE_ERR_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* rec = static_cast<uint8_t*>(ws) + kClockRecordOffset;
  cudaError_t e = cudaMemcpyAsync(counters_out, rec, 4 * sizeof(uint64_t),
                                  cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e == cudaSuccess && clear) {
    e = cudaMemsetAsync(rec, 0, 4 * sizeof(uint64_t), st);
    if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  }
  return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}

int moe_route(const moe_shape* shape, const void* x, const float* router_w, const float* bias,
              int32_t* topk_idx, float* topk_gate, int32_t* counts, void* ws, void* stream) {
  int rc = check(shape);
  if (rc) return rc;
  if (!ptr_ok(x) || !ptr_ok(router_w) || !ptr_ok(bias) || !ptr_ok(topk_idx) ||
      !ptr_ok(topk_gate) || !ptr_ok(counts))
    return MOE_ERR_ARG;
  if ((rc = ws_check(shape, ws))) return rc;
  return launch_route(*shape, x, router_w, bias, topk_idx, topk_gate, counts, ws,
                      static_cast<cudaStream_t>(stream));
}

int moe_route_softmax(const moe_shape* shape, const void* x, const float* router_w,
                      int32_t* topk_idx, float* topk_gate, int32_t* counts, float* prob_sum,
                      void* ws, void* stream) {
  int rc = check(shape);
  if (rc) return rc;
  if (shape->dtype == MOE_DTYPE_FP32) return MOE_ERR_UNSUPPORTED;
  if (!ptr_ok(x) || !ptr_ok(router_w) || !ptr_ok(topk_idx) || !ptr_ok(topk_gate) ||
      !ptr_ok(counts))
    return MOE_ERR_ARG;
  if (prob_sum != nullptr && !aligned16(prob_sum)) return MOE_ERR_ARG;
  if ((rc = ws_check(shape, ws))) return rc;
  return launch_route_softmax(*shape, x, router_w, topk_idx, topk_gate, counts, prob_sum, ws,
                              static_cast<cudaStream_t>(stream));
}

int moe_dispatch(const moe_shape* shape, const void* x, const int32_t* topk_idx,
                 const int32_t* counts, int32_t* offsets, int32_t* perm_tok, int32_t* slot,
                 void* x_perm, float* x_perm_scales, void* ws, void* stream) {
  int rc = check(shape);
  if (rc) return rc;
  if (!ptr_ok(x) || !ptr_ok(topk_idx) || !ptr_ok(counts) || !ptr_ok(offsets) ||
      !ptr_ok(perm_tok) || !ptr_ok(slot))
    return MOE_ERR_ARG;
  // x_perm may be NULL (rows not copied) except in E4M3 mode, which needs the codes
  if (x_perm != nullptr && !aligned16(x_perm)) return MOE_ERR_ARG;
  if (shape->dtype == MOE_DTYPE_E4M3 && (!ptr_ok(x_perm) || !ptr_ok(x_perm_scales)))
    return MOE_ERR_ARG;
  if ((rc = ws_check(shape, ws))) return rc;
  cudaError_t e = launch_dispatch(*shape, x, topk_idx, counts, offsets, perm_tok, slot, x_perm,
                                  x_perm_scales, ws, static_cast<cudaStream_t>(stream));
  if (e == cudaErrorNotSupported) return MOE_ERR_UNSUPPORTED;
  return cuda_status(e);
}

int moe_expert_ffn(const moe_shape* shape, const void* x_perm, const float* x_perm_scales,
                   const int32_t* offsets, const void* x, const void* w13, const void* w2,
                   const float* w13_scales, const float* w2_scales, void* y_perm,
                   void* y_shared, void* ws, void* stream) {
  int rc = check(shape);
  if (rc) return rc;
  if (!ptr_ok(x_perm) || !ptr_ok(offsets) || !ptr_ok(x) || !ptr_ok(w13) || !ptr_ok(w2) ||
      !ptr_ok(y_perm) || !ptr_ok(y_shared))
    return MOE_ERR_ARG;
  if (shape->dtype == MOE_DTYPE_E4M3 &&
      (!ptr_ok(x_perm_scales) || !ptr_ok(w13_scales) || !ptr_ok(w2_scales)))
    return MOE_ERR_ARG;
  if ((rc = ws_check(shape, ws))) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  switch (shape->dtype) {
    case MOE_DTYPE_FP32:
      return cuda_status(launch_ffn_simt(
          *shape, static_cast<const float*>(x_perm), offsets, static_cast<const float*>(x),
          static_cast<const float*>(w13), static_cast<const float*>(w2),
          static_cast<float*>(y_perm), static_cast<float*>(y_shared), ws, st));
    case MOE_DTYPE_BF16:
      return launch_ffn_tc_bf16(*shape, x_perm, nullptr, offsets, x, w13, w2, y_perm, y_shared,
                                ws, st);
    default:
      return launch_ffn_tc_e4m3(*shape, x_perm, x_perm_scales, offsets, x, w13, w2, w13_scales,
                                w2_scales, y_perm, y_shared, ws, st);
  }
}

int moe_expert_ffn_gathered(const moe_shape* shape, const void* x, const int32_t* perm_tok,
                            const int32_t* offsets, const void* w13, const void* w2,
                            void* y_perm, void* y_shared, void* ws, void* stream) {
  int rc = check(shape);
  if (rc) return rc;
  if (shape->dtype != MOE_DTYPE_BF16) return MOE_ERR_UNSUPPORTED;
  if (!ptr_ok(x) || !ptr_ok(perm_tok) || !ptr_ok(offsets) || !ptr_ok(w13) || !ptr_ok(w2) ||
      !ptr_ok(y_perm) || !ptr_ok(y_shared))
    return MOE_ERR_ARG;
  if ((rc = ws_check(shape, ws))) return rc;
  return launch_ffn_tc_bf16(*shape, nullptr, perm_tok, offsets, x, w13, w2, y_perm, y_shared,
                            ws, static_cast<cudaStream_t>(stream));
}

int moe_expert_ffn_combine(const moe_shape* shape, const void* x_perm, const int32_t* offsets,
                           const int32_t* perm_tok, const int32_t* slot, const float* topk_gate,
                           const void* x, const void* w13, const void* w2, void* y_perm,
                           void* y_shared, void* y, void* ws, void* stream) {
  int rc = check(shape);
  if (rc) return rc;
  if (shape->dtype != MOE_DTYPE_BF16) return MOE_ERR_UNSUPPORTED;
  if (!ptr_ok(x_perm) || !ptr_ok(offsets) || !ptr_ok(perm_tok) || !ptr_ok(slot) ||
      !ptr_ok(topk_gate) || !ptr_ok(x) || !ptr_ok(w13) || !ptr_ok(w2) || !ptr_ok(y_perm) ||
      !ptr_ok(y_shared) || !ptr_ok(y))
    return MOE_ERR_ARG;
  if ((rc = ws_check(shape, ws))) return rc;
  return launch_ffn_combine_bf16(*shape, x_perm, offsets, perm_tok, slot, topk_gate, x, w13, w2,
                                 y_perm, y_shared, y, ws, static_cast<cudaStream_t>(stream));
}

size_t moe_backward_workspace_size(const moe_shape* shape) {
  if (check(shape) != MOE_OK) return 0;
  if (shape->dtype == MOE_DTYPE_BF16) return backward_ws_bytes(*shape);
  if (shape->dtype == MOE_DTYPE_E4M3) return bwd_layout_fp8(*shape).total;
  return 0;
}

int moe_quantize_weights_transposed(const moe_shape* shape, const void* w13t, const void* w2t,
                                    void* w13t_q, float* w13t_scales, void* w2t_q,
                                    float* w2t_scales, void* stream) {
  int rc = check(shape);
  if (rc) return rc;
  if (shape->dtype != MOE_DTYPE_E4M3) return MOE_ERR_UNSUPPORTED;
  if (!ptr_ok(w13t) || !ptr_ok(w2t) || !ptr_ok(w13t_q) || !ptr_ok(w13t_scales) ||
      !ptr_ok(w2t_q) || !ptr_ok(w2t_scales))
    return MOE_ERR_ARG;
  return cuda_status(launch_quantize_weights_transposed(*shape, w13t, w2t, w13t_q, w13t_scales,
                                                        w2t_q, w2t_scales,
                                                        static_cast<cudaStream_t>(stream)));
}

int moe_expert_ffn_backward_dw_fp8(const moe_shape* shape, const int32_t* perm_tok,
                                   const int32_t* offsets, const void* x, const void* dy_perm,
                                   const void* dy_shared, void* dw13, void* dw2, void* ws_bwd,
                                   void* stream) {
  int rc = check(shape);
  if (rc) return rc;
  if (shape->dtype != MOE_DTYPE_E4M3 || shape->f % 256 != 0) return MOE_ERR_UNSUPPORTED;
  if (!ptr_ok(perm_tok) || !ptr_ok(offsets) || !ptr_ok(x) || !ptr_ok(dy_perm) ||
      !ptr_ok(dy_shared) || !ptr_ok(dw13) || !ptr_ok(dw2) || ws_check(shape, ws_bwd) != MOE_OK)
    return MOE_ERR_ARG;
  return launch_ffn_bwd_dw_e4m3(*shape, perm_tok, offsets, x, dy_perm, dy_shared, dw13, dw2,
                                ws_bwd, static_cast<cudaStream_t>(stream));
}

int moe_expert_ffn_backward_dx_fp8(const moe_shape* shape, const void* x_perm,
                                   const float* x_perm_scales, const int32_t* offsets,
                                   const void* x, const void* w13, const float* w13_scales,
                                   const void* w13t, const float* w13t_scales, const void* w2t,
                                   const float* w2t_scales, const void* dy_perm,
                                   const void* dy_shared, void* dx_perm, void* dx_shared,
                                   void* ws_bwd, void* stream) {
  int rc = check(shape);
  if (rc) return rc;
  if (shape->dtype != MOE_DTYPE_E4M3 || shape->f % 256 != 0) return MOE_ERR_UNSUPPORTED;
  if (!ptr_ok(x_perm) || !ptr_ok(x_perm_scales) || !ptr_ok(offsets) || !ptr_ok(x) ||
      !ptr_ok(w13) || !ptr_ok(w13_scales) || !ptr_ok(w13t) || !ptr_ok(w13t_scales) ||
      !ptr_ok(w2t) || !ptr_ok(w2t_scales) || !ptr_ok(dy_perm) || !ptr_ok(dy_shared) ||
      !ptr_ok(dx_perm) || !ptr_ok(dx_shared) || ws_check(shape, ws_bwd) != MOE_OK)
    return MOE_ERR_ARG;
  return launch_ffn_bwd_dx_e4m3(*shape, x_perm, x_perm_scales, offsets, x, w13, w13_scales, w13t,
                                w13t_scales, w2t, w2t_scales, dy_perm, dy_shared, dx_perm,
                                dx_shared, ws_bwd, static_cast<cudaStream_t>(stream));
}

int moe_transpose_weights(const moe_shape* shape, const void* w13, const void* w2, void* w13t,
                          void* w2t, void* stream) {
  int rc = check(shape);
  if (rc) return rc;
  if (shape->dtype == MOE_DTYPE_FP32) return MOE_ERR_UNSUPPORTED;  // bf16 weights
  if (!ptr_ok(w13) || !ptr_ok(w2) || !ptr_ok(w13t) || !ptr_ok(w2t)) return MOE_ERR_ARG;
  return cuda_status(launch_transpose_weights(*shape, w13, w2, w13t, w2t,
                                              static_cast<cudaStream_t>(stream)));
}

int moe_expert_ffn_backward_dx(const moe_shape* shape, const void* x_perm,
                               const int32_t* offsets, const void* x, const void* w13,
                               const void* w13t, const void* w2t, const void* dy_perm,
                               const void* dy_shared, void* dx_perm, void* dx_shared,
                               void* ws_bwd, void* stream) {
  int rc = check(shape);
  if (rc) return rc;
  if (shape->dtype != MOE_DTYPE_BF16) return MOE_ERR_UNSUPPORTED;
  if (!ptr_ok(x_perm) || !ptr_ok(offsets) || !ptr_ok(x) || !ptr_ok(w13) || !ptr_ok(w13t) ||
      !ptr_ok(w2t) || !ptr_ok(dy_perm) || !ptr_ok(dy_shared) || !ptr_ok(dx_perm) ||
      !ptr_ok(dx_shared) || !ptr_ok(ws_bwd))
    return MOE_ERR_ARG;
  return launch_ffn_bwd_dx_bf16(*shape, x_perm, offsets, x, w13, w13t, w2t, dy_perm, dy_shared,
                                dx_perm, dx_shared, ws_bwd, static_cast<cudaStream_t>(stream));
}

int moe_expert_ffn_backward_dw(const moe_shape* shape, const void* x_perm,
                               const int32_t* offsets, const void* x, const void* dy_perm,
                               const void* dy_shared, void* dw13, void* dw2, void* ws_bwd,
                               void* stream) {
  int rc = check(shape);
  if (rc) return rc;
  if (shape->dtype != MOE_DTYPE_BF16 || shape->f % 256 != 0) return MOE_ERR_UNSUPPORTED;
  if (!ptr_ok(x_perm) || !ptr_ok(offsets) || !ptr_ok(x) || !ptr_ok(dy_perm) ||
      !ptr_ok(dy_shared) || !ptr_ok(dw13) || !ptr_ok(dw2) || !ptr_ok(ws_bwd))
    return MOE_ERR_ARG;
  return launch_ffn_bwd_dw_bf16(*shape, x_perm, offsets, x, dy_perm, dy_shared, dw13, dw2,
                                ws_bwd, static_cast<cudaStream_t>(stream));
}

int moe_combine(const moe_shape* shape, const void* y_perm, const void* y_shared,
                const int32_t* slot, const float* topk_gate, void* y, void* stream) {
  int rc = check(shape);
  if (rc) return rc;
  if (!ptr_ok(y_perm) || !ptr_ok(y_shared) || !ptr_ok(slot) || !ptr_ok(topk_gate) ||
      !ptr_ok(y))
    return MOE_ERR_ARG;
  return cuda_status(launch_combine(*shape, y_perm, y_shared, slot, topk_gate, y,
                                    static_cast<cudaStream_t>(stream)));
}

int moe_combine_backward(const moe_shape* shape, const void* dy, const void* y_perm,
                         const int32_t* slot, const float* topk_gate, void* dy_perm,
                         float* dgate, void* stream) {
  int rc = check(shape);
  if (rc) return rc;
  if (!ptr_ok(dy) || !ptr_ok(y_perm) || !ptr_ok(slot) || !ptr_ok(topk_gate) ||
      !ptr_ok(dy_perm) || !ptr_ok(dgate))
    return MOE_ERR_ARG;
  return cuda_status(launch_combine_backward(*shape, dy, y_perm, slot, topk_gate, dy_perm, dgate,
                                             static_cast<cudaStream_t>(stream)));
}

int moe_route_backward(const moe_shape* shape, const void* x, const float* router_w,
                       const int32_t* topk_idx, const float* dgate, const int32_t* offsets,
                       const int32_t* perm_tok, const int32_t* slot, float* dlogit,
                       float* dx_route, float* drouter, void* stream) {
  int rc = check(shape);
  if (rc) return rc;
  if (!ptr_ok(x) || !ptr_ok(router_w) || !ptr_ok(topk_idx) || !ptr_ok(dgate) ||
      !ptr_ok(offsets) || !ptr_ok(perm_tok) || !ptr_ok(slot) || !ptr_ok(dlogit) ||
      !ptr_ok(dx_route) || !ptr_ok(drouter))
    return MOE_ERR_ARG;
  return cuda_status(launch_route_backward(*shape, x, router_w, topk_idx, dgate, offsets,
                                           perm_tok, slot, dlogit, dx_route, drouter,
                                           static_cast<cudaStream_t>(stream)));
}

int moe_dispatch_backward(const moe_shape* shape, const void* dx_perm, const void* dx_shared,
                          const int32_t* slot, const float* dx_route, void* dx, void* stream) {
  int rc = check(shape);
  if (rc) return rc;
  if (!ptr_ok(dx_perm) || !ptr_ok(dx_shared) || !ptr_ok(slot) || !ptr_ok(dx) ||
      (dx_route != nullptr && !ptr_ok(dx_route)))
    return MOE_ERR_ARG;
  return cuda_status(launch_dispatch_backward(*shape, dx_perm, dx_shared, slot, dx_route, dx,
                                              static_cast<cudaStream_t>(stream)));
}

int moe_quantize_rows_e5m2(const void* g, int64_t rows, int cols, uint8_t* codes,
                           float* scales, int64_t sc_ld, void* stream) {
  if (rows <= 0 || cols <= 0 || cols % 128 != 0 || sc_ld < rows) return MOE_ERR_ARG;
  if (rows > (int64_t{1} << 40) / cols) return MOE_ERR_UNSUPPORTED;
  if (!ptr_ok(g) || !ptr_ok(codes) || !ptr_ok(scales)) return MOE_ERR_ARG;
  return cuda_status(launch_quant_rows_e5m2(g, rows, cols, codes, scales, sc_ld,
                                            static_cast<cudaStream_t>(stream)));
}

int moe_bias_update(const moe_shape* shape, const int32_t* counts, float* bias, float gamma,
                    void* stream) {
  int rc = check(shape);
  if (rc) return rc;
  if (!ptr_ok(counts) || !ptr_ok(bias)) return MOE_ERR_ARG;
  if (!(gamma >= 0.f) || gamma != gamma) return MOE_ERR_ARG;
  return cuda_status(launch_bias_update(*shape, counts, bias, gamma,
                                        static_cast<cudaStream_t>(stream)));
}

int moe_pack_w13(const moe_shape* shape, const void* w1, const void* w3, void* w13,
                 void* stream) {
  int rc = check(shape);
  if (rc) return rc;
  if (!ptr_ok(w1) || !ptr_ok(w3) || !ptr_ok(w13)) return MOE_ERR_ARG;
  return cuda_status(launch_pack_w13(*shape, w1, w3, w13, static_cast<cudaStream_t>(stream)));
}

int moe_quantize_weights(const moe_shape* shape, const void* w13_bf16, const void* w2_bf16,
                         void* w13_q, float* w13_scales, void* w2_q, float* w2_scales,
                         void* stream) {
  int rc = check(shape);
  if (rc) return rc;
  if (shape->dtype != MOE_DTYPE_E4M3) return MOE_ERR_UNSUPPORTED;
  if (!ptr_ok(w13_bf16) || !ptr_ok(w2_bf16) || !ptr_ok(w13_q) || !ptr_ok(w13_scales) ||
      !ptr_ok(w2_q) || !ptr_ok(w2_scales))
    return MOE_ERR_ARG;
  cudaError_t e = launch_quantize_weights(*shape, w13_bf16, w2_bf16, w13_q, w13_scales, w2_q,
                                          w2_scales, static_cast<cudaStream_t>(stream));
  if (e == cudaErrorNotSupported) return MOE_ERR_UNSUPPORTED;
  return cuda_status(e);
}

int moe_forward(const moe_shape* shape, const void* x, const float* router_w, float* bias,
                float gamma, const void* w13, const void* w2, const float* w13_scales,
                const float* w2_scales, int32_t* topk_idx, float* topk_gate, int32_t* counts,
                int32_t* offsets, int32_t* perm_tok, int32_t* slot, void* x_perm,
                float* x_perm_scales, void* y_perm, void* y_shared, void* y, void* ws,
                void* stream) {
  int rc = moe_route(shape, x, router_w, bias, topk_idx, topk_gate, counts, ws, stream);
  if (rc) return rc;
  rc = moe_dispatch(shape, x, topk_idx, counts, offsets, perm_tok, slot, x_perm, x_perm_scales,
                    ws, stream);
  if (rc) return rc;
  rc = moe_expert_ffn(shape, x_perm, x_perm_scales, offsets, x, w13, w2, w13_scales, w2_scales,
                      y_perm, y_shared, ws, stream);
  if (rc) return rc;
  rc = moe_combine(shape, y_perm, y_shared, slot, topk_gate, y, stream);
  if (rc) return rc;
  return moe_bias_update(shape, counts, bias, gamma, stream);
}

}  // extern "C"
