// C-ABI entry points: argument validation, then the kernel launchers.
#include <string.h>

#include "common.cuh"

using namespace nvfp4;

namespace nvfp4 {
nvfp4_status launch_hessian_simt(float* H, const void* X, nvfp4_dtype xt, int64_t n_tok,
                                 int64_t d, int beta, cudaStream_t st);
}

namespace {

bool params_ok(const nvfp4_solve_params* p) {
  if (!p) return true;
  return p->n_candidates == kCand && p->cand_lo == -8 && p->lazy_batch == kLazyBatch &&
         p->scale_rule >= NVFP4_RULE_SCHUR_REPLAY && p->scale_rule <= NVFP4_RULE_BLOCK_MSE &&
         p->precision == NVFP4_PRECISION_FP64_REPLAY;
}

bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255) == 0; }
bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Largest dimension this build accepts; keeps every int index below 2^31.
constexpr int64_t kMaxDim = 1 << 17;
// Largest row count (output channels) accepted; keeps grid.y within 65535 tiles.
constexpr int64_t kMaxRows = 1 << 22;

}  // namespace

extern "C" {

void nvfp4_default_params(nvfp4_solve_params* p) {
  if (!p) return;
  p->n_candidates = kCand;
  p->cand_lo = -8;
  p->lazy_batch = kLazyBatch;
  p->scale_rule = NVFP4_RULE_SCHUR_REPLAY;
  p->precision = NVFP4_PRECISION_FP64_REPLAY;
}

const char* nvfp4_status_string(nvfp4_status s) {
  switch (s) {
    case NVFP4_OK: return "ok";
    case NVFP4_ERR_INVALID_ARG: return "invalid argument";
    case NVFP4_ERR_SHAPE: return "unsupported shape (dimension must be a multiple of 16)";
    case NVFP4_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case NVFP4_ERR_NONFINITE: return "non-finite value in the input";
    case NVFP4_ERR_NOT_PD: return "damped Hessian is not positive definite";
    case NVFP4_ERR_TIMEOUT: return "bounded device wait timed out";
    case NVFP4_ERR_CUDA: return "CUDA error";
    case NVFP4_ERR_UNSUPPORTED: return "unsupported parameter value";
    case NVFP4_ERR_BOUNDS: return "index left its array (debug build check)";
  }
  return "unknown status";
}

nvfp4_status nvfp4_workspace_status(const void* ws, nvfp4_stream_t stream) {
  if (!ws) return NVFP4_ERR_INVALID_ARG;
  int v = 0;
  NVFP4_CUDA_TRY(cudaMemcpyAsync(&v, ws, sizeof(int), cudaMemcpyDeviceToHost, as_cuda(stream)));
  NVFP4_CUDA_TRY(cudaStreamSynchronize(as_cuda(stream)));
  return static_cast<nvfp4_status>(v);
}

nvfp4_status nvfp4_hessian_accumulate(float* H, const void* X, nvfp4_dtype x_dtype,
                                      int64_t n_tok, int64_t d, int beta,
                                      nvfp4_stream_t stream) {
  if (!H || n_tok < 0 || d < 0 || (n_tok > 0 && !X)) return NVFP4_ERR_INVALID_ARG;
  if (x_dtype != NVFP4_BF16 && x_dtype != NVFP4_F32) return NVFP4_ERR_INVALID_ARG;
  if (beta != 0 && beta != 1) return NVFP4_ERR_INVALID_ARG;
  if (d % 16 || d > kMaxDim) return NVFP4_ERR_SHAPE;
  if (d == 0) return NVFP4_OK;
  ProfileScope ps(kPhaseHessian, as_cuda(stream));
  if (hessian_tc_supported(H, X, x_dtype, n_tok, d))
    return launch_hessian_tc(H, X, n_tok, d, beta, as_cuda(stream));
  return launch_hessian_simt(H, X, x_dtype, n_tok, d, beta, as_cuda(stream));
}

size_t nvfp4_hessian_host_workspace_size(int64_t d, int64_t chunk_tok, nvfp4_dtype x_dtype) {
  if (d < 0 || chunk_tok < 1 || (x_dtype != NVFP4_BF16 && x_dtype != NVFP4_F32)) return 0;
  return hessian_host_ws_bytes(d, chunk_tok, x_dtype);
}

nvfp4_status nvfp4_hessian_accumulate_host(float* H, const void* X_host, nvfp4_dtype x_dtype,
                                           int64_t n_tok, int64_t d, int beta,
                                           int64_t chunk_tok, void* ws, size_t ws_bytes,
                                           nvfp4_stream_t stream) {
  if (!H || n_tok < 0 || d < 0 || (n_tok > 0 && !X_host) || chunk_tok < 1)
    return NVFP4_ERR_INVALID_ARG;
  if (x_dtype != NVFP4_BF16 && x_dtype != NVFP4_F32) return NVFP4_ERR_INVALID_ARG;
  if (beta != 0 && beta != 1) return NVFP4_ERR_INVALID_ARG;
  if (d % 16 || d > kMaxDim) return NVFP4_ERR_SHAPE;
  if (d == 0) return NVFP4_OK;
  if (n_tok > 0 && (!ws || !aligned256(ws) ||
                    ws_bytes < hessian_host_ws_bytes(d, chunk_tok, x_dtype)))
    return NVFP4_ERR_WORKSPACE;
  ProfileScope ps(kPhaseHessian, as_cuda(stream));
  return launch_hessian_host(H, X_host, x_dtype, n_tok, d, beta, chunk_tok, ws,
                             as_cuda(stream));
}

nvfp4_status nvfp4_hessian_status(nvfp4_stream_t stream) {
  return static_cast<nvfp4_status>(hessian_tc_take_status(as_cuda(stream)));
}

size_t nvfp4_prepare_workspace_size(int64_t d) {
  if (d < 0) return 0;
  return prepare_ws_bytes(d);
}

nvfp4_status nvfp4_gptq_prepare(const float* H, int64_t d, float damp, float* U,
                                uint8_t* dead, float* lambda_out, void* ws, size_t ws_bytes,
                                nvfp4_stream_t stream) {
  if (!H || !U || d < 0 || !(damp >= 0.f)) return NVFP4_ERR_INVALID_ARG;
  if (d % 16 || d > kMaxDim) return NVFP4_ERR_SHAPE;
  if (!ws || !aligned256(ws) || ws_bytes < prepare_ws_bytes(d)) return NVFP4_ERR_WORKSPACE;
  if (d == 0) return NVFP4_OK;
  ProfileScope ps(kPhasePrepare, as_cuda(stream));
  return launch_prepare(H, false, d, damp, U, dead, lambda_out, ws, as_cuda(stream));
}

nvfp4_status nvfp4_gptq_prepare_f64(const double* H, int64_t d, float damp, float* U,
                                    uint8_t* dead, float* lambda_out, void* ws, size_t ws_bytes,
                                    nvfp4_stream_t stream) {
  if (!H || !U || d < 0 || !(damp >= 0.f)) return NVFP4_ERR_INVALID_ARG;
  if (d % 16 || d > kMaxDim) return NVFP4_ERR_SHAPE;
  if (!ws || !aligned256(ws) || ws_bytes < prepare_ws_bytes(d)) return NVFP4_ERR_WORKSPACE;
  if (d == 0) return NVFP4_OK;
  ProfileScope ps(kPhasePrepare, as_cuda(stream));
  return launch_prepare(H, true, d, damp, U, dead, lambda_out, ws, as_cuda(stream));
}

size_t nvfp4_hessian_f64_workspace_size(int64_t n_tok, int64_t d) {
  if (n_tok < 0 || d < 0) return 0;
  return hessian_f64_ws_bytes(n_tok, d);
}

nvfp4_status nvfp4_hessian_accumulate_f64(double* H, const void* X, nvfp4_dtype x_dtype,
                                          int64_t n_tok, int64_t d, int beta, void* ws,
                                          size_t ws_bytes, nvfp4_stream_t stream) {
  if (!H || n_tok < 0 || d < 0 || (n_tok > 0 && !X)) return NVFP4_ERR_INVALID_ARG;
  if (x_dtype != NVFP4_BF16 && x_dtype != NVFP4_F32) return NVFP4_ERR_INVALID_ARG;
  if (beta != 0 && beta != 1) return NVFP4_ERR_INVALID_ARG;
  if (d % 16 || d > kMaxDim) return NVFP4_ERR_SHAPE;
  if (d == 0) return NVFP4_OK;
  if (!ws || !aligned256(ws) || ws_bytes < hessian_f64_ws_bytes(n_tok, d))
    return NVFP4_ERR_WORKSPACE;
  ProfileScope ps(kPhaseHessian, as_cuda(stream));
  return launch_hessian_f64(H, X, x_dtype, n_tok, d, beta, ws, as_cuda(stream));
}

size_t nvfp4_quantize_workspace_size(int64_t d_out, int64_t d_in,
                                     const nvfp4_solve_params* params) {
  (void)params;
  if (d_out < 0 || d_in < 0) return 0;
  return quantize_ws_bytes(d_out, d_in);
}

nvfp4_status nvfp4_gptq_schur_replay_quantize(
    const void* W, nvfp4_dtype w_dtype, int64_t d_out, int64_t d_in, const float* U,
    const nvfp4_solve_params* params, const uint8_t* dead, uint8_t* codes, uint8_t* scales,
    float* global_scale, double* err_out, void* ws, size_t ws_bytes, nvfp4_stream_t stream) {
  if (d_out < 0 || d_in < 0 || !global_scale) return NVFP4_ERR_INVALID_ARG;
  if (d_out > 0 && d_in > 0 && (!W || !U || !codes || !scales)) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(W, 16) || !aligned(codes, 8)) return NVFP4_ERR_INVALID_ARG;
  if (w_dtype != NVFP4_BF16 && w_dtype != NVFP4_F32) return NVFP4_ERR_INVALID_ARG;
  if (!params_ok(params)) return NVFP4_ERR_UNSUPPORTED;
  if (d_in % 16 || d_in > kMaxDim || d_out > kMaxRows) return NVFP4_ERR_SHAPE;
  if (!ws || !aligned256(ws) || ws_bytes < quantize_ws_bytes(d_out, d_in))
    return NVFP4_ERR_WORKSPACE;
  const int rule = params ? params->scale_rule : NVFP4_RULE_SCHUR_REPLAY;
  return launch_quantize(W, w_dtype, d_out, d_in, U, dead, rule, codes, scales, global_scale,
                         err_out, ws, as_cuda(stream));
}

size_t nvfp4_export_scales_size(int64_t d_out, int64_t d_in) {
  if (d_out < 0 || d_in < 0 || d_in % 16) return 0;
  return scales_tiled_bytes(d_out, d_in);
}

nvfp4_status nvfp4_export_scales(const uint8_t* scales, int64_t d_out, int64_t d_in,
                                 uint8_t* out, nvfp4_stream_t stream) {
  if (d_out < 0 || d_in < 0) return NVFP4_ERR_INVALID_ARG;
  if (d_in % 16) return NVFP4_ERR_SHAPE;
  if (d_out > 0 && d_in > 0 && (!scales || !out)) return NVFP4_ERR_INVALID_ARG;
  return launch_scales_tiled(scales, d_out, d_in, out, as_cuda(stream));
}

nvfp4_status nvfp4_weight_amax(const void* W, nvfp4_dtype w_dtype, int64_t d_out, int64_t d_in,
                               const uint8_t* dead, float* amax_out, nvfp4_stream_t stream) {
  if (d_out < 0 || d_in < 0 || !amax_out || (d_out > 0 && d_in > 0 && !W))
    return NVFP4_ERR_INVALID_ARG;
  if (w_dtype != NVFP4_BF16 && w_dtype != NVFP4_F32) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(amax_out, 4)) return NVFP4_ERR_INVALID_ARG;
  return launch_weight_amax(W, w_dtype, d_out, d_in, dead, amax_out, as_cuda(stream));
}

nvfp4_status nvfp4_gptq_schur_replay_quantize_rows(
    const void* W, nvfp4_dtype w_dtype, int64_t d_out, int64_t d_in, const float* U,
    const nvfp4_solve_params* params, const uint8_t* dead, const float* amax,
    uint8_t* codes, uint8_t* scales, float* global_scale, double* err_out, void* ws,
    size_t ws_bytes, nvfp4_stream_t stream) {
  if (!amax) return NVFP4_ERR_INVALID_ARG;
  if (d_out < 0 || d_in < 0 || !global_scale) return NVFP4_ERR_INVALID_ARG;
  if (d_out > 0 && d_in > 0 && (!W || !U || !codes || !scales)) return NVFP4_ERR_INVALID_ARG;
  if (!aligned(W, 16) || !aligned(codes, 8)) return NVFP4_ERR_INVALID_ARG;
  if (w_dtype != NVFP4_BF16 && w_dtype != NVFP4_F32) return NVFP4_ERR_INVALID_ARG;
  if (!params_ok(params)) return NVFP4_ERR_UNSUPPORTED;
  if (d_in % 16 || d_in > kMaxDim || d_out > kMaxRows) return NVFP4_ERR_SHAPE;
  if (!ws || !aligned256(ws) || ws_bytes < quantize_ws_bytes(d_out, d_in))
    return NVFP4_ERR_WORKSPACE;
  const int rule = params ? params->scale_rule : NVFP4_RULE_SCHUR_REPLAY;
  return launch_quantize(W, w_dtype, d_out, d_in, U, dead, rule, codes, scales, global_scale,
                         err_out, ws, as_cuda(stream), amax);
}

nvfp4_status nvfp4_dequant(const uint8_t* codes, const uint8_t* scales,
                           const float* global_scale, int64_t d_out, int64_t d_in, void* out,
                           nvfp4_dtype out_dtype, nvfp4_stream_t stream) {
  if (d_out < 0 || d_in < 0) return NVFP4_ERR_INVALID_ARG;
  if (d_out > 0 && d_in > 0 && (!codes || !scales || !global_scale || !out))
    return NVFP4_ERR_INVALID_ARG;
  if (!aligned(codes, 8) || !aligned(out, 16)) return NVFP4_ERR_INVALID_ARG;
  if (out_dtype != NVFP4_BF16 && out_dtype != NVFP4_F32) return NVFP4_ERR_INVALID_ARG;
  if (d_in % 16) return NVFP4_ERR_SHAPE;
  ProfileScope ps(kPhaseDequant, as_cuda(stream));
  return launch_dequant(codes, scales, global_scale, d_out, d_in, out, out_dtype,
                        as_cuda(stream));
}

size_t nvfp4_layer_error_workspace_size(int64_t d_out, int64_t d_in) {
  if (d_out < 0 || d_in < 0) return 0;
  return layer_error_ws_bytes(d_out, d_in);
}

nvfp4_status nvfp4_layer_error(const void* W, nvfp4_dtype w_dtype, const uint8_t* codes,
                               const uint8_t* scales, const float* global_scale,
                               const float* H, int64_t d_out, int64_t d_in, double* err_out,
                               void* ws, size_t ws_bytes, nvfp4_stream_t stream) {
  if (d_out < 0 || d_in < 0 || !err_out) return NVFP4_ERR_INVALID_ARG;
  if (d_out > 0 && d_in > 0 && (!W || !codes || !scales || !global_scale || !H))
    return NVFP4_ERR_INVALID_ARG;
  if (!aligned(codes, 8)) return NVFP4_ERR_INVALID_ARG;
  if (w_dtype != NVFP4_BF16 && w_dtype != NVFP4_F32) return NVFP4_ERR_INVALID_ARG;
  if (d_in % 16 || d_in > kMaxDim || d_out > kMaxRows) return NVFP4_ERR_SHAPE;
  if (!ws || !aligned256(ws) || ws_bytes < layer_error_ws_bytes(d_out, d_in))
    return NVFP4_ERR_WORKSPACE;
  return launch_layer_error(W, w_dtype, codes, scales, global_scale, H, d_out, d_in, err_out,
                            ws, as_cuda(stream));
}

nvfp4_status nvfp4_gemm_nt_f32(int64_t M, int64_t N, int64_t K, float alpha, const float* P,
                               int64_t ldp, const float* Q, int64_t ldq, float beta, float* C,
                               int64_t ldc, int lower, int* status, nvfp4_stream_t stream) {
  if (M < 0 || N < 0 || K < 0 || !status || (lower && M != N)) return NVFP4_ERR_INVALID_ARG;
  if (M > kMaxRows || N > kMaxRows || K > kMaxDim) return NVFP4_ERR_SHAPE;
  if (M == 0 || N == 0) return NVFP4_OK;
  if (!P || !Q || !C || ldp < K || ldq < K || ldc < N) return NVFP4_ERR_INVALID_ARG;
  return gemm_nt_tc((int)M, (int)N, (int)K, alpha, P, ldp, 0, Q, ldq, 0, beta, C, ldc, 0,
                    nullptr, 0, 0, 1, lower ? 1 : 0, status, as_cuda(stream));
}

}  // extern "C"
