// Batched forms of the C-ABI calls: `count` independent problems in one call,
// e.g. the experts of a mixture-of-experts layer, each with its own Hessian,
// factor and weights.
//
// Problems of equal shape form a group (in their order of appearance, at most
// kMaxGroup per group) and every kernel launch of the call covers a whole
// group: the Hessian tiles of all its problems (ragged token counts), the
// factorisation's panels and GEMMs of all its problems (their matrices a
// uniform stride apart in the call's one workspace), the replay rows and
// update tiles of all its weight matrices.  A group runs exactly the kernels
// of the single-problem call with one more grid dimension, so every result
// equals the single call's bit for bit; the number of launches depends on the
// number of distinct shapes, not on the number of problems.
#include <vector>

#include "common.cuh"

namespace nvfp4 {
namespace {

// Problems grouped by key (first appearance order), at most kMaxGroup each.
template <typename Key>
std::vector<std::vector<int>> group_by(int count, Key key) {
  std::vector<std::vector<int>> groups;
  std::vector<int> open;   // index into groups of the open group of each key seen
  for (int i = 0; i < count; ++i) {
    int g = -1;
    for (int o : open)
      if (key(groups[o][0]) == key(i) && (int)groups[o].size() < kMaxGroup) {
        g = o;
        break;
      }
    if (g < 0) {
      groups.push_back({});
      g = (int)groups.size() - 1;
      open.push_back(g);
    }
    groups[g].push_back(i);
  }
  return groups;
}

bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255) == 0; }

__global__ void gather_status_kernel(int* batch_hdr, const int* gstatus,
                                     PtrArr<const int*> pstatus, PtrArr<int> idx, int P) {
  for (int i = threadIdx.x; i < P; i += blockDim.x) {
    int v = *pstatus.p[i];
    if (v == 0) v = *gstatus;   // a timed-out GEMM wait belongs to the whole group
    batch_hdr[1 + idx.p[i]] = v;
    if (v) atomicCAS(batch_hdr, 0, v);
  }
}

size_t prepare_batched_bytes(int count, const int64_t* d) {
  size_t b = batch_header_bytes(count);
  for (const auto& g : group_by(count, [&](int i) { return d[i]; }))
    b += prepare_group_ws_bytes(d[g[0]], (int)g.size());
  return b;
}

size_t layer_error_batched_bytes(int count, const int64_t* d_out, const int64_t* d_in) {
  size_t b = batch_header_bytes(count);
  for (const auto& g :
       group_by(count, [&](int i) { return std::make_pair(d_out[i], d_in[i]); }))
    b += layer_error_group_ws_bytes(d_out[g[0]], d_in[g[0]], (int)g.size());
  return b;
}

size_t quantize_batched_bytes(int count, const int64_t* d_out, const int64_t* d_in) {
  size_t b = batch_header_bytes(count);
  for (const auto& g :
       group_by(count, [&](int i) { return std::make_pair(d_out[i], d_in[i]); }))
    b += quantize_group_ws_bytes(d_out[g[0]], d_in[g[0]], (int)g.size());
  return b;
}

}  // namespace

nvfp4_status gather_group_status(int* batch_hdr, const int* group_status,
                                 const PtrArr<const int*>& per_problem_status,
                                 const PtrArr<int>& idx, int P, cudaStream_t st) {
  gather_status_kernel<<<1, 256, 0, st>>>(batch_hdr, group_status, per_problem_status, idx, P);
  NVFP4_LAUNCH_CHECK();
  count_launches(1);
  return NVFP4_OK;
}

}  // namespace nvfp4

using namespace nvfp4;

extern "C" {

size_t nvfp4_prepare_batched_workspace_size(int count, const int64_t* d) {
  if (count < 0 || (count > 0 && !d)) return 0;
  for (int i = 0; i < count; ++i)
    if (d[i] < 0) return 0;
  return prepare_batched_bytes(count, d);
}

size_t nvfp4_quantize_batched_workspace_size(int count, const int64_t* d_out,
                                             const int64_t* d_in,
                                             const nvfp4_solve_params* params) {
  (void)params;
  if (count < 0 || (count > 0 && (!d_out || !d_in))) return 0;
  for (int i = 0; i < count; ++i)
    if (d_out[i] < 0 || d_in[i] < 0) return 0;
  return quantize_batched_bytes(count, d_out, d_in);
}

nvfp4_status nvfp4_batched_workspace_status(const void* ws, int count, int* status,
                                            nvfp4_stream_t stream) {
  if (!ws || count < 0) return NVFP4_ERR_INVALID_ARG;
  std::vector<int> v((size_t)count + 1, 0);
  NVFP4_CUDA_TRY(cudaMemcpyAsync(v.data(), ws, sizeof(int) * v.size(), cudaMemcpyDeviceToHost,
                                 as_cuda(stream)));
  NVFP4_CUDA_TRY(cudaStreamSynchronize(as_cuda(stream)));
  if (status)
    for (int i = 0; i < count; ++i) status[i] = v[1 + i];
  return static_cast<nvfp4_status>(v[0]);
}

nvfp4_status nvfp4_hessian_accumulate_batched(int count, float* const* H, const void* const* X,
                                              nvfp4_dtype x_dtype, const int64_t* n_tok,
                                              const int64_t* d, int beta,
                                              nvfp4_stream_t stream) {
  if (count < 0 || (count > 0 && (!H || !X || !n_tok || !d))) return NVFP4_ERR_INVALID_ARG;
  if (x_dtype != NVFP4_BF16 && x_dtype != NVFP4_F32) return NVFP4_ERR_INVALID_ARG;
  if (beta != 0 && beta != 1) return NVFP4_ERR_INVALID_ARG;
  for (int i = 0; i < count; ++i) {
    if (!H[i] || n_tok[i] < 0 || d[i] < 0 || (n_tok[i] > 0 && !X[i]))
      return NVFP4_ERR_INVALID_ARG;
    if (d[i] % 16 || d[i] > (1 << 17)) return NVFP4_ERR_SHAPE;
  }
  cudaStream_t st = as_cuda(stream);
  ProfileScope ps(kPhaseHessian, st);
  // the tensor-core problems in groups of one dimension; the rest one by one
  std::vector<int> tc, other;
  for (int i = 0; i < count; ++i) {
    if (d[i] == 0) continue;
    (hessian_tc_supported(H[i], X[i], x_dtype, n_tok[i], d[i]) ? tc : other).push_back(i);
  }
  for (int i : other) {
    const nvfp4_status s =
        nvfp4_hessian_accumulate(H[i], X[i], x_dtype, n_tok[i], d[i], beta, stream);
    if (s != NVFP4_OK) return s;
  }
  const int n_tc = (int)tc.size();
  for (const auto& g : group_by(n_tc, [&](int k) { return d[tc[k]]; })) {
    std::vector<float*> h;
    std::vector<const void*> x;
    std::vector<int64_t> n;
    for (int k : g) {
      h.push_back(H[tc[k]]);
      x.push_back(X[tc[k]]);
      n.push_back(n_tok[tc[k]]);
    }
    const nvfp4_status s = launch_hessian_tc_group((int)g.size(), h.data(), x.data(), n.data(),
                                                   d[tc[g[0]]], beta, st);
    if (s != NVFP4_OK) return s;
  }
  return NVFP4_OK;
}

nvfp4_status nvfp4_gptq_prepare_batched(int count, const float* const* H, const int64_t* d,
                                        float damp, float* const* U, uint8_t* const* dead,
                                        float* const* lambda_out, void* ws, size_t ws_bytes,
                                        nvfp4_stream_t stream) {
  if (count < 0 || (count > 0 && (!H || !d || !U))) return NVFP4_ERR_INVALID_ARG;
  if (!(damp >= 0.f)) return NVFP4_ERR_INVALID_ARG;
  for (int i = 0; i < count; ++i) {
    if (!H[i] || !U[i] || d[i] < 0) return NVFP4_ERR_INVALID_ARG;
    if (d[i] % 16 || d[i] > (1 << 17)) return NVFP4_ERR_SHAPE;
  }
  if (count == 0) return NVFP4_OK;
  if (!ws || !aligned256(ws) || ws_bytes < prepare_batched_bytes(count, d))
    return NVFP4_ERR_WORKSPACE;
  cudaStream_t st = as_cuda(stream);
  int* bh = static_cast<int*>(ws);
  NVFP4_CUDA_TRY(cudaMemsetAsync(bh, 0, batch_header_bytes(count), st));
  char* region = static_cast<char*>(ws) + batch_header_bytes(count);
  ProfileScope ps(kPhasePrepare, st);
  for (const auto& g : group_by(count, [&](int i) { return d[i]; })) {
    const int P = (int)g.size();
    const int64_t dd = d[g[0]];
    if (dd > 0) {
      PtrArr<const void*> h;
      PtrArr<float*> u, lam;
      PtrArr<uint8_t*> de;
      for (int k = 0; k < P; ++k) {
        h.p[k] = H[g[k]];
        u.p[k] = U[g[k]];
        de.p[k] = dead ? dead[g[k]] : nullptr;
        lam.p[k] = lambda_out ? lambda_out[g[k]] : nullptr;
      }
      nvfp4_status s = launch_prepare_group(P, h, false, dd, damp, u, de, lam, region, st);
      if (s != NVFP4_OK) return s;
      PtrArr<const int*> ps_;
      PtrArr<int> idx;
      for (int k = 0; k < P; ++k) {
        ps_.p[k] = prepare_group_problem_status(region, k);
        idx.p[k] = g[k];
      }
      s = gather_group_status(bh, reinterpret_cast<const int*>(region), ps_, idx, P, st);
      if (s != NVFP4_OK) return s;
    }
    region += prepare_group_ws_bytes(dd, P);
  }
  return NVFP4_OK;
}

nvfp4_status nvfp4_gptq_schur_replay_quantize_batched(
    int count, const void* const* W, nvfp4_dtype w_dtype, const int64_t* d_out,
    const int64_t* d_in, const float* const* U, const nvfp4_solve_params* params,
    const uint8_t* const* dead, uint8_t* const* codes, uint8_t* const* scales,
    float* const* global_scale, double* const* err_out, void* ws, size_t ws_bytes,
    nvfp4_stream_t stream) {
  if (count < 0 ||
      (count > 0 && (!W || !d_out || !d_in || !U || !codes || !scales || !global_scale)))
    return NVFP4_ERR_INVALID_ARG;
  if (w_dtype != NVFP4_BF16 && w_dtype != NVFP4_F32) return NVFP4_ERR_INVALID_ARG;
  if (params) {
    nvfp4_solve_params def;
    nvfp4_default_params(&def);
    if (params->n_candidates != def.n_candidates || params->cand_lo != def.cand_lo ||
        params->lazy_batch != def.lazy_batch || params->scale_rule < NVFP4_RULE_SCHUR_REPLAY ||
        params->scale_rule > NVFP4_RULE_BLOCK_MSE || params->precision != def.precision)
      return NVFP4_ERR_UNSUPPORTED;
  }
  for (int i = 0; i < count; ++i) {
    if (d_out[i] < 0 || d_in[i] < 0 || !global_scale[i]) return NVFP4_ERR_INVALID_ARG;
    if (d_out[i] > 0 && d_in[i] > 0 && (!W[i] || !U[i] || !codes[i] || !scales[i]))
      return NVFP4_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(W[i]) & 15) || (reinterpret_cast<uintptr_t>(codes[i]) & 7))
      return NVFP4_ERR_INVALID_ARG;
    if (d_in[i] % 16 || d_in[i] > (1 << 17) || d_out[i] > (1 << 22)) return NVFP4_ERR_SHAPE;
  }
  if (count == 0) return NVFP4_OK;
  if (!ws || !aligned256(ws) || ws_bytes < quantize_batched_bytes(count, d_out, d_in))
    return NVFP4_ERR_WORKSPACE;
  const int rule = params ? params->scale_rule : NVFP4_RULE_SCHUR_REPLAY;
  cudaStream_t st = as_cuda(stream);
  int* bh = static_cast<int*>(ws);
  NVFP4_CUDA_TRY(cudaMemsetAsync(bh, 0, batch_header_bytes(count), st));
  char* region = static_cast<char*>(ws) + batch_header_bytes(count);
  for (const auto& g :
       group_by(count, [&](int i) { return std::make_pair(d_out[i], d_in[i]); })) {
    const int P = (int)g.size();
    const int64_t o = d_out[g[0]], n = d_in[g[0]];
    PtrArr<const void*> w;
    PtrArr<const float*> u, am;
    PtrArr<const uint8_t*> de;
    PtrArr<uint8_t*> c, sc;
    PtrArr<float*> gs;
    PtrArr<double*> e;
    for (int k = 0; k < P; ++k) {
      const int i = g[k];
      w.p[k] = W[i];
      u.p[k] = U[i];
      de.p[k] = dead ? dead[i] : nullptr;
      c.p[k] = codes[i];
      sc.p[k] = scales[i];
      gs.p[k] = global_scale[i];
      e.p[k] = err_out ? err_out[i] : nullptr;
      am.p[k] = nullptr;
    }
    nvfp4_status s =
        launch_quantize_group(P, w, w_dtype, o, n, u, de, rule, c, sc, gs, e, am, region, st);
    if (s != NVFP4_OK) return s;
    PtrArr<const int*> ps_;
    PtrArr<int> idx;
    for (int k = 0; k < P; ++k) {
      ps_.p[k] = quantize_group_problem_status(region, k);
      idx.p[k] = g[k];
    }
    s = gather_group_status(bh, reinterpret_cast<const int*>(region), ps_, idx, P, st);
    if (s != NVFP4_OK) return s;
    region += quantize_group_ws_bytes(o, n, P);
  }
  return NVFP4_OK;
}

size_t nvfp4_layer_error_batched_workspace_size(int count, const int64_t* d_out,
                                                const int64_t* d_in) {
  if (count < 0 || (count > 0 && (!d_out || !d_in))) return 0;
  for (int i = 0; i < count; ++i)
    if (d_out[i] < 0 || d_in[i] < 0) return 0;
  return layer_error_batched_bytes(count, d_out, d_in);
}

nvfp4_status nvfp4_layer_error_batched(int count, const void* const* W, nvfp4_dtype w_dtype,
                                       const uint8_t* const* codes, const uint8_t* const* scales,
                                       const float* const* global_scale, const float* const* H,
                                       const int64_t* d_out, const int64_t* d_in,
                                       double* const* err_out, void* ws, size_t ws_bytes,
                                       nvfp4_stream_t stream) {
  if (count < 0 || (count > 0 && (!W || !codes || !scales || !global_scale || !H || !d_out ||
                                  !d_in || !err_out)))
    return NVFP4_ERR_INVALID_ARG;
  if (w_dtype != NVFP4_BF16 && w_dtype != NVFP4_F32) return NVFP4_ERR_INVALID_ARG;
  for (int i = 0; i < count; ++i) {
    if (d_out[i] < 0 || d_in[i] < 0 || !err_out[i]) return NVFP4_ERR_INVALID_ARG;
    if (d_out[i] > 0 && d_in[i] > 0 &&
        (!W[i] || !codes[i] || !scales[i] || !global_scale[i] || !H[i]))
      return NVFP4_ERR_INVALID_ARG;
    if (reinterpret_cast<uintptr_t>(codes[i]) & 7) return NVFP4_ERR_INVALID_ARG;
    if (d_in[i] % 16 || d_in[i] > (1 << 17) || d_out[i] > (1 << 22)) return NVFP4_ERR_SHAPE;
  }
  if (count == 0) return NVFP4_OK;
  if (!ws || !aligned256(ws) || ws_bytes < layer_error_batched_bytes(count, d_out, d_in))
    return NVFP4_ERR_WORKSPACE;
  cudaStream_t st = as_cuda(stream);
  int* bh = static_cast<int*>(ws);
  NVFP4_CUDA_TRY(cudaMemsetAsync(bh, 0, batch_header_bytes(count), st));
  char* region = static_cast<char*>(ws) + batch_header_bytes(count);
  for (const auto& g :
       group_by(count, [&](int i) { return std::make_pair(d_out[i], d_in[i]); })) {
    const int P = (int)g.size();
    const int64_t o = d_out[g[0]], n = d_in[g[0]];
    PtrArr<const void*> w;
    PtrArr<const uint8_t*> c, sc;
    PtrArr<const float*> gs, h;
    PtrArr<double*> e;
    for (int k = 0; k < P; ++k) {
      const int i = g[k];
      w.p[k] = W[i];
      c.p[k] = codes[i];
      sc.p[k] = scales[i];
      gs.p[k] = global_scale[i];
      h.p[k] = H[i];
      e.p[k] = err_out[i];
    }
    nvfp4_status s =
        launch_layer_error_group(P, w, w_dtype, c, sc, gs, h, o, n, e, region, st);
    if (s != NVFP4_OK) return s;
    PtrArr<const int*> ps_;
    PtrArr<int> idx;
    for (int k = 0; k < P; ++k) {
      ps_.p[k] = reinterpret_cast<const int*>(region);   // one status word per group
      idx.p[k] = g[k];
    }
    s = gather_group_status(bh, reinterpret_cast<const int*>(region), ps_, idx, P, st);
    if (s != NVFP4_OK) return s;
    region += layer_error_group_ws_bytes(o, n, P);
  }
  return NVFP4_OK;
}

nvfp4_status nvfp4_dequant_batched(int count, const uint8_t* const* codes,
                                   const uint8_t* const* scales,
                                   const float* const* global_scale, const int64_t* d_out,
                                   const int64_t* d_in, void* const* out, nvfp4_dtype out_dtype,
                                   nvfp4_stream_t stream) {
  if (count < 0 || (count > 0 && (!codes || !scales || !global_scale || !d_out || !d_in || !out)))
    return NVFP4_ERR_INVALID_ARG;
  if (out_dtype != NVFP4_BF16 && out_dtype != NVFP4_F32) return NVFP4_ERR_INVALID_ARG;
  for (int i = 0; i < count; ++i) {
    if (d_out[i] < 0 || d_in[i] < 0) return NVFP4_ERR_INVALID_ARG;
    if (d_out[i] > 0 && d_in[i] > 0 && (!codes[i] || !scales[i] || !global_scale[i] || !out[i]))
      return NVFP4_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(codes[i]) & 7) || (reinterpret_cast<uintptr_t>(out[i]) & 15))
      return NVFP4_ERR_INVALID_ARG;
    if (d_in[i] % 16) return NVFP4_ERR_SHAPE;
  }
  cudaStream_t st = as_cuda(stream);
  ProfileScope ps(kPhaseDequant, st);
  for (const auto& g :
       group_by(count, [&](int i) { return std::make_pair(d_out[i], d_in[i]); })) {
    const int P = (int)g.size();
    PtrArr<const uint8_t*> c, s;
    PtrArr<const float*> gs;
    PtrArr<void*> o;
    for (int k = 0; k < P; ++k) {
      c.p[k] = codes[g[k]];
      s.p[k] = scales[g[k]];
      gs.p[k] = global_scale[g[k]];
      o.p[k] = out[g[k]];
    }
    const nvfp4_status r =
        launch_dequant_group(P, c, s, gs, o, d_out[g[0]], d_in[g[0]], out_dtype, st);
    if (r != NVFP4_OK) return r;
  }
  return NVFP4_OK;
}

}  // extern "C"
