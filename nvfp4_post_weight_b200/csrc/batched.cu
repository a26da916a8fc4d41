// Batched forms of the C-ABI calls: `count` independent problems in one call,
// e.g. the experts of a mixture-of-experts layer, each with its own Hessian,
// factor and weights.
//
// The problems are spread over a small pool of library streams that fork from
// and join back into the caller's stream (event dependencies, no host
// synchronisation), so that small problems run concurrently on the GPU.  Each
// problem has its own buffers and workspace, so they share nothing.
#include <mutex>

#include "common.cuh"

namespace nvfp4 {
namespace {

constexpr int kPoolStreams = 8;
constexpr int kMaxDevices = 64;

struct Pool {
  cudaStream_t s[kPoolStreams];
  cudaEvent_t fork, done[kPoolStreams];
  bool ready = false;
};

std::mutex g_pool_mu;
Pool g_pools[kMaxDevices];

// The current device's pool, created on first use.
nvfp4_status get_pool(Pool** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return NVFP4_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_pool_mu);
  Pool& p = g_pools[dev];
  if (!p.ready) {
    if (cudaEventCreateWithFlags(&p.fork, cudaEventDisableTiming) != cudaSuccess) {
      cudaGetLastError();
      return NVFP4_ERR_CUDA;
    }
    for (int i = 0; i < kPoolStreams; ++i) {
      if (cudaStreamCreateWithFlags(&p.s[i], cudaStreamNonBlocking) != cudaSuccess ||
          cudaEventCreateWithFlags(&p.done[i], cudaEventDisableTiming) != cudaSuccess) {
        cudaGetLastError();
        return NVFP4_ERR_CUDA;
      }
    }
    p.ready = true;
  }
  *out = &p;
  return NVFP4_OK;
}

// Runs fn(i, stream) for i < count on the pool's streams, ordered after the
// work already queued on `caller` and joined back into it.  The first failing
// status is returned.  Every pool stream that was forked is joined back into
// `caller` whatever failed in between, so that nothing queued on a pool
// stream can race with later work on the caller's stream; if the fork itself
// fails, no problem is issued.
template <typename F>
nvfp4_status fan_out(int count, cudaStream_t caller, F fn) {
  if (count <= 0) return NVFP4_OK;
  if (count == 1) return fn(0, caller);
  Pool* p = nullptr;
  nvfp4_status st = get_pool(&p);
  if (st != NVFP4_OK) return st;
  std::lock_guard<std::mutex> lock(g_pool_mu);   // one fan-out per device at a time
  NVFP4_CUDA_TRY(cudaEventRecord(p->fork, caller));
  const int want = count < kPoolStreams ? count : kPoolStreams;
  nvfp4_status first = NVFP4_OK;
  auto keep = [&](nvfp4_status s) {
    if (s != NVFP4_OK && first == NVFP4_OK) first = s;
  };
  int forked = 0;
  for (; forked < want; ++forked) {
    if (cudaStreamWaitEvent(p->s[forked], p->fork, 0) != cudaSuccess) {
      cudaGetLastError();
      keep(NVFP4_ERR_CUDA);
      break;
    }
  }
  if (forked == want) {
    for (int i = 0; i < count; ++i) keep(fn(i, p->s[i % kPoolStreams]));
  }
  for (int i = 0; i < forked; ++i) {
    if (cudaEventRecord(p->done[i], p->s[i]) != cudaSuccess ||
        cudaStreamWaitEvent(caller, p->done[i], 0) != cudaSuccess) {
      // no device-side join: wait on the host instead, so that the caller's
      // later work still cannot overlap this pool stream's
      cudaGetLastError();
      cudaStreamSynchronize(p->s[i]);
      cudaGetLastError();
      keep(NVFP4_ERR_CUDA);
    }
  }
  return first;
}

nvfp4_stream_t as_handle(cudaStream_t s) { return reinterpret_cast<nvfp4_stream_t>(s); }

}  // namespace
}  // namespace nvfp4

using namespace nvfp4;

extern "C" {

nvfp4_status nvfp4_hessian_accumulate_batched(int count, float* const* H, const void* const* X,
                                              nvfp4_dtype x_dtype, const int64_t* n_tok,
                                              const int64_t* d, int beta,
                                              nvfp4_stream_t stream) {
  if (count < 0 || (count > 0 && (!H || !X || !n_tok || !d))) return NVFP4_ERR_INVALID_ARG;
  return fan_out(count, as_cuda(stream), [&](int i, cudaStream_t s) {
    return nvfp4_hessian_accumulate(H[i], X[i], x_dtype, n_tok[i], d[i], beta, as_handle(s));
  });
}

nvfp4_status nvfp4_gptq_prepare_batched(int count, const float* const* H, const int64_t* d,
                                        float damp, float* const* U, uint8_t* const* dead,
                                        float* const* lambda_out, void* const* ws,
                                        const size_t* ws_bytes, nvfp4_stream_t stream) {
  if (count < 0 || (count > 0 && (!H || !d || !U || !ws || !ws_bytes)))
    return NVFP4_ERR_INVALID_ARG;
  return fan_out(count, as_cuda(stream), [&](int i, cudaStream_t s) {
    return nvfp4_gptq_prepare(H[i], d[i], damp, U[i], dead ? dead[i] : nullptr,
                              lambda_out ? lambda_out[i] : nullptr, ws[i], ws_bytes[i],
                              as_handle(s));
  });
}

nvfp4_status nvfp4_gptq_schur_replay_quantize_batched(
    int count, const void* const* W, nvfp4_dtype w_dtype, const int64_t* d_out,
    const int64_t* d_in, const float* const* U, const nvfp4_solve_params* params,
    const uint8_t* const* dead, uint8_t* const* codes, uint8_t* const* scales,
    float* const* global_scale, double* const* err_out, void* const* ws,
    const size_t* ws_bytes, nvfp4_stream_t stream) {
  if (count < 0 ||
      (count > 0 && (!W || !d_out || !d_in || !U || !codes || !scales || !global_scale ||
                     !ws || !ws_bytes)))
    return NVFP4_ERR_INVALID_ARG;
  return fan_out(count, as_cuda(stream), [&](int i, cudaStream_t s) {
    return nvfp4_gptq_schur_replay_quantize(W[i], w_dtype, d_out[i], d_in[i], U[i], params,
                                            dead ? dead[i] : nullptr, codes[i], scales[i],
                                            global_scale[i], err_out ? err_out[i] : nullptr,
                                            ws[i], ws_bytes[i], as_handle(s));
  });
}

nvfp4_status nvfp4_dequant_batched(int count, const uint8_t* const* codes,
                                   const uint8_t* const* scales,
                                   const float* const* global_scale, const int64_t* d_out,
                                   const int64_t* d_in, void* const* out, nvfp4_dtype out_dtype,
                                   nvfp4_stream_t stream) {
  if (count < 0 || (count > 0 && (!codes || !scales || !global_scale || !d_out || !d_in || !out)))
    return NVFP4_ERR_INVALID_ARG;
  return fan_out(count, as_cuda(stream), [&](int i, cudaStream_t s) {
    return nvfp4_dequant(codes[i], scales[i], global_scale[i], d_out[i], d_in[i], out[i],
                         out_dtype, as_handle(s));
  });
}

}  // extern "C"
