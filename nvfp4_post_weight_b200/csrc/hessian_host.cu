// a1 from host memory: H (+)= X^T X with the calibration tokens streamed in
// from the host, chunk by chunk.
//
// "Replay the Curvature", Abstract (infrastructure sentence): calibration
// activations are tiered across device, host and disk, and only the active
// layer stays resident.  This is the device/host slice of that tiering for the
// second-order state: the tokens of a layer live in host memory and pass
// through two device staging buffers; the copy of chunk c + 1 (on a library
// copy stream) overlaps the tensor-core Hessian of chunk c (on the caller's
// stream), and H accumulates over the chunks in fp32.
#include <mutex>

#include "common.cuh"

namespace nvfp4 {

nvfp4_status launch_hessian_tc(float* H, const void* X, int64_t n_tok, int64_t d, int beta,
                               cudaStream_t st);
nvfp4_status launch_hessian_simt(float* H, const void* X, nvfp4_dtype xt, int64_t n_tok,
                                 int64_t d, int beta, cudaStream_t st);

namespace {

constexpr int kMaxDevices = 64;
std::mutex g_copy_mu;
cudaStream_t g_copy_stream[kMaxDevices];

// The current device's copy stream (non-blocking, created on first use).
nvfp4_status copy_stream(cudaStream_t* out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    cudaGetLastError();
    return NVFP4_ERR_CUDA;
  }
  std::lock_guard<std::mutex> lock(g_copy_mu);
  if (!g_copy_stream[dev]) {
    if (cudaStreamCreateWithFlags(&g_copy_stream[dev], cudaStreamNonBlocking) != cudaSuccess) {
      cudaGetLastError();
      g_copy_stream[dev] = nullptr;
      return NVFP4_ERR_CUDA;
    }
  }
  *out = g_copy_stream[dev];
  return NVFP4_OK;
}

size_t elem_bytes(nvfp4_dtype xt) { return xt == NVFP4_BF16 ? 2 : 4; }

// The event handles of one call; destroyed when the call has been enqueued
// (CUDA releases them once the work that references them is done).
struct Events {
  cudaEvent_t e[5] = {};
  bool ok = true;
  Events() {
    for (auto& x : e)
      if (cudaEventCreateWithFlags(&x, cudaEventDisableTiming) != cudaSuccess) {
        cudaGetLastError();
        x = nullptr;
        ok = false;
      }
  }
  ~Events() {
    for (auto& x : e)
      if (x) cudaEventDestroy(x);
  }
};

}  // namespace

size_t hessian_host_ws_bytes(int64_t d, int64_t chunk_tok, nvfp4_dtype xt) {
  return 2 * align256(elem_bytes(xt) * (size_t)chunk_tok * (size_t)d);
}

nvfp4_status launch_hessian_host(float* H, const void* X_host, nvfp4_dtype xt, int64_t n_tok,
                                 int64_t d, int beta, int64_t chunk_tok, void* ws,
                                 cudaStream_t st) {
  if (n_tok == 0) return launch_hessian_simt(H, nullptr, xt, 0, d, beta, st);
  cudaStream_t cs = nullptr;
  nvfp4_status s = copy_stream(&cs);
  if (s != NVFP4_OK) return s;
  Events ev;
  if (!ev.ok) return NVFP4_ERR_CUDA;
  cudaEvent_t fork = ev.e[0], filled[2] = {ev.e[1], ev.e[2]}, freed[2] = {ev.e[3], ev.e[4]};
  const size_t esz = elem_bytes(xt);
  char* buf[2] = {static_cast<char*>(ws),
                  static_cast<char*>(ws) + align256(esz * (size_t)chunk_tok * (size_t)d)};
  // the copies start after everything already queued on the caller's stream
  // (a previous call may still be reading the staging buffers)
  NVFP4_CUDA_TRY(cudaEventRecord(fork, st));
  NVFP4_CUDA_TRY(cudaStreamWaitEvent(cs, fork, 0));
  const char* src = static_cast<const char*>(X_host);
  const int64_t n_chunks = (n_tok + chunk_tok - 1) / chunk_tok;
  for (int64_t c = 0; c < n_chunks; ++c) {
    const int b = (int)(c & 1);
    const int64_t t0 = c * chunk_tok;
    const int64_t rows = (n_tok - t0) < chunk_tok ? (n_tok - t0) : chunk_tok;
    // buffer b is free once the Hessian of chunk c - 2 has read it
    if (c >= 2) NVFP4_CUDA_TRY(cudaStreamWaitEvent(cs, freed[b], 0));
    NVFP4_CUDA_TRY(cudaMemcpyAsync(buf[b], src + esz * (size_t)t0 * (size_t)d,
                                   esz * (size_t)rows * (size_t)d, cudaMemcpyHostToDevice, cs));
    NVFP4_CUDA_TRY(cudaEventRecord(filled[b], cs));
    NVFP4_CUDA_TRY(cudaStreamWaitEvent(st, filled[b], 0));
    const int bt = c > 0 ? 1 : beta;
    s = hessian_tc_supported(H, buf[b], xt, rows, d)
            ? launch_hessian_tc(H, buf[b], rows, d, bt, st)
            : launch_hessian_simt(H, buf[b], xt, rows, d, bt, st);
    if (s != NVFP4_OK) return s;
    NVFP4_CUDA_TRY(cudaEventRecord(freed[b], st));
  }
  return NVFP4_OK;
}

}  // namespace nvfp4
