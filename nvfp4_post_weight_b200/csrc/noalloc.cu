// Allocation-free form of the Schur Replay quantize call.
//
// Some callers cannot allocate device memory at the point where they quantize:
// an engine that owns every byte of the GPU through its own fixed pool and
// forbids allocations outside it, or a host loop that must not take the
// device-wide synchronisation cudaMalloc/cudaFree may imply.  For them this
// file keeps the quantize call's scratch in a fixed device array compiled into
// the library, so the call allocates nothing; the caller still passes its
// inputs and outputs.
//
// The array is kNoAllocScratchBytes (16 MiB) on every GPU that loads the
// library, held until the process exits.  Every call on a device shares it and
// it keeps the last call's contents, so calls whose GPU work overlaps (on two
// streams, say) race; the quantize kernels themselves clear what must start at
// zero (status word, amax, per-row error sums) before use.
#include <mutex>

#include "common.cuh"

namespace nvfp4 {
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of g_noalloc_scratch per device.  In host code the symbol is
// only a host-side stand-in, so the address must be looked up with the device
// current, once per device.
std::mutex g_noalloc_mu;
void* g_noalloc_addr[kMaxDevices] = {};

nvfp4_status noalloc_scratch(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) {
    cudaGetLastError();
    return NVFP4_ERR_CUDA;
  }
  if (dev < 0 || dev >= kMaxDevices) return NVFP4_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
      cudaGetLastError();
      return NVFP4_ERR_CUDA;
    }
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return NVFP4_OK;
}

}  // namespace
}  // namespace nvfp4

using namespace nvfp4;

extern "C" {

nvfp4_status nvfp4_gptq_schur_replay_quantize_noalloc(
    const void* W, nvfp4_dtype w_dtype, int64_t d_out, int64_t d_in, const float* U,
    const nvfp4_solve_params* params, const uint8_t* dead, uint8_t* codes, uint8_t* scales,
    float* global_scale, double* err_out, int* status_out, nvfp4_stream_t stream) {
  if (d_out < 0 || d_in < 0) return NVFP4_ERR_INVALID_ARG;
  if (d_in % 16) return NVFP4_ERR_SHAPE;
  if (nvfp4_quantize_workspace_size(d_out, d_in, params) > kNoAllocScratchBytes)
    return NVFP4_ERR_WORKSPACE;
  void* ws = nullptr;
  nvfp4_status s = noalloc_scratch(&ws);
  if (s != NVFP4_OK) return s;
  s = nvfp4_gptq_schur_replay_quantize(W, w_dtype, d_out, d_in, U, params, dead, codes, scales,
                                       global_scale, err_out, ws, kNoAllocScratchBytes, stream);
  if (s != NVFP4_OK) return s;
  if (status_out)  // the sticky status word is the scratch's first int
    NVFP4_CUDA_TRY(cudaMemcpyAsync(status_out, ws, sizeof(int), cudaMemcpyDeviceToDevice,
                                   as_cuda(stream)));
  return NVFP4_OK;
}

}  // extern "C"
