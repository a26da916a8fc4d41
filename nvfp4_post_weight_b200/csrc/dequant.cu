// a9: dequantization Q = e2m1(code) * e4m3(scale) * s_g, and a10: the layer
// error tr((W - Q) H (W - Q)^T).
//
// "Replay the Curvature", Abstract: every 16 E2M1 weights share one E4M3 block
// scale; the per-tensor fp32 global scale s_g multiplies both.  e2m1 * e4m3 has
// at most 6 significant bits and is exact in fp32, so the fp32 result
// (e2m1 * e4m3) * s_g is the correctly rounded full product.  For bf16 output
// the product is formed with round-to-odd in fp32 (round toward zero, then the
// sticky bit from the exact residual) and then rounded to bf16, which is again
// the correctly rounded full product (24 >= 8 + 2 bits).
#include <cuda_bf16.h>

#include "common.cuh"
#include "nvfp4_format.cuh"

namespace nvfp4 {
namespace {

__device__ __forceinline__ uint16_t bf16_of_product(float cs, float sg) {
  float hi = __fmul_rz(cs, sg);
  const float lo = fmaf(cs, sg, -hi);  // exact residual
  if (lo != 0.f) hi = __uint_as_float(__float_as_uint(hi) | 1u);
  return __bfloat16_as_ushort(__float2bfloat16_rn(hi));
}

// One thread per 16-weight block: 8 code bytes + 1 scale byte in, 16 values out.
template <bool kBF16>
__global__ void dequant_kernel(const uint8_t* __restrict__ codes,
                               const uint8_t* __restrict__ scales,
                               const float* __restrict__ sg_ptr, int64_t nblocks,
                               void* __restrict__ out) {
  const float sg = *sg_ptr;
  for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < nblocks;
       b += (int64_t)gridDim.x * blockDim.x) {
    const uint2 c = reinterpret_cast<const uint2*>(codes)[b];
    const float sb = (float)e4m3_value(scales[b] & 0x7F);
    const uint64_t p = ((uint64_t)c.y << 32) | c.x;
    float cs[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) cs[j] = e2m1_value((uint32_t)(p >> (4 * j)) & 0xF) * sb;
    if constexpr (kBF16) {
      uint32_t h[8];
#pragma unroll
      for (int j = 0; j < 8; ++j)
        h[j] = (uint32_t)bf16_of_product(cs[2 * j], sg) |
               ((uint32_t)bf16_of_product(cs[2 * j + 1], sg) << 16);
      uint4* o = reinterpret_cast<uint4*>(out) + 2 * b;
      o[0] = make_uint4(h[0], h[1], h[2], h[3]);
      o[1] = make_uint4(h[4], h[5], h[6], h[7]);
    } else {
      float4* o = reinterpret_cast<float4*>(out) + 4 * b;
#pragma unroll
      for (int q = 0; q < 4; ++q)
        o[q] = make_float4(cs[4 * q] * sg, cs[4 * q + 1] * sg, cs[4 * q + 2] * sg,
                           cs[4 * q + 3] * sg);
    }
  }
}

// E = W - Q in fp32 (W bf16 or fp32).
template <typename T>
__global__ void error_matrix_kernel(const T* __restrict__ W, const uint8_t* __restrict__ codes,
                                    const uint8_t* __restrict__ scales,
                                    const float* __restrict__ sg_ptr, int64_t nblocks,
                                    float* __restrict__ E) {
  const float sg = *sg_ptr;
  for (int64_t b = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; b < nblocks;
       b += (int64_t)gridDim.x * blockDim.x) {
    const uint2 c = reinterpret_cast<const uint2*>(codes)[b];
    const float sb = (float)e4m3_value(scales[b] & 0x7F);
    const uint64_t p = ((uint64_t)c.y << 32) | c.x;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      float w;
      if constexpr (sizeof(T) == 2)
        w = __uint_as_float((uint32_t)W[16 * b + j] << 16);
      else
        w = W[16 * b + j];
      // w - (e2m1 * e4m3) * s_g with a single rounding
      E[16 * b + j] = fmaf(-e2m1_value((uint32_t)(p >> (4 * j)) & 0xF) * sb, sg, w);
    }
  }
}

// sum_ij EH_ij * E_ij in fp64
__global__ void dot_kernel(const float* __restrict__ A, const float* __restrict__ B, int64_t n,
                           double* __restrict__ partial) {
  __shared__ double part[32];
  double s = 0.0;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (int64_t)gridDim.x * blockDim.x)
    s += (double)A[i] * (double)B[i];
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x < 32) {
    s = (threadIdx.x < (blockDim.x >> 5)) ? part[threadIdx.x] : 0.0;
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (threadIdx.x == 0) partial[blockIdx.x] = s;
  }
}

__global__ void sum_partials_kernel(const double* __restrict__ p, int n, double* __restrict__ out) {
  if (threadIdx.x == 0) {
    double s = 0.0;
    for (int i = 0; i < n; ++i) s += p[i];
    *out = s;
  }
}

int grid_for(int64_t n, int threads) {
  int64_t b = (n + threads - 1) / threads;
  return (int)(b < 8 * kNumSMs ? (b < 1 ? 1 : b) : 8 * kNumSMs);
}

constexpr int kDotBlocks = 2 * kNumSMs;

}  // namespace

nvfp4_status launch_dequant(const uint8_t* codes, const uint8_t* scales, const float* sg,
                            int64_t d_out, int64_t d_in, void* out, nvfp4_dtype ot,
                            cudaStream_t st) {
  const int64_t nb = d_out * (d_in / kBlock);
  if (nb == 0) return NVFP4_OK;
  if (ot == NVFP4_BF16)
    dequant_kernel<true><<<grid_for(nb, 256), 256, 0, st>>>(codes, scales, sg, nb, out);
  else
    dequant_kernel<false><<<grid_for(nb, 256), 256, 0, st>>>(codes, scales, sg, nb, out);
  NVFP4_LAUNCH_CHECK();
  count_launches(1);
  return NVFP4_OK;
}

size_t layer_error_ws_bytes(int64_t d_out, int64_t d_in) {
  return kWsHeader + 2 * align256(sizeof(float) * d_out * d_in) +
         align256(sizeof(double) * kDotBlocks);
}

nvfp4_status launch_layer_error(const void* W, nvfp4_dtype wt, const uint8_t* codes,
                                const uint8_t* scales, const float* sg, const float* H,
                                int64_t d_out, int64_t d_in, double* err, void* ws,
                                cudaStream_t st) {
  char* p = static_cast<char*>(ws) + kWsHeader;
  float* E = reinterpret_cast<float*>(p);
  float* EH = reinterpret_cast<float*>(p + align256(sizeof(float) * d_out * d_in));
  double* part =
      reinterpret_cast<double*>(p + 2 * align256(sizeof(float) * d_out * d_in));
  const int64_t nb = d_out * (d_in / kBlock);
  if (nb == 0) {
    NVFP4_CUDA_TRY(cudaMemsetAsync(err, 0, sizeof(double), st));
    return NVFP4_OK;
  }
  if (wt == NVFP4_BF16)
    error_matrix_kernel<uint16_t><<<grid_for(nb, 256), 256, 0, st>>>(
        static_cast<const uint16_t*>(W), codes, scales, sg, nb, E);
  else
    error_matrix_kernel<float><<<grid_for(nb, 256), 256, 0, st>>>(
        static_cast<const float*>(W), codes, scales, sg, nb, E);
  NVFP4_LAUNCH_CHECK();
  count_launches(1);
  // EH = E H^T = E H (H symmetric) on the tensor cores
  int* status = static_cast<int*>(ws);
  NVFP4_CUDA_TRY(cudaMemsetAsync(status, 0, sizeof(int), st));
  nvfp4_status s = gemm_nt_tc((int)d_out, (int)d_in, (int)d_in, 1.f, E, d_in, 0, H, d_in, 0,
                              0.f, EH, d_in, 0, nullptr, 0, 0, 1, 0, status, st);
  if (s != NVFP4_OK) return s;
  dot_kernel<<<kDotBlocks, 256, 0, st>>>(E, EH, d_out * d_in, part);
  NVFP4_LAUNCH_CHECK();
  sum_partials_kernel<<<1, 32, 0, st>>>(part, kDotBlocks, err);
  NVFP4_LAUNCH_CHECK();
  count_launches(2);
  return NVFP4_OK;
}

}  // namespace nvfp4
