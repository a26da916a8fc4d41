// a1 (CUDA-core variant): H (+)= X^T X for fp32 activations.
//
// "Replay the Curvature", Abstract: the second-order state of a layer is built
// from its calibration activations.  fp32 inputs take this path (their
// products are not exact on the bf16 tensor-core path); bf16 inputs take the
// tcgen05 kernel.  Only tiles on or below the diagonal are computed and each
// is mirrored, so both triangles of H are written.
#include "common.cuh"

namespace nvfp4 {
namespace {

constexpr int BM = 128, BK = 16, TM = 8;
constexpr int kThreads = (BM / TM) * (BM / TM);

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <>
__device__ __forceinline__ float to_f32<uint16_t>(uint16_t v) {
  return __uint_as_float((uint32_t)v << 16);
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
    syrk_simt_kernel(float* __restrict__ H, const T* __restrict__ X, int64_t n_tok, int64_t d,
                     int beta) {
  // lower-triangular tile index -> (ti, tj), tj <= ti
  const int64_t t = blockIdx.x;
  int64_t ti = (int64_t)((sqrt(8.0 * (double)t + 1.0) - 1.0) / 2.0);
  while (ti * (ti + 1) / 2 > t) --ti;
  while ((ti + 1) * (ti + 2) / 2 <= t) ++ti;
  const int64_t tj = t - ti * (ti + 1) / 2;
  const int64_t bm = ti * BM, bn = tj * BM;

  __shared__ float As[BK][BM];
  __shared__ float Bs[BK][BM];
  const int tid = threadIdx.x, tr = tid / (BM / TM), tc = tid % (BM / TM);
  float acc[TM][TM];
#pragma unroll
  for (int i = 0; i < TM; ++i)
#pragma unroll
    for (int j = 0; j < TM; ++j) acc[i][j] = 0.f;

  for (int64_t k0 = 0; k0 < n_tok; k0 += BK) {
#pragma unroll
    for (int e = 0; e < (BK * BM) / kThreads; ++e) {
      const int idx = tid + e * kThreads;
      const int k = idx / BM, m = idx % BM;
      const int64_t kk = k0 + k;
      As[k][m] = (kk < n_tok && bm + m < d) ? to_f32<T>(X[kk * d + bm + m]) : 0.f;
      Bs[k][m] = (kk < n_tok && bn + m < d) ? to_f32<T>(X[kk * d + bn + m]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int k = 0; k < BK; ++k) {
      float a[TM], b[TM];
#pragma unroll
      for (int i = 0; i < TM; ++i) a[i] = As[k][tr + i * (BM / TM)];
#pragma unroll
      for (int j = 0; j < TM; ++j) b[j] = Bs[k][tc + j * (BM / TM)];
#pragma unroll
      for (int i = 0; i < TM; ++i)
#pragma unroll
        for (int j = 0; j < TM; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
  const bool diag = (ti == tj);
#pragma unroll
  for (int i = 0; i < TM; ++i) {
    const int64_t m = bm + tr + i * (BM / TM);
    if (m >= d) continue;
#pragma unroll
    for (int j = 0; j < TM; ++j) {
      const int64_t n = bn + tc + j * (BM / TM);
      if (n >= d || (diag && n > m)) continue;
      float v = acc[i][j];
      if (beta) v += H[m * d + n];
      H[m * d + n] = v;
      if (m != n) H[n * d + m] = v;
    }
  }
}

}  // namespace

nvfp4_status launch_hessian_simt(float* H, const void* X, nvfp4_dtype xt, int64_t n_tok,
                                 int64_t d, int beta, cudaStream_t st) {
  const int64_t nt = (d + BM - 1) / BM;
  const int64_t tiles = nt * (nt + 1) / 2;
  if (xt == NVFP4_F32)
    syrk_simt_kernel<float><<<(unsigned)tiles, kThreads, 0, st>>>(
        H, static_cast<const float*>(X), n_tok, d, beta);
  else
    syrk_simt_kernel<uint16_t><<<(unsigned)tiles, kThreads, 0, st>>>(
        H, static_cast<const uint16_t*>(X), n_tok, d, beta);
  NVFP4_LAUNCH_CHECK();
  count_launches(1);
  return NVFP4_OK;
}

}  // namespace nvfp4
