// a1 at fp64 accuracy: H (+)= X^T X stored in fp64, for layers whose damped
// Hessian is so ill-conditioned (fewer calibration tokens than channels) that
// the fp32 storage of H alone moves the factor's decisions.
//
// "Replay the Curvature" (arXiv 2609.36654v1), Abstract: the second-order state
// is accumulated from the calibration activations.  Here every product of two
// bf16 (or fp32) activations and their sums are kept to fp64 accuracy: the
// tokens are transposed into fp64 rows (one per channel, tokens contiguous,
// zero-padded to a multiple of 16) and the product X^T X goes through the
// int8-slice tensor-core GEMM (dgemm_i8: each channel's row scaled by a power
// of two and cut into 7-bit slices, slice products exact in int32, levels
// combined in fp64); only the tiles on or below the diagonal are formed, then
// the lower triangle is mirrored.  A bf16 value has 8 significant bits, so the
// slices hold every token value within 2^-34 of its channel's largest exactly;
// the result's error is below 2^-39 of the channel maxima per product.
#include "common.cuh"

namespace nvfp4 {
namespace {

constexpr int kT = 32;   // transpose tile

// XT[c][t] = X[t][c] in fp64 for t < n_tok, 0 for n_tok <= t < kp.
template <typename T>
__global__ void transpose_f64_kernel(const T* __restrict__ X, int64_t n_tok, int64_t d,
                                     int64_t kp, double* __restrict__ XT) {
  __shared__ double tile[kT][kT + 1];
  const int64_t t0 = (int64_t)blockIdx.x * kT, c0 = (int64_t)blockIdx.y * kT;
  const int tx = threadIdx.x, ty = threadIdx.y;   // 32 x 8
  for (int r = ty; r < kT; r += 8) {
    const int64_t t = t0 + r, c = c0 + tx;
    double v = 0.0;
    if (t < n_tok && c < d) {
      if constexpr (sizeof(T) == 2)
        v = (double)__uint_as_float((uint32_t)X[t * d + c] << 16);
      else
        v = (double)X[t * d + c];
    }
    tile[r][tx] = v;
  }
  __syncthreads();
  for (int r = ty; r < kT; r += 8) {
    const int64_t c = c0 + r, t = t0 + tx;
    if (c < d && t < kp) XT[c * kp + t] = tile[tx][r];
  }
}

// H[i][j] = H[j][i] for i < j (the upper triangle from the lower), 32 x 32
// tiles through shared memory: tile (bi, bj), bj >= bi, of the upper part is
// the transpose of tile (bj, bi).
__global__ void mirror_lower_kernel(double* __restrict__ H, int64_t d) {
  __shared__ double tile[kT][kT + 1];
  const int bi = blockIdx.y, bj = blockIdx.x;
  if (bj < bi) return;
  const int tx = threadIdx.x, ty = threadIdx.y;
  for (int r = ty; r < kT; r += 8) {
    const int64_t i = (int64_t)bj * kT + r, j = (int64_t)bi * kT + tx;   // lower block (bj, bi)
    tile[r][tx] = (i < d && j < d) ? H[i * d + j] : 0.0;
  }
  __syncthreads();
  for (int r = ty; r < kT; r += 8) {
    const int64_t i = (int64_t)bi * kT + r, j = (int64_t)bj * kT + tx;   // upper block (bi, bj)
    if (i < d && j < d && j > i) H[i * d + j] = tile[tx][r];
  }
}

// Tokens per pass: each pass transposes a chunk and adds its product (fp64
// accumulation across passes), which bounds the workspace and keeps the int32
// slice sums exact (K < 2^16).
constexpr int64_t kChunk = 8192;

int64_t padded(int64_t n) { return (n + 15) / 16 * 16; }

}  // namespace

size_t hessian_f64_ws_bytes(int64_t n_tok, int64_t d) {
  const int64_t kp = padded(n_tok < kChunk ? n_tok : kChunk);
  return kWsHeader + align256(sizeof(double) * d * kp) +
         align256(dgemm_i8_scratch_bytes(d, d, kp, 1));
}

nvfp4_status launch_hessian_f64(double* H, const void* X, nvfp4_dtype xt, int64_t n_tok,
                                int64_t d, int beta, void* ws, cudaStream_t st) {
  char* p = static_cast<char*>(ws);
  int* status = reinterpret_cast<int*>(p);
  NVFP4_CUDA_TRY(cudaMemsetAsync(status, 0, sizeof(int), st));
  if (n_tok == 0) {   // no tokens: H = 0 (beta = 0) or unchanged
    if (!beta) NVFP4_CUDA_TRY(cudaMemsetAsync(H, 0, sizeof(double) * d * d, st));
    return NVFP4_OK;
  }
  double* XT = reinterpret_cast<double*>(p + kWsHeader);
  const int64_t kmax = padded(n_tok < kChunk ? n_tok : kChunk);
  void* S8 = p + kWsHeader + align256(sizeof(double) * d * kmax);
  const size_t s8_bytes = dgemm_i8_scratch_bytes(d, d, kmax, 1);
  const size_t esize = xt == NVFP4_BF16 ? 2 : 4;
  for (int64_t t0 = 0; t0 < n_tok; t0 += kChunk) {
    const int64_t n = (n_tok - t0) < kChunk ? (n_tok - t0) : kChunk;
    const int64_t kp = padded(n);
    const void* Xc = static_cast<const char*>(X) + (size_t)t0 * d * esize;
    const dim3 tg((unsigned)((kp + kT - 1) / kT), (unsigned)((d + kT - 1) / kT));
    if (xt == NVFP4_BF16)
      transpose_f64_kernel<uint16_t><<<tg, dim3(32, 8), 0, st>>>(
          static_cast<const uint16_t*>(Xc), n, d, kp, XT);
    else
      transpose_f64_kernel<float><<<tg, dim3(32, 8), 0, st>>>(static_cast<const float*>(Xc), n,
                                                              d, kp, XT);
    NVFP4_LAUNCH_CHECK();
    count_launches(1);
    const double b = (t0 > 0 || beta) ? 1.0 : 0.0;
    nvfp4_status s = dgemm_i8((int)d, (int)d, (int)kp, 1.0, XT, kp, 0, XT, kp, 0, b, H, d, 0,
                              nullptr, 0, 0, 1, 1, 0, S8, s8_bytes, status, st);
    if (s != NVFP4_OK) return s;
  }
  const dim3 mg((unsigned)((d + kT - 1) / kT), (unsigned)((d + kT - 1) / kT));
  mirror_lower_kernel<<<mg, dim3(32, 8), 0, st>>>(H, d);
  NVFP4_LAUNCH_CHECK();
  count_launches(1);
  return NVFP4_OK;
}

}  // namespace nvfp4
