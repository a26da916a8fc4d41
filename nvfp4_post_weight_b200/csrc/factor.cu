// a2-a4: damping and the upper Cholesky factor U of the damped inverse Hessian.
//
// GPTQ ("Replay the Curvature", Abstract: quantizing one column updates the
// columns that follow it) propagates each column's error with the rows of U,
// the upper triangular factor with positive diagonal and (H + lambda I)^-1 =
// U^T U.  Route taken here (no explicit inverse of H is formed):
//   A = J H_d J                 J reverses the index order
//   A = L L^T                   blocked right-looking Cholesky, lower L
//   X = L^-1                    recursive doubling over diagonal blocks
//   U = J X J                   then H_d = (J L J)(J L J)^T with J L J upper,
//                               so H_d^-1 = (J X J)^T (J X J) and J X J is upper.
// Diagonal blocks are factored and inverted in fp64 in shared memory; the
// off-diagonal work is fp32 GEMMs.
#include <math.h>

#include "common.cuh"

namespace nvfp4 {
namespace {

constexpr int NB = 64;  // diagonal block (panel) width

struct PrepHeader {   // lives in the workspace header (first 256 bytes)
  int status;
  int pad;
  double diag_sum;
  float lambda;
};

// Sum of the diagonal (dead entries counted as 1), dead flags, lambda.
__global__ void diag_stats_kernel(const float* __restrict__ H, int64_t d, float damp,
                                  uint8_t* __restrict__ dead, float* __restrict__ lambda_out,
                                  PrepHeader* hdr) {
  __shared__ double part[32];
  double s = 0.0;
  for (int64_t i = threadIdx.x; i < d; i += blockDim.x) {
    const float h = H[i * d + i];
    const bool is_dead = (h == 0.f);
    if (dead) dead[i] = is_dead ? 1 : 0;
    if (!isfinite(h)) flag_status(&hdr->status, NVFP4_ERR_NONFINITE);
    s += is_dead ? 1.0 : (double)h;
  }
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if ((threadIdx.x & 31) == 0) part[threadIdx.x >> 5] = s;
  __syncthreads();
  if (threadIdx.x < 32) {
    s = (threadIdx.x < (blockDim.x >> 5)) ? part[threadIdx.x] : 0.0;
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (threadIdx.x == 0) {
      hdr->diag_sum = s;
      const float lam = (float)((double)damp * (s / (double)d));
      hdr->lambda = lam;
      if (lambda_out) *lambda_out = lam;
    }
  }
}

// A[i][j] = H_d[d-1-i][d-1-j]; dead diagonal entries become 1 + lambda.
// Also zero-fills X (the inverse is built from its block diagonal outward).
__global__ void reverse_damp_kernel(const float* __restrict__ H, int64_t d,
                                    float* __restrict__ A, float* __restrict__ X,
                                    PrepHeader* hdr) {
  const float lam = hdr->lambda;
  const int64_t total = d * d;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int64_t i = idx / d, j = idx - i * d;
    float h = H[(d - 1 - i) * d + (d - 1 - j)];
    if (!isfinite(h)) flag_status(&hdr->status, NVFP4_ERR_NONFINITE);
    if (i == j) h = (h == 0.f ? 1.f : h) + lam;
    A[idx] = h;
    X[idx] = 0.f;
  }
}

// Factors the kb x kb diagonal block at (k, k) of A in fp64: A_kk = L11 L11^T,
// writes L11 back into A and L11^-1 into the same block of X.
__global__ void __launch_bounds__(256) chol_diag_block_kernel(float* __restrict__ A, int64_t d,
                                                              int64_t k, int kb,
                                                              float* __restrict__ X,
                                                              PrepHeader* hdr) {
  extern __shared__ double dsm[];
  double(*S)[NB + 1] = reinterpret_cast<double(*)[NB + 1]>(dsm);
  double(*V)[NB + 1] = reinterpret_cast<double(*)[NB + 1]>(dsm + NB * (NB + 1));
  const int tid = threadIdx.x;
  for (int idx = tid; idx < kb * kb; idx += blockDim.x) {
    const int i = idx / kb, j = idx % kb;
    S[i][j] = (j <= i) ? (double)A[(k + i) * d + k + j] : 0.0;
  }
  __syncthreads();
  for (int j = 0; j < kb; ++j) {
    if (tid == 0) {
      double p = S[j][j];
      if (!(p > 0.0)) {           // also catches NaN
        flag_status(&hdr->status, NVFP4_ERR_NOT_PD);
        p = 1.0;
      }
      S[j][j] = sqrt(p);
    }
    __syncthreads();
    const double piv = S[j][j];
    for (int i = j + 1 + tid; i < kb; i += blockDim.x) S[i][j] /= piv;
    __syncthreads();
    const int w = kb - j - 1;
    for (int idx = tid; idx < w * w; idx += blockDim.x) {
      const int i = j + 1 + idx / w, l = j + 1 + idx % w;
      if (l <= i) S[i][l] -= S[i][j] * S[l][j];
    }
    __syncthreads();
  }
  // inverse of the lower triangle, one column per thread (forward substitution)
  if (tid < kb) {
    const int c = tid;
    for (int i = 0; i < c; ++i) V[i][c] = 0.0;
    V[c][c] = 1.0 / S[c][c];
    for (int i = c + 1; i < kb; ++i) {
      double acc = 0.0;
      for (int l = c; l < i; ++l) acc += S[i][l] * V[l][c];
      V[i][c] = -acc / S[i][i];
    }
  }
  __syncthreads();
  for (int idx = tid; idx < kb * kb; idx += blockDim.x) {
    const int i = idx / kb, j = idx % kb;
    if (j <= i) A[(k + i) * d + k + j] = (float)S[i][j];
    X[(k + i) * d + k + j] = (float)V[i][j];
  }
}

// U[i][j] = X[d-1-i][d-1-j] for j >= i, 0 below the diagonal.
__global__ void reverse_to_upper_kernel(const float* __restrict__ X, int64_t d,
                                        float* __restrict__ U) {
  const int64_t total = d * d;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int64_t i = idx / d, j = idx - i * d;
    U[idx] = (j >= i) ? X[(d - 1 - i) * d + (d - 1 - j)] : 0.f;
  }
}

struct PrepLayout {
  PrepHeader* hdr;
  float* A;
  float* X;
  float* T;
};

PrepLayout prep_layout(void* ws, int64_t d) {
  char* p = static_cast<char*>(ws);
  PrepLayout L;
  L.hdr = reinterpret_cast<PrepHeader*>(p);
  size_t off = kWsHeader;
  L.A = reinterpret_cast<float*>(p + off);
  off += align256(sizeof(float) * d * d);
  L.X = reinterpret_cast<float*>(p + off);
  off += align256(sizeof(float) * d * d);
  L.T = reinterpret_cast<float*>(p + off);
  return L;
}

int grid_for(int64_t n, int threads) {
  int64_t b = (n + threads - 1) / threads;
  return (int)(b < 8 * kNumSMs ? (b < 1 ? 1 : b) : 8 * kNumSMs);
}

}  // namespace

size_t prepare_ws_bytes(int64_t d) {
  return kWsHeader + 2 * align256(sizeof(float) * d * d) +
         align256(sizeof(float) * (size_t)((d * d + 3) / 4 + d * NB));
}

nvfp4_status launch_prepare(const float* H, int64_t d, float damp, float* U, uint8_t* dead,
                            float* lambda_out, void* ws, cudaStream_t st) {
  PrepLayout L = prep_layout(ws, d);
  NVFP4_CUDA_TRY(cudaMemsetAsync(L.hdr, 0, sizeof(PrepHeader), st));
  diag_stats_kernel<<<1, 1024, 0, st>>>(H, d, damp, dead, lambda_out, L.hdr);
  NVFP4_LAUNCH_CHECK();
  count_launches(1);
  reverse_damp_kernel<<<grid_for(d * d, 256), 256, 0, st>>>(H, d, L.A, L.X, L.hdr);
  NVFP4_LAUNCH_CHECK();
  count_launches(1);

  // Blocked right-looking Cholesky of A (lower).
  const size_t diag_smem = 2 * sizeof(double) * NB * (NB + 1);
  NVFP4_CUDA_TRY(cudaFuncSetAttribute(chol_diag_block_kernel,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)diag_smem));
  for (int64_t k = 0; k < d; k += NB) {
    const int kb = (int)((d - k) < NB ? (d - k) : NB);
    chol_diag_block_kernel<<<1, 256, diag_smem, st>>>(L.A, d, k, kb, L.X, L.hdr);
    NVFP4_LAUNCH_CHECK();
  count_launches(1);
    const int64_t m = d - k - kb;
    if (m <= 0) break;
    float* A21 = L.A + (k + kb) * d + k;
    // L21 = A21 L11^-T, in place: each CTA owns whole rows of the panel.
    nvfp4_status s = sgemm_simt((int)m, kb, kb, 1.f, A21, d, 0, L.X + k * d + k, d, 1, 0.f,
                                A21, d, 0, st);
    if (s != NVFP4_OK) return s;
    // A22 -= L21 L21^T (lower tiles)
    s = sgemm_simt((int)m, (int)m, kb, -1.f, A21, d, 0, A21, d, 1, 1.f,
                   L.A + (k + kb) * d + (k + kb), d, 1, st);
    if (s != NVFP4_OK) return s;
  }

  // X = L^-1 by recursive doubling: for adjacent diagonal blocks of size b,
  // X21 = -X22 (L21 X11).  All pairs of one level are independent.
  for (int64_t b = NB; b < d; b *= 2) {
    const int64_t npairs_full = d / (2 * b);
    const int64_t stride = 2 * b * (d + 1);
    if (npairs_full > 0) {
      // T_p = L21 X11   (b x b each)
      nvfp4_status s = sgemm_simt_batched((int)b, (int)b, (int)b, 1.f, L.A + b * d, d, stride,
                                          0, L.X, d, stride, 0, 0.f, L.T, b, b * b, 0,
                                          (int)npairs_full, st);
      if (s != NVFP4_OK) return s;
      // X21 = -X22 T_p
      s = sgemm_simt_batched((int)b, (int)b, (int)b, -1.f, L.X + b * d + b, d, stride, 0,
                             L.T, b, b * b, 0, 0.f, L.X + b * d, d, stride, 0,
                             (int)npairs_full, st);
      if (s != NVFP4_OK) return s;
    }
    const int64_t r0 = npairs_full * 2 * b;         // start of a ragged pair
    const int64_t rr = d - r0 - b;                  // rows in its right block
    if (rr > 0) {
      const int64_t o = r0 * (d + 1);
      nvfp4_status s = sgemm_simt((int)rr, (int)b, (int)b, 1.f, L.A + o + b * d, d, 0, L.X + o,
                                  d, 0, 0.f, L.T, b, 0, st);
      if (s != NVFP4_OK) return s;
      s = sgemm_simt((int)rr, (int)b, (int)rr, -1.f, L.X + o + b * d + b, d, 0, L.T, b, 0, 0.f,
                     L.X + o + b * d, d, 0, st);
      if (s != NVFP4_OK) return s;
    }
  }
  reverse_to_upper_kernel<<<grid_for(d * d, 256), 256, 0, st>>>(L.X, d, U);
  NVFP4_LAUNCH_CHECK();
  count_launches(1);
  return NVFP4_OK;
}

}  // namespace nvfp4
