// a8 trailing update on the CUDA cores in fp64: C -= A B.
//
// GPTQ ("Replay the Curvature", Abstract: quantizing one column updates the
// columns that follow it) applies a whole lazy batch of column errors to every
// later column at once: W~[:, e:] -= Delta U[batch, e:].  W~ and Delta are
// fp64 and U is fp32 (widened exactly), so every product is exact and the sum
// carries fp64 rounding only.
//
// 128 x 128 output tile per CTA, K staged through shared memory 16 at a time
// (next slab prefetched into registers), 8 x 8 outputs per thread.
#include "common.cuh"

namespace nvfp4 {
namespace {

constexpr int BM = 128, BN = 128, BK = 16, TM = 8, TN = 8;
constexpr int kThreads = (BM / TM) * (BN / TN);  // 256
constexpr int kPad = 2;                          // breaks bank conflicts of the A stores

__global__ void __launch_bounds__(kThreads, 1)
    dgemm_update_kernel(int M, int N, int K, const double* __restrict__ A, int64_t lda,
                        const float* __restrict__ B, int64_t ldb, double* __restrict__ C,
                        int64_t ldc) {
  __shared__ double As[BK][BM + kPad];
  __shared__ double Bs[BK][BN];
  const int bm = blockIdx.y * BM, bn = blockIdx.x * BN;
  const int tid = threadIdx.x;
  const int tr = tid / (BN / TN), tc = tid % (BN / TN);

  double acc[TM][TN];
#pragma unroll
  for (int i = 0; i < TM; ++i)
#pragma unroll
    for (int j = 0; j < TN; ++j) acc[i][j] = 0.0;

  // A slab: 128 rows x 16 k, thread -> (m = idx / 16, k = idx % 16), 8 per thread.
  // B slab: 16 k x 128 cols, thread -> (k = idx / 128, n = idx % 128), 8 per thread.
  double ra[8];
  float rb[8];
  auto load = [&](int k0) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int idx = tid + e * kThreads;
      const int m = idx >> 4, k = idx & 15;
      ra[e] = (bm + m < M && k0 + k < K) ? A[(int64_t)(bm + m) * lda + k0 + k] : 0.0;
      const int kk = idx >> 7, n = idx & 127;
      rb[e] = (k0 + kk < K && bn + n < N) ? B[(int64_t)(k0 + kk) * ldb + bn + n] : 0.f;
    }
  };
  auto store = [&]() {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int idx = tid + e * kThreads;
      As[idx & 15][idx >> 4] = ra[e];
      Bs[idx >> 7][idx & 127] = (double)rb[e];
    }
  };

  const int nk = (K + BK - 1) / BK;
  load(0);
  for (int t = 0; t < nk; ++t) {
    store();
    __syncthreads();
    if (t + 1 < nk) load((t + 1) * BK);
#pragma unroll
    for (int k = 0; k < BK; ++k) {
      double a[TM], b[TN];
#pragma unroll
      for (int i = 0; i < TM; ++i) a[i] = As[k][tr + i * (BM / TM)];
#pragma unroll
      for (int j = 0; j < TN; ++j) b[j] = Bs[k][tc + j * (BN / TN)];
#pragma unroll
      for (int i = 0; i < TM; ++i)
#pragma unroll
        for (int j = 0; j < TN; ++j) acc[i][j] = fma(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }

#pragma unroll
  for (int i = 0; i < TM; ++i) {
    const int m = bm + tr + i * (BM / TM);
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < TN; ++j) {
      const int n = bn + tc + j * (BN / TN);
      if (n >= N) continue;
      double* c = C + (int64_t)m * ldc + n;
      *c -= acc[i][j];
    }
  }
}

}  // namespace

nvfp4_status dgemm_update(int M, int N, int K, const double* A, int64_t lda, const float* B,
                          int64_t ldb, double* C, int64_t ldc, cudaStream_t st) {
  if (M <= 0 || N <= 0 || K <= 0) return NVFP4_OK;
  dim3 grid((N + BN - 1) / BN, (M + BM - 1) / BM);
  dgemm_update_kernel<<<grid, kThreads, 0, st>>>(M, N, K, A, lda, B, ldb, C, ldc);
  NVFP4_LAUNCH_CHECK();
  count_launches(1);
  return NVFP4_OK;
}

}  // namespace nvfp4
