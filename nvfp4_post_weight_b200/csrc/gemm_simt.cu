// fp32 GEMM on the CUDA cores: C = alpha * op(A) op(B) + beta * C.
//
// Used where the factorization needs exact-fp32 products of fp32 operands
// (diagonal-block solves, small batched products).  128 x 128 output tile per
// CTA, K staged through shared memory 16 at a time (double buffered), 8 x 8
// outputs per thread.  Batched over blockIdx.z with element strides.
#include "common.cuh"

namespace nvfp4 {
namespace {

constexpr int BM = 128, BN = 128, BK = 16, TM = 8, TN = 8;
constexpr int kThreads = (BM / TM) * (BN / TN);  // 256

struct GemmArgs {
  int M, N, K;
  float alpha, beta;
  const float* A;
  int64_t lda, sA;
  const float* B;
  int64_t ldb, sB;
  float* C;
  int64_t ldc, sC;
  int ta, tb, tri;
};

__device__ __forceinline__ float ldA(const GemmArgs& g, const float* A, int m, int k) {
  if (m >= g.M || k >= g.K) return 0.f;
  return g.ta ? A[(int64_t)k * g.lda + m] : A[(int64_t)m * g.lda + k];
}
__device__ __forceinline__ float ldB(const GemmArgs& g, const float* B, int k, int n) {
  if (k >= g.K || n >= g.N) return 0.f;
  return g.tb ? B[(int64_t)n * g.ldb + k] : B[(int64_t)k * g.ldb + n];
}

__global__ void __launch_bounds__(kThreads) sgemm_kernel(GemmArgs g) {
  const int bm = blockIdx.y * BM, bn = blockIdx.x * BN;
  if (g.tri == 1 && bn > bm + BM - 1) return;   // tile strictly above the diagonal
  if (g.tri == 2 && bm > bn + BN - 1) return;   // tile strictly below the diagonal
  const float* A = g.A + (int64_t)blockIdx.z * g.sA;
  const float* B = g.B + (int64_t)blockIdx.z * g.sB;
  float* C = g.C + (int64_t)blockIdx.z * g.sC;

  __shared__ float As[2][BK][BM];
  __shared__ float Bs[2][BK][BN];
  const int tid = threadIdx.x;
  const int tr = tid / (BN / TN), tc = tid % (BN / TN);

  float acc[TM][TN];
#pragma unroll
  for (int i = 0; i < TM; ++i)
#pragma unroll
    for (int j = 0; j < TN; ++j) acc[i][j] = 0.f;

  // Each thread stages 8 A and 8 B elements per K-slab.  The mapping keeps the
  // global reads along the contiguous dimension of the stored matrix.
  float ra[8], rb[8];
  auto load = [&](int k0) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int idx = tid + e * kThreads;  // 0 .. 2047
      int m, k;
      if (g.ta) { k = idx / BM; m = idx % BM; } else { m = idx / BK; k = idx % BK; }
      ra[e] = ldA(g, A, bm + m, k0 + k);
      int n, kk;
      if (g.tb) { n = idx / BK; kk = idx % BK; } else { kk = idx / BN; n = idx % BN; }
      rb[e] = ldB(g, B, k0 + kk, bn + n);
    }
  };
  auto store = [&](int buf) {
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int idx = tid + e * kThreads;
      int m, k;
      if (g.ta) { k = idx / BM; m = idx % BM; } else { m = idx / BK; k = idx % BK; }
      As[buf][k][m] = ra[e];
      int n, kk;
      if (g.tb) { n = idx / BK; kk = idx % BK; } else { kk = idx / BN; n = idx % BN; }
      Bs[buf][kk][n] = rb[e];
    }
  };

  const int nk = (g.K + BK - 1) / BK;
  if (nk > 0) {
    load(0);
    store(0);
  }
  __syncthreads();
  for (int t = 0; t < nk; ++t) {
    const int buf = t & 1;
    if (t + 1 < nk) load((t + 1) * BK);
#pragma unroll
    for (int k = 0; k < BK; ++k) {
      float a[TM], b[TN];
#pragma unroll
      for (int i = 0; i < TM; ++i) a[i] = As[buf][k][tr + i * (BM / TM)];
#pragma unroll
      for (int j = 0; j < TN; ++j) b[j] = Bs[buf][k][tc + j * (BN / TN)];
#pragma unroll
      for (int i = 0; i < TM; ++i)
#pragma unroll
        for (int j = 0; j < TN; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    if (t + 1 < nk) store(buf ^ 1);
    __syncthreads();
  }

#pragma unroll
  for (int i = 0; i < TM; ++i) {
    const int m = bm + tr + i * (BM / TM);
    if (m >= g.M) continue;
#pragma unroll
    for (int j = 0; j < TN; ++j) {
      const int n = bn + tc + j * (BN / TN);
      if (n >= g.N) continue;
      if (g.tri == 1 && n > m) continue;
      if (g.tri == 2 && m > n) continue;
      float* c = C + (int64_t)m * g.ldc + n;
      *c = g.beta == 0.f ? g.alpha * acc[i][j] : fmaf(g.alpha, acc[i][j], g.beta * *c);
    }
  }
}

}  // namespace

nvfp4_status sgemm_simt_batched(int M, int N, int K, float alpha, const float* A,
                                int64_t lda, int64_t sA, int ta, const float* B,
                                int64_t ldb, int64_t sB, int tb, float beta, float* C,
                                int64_t ldc, int64_t sC, int tri, int batch,
                                cudaStream_t st) {
  if (M <= 0 || N <= 0 || batch <= 0) return NVFP4_OK;
  GemmArgs g{M, N, K, alpha, beta, A, lda, sA, B, ldb, sB, C, ldc, sC, ta, tb, tri};
  dim3 grid((N + BN - 1) / BN, (M + BM - 1) / BM, batch);
  sgemm_kernel<<<grid, kThreads, 0, st>>>(g);
  NVFP4_LAUNCH_CHECK();
  count_launches(1);
  return NVFP4_OK;
}

nvfp4_status sgemm_simt(int M, int N, int K, float alpha, const float* A, int64_t lda,
                        int ta, const float* B, int64_t ldb, int tb, float beta, float* C,
                        int64_t ldc, int tri, cudaStream_t st) {
  return sgemm_simt_batched(M, N, K, alpha, A, lda, 0, ta, B, ldb, 0, tb, beta, C, ldc, 0,
                            tri, 1, st);
}

}  // namespace nvfp4
