// fp64 GEMM on the CUDA cores:  C = beta C + alpha P Q^T
// (P: M x K, Q: N x K, row-major with K contiguous; C: M x N row-major),
// optionally batched (blockIdx.z, element strides) and optionally restricted
// to the 64 x 64 tiles on or below the diagonal (M == N); optionally writes
// C^T into C2 as well (beta == 0).
//
// Used by the factorisation, whose accuracy sets how faithfully the GPTQ
// decisions follow an exact solve: the damped Hessian of a layer calibrated on
// few tokens is ill-conditioned (1e4 and more), and a factor carried in fp32
// arithmetic moves block decisions that sit a few 1e-5 from a tie.  The
// 5th-generation tensor cores have no fp64 kind, and B200's fp64 tensor and
// CUDA-core rates are the same, so this is a register-tiled DFMA kernel:
// 64 x 64 tiles, 256 threads with 4 x 4 outputs each, K in steps of 16
// staged transposed in shared memory (double buffered through registers).
#include "common.cuh"

namespace nvfp4 {
namespace {

constexpr int DM = 64, DN = 64, DK = 16;
constexpr int kDThreads = 256;

__global__ void __launch_bounds__(kDThreads)
    dgemm_nt_kernel(int M, int N, int K, double alpha, const double* __restrict__ P,
                    int64_t ldp, int64_t strideP, const double* __restrict__ Q, int64_t ldq,
                    int64_t strideQ, double beta, double* __restrict__ C, int64_t ldc,
                    int64_t strideC, double* __restrict__ C2, int64_t ldc2, int64_t strideC2,
                    int lower) {
  __shared__ double Ps[2][DK][DM + 2];
  __shared__ double Qs[2][DK][DN + 2];
  int tm = blockIdx.y, tn = blockIdx.x;
  if (lower && tn > tm) return;
  const int b = blockIdx.z;
  P += b * strideP;
  Q += b * strideQ;
  C += b * strideC;
  if (C2) C2 += b * strideC2;
  const int tid = threadIdx.x, ty = tid >> 4, tx = tid & 15;
  const int m0 = tm * DM, n0 = tn * DN;
  // loader mapping: 64 rows x 16 k per operand = 1024 values, 4 per thread
  const int lr = tid >> 2, lk = (tid & 3) * 4;
  double pr[4], qr[4];
  auto load = [&](int k0) {
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const int k = k0 + lk + t;
      pr[t] = (m0 + lr < M && k < K) ? P[(int64_t)(m0 + lr) * ldp + k] : 0.0;
      qr[t] = (n0 + lr < N && k < K) ? Q[(int64_t)(n0 + lr) * ldq + k] : 0.0;
    }
  };
  auto stash = [&](int buf) {
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      Ps[buf][lk + t][lr] = pr[t];
      Qs[buf][lk + t][lr] = qr[t];
    }
  };
  double acc[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = 0.0;
  const int nk = (K + DK - 1) / DK;
  if (nk > 0) {
    load(0);
    stash(0);
  }
  __syncthreads();
  for (int kt = 0; kt < nk; ++kt) {
    const int cur = kt & 1;
    if (kt + 1 < nk) load((kt + 1) * DK);
#pragma unroll
    for (int k = 0; k < DK; ++k) {
      double a[4], c[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = Ps[cur][k][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) c[j] = Qs[cur][k][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fma(a[i], c[j], acc[i][j]);
    }
    if (kt + 1 < nk) stash(cur ^ 1);
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty + 16 * i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx + 16 * j;
      if (n >= N) continue;
      double x = alpha * acc[i][j];
      if (beta != 0.0) x = fma(beta, C[(int64_t)m * ldc + n], x);
      C[(int64_t)m * ldc + n] = x;
      if (C2) C2[(int64_t)n * ldc2 + m] = x;
    }
  }
}

}  // namespace

nvfp4_status dgemm_nt(int M, int N, int K, double alpha, const double* P, int64_t ldp,
                      int64_t strideP, const double* Q, int64_t ldq, int64_t strideQ,
                      double beta, double* C, int64_t ldc, int64_t strideC, double* C2,
                      int64_t ldc2, int64_t strideC2, int batch, int lower, cudaStream_t st) {
  if (M <= 0 || N <= 0 || batch <= 0) return NVFP4_OK;
  if ((C2 && beta != 0.0) || (lower && M != N) || batch > 65535) return NVFP4_ERR_INVALID_ARG;
  const dim3 grid((unsigned)((N + DN - 1) / DN), (unsigned)((M + DM - 1) / DM), (unsigned)batch);
  if (grid.y > 65535) return NVFP4_ERR_SHAPE;
  dgemm_nt_kernel<<<grid, kDThreads, 0, st>>>(M, N, K, alpha, P, ldp, strideP, Q, ldq, strideQ,
                                              beta, C, ldc, strideC, C2, ldc2, strideC2, lower);
  NVFP4_LAUNCH_CHECK();
  count_launches(1);
  return NVFP4_OK;
}

}  // namespace nvfp4
