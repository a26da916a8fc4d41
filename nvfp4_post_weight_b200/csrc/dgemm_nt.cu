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
// 5th-generation tcgen05 instructions have no fp64 kind; fp64 runs on the
// warp-level mma.sync m8n8k4 (measured at ~36.7 TF/s on B200, its fp64 peak,
// with 8 warps per SM, and 8x fewer instructions than fp64 FMAs):
// 64 x 64 or 128 x 128 CTA tiles, 8 warps of 32 x 16 or 64 x 32, K in steps
// of 16 staged in shared memory (double buffered through registers); a
// triangular P skips its zero half of K.
#include "common.cuh"

namespace nvfp4 {
namespace {

constexpr int DK = 16;
constexpr int kDThreads = 256;   // 8 warps: 2 along M x 4 along N

// CTA tile (16 T) x (32 T) ... see below; T = 4: 64 x 64 (each warp 32 x 16),
// T = 8: 128 x 128 (each warp 64 x 32).  ktri: 0 dense P; 1 P upper triangular
// (P[m][k] = 0 for k < m), so a tile's K range starts at its first row; 2 P
// lower triangular (P[m][k] = 0 for k > m), so it ends after its last row.
template <int T>
__global__ void __launch_bounds__(kDThreads)
    dgemm_nt_kernel(int M, int N, int K, double alpha, const double* __restrict__ P,
                    int64_t ldp, int64_t strideP, const double* __restrict__ Q, int64_t ldq,
                    int64_t strideQ, double beta, double* __restrict__ C, int64_t ldc,
                    int64_t strideC, double* __restrict__ C2, int64_t ldc2, int64_t strideC2,
                    int lower, int ktri) {
  constexpr int TL = 16 * T;            // CTA tile side (64 or 128)
  constexpr int WM = TL / 2, WN = TL / 4;   // warp tile
  constexpr int MT = WM / 8, NT = WN / 8;   // 8x8 MMA tiles per warp
  constexpr int PITCH = DK + 4;         // 20 doubles: fragment loads at the 2-wavefront minimum
  constexpr int PER = TL * DK / kDThreads;  // values per thread per operand and K step
  extern __shared__ double dsm[];
  double(*Ps)[TL][PITCH] = reinterpret_cast<double(*)[TL][PITCH]>(dsm);
  double(*Qs)[TL][PITCH] = reinterpret_cast<double(*)[TL][PITCH]>(dsm + 2 * TL * PITCH);
  const int tm = blockIdx.y, tn = blockIdx.x;
  if (lower && tn > tm) return;
  const int b = blockIdx.z;
  P += b * strideP;
  Q += b * strideQ;
  C += b * strideC;
  if (C2) C2 += b * strideC2;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int m0 = tm * TL, n0 = tn * TL;
  const int wm0 = (warp & 1) * WM, wn0 = (warp >> 1) * WN;
  int kbeg = 0, kend = K;
  if (ktri == 1) kbeg = (m0 / DK) * DK;
  if (ktri == 2) kend = (m0 + TL) < K ? (m0 + TL) : K;
  // loader: row lr, PER consecutive k values from lk
  constexpr int KG = DK / PER;
  const int lr = tid / KG, lk = (tid % KG) * PER;
  double pr[PER], qr[PER];
  auto load = [&](int k0) {
#pragma unroll
    for (int t = 0; t < PER; ++t) {
      const int k = k0 + lk + t;
      pr[t] = (m0 + lr < M && k < kend) ? P[(int64_t)(m0 + lr) * ldp + k] : 0.0;
      qr[t] = (n0 + lr < N && k < kend) ? Q[(int64_t)(n0 + lr) * ldq + k] : 0.0;
    }
  };
  auto stash = [&](int buf) {
#pragma unroll
    for (int t = 0; t < PER; ++t) {
      Ps[buf][lr][lk + t] = pr[t];
      Qs[buf][lr][lk + t] = qr[t];
    }
  };
  double acc[MT][NT][2];
#pragma unroll
  for (int i = 0; i < MT; ++i)
#pragma unroll
    for (int j = 0; j < NT; ++j) acc[i][j][0] = acc[i][j][1] = 0.0;
  const int nk = kend > kbeg ? (kend - kbeg + DK - 1) / DK : 0;
  if (nk > 0) {
    load(kbeg);
    stash(0);
  }
  __syncthreads();
  const int fr = lane >> 2, fc = lane & 3;
  for (int kt = 0; kt < nk; ++kt) {
    const int cur = kt & 1;
    if (kt + 1 < nk) load(kbeg + (kt + 1) * DK);
#pragma unroll
    for (int k4 = 0; k4 < DK; k4 += 4) {
      double af[MT], bf[NT];
#pragma unroll
      for (int i = 0; i < MT; ++i) af[i] = Ps[cur][wm0 + 8 * i + fr][k4 + fc];
#pragma unroll
      for (int j = 0; j < NT; ++j) bf[j] = Qs[cur][wn0 + 8 * j + fr][k4 + fc];
#pragma unroll
      for (int i = 0; i < MT; ++i)
#pragma unroll
        for (int j = 0; j < NT; ++j) dmma_m8n8k4(acc[i][j][0], acc[i][j][1], af[i], bf[j]);
    }
    if (kt + 1 < nk) stash(cur ^ 1);
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < MT; ++i) {
    const int m = m0 + wm0 + 8 * i + fr;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < NT; ++j)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int n = n0 + wn0 + 8 * j + 2 * fc + h;
        if (n >= N) continue;
        double x = alpha * acc[i][j][h];
        if (beta != 0.0) x = fma(beta, C[(int64_t)m * ldc + n], x);
        C[(int64_t)m * ldc + n] = x;
        if (C2) C2[(int64_t)n * ldc2 + m] = x;
      }
  }
}

template <int T>
nvfp4_status launch_dgemm(int M, int N, int K, double alpha, const double* P, int64_t ldp,
                          int64_t strideP, const double* Q, int64_t ldq, int64_t strideQ,
                          double beta, double* C, int64_t ldc, int64_t strideC, double* C2,
                          int64_t ldc2, int64_t strideC2, int batch, int lower, int ktri,
                          cudaStream_t st) {
  constexpr int TL = 16 * T;
  const size_t smem = sizeof(double) * 4 * TL * (DK + 4);
  const dim3 grid((unsigned)((N + TL - 1) / TL), (unsigned)((M + TL - 1) / TL), (unsigned)batch);
  if (grid.y > 65535) return NVFP4_ERR_SHAPE;
  NVFP4_CUDA_TRY(cudaFuncSetAttribute(dgemm_nt_kernel<T>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
  dgemm_nt_kernel<T><<<grid, kDThreads, smem, st>>>(M, N, K, alpha, P, ldp, strideP, Q, ldq,
                                                    strideQ, beta, C, ldc, strideC, C2, ldc2,
                                                    strideC2, lower, ktri);
  NVFP4_LAUNCH_CHECK();
  count_launches(1);
  return NVFP4_OK;
}

}  // namespace

nvfp4_status dgemm_nt(int M, int N, int K, double alpha, const double* P, int64_t ldp,
                      int64_t strideP, const double* Q, int64_t ldq, int64_t strideQ,
                      double beta, double* C, int64_t ldc, int64_t strideC, double* C2,
                      int64_t ldc2, int64_t strideC2, int batch, int lower, int ktri,
                      cudaStream_t st) {
  if (M <= 0 || N <= 0 || batch <= 0) return NVFP4_OK;
  if ((C2 && beta != 0.0) || (lower && M != N) || batch > 65535 || ktri < 0 || ktri > 2)
    return NVFP4_ERR_INVALID_ARG;
  // 128 x 128 tiles once there are enough of them to fill the GPU, else 64 x 64
  const int64_t big_tiles = (int64_t)((M + 127) / 128) * ((N + 127) / 128) * batch;
  if (big_tiles >= 2 * kNumSMs)
    return launch_dgemm<8>(M, N, K, alpha, P, ldp, strideP, Q, ldq, strideQ, beta, C, ldc,
                           strideC, C2, ldc2, strideC2, batch, lower, ktri, st);
  return launch_dgemm<4>(M, N, K, alpha, P, ldp, strideP, Q, ldq, strideQ, beta, C, ldc,
                         strideC, C2, ldc2, strideC2, batch, lower, ktri, st);
}

}  // namespace nvfp4
