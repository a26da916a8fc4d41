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
  float lambda;       // fp32 copy for the caller
  double lambda64;    // used for the damping
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
      const double lam64 = (double)damp * (s / (double)d);
      const float lam = (float)lam64;
      hdr->lambda = lam;
      hdr->lambda64 = lam64;
      if (lambda_out) *lambda_out = lam;
    }
  }
}

// A[i][j] = H_d[d-1-i][d-1-j]; dead diagonal entries become 1 + lambda.
// Also zero-fills X (the inverse is built from its block diagonal outward).
__global__ void reverse_damp_kernel(const float* __restrict__ H, int64_t d,
                                    double* __restrict__ A, double* __restrict__ X,
                                    PrepHeader* hdr) {
  const double lam = hdr->lambda64;
  const int64_t total = d * d;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int64_t i = idx / d, j = idx - i * d;
    const float h = H[(d - 1 - i) * d + (d - 1 - j)];
    if (!isfinite(h)) flag_status(&hdr->status, NVFP4_ERR_NONFINITE);
    double a = (double)h;
    if (i == j) a = (h == 0.f ? 1.0 : a) + lam;
    A[idx] = a;
    X[idx] = 0.0;
  }
}

// One panel of the right-looking Cholesky: columns k .. k+kb-1 of A (lower,
// already updated by the earlier panels).  Every CTA factors the 64 x 64
// diagonal block A11 = L11 L11^T and inverts L11 in fp64 (redundantly: no CTA
// waits for another); CTA 0 then writes X11 = L11^-1 and Y11 = X11^T into the
// diagonal blocks of X and Y (A11 stays as it is: the other CTAs of the launch
// may still be reading it), every other CTA solves its own 64-row slice of the
// panel below, L21 = A21 X11^T, in place.
//
// The 64 x 64 block is itself blocked by 16 (a per-column CTA barrier costs
// far more than the arithmetic of a column):
//   for each 16-column sub-panel K:
//     one warp factors and inverts the 16 x 16 diagonal block in registers,
//       exchanging values by shuffles (lane i holds row i);
//     all threads solve the rows below it, L[r][K] = S[r][K] inv(L_KK)^T,
//     and update the trailing lower part, S -= L[:,K] L[:,K]^T;
//   the inverse of L is assembled from the four 16 x 16 inverses by two
//   doubling steps, X21 = -X22 (L21 X11), as small products.
constexpr int kPanelThreads = 256;
constexpr int kPitch = NB + 1;
constexpr int kSub = 16;

// 1/p for p > 0: the hardware's approximate fp64 reciprocal refined by two
// Newton-Raphson steps (x <- x + x (1 - p x)), which square the relative
// error each time.
__device__ __forceinline__ double recip_nr(double p) {
  double x;
  asm("rcp.approx.ftz.f64 %0, %1;" : "=d"(x) : "d"(p));
  x = fma(x, fma(-p, x, 1.0), x);
  x = fma(x, fma(-p, x, 1.0), x);
  return x;
}

constexpr size_t kPanelSmem = sizeof(double) * (4 * NB * kPitch);

// One warp, lanes 0..15 meaningful: factor the 16 x 16 block at (o, o) of S
// (lower part), write L_KK back into S and inv(L_KK) into the same block of
// Xd (lower, zeros above).  A non-positive pivot is flagged and taken as 1.
__device__ __forceinline__ void factor_invert_16(double (*S)[kPitch], double (*Xd)[kPitch],
                                                 int o, PrepHeader* hdr) {
  const int lane = threadIdx.x & 31;
  const int i = lane & 15;
  const unsigned full = 0xffffffffu;
  double r[kSub];   // row i of the block
#pragma unroll
  for (int l = 0; l < kSub; ++l) r[l] = (l <= i) ? S[o + i][o + l] : 0.0;
  double sq[kSub];  // sqrt(pivot_j), the same in every lane
#pragma unroll
  for (int j = 0; j < kSub; ++j) {
    double p = __shfl_sync(full, r[j], j, 16);
    const bool ok = p > 0.0;
    if (!ok) {
      if (lane == 0) flag_status(&hdr->status, NVFP4_ERR_NOT_PD);
      p = 1.0;
    }
    sq[j] = p;   // square root taken below, off the per-column chain
    const double a = (i > j) ? r[j] * recip_nr(p) : 0.0;
#pragma unroll
    for (int l = j + 1; l < kSub; ++l) {
      const double cl = __shfl_sync(full, r[j], l, 16);   // S[l][j]
      r[l] = fma(-a, cl, r[l]);
    }
  }
  // L[i][l] = r[l] / sqrt(p_l) (l < i), L[i][i] = sqrt(p_i)
  double isq[kSub];
#pragma unroll
  for (int l = 0; l < kSub; ++l) {
    sq[l] = sqrt(sq[l]);
    isq[l] = recip_nr(sq[l]);
  }
#pragma unroll
  for (int l = 0; l < kSub; ++l) r[l] = l < i ? r[l] * isq[l] : (l == i ? sq[i] : 0.0);
  // column c = i of inv(L): x[m] = -(sum_{l<m} L[m][l] x[l]) / L[m][m] for m > c
  double x[kSub];
#pragma unroll
  for (int m = 0; m < kSub; ++m) {
    double acc = 0.0;
#pragma unroll
    for (int l = 0; l < m; ++l) acc = fma(__shfl_sync(full, r[l], m, 16), x[l], acc);
    x[m] = m < i ? 0.0 : (m == i ? isq[m] : -acc * isq[m]);
  }
  if (lane < kSub) {
#pragma unroll
    for (int l = 0; l < kSub; ++l) {
      S[o + i][o + l] = l <= i ? r[l] : 0.0;
      Xd[o + l][o + i] = x[l];   // column i of the inverse
    }
  }
}

__global__ void __launch_bounds__(kPanelThreads)
    chol_panel_kernel(double* __restrict__ A, int64_t d, int64_t k, int kb,
                      double* __restrict__ X, double* __restrict__ Y, PrepHeader* hdr) {
  extern __shared__ double dsm[];
  double(*S)[kPitch] = reinterpret_cast<double(*)[kPitch]>(dsm);             // A11 -> L11
  double(*Xd)[kPitch] = reinterpret_cast<double(*)[kPitch]>(dsm + NB * kPitch);   // X11
  double(*R)[kPitch] = reinterpret_cast<double(*)[kPitch]>(dsm + 2 * NB * kPitch);
  double(*T)[kPitch] = reinterpret_cast<double(*)[kPitch]>(dsm + 3 * NB * kPitch);  // scratch
  const int tid = threadIdx.x, warp = tid >> 5;
  const int64_t r0 = k + kb + (int64_t)(blockIdx.x - 1) * NB;   // slice rows (CTA >= 1)
  const int64_t rem = d - r0;
  const int rows = blockIdx.x == 0 ? 0 : (int)(rem < NB ? rem : NB);

  {   // all global loads of a thread are issued before any is used
    constexpr int kPer = NB * NB / kPanelThreads;   // 16
    double a11[kPer], a21[kPer];
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
      const int idx = tid + q * kPanelThreads, i = idx / NB, l = idx % NB;
      a11[q] = (i < kb && l <= i) ? A[(k + i) * d + k + l] : 0.0;
      a21[q] = (i < rows && l < kb) ? A[(r0 + i) * d + k + l] : 0.0;
    }
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
      const int idx = tid + q * kPanelThreads, i = idx / NB, l = idx % NB;
      S[i][l] = (i < kb && l < kb) ? a11[q] : (i == l ? 1.0 : 0.0);
      Xd[i][l] = 0.0;
      R[i][l] = a21[q];
    }
  }
  __syncthreads();

  // ---- factor, 16 columns at a time
  for (int K = 0; K < NB / kSub; ++K) {
    const int o = K * kSub;
    if (warp == 0) factor_invert_16(S, Xd, o, hdr);
    __syncthreads();
    // rows below the sub-block: T[r][c] = sum_{l <= c} S[r][o+l] inv(L_KK)[c][l]
    const int nb = NB - o - kSub;   // rows below (0, 16, 32 or 48)
    for (int idx = tid; idx < nb * kSub; idx += blockDim.x) {
      const int rr = o + kSub + idx / kSub, c = idx % kSub;
      double acc = 0.0;
#pragma unroll
      for (int l = 0; l < kSub; ++l) acc = fma(S[rr][o + l], Xd[o + c][o + l], acc);
      T[rr][c] = acc;
    }
    __syncthreads();
    for (int idx = tid; idx < nb * kSub; idx += blockDim.x) {
      const int rr = o + kSub + idx / kSub, c = idx % kSub;
      S[rr][o + c] = T[rr][c];
    }
    __syncthreads();
    // trailing lower part: S[r][l] -= sum_m L[r][o+m] L[l][o+m], o+16 <= l <= r
    for (int idx = tid; idx < nb * nb; idx += blockDim.x) {
      const int rr = o + kSub + idx / nb, l = o + kSub + idx % nb;
      if (l <= rr) {
        double acc = S[rr][l];
#pragma unroll
        for (int m = 0; m < kSub; ++m) acc = fma(-S[rr][o + m], S[l][o + m], acc);
        S[rr][l] = acc;
      }
    }
    __syncthreads();
  }

  // ---- inverse by doubling: blocks of 16 -> 32 -> 64.  For a pair of
  // diagonal blocks of size b at offset q: X21 = -X22 (L21 X11).
  for (int b = kSub; b < NB; b *= 2) {
    const int npairs = NB / (2 * b);
    // T = L21 X11 for every pair (b x b each)
    for (int idx = tid; idx < npairs * b * b; idx += blockDim.x) {
      const int pq = idx / (b * b), e = idx % (b * b), i = e / b, j = e % b;
      const int q = pq * 2 * b;
      double acc = 0.0;
      for (int l = j; l < b; ++l) acc = fma(S[q + b + i][q + l], Xd[q + l][q + j], acc);
      T[q + b + i][q + j] = acc;
    }
    __syncthreads();
    for (int idx = tid; idx < npairs * b * b; idx += blockDim.x) {
      const int pq = idx / (b * b), e = idx % (b * b), i = e / b, j = e % b;
      const int q = pq * 2 * b;
      double acc = 0.0;
      for (int l = 0; l <= i; ++l) acc = fma(Xd[q + b + i][q + b + l], T[q + b + l][q + j], acc);
      Xd[q + b + i][q + j] = -acc;
    }
    __syncthreads();
  }

  if (blockIdx.x == 0) {
    for (int idx = tid; idx < kb * kb; idx += blockDim.x) {
      const int i = idx / kb, j = idx % kb;
      // L11 itself is not written back: nothing reads the diagonal blocks of L
      // later, and the other CTAs of this launch may still be reading A11.
      const double x = Xd[i][j];
      X[(k + i) * d + k + j] = x;            // lower (zeros above)
      Y[(k + j) * d + k + i] = x;            // its transpose, upper
    }
    return;
  }
  // ---- L21 slice = A21 slice X11^T: thread (ty, tx) computes a 4 x 4 tile,
  // L21[i][c] = sum_l R[i][l] X11[c][l]; X11 is staged transposed in T first
  // so that the loop reads it along rows (free of bank conflicts).
  for (int idx = tid; idx < NB * NB; idx += blockDim.x) {
    const int c = idx / NB, l = idx % NB;
    T[l][c] = Xd[c][l];
  }
  __syncthreads();
  const int ty = tid >> 4, tx = tid & 15, i0 = 4 * ty, l0 = 4 * tx;
  double acc[4][4] = {};
  for (int l = 0; l < NB; ++l) {
    double rv[4], xv[4];
#pragma unroll
    for (int a = 0; a < 4; ++a) rv[a] = R[i0 + a][l];
#pragma unroll
    for (int b = 0; b < 4; ++b) xv[b] = T[l][l0 + b];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) acc[a][b] = fma(rv[a], xv[b], acc[a][b]);
  }
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int b = 0; b < 4; ++b)
      if (i0 + a < rows && l0 + b < kb)
        A[(r0 + i0 + a) * d + k + l0 + b] = acc[a][b];
}

// U[i][j] = X[d-1-i][d-1-j] for j >= i, 0 below the diagonal.
__global__ void reverse_to_upper_kernel(const double* __restrict__ X, int64_t d,
                                        float* __restrict__ U) {
  const int64_t total = d * d;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int64_t i = idx / d, j = idx - i * d;
    U[idx] = (j >= i) ? (float)X[(d - 1 - i) * d + (d - 1 - j)] : 0.f;
  }
}

struct PrepLayout {
  PrepHeader* hdr;
  double* A;   // J H_d J, then its Cholesky factor L (lower)
  double* X;   // L^-1 (lower)
  double* Y;   // L^-T (upper)
  double* T;   // scratch of the inverse doubling
};

PrepLayout prep_layout(void* ws, int64_t d) {
  char* p = static_cast<char*>(ws);
  PrepLayout L;
  L.hdr = reinterpret_cast<PrepHeader*>(p);
  size_t off = kWsHeader;
  L.A = reinterpret_cast<double*>(p + off);
  off += align256(sizeof(double) * d * d);
  L.X = reinterpret_cast<double*>(p + off);
  off += align256(sizeof(double) * d * d);
  L.Y = reinterpret_cast<double*>(p + off);
  off += align256(sizeof(double) * d * d);
  L.T = reinterpret_cast<double*>(p + off);
  return L;
}

int grid_for(int64_t n, int threads) {
  int64_t b = (n + threads - 1) / threads;
  return (int)(b < 8 * kNumSMs ? (b < 1 ? 1 : b) : 8 * kNumSMs);
}

}  // namespace

size_t prepare_ws_bytes(int64_t d) {
  return kWsHeader + 3 * align256(sizeof(double) * d * d) +
         align256(sizeof(double) * (size_t)((d * d + 3) / 4 + d * NB));
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

  NVFP4_CUDA_TRY(cudaMemsetAsync(L.Y, 0, sizeof(double) * d * d, st));

  // Blocked right-looking Cholesky of A (lower), two levels: 64-column panels
  // (one fused panel kernel each: diagonal factor + inverse + panel solve)
  // inside 256-column outer blocks.  A panel updates only the rest of its outer
  // block right away; the trailing matrix beyond the block is updated once per
  // block, A22 -= L21 L21^T with K = 256, which reads and writes it 4x less
  // often than per-panel updates would.
  constexpr int64_t OB = 4 * NB;
  NVFP4_CUDA_TRY(cudaFuncSetAttribute(chol_panel_kernel,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)kPanelSmem));
  for (int64_t k0 = 0; k0 < d; k0 += OB) {
    const int64_t kend = (d - k0) < OB ? d : k0 + OB;
    for (int64_t k = k0; k < kend; k += NB) {
      const int kb = (int)((d - k) < NB ? (d - k) : NB);
      const int64_t m = d - k - kb;
      const int grid = 1 + (int)((m + NB - 1) / NB);
      chol_panel_kernel<<<grid, kPanelThreads, kPanelSmem, st>>>(L.A, d, k, kb, L.X, L.Y, L.hdr);
      NVFP4_LAUNCH_CHECK();
      count_launches(1);
      const int64_t nc = kend - (k + kb);   // columns of the outer block still to come
      if (m <= 0 || nc <= 0) continue;
      const double* L21 = L.A + (k + kb) * d + k;
      nvfp4_status s = dgemm_nt((int)m, (int)nc, kb, -1.0, L21, d, 0, L21, d, 0, 1.0,
                                L.A + (k + kb) * (d + 1), d, 0, nullptr, 0, 0, 1, 0, 0, st);
      if (s != NVFP4_OK) return s;
    }
    const int64_t m2 = d - kend;
    if (m2 > 0) {
      const double* Lb = L.A + kend * d + k0;
      nvfp4_status s = dgemm_nt((int)m2, (int)m2, (int)(kend - k0), -1.0, Lb, d, 0, Lb, d, 0,
                                1.0, L.A + kend * (d + 1), d, 0, nullptr, 0, 0, 1, 1, 0, st);
      if (s != NVFP4_OK) return s;
    }
  }

  // X = L^-1 by recursive doubling over pairs of adjacent diagonal blocks of
  // size b (all pairs of one level at once):  with L = [L11 0; L21 L22],
  //   T^T = Y11 L21^T,  X21 = -X22 T,  Y12 = X21^T   (Y = X^T throughout),
  // so every product is of the form P Q^T with K-contiguous operands.
  for (int64_t b = NB; b < d; b *= 2) {
    const int64_t npairs = d / (2 * b);
    const int64_t stride = 2 * b * (d + 1);
    if (npairs > 0) {
      nvfp4_status s = dgemm_nt((int)b, (int)b, (int)b, 1.0, L.Y, d, stride, L.A + b * d, d,
                                  stride, 0.0, L.T, b, b * b, nullptr, 0, 0, (int)npairs, 0, 1, st);
      if (s != NVFP4_OK) return s;
      s = dgemm_nt((int)b, (int)b, (int)b, -1.0, L.X + b * (d + 1), d, stride, L.T, b, b * b,
                     0.0, L.X + b * d, d, stride, L.Y + b, d, stride, (int)npairs, 0, 2,
                     st);
      if (s != NVFP4_OK) return s;
    }
    const int64_t r0 = npairs * 2 * b;   // a ragged pair: full left block, rr rows right
    const int64_t rr = d - r0 - b;
    if (rr > 0) {
      const int64_t o = r0 * (d + 1);
      nvfp4_status s = dgemm_nt((int)b, (int)rr, (int)b, 1.0, L.Y + o, d, 0,
                                  L.A + o + b * d, d, 0, 0.0, L.T, rr, 0, nullptr, 0, 0, 1, 0, 1, st);
      if (s != NVFP4_OK) return s;
      // X21 (rr x b) = -X22 (rr x rr) T (rr x b): P = X22, Q = T^T (b x rr)
      s = dgemm_nt((int)rr, (int)b, (int)rr, -1.0, L.X + o + b * (d + 1), d, 0, L.T, rr, 0,
                     0.0, L.X + o + b * d, d, 0, L.Y + o + b, d, 0, 1, 0, 2, st);
      if (s != NVFP4_OK) return s;
    }
  }
  reverse_to_upper_kernel<<<grid_for(d * d, 256), 256, 0, st>>>(L.X, d, U);
  NVFP4_LAUNCH_CHECK();
  count_launches(1);
  return NVFP4_OK;
}

}  // namespace nvfp4
