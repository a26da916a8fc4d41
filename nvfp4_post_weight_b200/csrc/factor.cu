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

struct PrepHeader {   // one per problem of a group
  int status;
  int pad;
  double diag_sum;
  float lambda;       // fp32 copy for the caller
  double lambda64;    // used for the damping
};

// Sum of the diagonal (dead entries counted as 1), dead flags, lambda.  One
// CTA per problem of the group (blockIdx.x).  H is fp32 or fp64 (T).
template <typename T>
__global__ void diag_stats_kernel(PtrArr<const void*> Hs, int64_t d, float damp,
                                  PtrArr<uint8_t*> deads, PtrArr<float*> lambdas,
                                  PrepHeader* hdrs, int* gstatus) {
  __shared__ double part[32];
  const int pb = blockIdx.x;
  const T* __restrict__ H = static_cast<const T*>(Hs.p[pb]);
  uint8_t* dead = deads.p[pb];
  PrepHeader* hdr = hdrs + pb;
  double s = 0.0;
  for (int64_t i = threadIdx.x; i < d; i += blockDim.x) {
    const T h = H[i * d + i];
    const bool is_dead = (h == T(0));
    if (dead) dead[i] = is_dead ? 1 : 0;
    if (!isfinite(h)) {
      flag_status(&hdr->status, NVFP4_ERR_NONFINITE);
      flag_status(gstatus, NVFP4_ERR_NONFINITE);
    }
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
      if (lambdas.p[pb]) *lambdas.p[pb] = lam;
    }
  }
}

// A[i][j] = H_d[d-1-i][d-1-j]; dead diagonal entries become 1 + lambda.
// Also zero-fills X and Y (the inverse is built from its block diagonal
// outward).  Rows blockIdx.y, + gridDim.y, ...; four consecutive columns per
// thread (d is a multiple of 16); an fp32 H is read as float4 when it is
// 16-byte aligned.  Problem blockIdx.z of the group: its matrices sa elements
// after the previous problem's.  H is fp32 or fp64 (T).
template <typename T>
__global__ void reverse_damp_kernel(PtrArr<const void*> Hs, int64_t d, double* __restrict__ A,
                                    double* __restrict__ X, double* __restrict__ Y, int64_t sa,
                                    PrepHeader* hdrs, int* gstatus) {
  const int pb = blockIdx.z;
  const T* __restrict__ H = static_cast<const T*>(Hs.p[pb]);
  PrepHeader* hdr = hdrs + pb;
  A += pb * sa;
  X += pb * sa;
  Y += pb * sa;
  const bool vec = sizeof(T) == 4 && (reinterpret_cast<uintptr_t>(H) & 15) == 0;
  const double lam = hdr->lambda64;
  const int64_t j = 4 * ((int64_t)blockIdx.x * blockDim.x + threadIdx.x);
  if (j >= d) return;
  for (int64_t i = blockIdx.y; i < d; i += gridDim.y) {
    // H row d-1-i, columns d-4-j .. d-1-j, i.e. hv[3..0] for A's columns j .. j+3
    const T* hr = H + (d - 1 - i) * d + (d - 4 - j);
    double hv[4];
    if (vec) {
      const float4 h4 = *reinterpret_cast<const float4*>(hr);
      hv[0] = h4.w, hv[1] = h4.z, hv[2] = h4.y, hv[3] = h4.x;
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q) hv[q] = (double)hr[3 - q];
    }
    double a[4];
    bool bad = false;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      bad |= !isfinite(hv[q]);
      a[q] = hv[q];
      if (i == j + q) a[q] = (hv[q] == 0.0 ? 1.0 : a[q]) + lam;
    }
    if (bad) {
      flag_status(&hdr->status, NVFP4_ERR_NONFINITE);
      flag_status(gstatus, NVFP4_ERR_NONFINITE);
    }
    double2* Ar = reinterpret_cast<double2*>(A + i * d + j);   // workspace: aligned
    double2* Xr = reinterpret_cast<double2*>(X + i * d + j);
    double2* Yr = reinterpret_cast<double2*>(Y + i * d + j);
    Ar[0] = make_double2(a[0], a[1]);
    Ar[1] = make_double2(a[2], a[3]);
    Xr[0] = make_double2(0.0, 0.0);
    Xr[1] = make_double2(0.0, 0.0);
    Yr[0] = make_double2(0.0, 0.0);
    Yr[1] = make_double2(0.0, 0.0);
  }
}

// One panel of the right-looking Cholesky: columns k .. k+kb-1 of A (lower,
// already updated by the earlier panels).  Every CTA factors the 64 x 64
// diagonal block A11 = L11 L11^T and inverts L11 in fp64 (redundantly: no CTA
// waits for another); CTA 0 then writes X11 = L11^-1 and Y11 = X11^T into the
// diagonal blocks of X and Y (A11 stays as it is: the other CTAs of the launch
// may still be reading it), every other CTA solves its own 32-row slice of the
// panel below, L21 = A21 X11^T, in place.
//
// The 64 x 64 block is blocked by 16 (a per-column CTA barrier costs far more
// than the arithmetic of a column):
//   for each 16-column sub-panel K:
//     one warp factors the 16 x 16 diagonal block in registers, exchanging
//       values by shuffles (lane i holds row i) -- the only serial chain;
//     one thread per row below solves L[r][K] L_KK^T = S[r][K] by forward
//       substitution;
//     the warps update the trailing lower part, S -= L[:,K] L[:,K]^T, as
//       8 x 8 fp64 tensor-core tiles (mma.sync m8n8k4);
//   four warps then invert the four 16 x 16 diagonal blocks at once, and two
//   doubling steps, X21 = -X22 (L21 X11), assemble the inverse of L11; the
//   doubling products and the slice solve are tensor-core tiles too.
constexpr int kPanelThreads = 256;
constexpr int kPitch = NB + 4;   // 68: an 8 x 4 fragment (two half-warps) is conflict-free
constexpr int kSub = 16;
constexpr int kSlice = 32;       // rows of the panel below the diagonal block per CTA

// 1/p for p > 0: the hardware's approximate fp64 reciprocal refined by one
// Newton-Raphson step (x <- x + x (1 - p x)), which squares its relative
// error (2^-23 -> 2^-46: far below what the fp32 factor U keeps).
__device__ __forceinline__ double recip_nr1(double p) {
  double x;
  asm("rcp.approx.ftz.f64 %0, %1;" : "=d"(x) : "d"(p));
  return fma(x, fma(-p, x, 1.0), x);
}

// sqrt(p) and 1/sqrt(p) for p > 0 by Newton-Raphson on the reciprocal square
// root, y <- y + y (1/2 - (p/2) y^2), from the hardware approximation (two
// steps), then one Newton correction of the square root s = p y,
// s <- s + (y/2) (p - s^2).
__device__ __forceinline__ void sqrt_rsqrt(double p, double& sq, double& isq) {
  double y;
  asm("rsqrt.approx.ftz.f64 %0, %1;" : "=d"(y) : "d"(p));
  const double h = 0.5 * p;
  y = fma(y, fma(-h * y, y, 0.5), y);
  y = fma(y, fma(-h * y, y, 0.5), y);
  const double s0 = p * y;
  sq = fma(0.5 * y, fma(-s0, s0, p), s0);
  isq = y;
}

constexpr size_t kPanelSmem = sizeof(double) * ((3 * NB + kSlice) * kPitch + NB);

// One warp, lanes 0..15 meaningful: factor the 16 x 16 block at (o, o) of S
// (lower part) and write L_KK back into S (zeros above) and 1/L_jj into invd.
// A non-positive pivot is flagged and taken as 1.
__device__ __forceinline__ void factor_16(double (*S)[kPitch], double* invd, int o,
                                          PrepHeader* hdr, int* gstatus) {
  const int lane = threadIdx.x & 31;
  const int i = lane & 15;
  const unsigned full = 0xffffffffu;
  double r[kSub];   // row i of the block
#pragma unroll
  for (int l = 0; l < kSub; ++l) r[l] = (l <= i) ? S[o + i][o + l] : 0.0;
  double pv[kSub];  // the pivots, the same in every lane
  bool bad = false;
#pragma unroll
  for (int j = 0; j < kSub; ++j) {
    // branch-free: a (never taken) branch per pivot costs more than the pivot
    double p = __shfl_sync(full, r[j], j, 16);
    bad |= !(p > 0.0);
    p = p > 0.0 ? p : 1.0;
    pv[j] = p;
    const double a = (i > j) ? r[j] * recip_nr1(p) : 0.0;
#pragma unroll
    for (int l = j + 1; l < kSub; ++l) {
      const double cl = __shfl_sync(full, r[j], l, 16);   // S[l][j]
      r[l] = fma(-a, cl, r[l]);
    }
  }
  if (bad && lane == 0) {
    flag_status(&hdr->status, NVFP4_ERR_NOT_PD);
    flag_status(gstatus, NVFP4_ERR_NOT_PD);
  }
  // L[i][l] = r[l] / sqrt(p_l) (l < i), L[i][i] = sqrt(p_i)
  double sq[kSub], isq[kSub];
#pragma unroll
  for (int l = 0; l < kSub; ++l) sqrt_rsqrt(pv[l], sq[l], isq[l]);
  if (lane < kSub) {
    double isq_i = 0.0;   // isq[i] without a dynamic register index
#pragma unroll
    for (int l = 0; l < kSub; ++l) {
      S[o + i][o + l] = l < i ? r[l] * isq[l] : (l == i ? sq[l] : 0.0);
      isq_i = l == i ? isq[l] : isq_i;
    }
    invd[o + i] = isq_i;
  }
}

// One warp, lanes 0..15 meaningful: column i of inv(L_KK) for the factored
// block at (o, o) of S, by right-looking forward substitution (each x[m]
// updates the later sums at once, so the serial chain is one fma per m),
// written into the same block of Xd (lower, zeros above).  L[n][m] is read
// from shared memory (the same address in every lane: a broadcast), not
// passed between lanes.
__device__ __forceinline__ void invert_16(double (*S)[kPitch], double (*Xd)[kPitch],
                                          const double* invd, int o) {
  const int i = threadIdx.x & 15;
  double x[kSub], acc[kSub];
#pragma unroll
  for (int l = 0; l < kSub; ++l) acc[l] = 0.0;
#pragma unroll
  for (int m = 0; m < kSub; ++m) {
    const double id = invd[o + m];
    x[m] = m < i ? 0.0 : (m == i ? id : -acc[m] * id);
#pragma unroll
    for (int n = m + 1; n < kSub; ++n) acc[n] = fma(S[o + n][o + m], x[m], acc[n]);
  }
  if ((threadIdx.x & 31) < kSub) {
#pragma unroll
    for (int l = 0; l < kSub; ++l) Xd[o + l][o + i] = x[l];   // column i of the inverse
  }
}

// acc (8 x 8 tile, fragment layout of dmma_m8n8k4) += sgn * P[pm.., k] Q[qn.., k]^T
// summed over k in [k0, k1) (steps of 4), P and Q row-major in shared memory.
__device__ __forceinline__ void tile_pqt(double& d0, double& d1, double (*P)[kPitch], int pm,
                                         double (*Q)[kPitch], int qn, int k0, int k1,
                                         double sgn) {
  const int lane = threadIdx.x & 31, fr = lane >> 2, fc = lane & 3;
  for (int k = k0; k < k1; k += 4)
    dmma_m8n8k4(d0, d1, sgn * P[pm + fr][k + fc], Q[qn + fr][k + fc]);
}

// acc += sgn * P[pm.., k] B[k, bn..] summed over k in [k0, k1), with B read
// in place (row-major, N contiguous): no transposed copy needed.
__device__ __forceinline__ void tile_pb(double& d0, double& d1, double (*P)[kPitch], int pm,
                                        double (*Bm)[kPitch], int bn, int k0, int k1,
                                        double sgn) {
  const int lane = threadIdx.x & 31, fr = lane >> 2, fc = lane & 3;
  for (int k = k0; k < k1; k += 4)
    dmma_m8n8k4(d0, d1, sgn * P[pm + fr][k + fc], Bm[k + fc][bn + fr]);
}

// One level of the inverse doubling for every pair of adjacent b x b diagonal
// blocks at offset q:  T = L21 X11,  X21 = -X22 T.  The triangular factors
// are stored with zeros above their diagonals, so full-length sums are exact.
// 8 x 8 output tiles spread over the 8 warps.
template <int b>
__device__ __forceinline__ void doubling_level(double (*S)[kPitch], double (*Xd)[kPitch],
                                               double (*T)[kPitch]) {
  constexpr int kPairs = NB / (2 * b);
  constexpr int kTb = b / 8;                        // tiles per side of a block
  constexpr int kTiles = kPairs * kTb * kTb;        // 8 (b = 16) or 16 (b = 32)
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int fr = lane >> 2, fc2 = 2 * (lane & 3);
  for (int t = warp; t < kTiles; t += kPanelThreads / 32) {
    const int q = (t / (kTb * kTb)) * 2 * b, ti = (t / kTb) % kTb, tj = t % kTb;
    double d0 = 0.0, d1 = 0.0;
    tile_pb(d0, d1, S, q + b + 8 * ti, Xd, q + 8 * tj, q, q + b, 1.0);
    T[q + b + 8 * ti + fr][q + 8 * tj + fc2] = d0;
    T[q + b + 8 * ti + fr][q + 8 * tj + fc2 + 1] = d1;
  }
  __syncthreads();
  for (int t = warp; t < kTiles; t += kPanelThreads / 32) {
    const int q = (t / (kTb * kTb)) * 2 * b, ti = (t / kTb) % kTb, tj = t % kTb;
    double d0 = 0.0, d1 = 0.0;
    // P = X22 (rows and columns q+b ..), B = T (rows q+b .., columns q ..)
    tile_pb(d0, d1, Xd, q + b + 8 * ti, T, q + 8 * tj, q + b, q + 2 * b, -1.0);
    Xd[q + b + 8 * ti + fr][q + 8 * tj + fc2] = d0;
    Xd[q + b + 8 * ti + fr][q + 8 * tj + fc2 + 1] = d1;
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kPanelThreads)
    chol_panel_kernel(double* __restrict__ A, int64_t d, int64_t k, int kb,
                      double* __restrict__ X, double* __restrict__ Y, int64_t sa,
                      PrepHeader* hdrs, int* gstatus) {
  // problem blockIdx.y of the group
  A += blockIdx.y * sa;
  X += blockIdx.y * sa;
  Y += blockIdx.y * sa;
  PrepHeader* hdr = hdrs + blockIdx.y;
  extern __shared__ double dsm[];
  double(*S)[kPitch] = reinterpret_cast<double(*)[kPitch]>(dsm);             // A11 -> L11
  double(*Xd)[kPitch] = reinterpret_cast<double(*)[kPitch]>(dsm + NB * kPitch);   // X11
  double(*T)[kPitch] = reinterpret_cast<double(*)[kPitch]>(dsm + 2 * NB * kPitch);  // scratch
  double(*R)[kPitch] = reinterpret_cast<double(*)[kPitch]>(dsm + 3 * NB * kPitch);  // A21 slice
  double* invd = dsm + (3 * NB + kSlice) * kPitch;                             // 1 / L_jj
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int fr = lane >> 2, fc2 = 2 * (lane & 3);
  const int64_t r0 = k + kb + (int64_t)(blockIdx.x - 1) * kSlice;   // slice rows (CTA >= 1)
  const int64_t rem = d - r0;
  const int rows = blockIdx.x == 0 ? 0 : (int)(rem < kSlice ? rem : kSlice);
  pdl_wait();

  {   // all global loads of a thread are issued before any is used
    constexpr int kPer = NB * NB / kPanelThreads;        // 16
    constexpr int kPerS = kSlice * NB / kPanelThreads;   // 8
    double a11[kPer], a21[kPerS];
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
      const int idx = tid + q * kPanelThreads, i = idx / NB, l = idx % NB;
      a11[q] = (i < kb && l <= i) ? A[(k + i) * d + k + l] : 0.0;
    }
#pragma unroll
    for (int q = 0; q < kPerS; ++q) {
      const int idx = tid + q * kPanelThreads, i = idx / NB, l = idx % NB;
      a21[q] = (i < rows && l < kb) ? A[(r0 + i) * d + k + l] : 0.0;
    }
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
      const int idx = tid + q * kPanelThreads, i = idx / NB, l = idx % NB;
      S[i][l] = (i < kb && l < kb) ? a11[q] : (i == l ? 1.0 : 0.0);
      Xd[i][l] = 0.0;
    }
#pragma unroll
    for (int q = 0; q < kPerS; ++q) {
      const int idx = tid + q * kPanelThreads, i = idx / NB, l = idx % NB;
      R[i][l] = a21[q];
    }
  }
  __syncthreads();

  // ---- factor, 16 columns at a time (not unrolled: inlined copies of the
  // warp factor overflow the instruction cache)
#pragma unroll 1
  for (int K = 0; K < NB / kSub; ++K) {
    const int o = K * kSub;
    if (warp == 0) factor_16(S, invd, o, hdr, gstatus);
    __syncthreads();
    const int nb = NB - o - kSub;   // rows below the sub-block (48, 32, 16 or 0)
    if (nb == 0) break;
    // rows below: solve x L_KK^T = S[r][K] for the row's new L values, one
    // thread per row, right-looking (one fma per step on the serial chain)
    if (tid >= 32 && tid < 32 + nb) {
      const int rr = o + kSub + tid - 32;
      double x[kSub];
#pragma unroll
      for (int c = 0; c < kSub; ++c) x[c] = S[rr][o + c];
#pragma unroll
      for (int c = 0; c < kSub; ++c) {
        x[c] *= invd[o + c];
#pragma unroll
        for (int c2 = c + 1; c2 < kSub; ++c2) x[c2] = fma(-x[c], S[o + c2][o + c], x[c2]);
      }
#pragma unroll
      for (int c = 0; c < kSub; ++c) S[rr][o + c] = x[c];
    }
    __syncthreads();
    // trailing lower part: S[r][l] -= sum_m L[r][o+m] L[l][o+m] for
    // o+16 <= l <= r, as 8 x 8 tiles on or below the diagonal
    {
      const int nt = nb / 8, ntiles = nt * (nt + 1) / 2, b0 = o + kSub;
      for (int t = warp; t < ntiles; t += kPanelThreads / 32) {
        int ti = 0, tt = t;
        while (tt > ti) tt -= ++ti;   // t -> (ti, tj), tj <= ti
        const int tj = tt;
        const int row = b0 + 8 * ti + fr, col = b0 + 8 * tj + fc2;
        double d0 = S[row][col], d1 = S[row][col + 1];
        tile_pqt(d0, d1, S, b0 + 8 * ti, S, b0 + 8 * tj, o, o + kSub, -1.0);
        if (col <= row) S[row][col] = d0;
        if (col + 1 <= row) S[row][col + 1] = d1;
      }
    }
    __syncthreads();
  }

  // ---- inverse: the four 16 x 16 diagonal inverses at once, then doubling
  // 16 -> 32 -> 64
  if (warp < NB / kSub) invert_16(S, Xd, invd, warp * kSub);
  __syncthreads();
  doubling_level<16>(S, Xd, T);
  doubling_level<32>(S, Xd, T);

  if (blockIdx.x == 0) {
    // L11 itself is not written back: nothing reads the diagonal blocks of L
    // later, and the other CTAs of this launch may still be reading A11.
    // X11 (lower, zeros above) and its transpose into Y, row by row; all
    // shared-memory reads of a thread before its stores, no division
    constexpr int kPer = NB * NB / kPanelThreads;   // 16
    double xv[kPer], yv[kPer];
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
      const int idx = tid + q * kPanelThreads, i = idx >> 6, j = idx & (NB - 1);
      xv[q] = Xd[i][j];
      yv[q] = Xd[j][i];   // Y[i][j] = X[j][i]
    }
#pragma unroll
    for (int q = 0; q < kPer; ++q) {
      const int idx = tid + q * kPanelThreads, i = idx >> 6, j = idx & (NB - 1);
      if (i < kb && j < kb) {
        X[(k + i) * d + k + j] = xv[q];
        Y[(k + i) * d + k + j] = yv[q];
      }
    }
    return;
  }
  // ---- L21 slice = A21 slice X11^T: 32 x 64 = 4 x 8 tiles, 4 per warp; then
  // the CTA's further slices (gridDim.x - 1 slices apart), each loaded after
  // the previous one is written (the diagonal block is factored once per CTA)
  int64_t rs = r0;
  int nrows = rows;
  const int64_t slice_step = (int64_t)(gridDim.x - 1) * kSlice;
  for (;;) {
    const int ti = warp & 3, tj0 = (warp >> 2) * 4;
    double acc[4][2] = {};
    for (int kk = 0; kk < NB; kk += 4) {
      const double a = R[8 * ti + fr][kk + (lane & 3)];
#pragma unroll
      for (int j = 0; j < 4; ++j)
        dmma_m8n8k4(acc[j][0], acc[j][1], a, Xd[8 * (tj0 + j) + fr][kk + (lane & 3)]);
    }
    const int i = 8 * ti + fr;
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int c = 8 * (tj0 + j) + fc2 + h;
        if (i < nrows && c < kb) A[(rs + i) * d + k + c] = acc[j][h];
      }
    rs += slice_step;
    if (rs >= d) break;
    nrows = (int)((d - rs) < kSlice ? (d - rs) : kSlice);
    constexpr int kPerS = kSlice * NB / kPanelThreads;   // 8
    double a21[kPerS];
#pragma unroll
    for (int q = 0; q < kPerS; ++q) {
      const int idx = tid + q * kPanelThreads, ii = idx / NB, l = idx % NB;
      a21[q] = (ii < nrows && l < kb) ? A[(rs + ii) * d + k + l] : 0.0;
    }
    __syncthreads();   // every warp is done reading the previous slice
#pragma unroll
    for (int q = 0; q < kPerS; ++q) {
      const int idx = tid + q * kPanelThreads, ii = idx / NB, l = idx % NB;
      R[ii][l] = a21[q];
    }
    __syncthreads();
  }
}

// CTAs that solve a panel's slices, per problem of a group of P: every CTA
// factors the diagonal block (a fixed chain of about kChainUnits time units)
// before it solves its slices (about one unit each), and the panel kernel
// runs one CTA per SM; so take the count of slice CTAs that minimises waves x
// time per CTA.
constexpr int kChainUnits = 8;
int panel_slice_ctas(int64_t nslices, int P, int sms) {
  if (nslices <= 0) return 0;
  int best = 1;
  double best_t = 1e300;
  for (int64_t c = 1; c <= nslices; ++c) {
    const int64_t waves = ((int64_t)P * (1 + c) + sms - 1) / sms;
    const double t = (double)waves * (kChainUnits + (double)((nslices + c - 1) / c));
    if (t < best_t) {
      best_t = t;
      best = (int)c;
    }
    if ((int64_t)P * (1 + c) > 64LL * sms) break;
  }
  return best;
}

// U[i][j] = X[d-1-i][d-1-j] for j >= i, 0 below the diagonal.  Rows
// blockIdx.y, + gridDim.y, ...; four consecutive columns per thread, U
// written as float4 when it is 16-byte aligned (vec).
__global__ void reverse_to_upper_kernel(const double* __restrict__ X, int64_t d, int64_t sa,
                                        PtrArr<float*> Us) {
  float* __restrict__ U = Us.p[blockIdx.z];   // problem blockIdx.z of the group
  X += blockIdx.z * sa;
  const bool vec = (reinterpret_cast<uintptr_t>(U) & 15) == 0;
  const int64_t j = 4 * ((int64_t)blockIdx.x * blockDim.x + threadIdx.x);
  if (j >= d) return;
  for (int64_t i = blockIdx.y; i < d; i += gridDim.y) {
    float u[4] = {0.f, 0.f, 0.f, 0.f};
    if (j + 3 >= i) {   // some of the four are on or above the diagonal
      // X row d-1-i, columns d-4-j .. d-1-j (workspace: 16-byte aligned pairs)
      const double2* xr = reinterpret_cast<const double2*>(X + (d - 1 - i) * d + (d - 4 - j));
      const double2 p = xr[0], q2 = xr[1];
      const double xv[4] = {q2.y, q2.x, p.y, p.x};   // columns j .. j+3 of the reversed row
#pragma unroll
      for (int q = 0; q < 4; ++q) u[q] = (j + q >= i) ? (float)xv[q] : 0.f;
    }
    float* ur = U + i * d + j;
    if (vec) {
      *reinterpret_cast<float4*>(ur) = make_float4(u[0], u[1], u[2], u[3]);
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q) ur[q] = u[q];
    }
  }
}

// A group region of the prepare: the group header (its first int the status
// word), P problem headers, then P copies each of A, X, Y (sa = d (d + 1)
// elements apart: one d x d matrix and d elements of padding, so that the
// pairs of the inverse doubling of all P problems sit one stride apart when
// 2b divides d), the doubling scratch T and the int8-slice scratch.
struct PrepLayout {
  int* gstatus;
  PrepHeader* hdr;
  int64_t sa;   // elements between the problems' A (X, Y) matrices
  double* A;    // J H_d J, then its Cholesky factor L (lower)
  double* X;    // L^-1 (lower)
  double* Y;    // L^-T (upper)
  double* T;    // scratch of the inverse doubling
  void* S8;     // int8 slices of the tensor-core fp64 GEMMs
  size_t s8_bytes;
};

// Doubling scratch per problem: a level's pairs (d / 2b of b x b) or its
// ragged pair (b x rr, rr < b), at most d^2 / 4; plus room for d x NB.
int64_t t_elems(int64_t d) { return (d * d + 3) / 4 + d * NB; }

// Slice scratch of the int8-slice GEMMs for P problems: the largest operand
// pair of a call (trailing update: d x 512 twice; doubling level b: d/2b
// pairs of b x b, twice) per problem is below the bound for M = N = d,
// K = d/2.
size_t slice_scratch_bytes(int64_t d, int P) {
  return dgemm_i8_scratch_bytes(d, d, (d / 2 + 15) / 16 * 16 + 256, P);
}

size_t prep_group_bytes(int64_t d, int P) {
  const int64_t sa = d * (d + 1);
  return kWsHeader + align256(sizeof(PrepHeader) * P) + 3 * align256(sizeof(double) * sa * P) +
         align256(sizeof(double) * (size_t)t_elems(d) * P) + align256(slice_scratch_bytes(d, P));
}

PrepLayout prep_layout(void* ws, int64_t d, int P) {
  char* p = static_cast<char*>(ws);
  PrepLayout L;
  L.gstatus = reinterpret_cast<int*>(p);
  size_t off = kWsHeader;
  L.hdr = reinterpret_cast<PrepHeader*>(p + off);
  off += align256(sizeof(PrepHeader) * P);
  L.sa = d * (d + 1);
  L.A = reinterpret_cast<double*>(p + off);
  off += align256(sizeof(double) * L.sa * P);
  L.X = reinterpret_cast<double*>(p + off);
  off += align256(sizeof(double) * L.sa * P);
  L.Y = reinterpret_cast<double*>(p + off);
  off += align256(sizeof(double) * L.sa * P);
  L.T = reinterpret_cast<double*>(p + off);
  off += align256(sizeof(double) * (size_t)t_elems(d) * P);
  L.S8 = p + off;
  L.s8_bytes = slice_scratch_bytes(d, P);
  return L;
}

}  // namespace

size_t prepare_ws_bytes(int64_t d) { return prep_group_bytes(d, 1); }
size_t prepare_group_ws_bytes(int64_t d, int P) { return prep_group_bytes(d, P); }

// The prepare of a group of P problems of dimension d (every launch covers all
// P): ws is the group region (prepare_group_ws_bytes(d, P) bytes).  A problem
// whose factor meets a non-positive pivot or a non-finite H has its own
// header's status set; the group word at the start of ws collects the first
// status of any problem and the GEMMs' timeouts.
nvfp4_status launch_prepare_group(int P, const PtrArr<const void*>& H, bool h64, int64_t d,
                                  float damp, const PtrArr<float*>& U,
                                  const PtrArr<uint8_t*>& dead, const PtrArr<float*>& lambda_out,
                                  void* ws, cudaStream_t st) {
  if (P < 1 || P > kMaxGroup) return NVFP4_ERR_INVALID_ARG;
  PrepLayout L = prep_layout(ws, d, P);
  NVFP4_CUDA_TRY(cudaMemsetAsync(ws, 0, kWsHeader + align256(sizeof(PrepHeader) * P), st));
  if (h64)
    diag_stats_kernel<double><<<P, 1024, 0, st>>>(H, d, damp, dead, lambda_out, L.hdr,
                                                  L.gstatus);
  else
    diag_stats_kernel<float><<<P, 1024, 0, st>>>(H, d, damp, dead, lambda_out, L.hdr,
                                                 L.gstatus);
  NVFP4_LAUNCH_CHECK();
  count_launches(1);
  const dim3 rgrid((unsigned)((d / 4 + 255) / 256), (unsigned)(d < 65535 ? d : 65535),
                   (unsigned)P);
  if (h64)
    reverse_damp_kernel<double><<<rgrid, 256, 0, st>>>(H, d, L.A, L.X, L.Y, L.sa, L.hdr,
                                                       L.gstatus);
  else
    reverse_damp_kernel<float><<<rgrid, 256, 0, st>>>(H, d, L.A, L.X, L.Y, L.sa, L.hdr,
                                                      L.gstatus);
  NVFP4_LAUNCH_CHECK();
  count_launches(1);
  const int64_t sa = L.sa;

  // Blocked right-looking Cholesky of A (lower), two levels: 64-column panels
  // (one fused panel kernel each: diagonal factor + inverse + panel solve)
  // inside 512-column outer blocks.  A panel updates only the rest of its outer
  // block right away; the trailing matrix beyond the block is updated once per
  // block, A22 -= L21 L21^T with K = 512, which reads and writes it 8x less
  // often than per-panel updates would (measured: 512-column blocks beat 256
  // and 1024 on the 4096-wide layer).
  constexpr int64_t OB = 8 * NB;
  // the large products (trailing updates of at least 512 rows, doubling
  // levels from 256) go to the int8-slice tensor-core engine, the small and
  // narrow ones to mma.sync fp64, whose latency is lower
  constexpr int64_t kBigGemm = 512;
  auto gemm = [&](bool big, int M, int N, int K, double alpha, const double* Pm, int64_t ldp,
                  int64_t sP, const double* Q, int64_t ldq, int64_t sQ, double beta, double* C,
                  int64_t ldc, int64_t sC, double* C2, int64_t ldc2, int64_t sC2, int batch,
                  int lower, int ktri) {
    if (big && K < (1 << 16))
      return dgemm_i8(M, N, K, alpha, Pm, ldp, sP, Q, ldq, sQ, beta, C, ldc, sC, C2, ldc2, sC2,
                      batch, lower, ktri, L.S8, L.s8_bytes, L.gstatus, st);
    return dgemm_nt(M, N, K, alpha, Pm, ldp, sP, Q, ldq, sQ, beta, C, ldc, sC, C2, ldc2, sC2,
                    batch, lower, ktri, L.gstatus, st);
  };
  NVFP4_CUDA_TRY(cudaFuncSetAttribute(chol_panel_kernel,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)kPanelSmem));
  for (int64_t k0 = 0; k0 < d; k0 += OB) {
    const int64_t kend = (d - k0) < OB ? d : k0 + OB;
    for (int64_t k = k0; k < kend; k += NB) {
      const int kb = (int)((d - k) < NB ? (d - k) : NB);
      const int64_t m = d - k - kb;
      const int grid = 1 + panel_slice_ctas((m + kSlice - 1) / kSlice, P, num_sms());
      {
        ProfileScope ps(kPhasePanel, st);
        // Cholesky and inverse of the kb x kb block, and the m x kb slice solve
        add_phase_work(P * (2.0 * kb * kb * kb / 3.0 + (double)m * kb * kb));
        NVFP4_CUDA_TRY(launch_chained(chol_panel_kernel, dim3(grid, P), dim3(kPanelThreads),
                                      kPanelSmem, st, L.A, d, k, kb, L.X, L.Y, sa, L.hdr,
                                      L.gstatus));
        count_launches(1);
      }
      const int64_t nc = kend - (k + kb);   // columns of the outer block still to come
      if (m <= 0 || nc <= 0) continue;
      const double* L21 = L.A + (k + kb) * d + k;
      nvfp4_status s = dgemm_nt((int)m, (int)nc, kb, -1.0, L21, d, sa, L21, d, sa, 1.0,
                                L.A + (k + kb) * (d + 1), d, sa, nullptr, 0, 0, P, 0, 0,
                                L.gstatus, st);
      if (s != NVFP4_OK) return s;
    }
    const int64_t m2 = d - kend;
    if (m2 > 0) {
      const double* Lb = L.A + kend * d + k0;
      nvfp4_status s = gemm(m2 >= kBigGemm, (int)m2, (int)m2, (int)(kend - k0), -1.0, Lb, d, sa,
                            Lb, d, sa, 1.0, L.A + kend * (d + 1), d, sa, nullptr, 0, 0, P, 1, 0);
      if (s != NVFP4_OK) return s;
    }
  }

  // X = L^-1 by recursive doubling over pairs of adjacent diagonal blocks of
  // size b (all pairs of one level, of all P problems, at once):  with
  // L = [L11 0; L21 L22],
  //   T^T = Y11 L21^T,  X21 = -X22 T,  Y12 = X21^T   (Y = X^T throughout),
  // so every product is of the form P Q^T with K-contiguous operands.  The
  // pairs of a level lie 2b (d + 1) apart inside a problem; across problems
  // that is still one stride when 2b divides d (sa = (d / 2b) 2b (d + 1)) or
  // when there is one pair per problem (stride sa); otherwise the level runs
  // problem by problem.
  auto level = [&](int64_t b, int64_t npairs, const double* base_off_A, int nbatch,
                   int64_t stride, double* T) -> nvfp4_status {
    const bool big = b >= kBigGemm / 2;
    const int64_t o = base_off_A - L.A;   // element offset of the first pair's block
    nvfp4_status s = gemm(big, (int)b, (int)b, (int)b, 1.0, L.Y + o, d, stride,
                          L.A + o + b * d, d, stride, 0.0, T, b, b * b, nullptr, 0, 0, nbatch,
                          0, 1);
    if (s != NVFP4_OK) return s;
    (void)npairs;
    return gemm(big, (int)b, (int)b, (int)b, -1.0, L.X + o + b * (d + 1), d, stride, T, b,
                b * b, 0.0, L.X + o + b * d, d, stride, L.Y + o + b, d, stride, nbatch, 0, 2);
  };
  for (int64_t b = NB; b < d; b *= 2) {
    const int64_t npairs = d / (2 * b);
    const int64_t stride = 2 * b * (d + 1);
    if (npairs > 0) {
      nvfp4_status s;
      if (P == 1 || d % (2 * b) == 0) {
        s = level(b, npairs, L.A, (int)(npairs * P), stride, L.T);
      } else if (npairs == 1) {
        s = level(b, npairs, L.A, P, sa, L.T);
      } else {
        s = NVFP4_OK;
        for (int pb = 0; pb < P && s == NVFP4_OK; ++pb)
          s = level(b, npairs, L.A + pb * sa, (int)npairs, stride, L.T + pb * npairs * b * b);
      }
      if (s != NVFP4_OK) return s;
    }
    const int64_t r0 = npairs * 2 * b;   // a ragged pair: full left block, rr rows right
    const int64_t rr = d - r0 - b;
    if (rr > 0) {
      const int64_t o = r0 * (d + 1);
      nvfp4_status s = gemm(b >= kBigGemm / 2, (int)b, (int)rr, (int)b, 1.0, L.Y + o, d, sa,
                            L.A + o + b * d, d, sa, 0.0, L.T, rr, b * rr, nullptr, 0, 0, P, 0,
                            1);
      if (s != NVFP4_OK) return s;
      // X21 (rr x b) = -X22 (rr x rr) T (rr x b): P = X22, Q = T^T (b x rr)
      s = gemm(b >= kBigGemm / 2, (int)rr, (int)b, (int)rr, -1.0, L.X + o + b * (d + 1), d, sa,
               L.T, rr, b * rr, 0.0, L.X + o + b * d, d, sa, L.Y + o + b, d, sa, P, 0, 2);
      if (s != NVFP4_OK) return s;
    }
  }
  reverse_to_upper_kernel<<<rgrid, 256, 0, st>>>(L.X, d, sa, U);
  NVFP4_LAUNCH_CHECK();
  count_launches(1);
  return NVFP4_OK;
}

// The single-problem prepare: a group of one whose region is ws; H is fp32,
// or fp64 when h64.
nvfp4_status launch_prepare(const void* H, bool h64, int64_t d, float damp, float* U,
                            uint8_t* dead, float* lambda_out, void* ws, cudaStream_t st) {
  PtrArr<const void*> h;
  PtrArr<float*> u, lam;
  PtrArr<uint8_t*> dd;
  h.p[0] = H;
  u.p[0] = U;
  dd.p[0] = dead;
  lam.p[0] = lambda_out;
  return launch_prepare_group(1, h, h64, d, damp, u, dd, lam, ws, st);
}

// Problem i's status word of a prepare group region.
const int* prepare_group_problem_status(const void* ws, int i) {
  const char* p = static_cast<const char*>(ws) + kWsHeader;
  return reinterpret_cast<const int*>(p + sizeof(PrepHeader) * i);
}

}  // namespace nvfp4
