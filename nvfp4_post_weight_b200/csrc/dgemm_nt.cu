// fp64 GEMM on the tensor cores:  C = beta C + alpha P Q^T
// (P: M x K, Q: N x K, row-major with K contiguous; C: M x N row-major),
// optionally batched (blockIdx.z, element strides) and optionally restricted
// to the tiles on or below the diagonal (M == N); optionally writes C^T into
// C2 as well (beta == 0).
//
// Used by the factorisation, whose accuracy sets how faithfully the GPTQ
// decisions follow an exact solve: the damped Hessian of a layer calibrated on
// few tokens is ill-conditioned (1e4 and more), and a factor carried in fp32
// arithmetic moves block decisions that sit a few 1e-5 from a tie.  The
// 5th-generation tcgen05 instructions have no fp64 kind; fp64 runs on the
// warp-level mma.sync m8n8k4 (measured at ~36.7 TF/s on B200, its fp64 peak,
// with 8 warps per SM).
//
// Pipeline per CTA (one output tile of TL x TL, TL = 64 or 128):
//   warp 16     TMA producer: 16-wide K slices of P and Q (128 bytes of fp64
//               per row, 128-byte swizzle) into a 4-stage ring;
//   warps 0-15  consumers: fragments straight from the swizzled ring into
//               mma.sync; each warp owns a (TL/4) x (TL/4) block of C.
// A triangular P skips its zero half of K (ktri).  Every wait is bounded; a
// wait that runs out records NVFP4_ERR_TIMEOUT in *status.
#include <cuda.h>

#include "common.cuh"
#include "sm100.cuh"

namespace nvfp4 {
namespace {

using namespace sm100;

constexpr int DK = 16;                      // K per stage: 16 fp64 = 128 bytes per row
constexpr int kStages = 4;

// 16 consumer warps in a 4 x 4 grid (warp blocks of 32 x 32 for 128 x 128
// tiles, 16 x 16 for 64 x 64), so that each SM sub-partition interleaves four
// warps' mma.sync chains (measured faster than 8 warps of twice the block).
template <int TL>
struct Cfg {
  static constexpr int WGM = 4, WGN = 4;   // consumer warp grid
  static constexpr int kConsumerWarps = WGM * WGN;
  static constexpr int kThreads = 32 * (kConsumerWarps + 1);
  static constexpr int WM = TL / WGM, WN = TL / WGN;        // warp block of C
  static constexpr int MT = WM / 8, NT = WN / 8;            // 8 x 8 MMA tiles per warp
  static constexpr uint32_t kTile = TL * DK * 8;  // bytes of P (or Q) per stage
  static constexpr uint32_t kStage = 2 * kTile;
  static constexpr size_t kSmem = kStages * kStage + 1024 + 128;
};

struct Bars {
  uint64_t full[kStages], empty[kStages];
  int abort;
};

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// Byte offset, inside an 8-row group, of element (row fr, k) of a
// 128-byte-swizzled stage tile: the 16-byte chunk k/2 of row r sits at chunk
// position (k/2) ^ (r % 8).
//
// Fragment k mapping: the four k of m8n8k4 step s (0..3) are
// {2s, 2s+1, 2s+8, 2s+9}, lane column fc taking 2s + (fc & 1) + 8 (fc >> 1).
// The two chunks a half-warp touches, s and s ^ 4, then land on 8 distinct
// chunk positions across its 4 rows: every fragment load is conflict-free.
// A and B use the same mapping, so each step still sums four matching
// products.
__device__ __forceinline__ uint32_t frag_off(int fr, int fc, int s) {
  const int k = 2 * s + (fc & 1) + 8 * (fc >> 1);
  return (uint32_t)(fr * 128 + ((((k >> 1) ^ fr) & 7) << 4) + ((k & 1) << 3));
}

template <int TL>
__global__ void __launch_bounds__(Cfg<TL>::kThreads)
    dgemm_nt_kernel(const __grid_constant__ CUtensorMap tmP,
                    const __grid_constant__ CUtensorMap tmQ, int M, int N, int K, double alpha,
                    double beta, double* __restrict__ C, int64_t ldc, int64_t strideC,
                    double* __restrict__ C2, int64_t ldc2, int64_t strideC2, int lower,
                    int ktri, int* status) {
  using G = Cfg<TL>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  Bars* bars = reinterpret_cast<Bars*>(ring + kStages * G::kStage);
  // a lower-triangular P (ktri 2) gives the last row blocks the longest K
  // range: schedule them first, so that the long tiles do not form the tail
  const int tm = ktri == 2 ? (int)gridDim.y - 1 - (int)blockIdx.y : (int)blockIdx.y;
  const int tn = blockIdx.x, bz = blockIdx.z;
  if (lower && tn > tm) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = tm * TL, n0 = tn * TL;
  int kbeg = 0, kend = K;
  if (ktri == 1) kbeg = (m0 / DK) * DK;
  if (ktri == 2) kend = (m0 + TL) < K ? (m0 + TL) : K;
  const int kt0 = kbeg / DK;
  const int nk = kend > kbeg ? (kend - kbeg + DK - 1) / DK : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&bars->full[s], 1);
      mbar_init(&bars->empty[s], G::kConsumerWarps);
    }
    bars->abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  pdl_wait();

  if (warp == G::kConsumerWarps) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      tma_prefetch(&tmP);
      tma_prefetch(&tmQ);
      int issued = 0;
      for (int i = 0; i < nk; ++i) {
        const int s = i % kStages;
        if (i >= kStages && !mbar_wait(&bars->empty[s], ((i / kStages) - 1) & 1)) {
          atomicExch(&bars->abort, 1);
          atomicCAS(status, 0, (int)NVFP4_ERR_TIMEOUT);
          break;
        }
        if (*reinterpret_cast<volatile int*>(&bars->abort)) break;
        uint8_t* st = ring + s * G::kStage;
        mbar_arrive_expect_tx(&bars->full[s], G::kStage);
        tma_load_3d(st, &tmP, &bars->full[s], (kt0 + i) * DK, m0, bz);
        tma_load_3d(st + G::kTile, &tmQ, &bars->full[s], (kt0 + i) * DK, n0, bz);
        ++issued;
      }
      // whatever happened, no copy may still be in flight when the CTA exits
      for (int i = issued - kStages < 0 ? 0 : issued - kStages; i < issued; ++i)
        mbar_wait_drain(&bars->full[i % kStages], (i / kStages) & 1);
    }
    return;
  }

  // -------------------------------------------------------------- consumers
  const int fr = lane >> 2, fc = lane & 3;
  const int wm0 = (warp % G::WGM) * G::WM, wn0 = (warp / G::WGM) * G::WN;
  double acc[G::MT][G::NT][2];
#pragma unroll
  for (int i = 0; i < G::MT; ++i)
#pragma unroll
    for (int j = 0; j < G::NT; ++j) acc[i][j][0] = acc[i][j][1] = 0.0;
  uint32_t off[4];
#pragma unroll
  for (int s = 0; s < 4; ++s) off[s] = frag_off(fr, fc, s);
  bool ok = true;
  for (int i = 0; i < nk; ++i) {
    const int s = i % kStages;
    if (!mbar_wait(&bars->full[s], (i / kStages) & 1)) {
      atomicExch(&bars->abort, 1);
      atomicCAS(status, 0, (int)NVFP4_ERR_TIMEOUT);
      ok = false;
      break;
    }
    const uint8_t* Pb = ring + s * G::kStage + wm0 * 128;
    const uint8_t* Qb = ring + s * G::kStage + G::kTile + wn0 * 128;
#pragma unroll
    for (int k4 = 0; k4 < 4; ++k4) {
      double af[G::MT], bf[G::NT];
#pragma unroll
      for (int t = 0; t < G::MT; ++t)
        af[t] = *reinterpret_cast<const double*>(Pb + t * 8 * 128 + off[k4]);
#pragma unroll
      for (int t = 0; t < G::NT; ++t)
        bf[t] = *reinterpret_cast<const double*>(Qb + t * 8 * 128 + off[k4]);
#pragma unroll
      for (int a = 0; a < G::MT; ++a)
#pragma unroll
        for (int b = 0; b < G::NT; ++b) dmma_m8n8k4(acc[a][b][0], acc[a][b][1], af[a], bf[b]);
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&bars->empty[s]);
  }
  if (!__all_sync(0xffffffffu, ok)) return;

  C += bz * strideC;
  if (C2) C2 += bz * strideC2;
#pragma unroll
  for (int a = 0; a < G::MT; ++a) {
    const int m = m0 + wm0 + 8 * a + fr;
    if (m >= M) continue;
#pragma unroll
    for (int b = 0; b < G::NT; ++b)
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int n = n0 + wn0 + 8 * b + 2 * fc + h;
        if (n >= N) continue;
        double x = alpha * acc[a][b][h];
        if (beta != 0.0) x = fma(beta, C[(int64_t)m * ldc + n], x);
        C[(int64_t)m * ldc + n] = x;
        if (C2) C2[(int64_t)n * ldc2 + m] = x;
      }
  }
}

// 3-D map (K, rows, batch) of fp64 with a {16, TL, 1} box, 128-byte swizzle.
bool encode_map(CUtensorMap* map, const double* base, int64_t K, int64_t rows, int64_t ld,
                int64_t batch, int64_t stride, int TL) {
  const uint64_t dims[3] = {(uint64_t)K, (uint64_t)rows, (uint64_t)batch};
  const uint64_t strides[2] = {(uint64_t)ld * 8, (uint64_t)(batch > 1 ? stride : rows * ld) * 8};
  const uint32_t box[3] = {(uint32_t)DK, (uint32_t)TL, 1u};
  return encode_tmap_nd(map, base, CU_TENSOR_MAP_DATA_TYPE_FLOAT64, 3, dims, strides, box,
                        CU_TENSOR_MAP_SWIZZLE_128B);
}

template <int TL>
nvfp4_status launch_dgemm(int M, int N, int K, double alpha, const double* P, int64_t ldp,
                          int64_t strideP, const double* Q, int64_t ldq, int64_t strideQ,
                          double beta, double* C, int64_t ldc, int64_t strideC, double* C2,
                          int64_t ldc2, int64_t strideC2, int batch, int lower, int ktri,
                          int* status, cudaStream_t st) {
  using G = Cfg<TL>;
  CUtensorMap mp, mq;
  if (!encode_map(&mp, P, K, M, ldp, batch, strideP, TL) ||
      !encode_map(&mq, Q, K, N, ldq, batch, strideQ, TL))
    return NVFP4_ERR_CUDA;
  const dim3 grid((unsigned)((N + TL - 1) / TL), (unsigned)((M + TL - 1) / TL), (unsigned)batch);
  if (grid.y > 65535) return NVFP4_ERR_SHAPE;
  NVFP4_CUDA_TRY(cudaFuncSetAttribute(dgemm_nt_kernel<TL>,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      (int)G::kSmem));
  NVFP4_CUDA_TRY(launch_chained(dgemm_nt_kernel<TL>, grid, dim3(G::kThreads), G::kSmem, st, mp, mq,
                                M, N, K, alpha, beta, C, ldc, strideC, C2, ldc2, strideC2, lower,
                                ktri, status));
  count_launches(1);
  return NVFP4_OK;
}

}  // namespace

nvfp4_status dgemm_nt(int M, int N, int K, double alpha, const double* P, int64_t ldp,
                      int64_t strideP, const double* Q, int64_t ldq, int64_t strideQ,
                      double beta, double* C, int64_t ldc, int64_t strideC, double* C2,
                      int64_t ldc2, int64_t strideC2, int batch, int lower, int ktri,
                      int* status, cudaStream_t st) {
  if (M <= 0 || N <= 0 || batch <= 0) return NVFP4_OK;
  if ((C2 && beta != 0.0) || (lower && M != N) || batch > 65535 || ktri < 0 || ktri > 2 ||
      !status)
    return NVFP4_ERR_INVALID_ARG;
  // TMA: 16-byte aligned bases and row / batch strides; K a multiple of 16
  if (((ldp | ldq) & 1) != 0 || (batch > 1 && ((strideP | strideQ) & 1) != 0) || (K % DK) != 0 ||
      ((reinterpret_cast<uintptr_t>(P) | reinterpret_cast<uintptr_t>(Q)) & 15) != 0)
    return NVFP4_ERR_INVALID_ARG;
  ProfileScope ps(kPhaseFactorGemm, st);
  {
    // useful flops: only C's lower triangle when lower; a triangular P has
    // sum over rows of its nonzero K range (M <= K: M (M + 1) / 2 products per column)
    double f = 2.0 * M * N * K;
    if (lower) f = 2.0 * ((double)N * (N + 1) / 2) * K;
    if (ktri != 0 && M <= K) f = 2.0 * N * ((double)M * (M + 1) / 2 + (double)M * (K - M) * (ktri == 1));
    add_phase_work(f * batch);
  }
  // 128 x 128 tiles once there are enough of them to fill the GPU, else 64 x 64
  const int64_t big_tiles = (int64_t)((M + 127) / 128) * ((N + 127) / 128) * batch;
  if (big_tiles >= kNumSMs)
    return launch_dgemm<128>(M, N, K, alpha, P, ldp, strideP, Q, ldq, strideQ, beta, C, ldc,
                             strideC, C2, ldc2, strideC2, batch, lower, ktri, status, st);
  return launch_dgemm<64>(M, N, K, alpha, P, ldp, strideP, Q, ldq, strideQ, beta, C, ldc,
                          strideC, C2, ldc2, strideC2, batch, lower, ktri, status, st);
}

}  // namespace nvfp4
