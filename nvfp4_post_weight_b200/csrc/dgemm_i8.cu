// fp64-accurate GEMM on the 5th-generation tensor cores through int8 slices:
//   C = beta C + alpha P Q^T   (P: M x K, Q: N x K row-major fp64, C: M x N)
// with the options of dgemm_nt (batch, lower tiles, triangular P, C2 = C^T).
//
// tcgen05 has no fp64 kind, but its int8 kind multiplies exactly into int32.
// Each row of P (and of Q) is scaled by a power of two so that its largest
// entry lies in [1/4, 1/2), and the scaled values are cut into S signed 7-bit
// slices:  x = sum_t a_t 2^(-7 (t + 1)) + r,  a_t in [-64, 64] (balanced
// base-128 digits of x rounded to a multiple of 2^(-7 S)), |r| <= 2^(-7 S - 1)
// (the splitting of Ozaki et al., "Error-free
// transformations of matrix multiplication by using fast routines of matrix
// multiplication and its applications", Numer. Algorithms 59 (2012), with
// integer slices).  Then
//   (P Q^T)_mn = 2^(e_m + e_n) sum_{t,u} 2^(-7 (t + u + 2)) (A_t B_u^T)_mn,
// every slice product is exact in int32, and the products of one level
// l = t + u share an int32 TMEM accumulator (exact: |sum| < 2^31 for K < 2^16).
// Levels l > S - 1 are dropped: together they weigh less than 2^(-7 S + 3)
// of the row and column maxima, i.e. about 2^-46 for S = 7 -- far below what
// the fp32 factor U keeps after the condition number of the damped Hessian
// amplifies it.  The levels are combined in fp64 in the epilogue.
//
// Pipeline per 128 x 64 output tile, K in 64-byte chunks (SWIZZLE_64B, all S
// slices of a chunk in one 3-D TMA load per operand):
//   warp 0     TMA producer (2-stage ring of A and B slices)
//   warp 1     MMA issuer: S (S + 1) / 2 slice pairs x 2 K-steps of 32 per chunk
//   warps 2-5  epilogue: TMEM -> registers, levels summed in fp64, scaled by
//              the row and column exponents, C written (beta, C2, alpha).
// Every wait is bounded; a wait that runs out records NVFP4_ERR_TIMEOUT.
#include <cuda.h>

#include "common.cuh"
#include "sm100.cuh"

namespace nvfp4 {
namespace {

using namespace sm100;

constexpr int S = 7;                     // slices per value
constexpr int IM = 128, IN = 64;         // output tile
constexpr int KC = 64;                   // K bytes (int8 values) per stage
constexpr int kIStages = 2;
constexpr uint32_t kASlice = IM * KC;    // 8 KB
constexpr uint32_t kBSlice = IN * KC;    // 4 KB
constexpr uint32_t kIStage = S * (kASlice + kBSlice);   // 84 KB
constexpr int kIThreads = 192;
constexpr uint32_t kITmemCols = 512;     // S levels x IN columns = 448
constexpr size_t kISmem = kIStages * kIStage + 1024 + 256;

struct IBars {
  uint64_t full[kIStages], empty[kIStages], done;
  uint32_t tmem;
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

// K-major operand in the canonical 64-byte-swizzled layout: rows of 64 bytes,
// 8-row groups 512 bytes apart.
__device__ __forceinline__ uint64_t desc_sw64(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFF);
  d |= (uint64_t)1 << 16;             // leading byte offset (unused when K fits a row)
  d |= (uint64_t)(512 >> 4) << 32;    // stride byte offset: 8 rows x 64 B
  d |= (uint64_t)1 << 46;             // descriptor version (sm_100)
  d |= (uint64_t)4 << 61;             // SWIZZLE_64B
  return d;
}

__device__ __forceinline__ void mma_i8(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 64 consecutive 32-bit columns of this thread's TMEM lane (warp-wide), one
// load and its wait in one statement.
__device__ __forceinline__ void tmem_ld64_raw(uint32_t taddr, uint32_t (&r)[64]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
      : "r"(taddr)
      : "memory");
}

// D = s32, A and B signed 8-bit, both K-major, M = 128, N = 64.
constexpr uint32_t kIdescI8 = (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(IN >> 3) << 17) |
                              ((uint32_t)(IM >> 4) << 24);

// Slices of one fp64 matrix (rows x K, leading dimension ld, batch entries
// `stride` apart): slice t of row r (batch b) at out + t * plane +
// (b * rows + r) * kp, exponent at e[b * rows + r].  One warp per row.
__global__ void __launch_bounds__(256) slice_rows_kernel(const double* __restrict__ X,
                                                         int64_t rows, int64_t K, int64_t ld,
                                                         int64_t stride, int64_t kp,
                                                         int64_t plane,
                                                         int8_t* __restrict__ out,
                                                         int* __restrict__ e) {
  pdl_wait();
  const int lane = threadIdx.x & 31;
  const int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int b = blockIdx.y;
  if (r >= rows) return;
  const double* x = X + b * stride + r * ld;
  double m = 0.0;
  for (int64_t k = lane; k < K; k += 32) m = fmax(m, fabs(x[k]));
  for (int o = 16; o > 0; o >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, o));
  // 2^-ex m in [1/4, 1/2): the first slice rint(128 x) stays within [-64, 64]
  const int ex = m > 0.0 ? ilogb(m) + 2 : 0;
  const double scale = scalbn(1.0, -ex);   // exact power of two
  const int64_t row = b * rows + r;
  if (lane == 0) e[row] = ex;
  int8_t* o = out + row * kp;
  // eight consecutive values per lane and step (K and kp are multiples of 16).
  // Each scaled value is rounded once to an integer multiple of 2^(-7 S)
  // (|v| < 2^(7 S - 1)) and cut into balanced base-128 digits from the bottom:
  // digit t in [-64, 63] for t > 0, the top digit in [-64, 64].
  const double to_int = scalbn(scale, 7 * S);
  for (int64_t k = 8 * lane; k < kp; k += 256) {
    long long v[8];
    if (k + 8 <= K && ((reinterpret_cast<uintptr_t>(x + k) & 15) == 0)) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const double2 p2 = reinterpret_cast<const double2*>(x + k)[q];
        v[2 * q] = __double2ll_rn(p2.x * to_int);
        v[2 * q + 1] = __double2ll_rn(p2.y * to_int);
      }
    } else {
#pragma unroll
      for (int q = 0; q < 8; ++q) v[q] = k + q < K ? __double2ll_rn(x[k + q] * to_int) : 0ll;
    }
    uint32_t w[S][2];
#pragma unroll
    for (int t = 0; t < S; ++t) w[t][0] = w[t][1] = 0u;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      long long dgt = v[q];
#pragma unroll
      for (int t = S - 1; t >= 0; --t) {
        const long long a = t > 0 ? ((dgt + 64) & 127) - 64 : dgt;
        dgt = (dgt - a) >> 7;   // exact: dgt - a is a multiple of 128
        w[t][q >> 2] |= ((uint32_t)(int)a & 0xFFu) << (8 * (q & 3));
      }
    }
#pragma unroll
    for (int t = 0; t < S; ++t)
      *reinterpret_cast<uint2*>(o + t * plane + k) = make_uint2(w[t][0], w[t][1]);
  }
}

struct ITiles {
  int mt, nt, lower, ktri;
};

__global__ void __launch_bounds__(kIThreads, 1)
    dgemm_i8_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const int* __restrict__ eA, const int* __restrict__ eB, int M, int N, int K,
                    double alpha, double beta, double* __restrict__ C, int64_t ldc,
                    int64_t strideC, double* __restrict__ C2, int64_t ldc2, int64_t strideC2,
                    ITiles ts, int* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  IBars* sm = reinterpret_cast<IBars*>(ring + kIStages * kIStage);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tm = ts.ktri == 2 ? (int)gridDim.y - 1 - (int)blockIdx.y : (int)blockIdx.y;
  const int tn = blockIdx.x, bz = blockIdx.z;
  const int m0 = tm * IM, n0 = tn * IN;
  if (ts.lower && n0 > m0 + IM - 1) return;   // wholly above the diagonal
  int kbeg = 0, kend = K;
  if (ts.ktri == 1) kbeg = (m0 / KC) * KC;
  if (ts.ktri == 2) kend = (m0 + IM) < K ? (m0 + IM) : K;
  const int kc0 = kbeg / KC;
  const int nk = kend > kbeg ? (kend - kbeg + KC - 1) / KC : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kIStages; ++s) {
      mbar_init(&sm->full[s], 1);
      mbar_init(&sm->empty[s], 1);
    }
    mbar_init(&sm->done, 1);
    sm->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&sm->tmem, kITmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm->tmem;
  pdl_wait();

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ producer
    tma_prefetch(&tmA);
    tma_prefetch(&tmB);
    int issued = 0;
    for (int i = 0; i < nk; ++i) {
      const int s = i % kIStages;
      if (i >= kIStages && !mbar_wait(&sm->empty[s], ((i / kIStages) - 1) & 1)) {
        atomicExch(&sm->abort, 1);
        atomicCAS(status, 0, (int)NVFP4_ERR_TIMEOUT);
        break;
      }
      uint8_t* st = ring + s * kIStage;
      mbar_arrive_expect_tx(&sm->full[s], kIStage);
      tma_load_3d(st, &tmA, &sm->full[s], (kc0 + i) * KC, bz * M + m0, 0);
      tma_load_3d(st + S * kASlice, &tmB, &sm->full[s], (kc0 + i) * KC, bz * N + n0, 0);
      ++issued;
    }
    for (int i = issued - kIStages < 0 ? 0 : issued - kIStages; i < issued; ++i)
      mbar_wait(&sm->full[i % kIStages], (i / kIStages) & 1);
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    bool ok = true;
    for (int i = 0; ok && i < nk; ++i) {
      const int s = i % kIStages;
      if (!mbar_wait(&sm->full[s], (i / kIStages) & 1)) {
        atomicExch(&sm->abort, 1);
        atomicCAS(status, 0, (int)NVFP4_ERR_TIMEOUT);
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t a0 = smem_u32(ring + s * kIStage), b0 = a0 + S * kASlice;
#pragma unroll
      for (int l = 0; l < S; ++l) {
#pragma unroll
        for (int t = 0; t <= l; ++t) {
          const int u = l - t;
#pragma unroll
          for (int kk = 0; kk < KC / 32; ++kk)
            mma_i8(tmem + l * IN, desc_sw64(a0 + t * kASlice + 32 * kk),
                   desc_sw64(b0 + u * kBSlice + 32 * kk), kIdescI8,
                   (i > 0 || t > 0 || kk > 0) ? 1u : 0u);
        }
      }
      mma_commit(&sm->empty[s]);
    }
    mma_commit(&sm->done);
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue
    // (1) each thread sums the levels of its row in fp64 and stages the row,
    // scaled by 2^(e_m - 14), in shared memory (the ring is free once the
    // MMAs are done); (2) the four warps write C row by row and C2 column by
    // column, both coalesced, with the column factors 2^(e_n).
    constexpr int kPitch = IN + 1;
    double* tile = reinterpret_cast<double*>(ring);   // IM x kPitch
    const int q = warp & 3;
    const int r = q * 32 + lane;   // tile row = TMEM lane
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&sm->done, 0)) &&
                    !*reinterpret_cast<volatile int*>(&sm->abort);
    if (!ok && lane == 0) atomicCAS(status, 0, (int)NVFP4_ERR_TIMEOUT);
    if (ok) {
      tc_fence_after();
      double acc[IN];
#pragma unroll
      for (int j = 0; j < IN; ++j) acc[j] = 0.0;
      if (nk > 0) {
        // levels from the smallest weight up: acc = sum_l 2^(-7 l) v_l
#pragma unroll 1
        for (int l = S - 1; l >= 0; --l) {
          const uint32_t ta = tmem + ((uint32_t)(q * 32) << 16) + l * IN;
          uint32_t v[IN];
          tmem_ld64_raw(ta, v);
#pragma unroll
          for (int j = 0; j < IN; ++j)
            acc[j] = fma(acc[j], 0.0078125 /* 2^-7 */, (double)(int)v[j]);
        }
      }
      // level 0 weighs 2^-14 relative to 2^(e_m + e_n)
      const int m = m0 + r;
      const double fm = m < M ? scalbn(alpha, eA[bz * M + m] - 14) : 0.0;
#pragma unroll
      for (int j = 0; j < IN; ++j) tile[r * kPitch + j] = acc[j] * fm;
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (ok) {
      double fn[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int n = n0 + lane + 32 * h;
        fn[h] = n < N ? scalbn(1.0, eB[bz * N + n]) : 0.0;
      }
      double* __restrict__ Cb = C + bz * strideC;
      // the warp's 32 rows: all their C loads are issued before any store
      double old[IM / 4][2];
#pragma unroll
      for (int i = 0; i < IM / 4; ++i) {
        const int m = m0 + q + 4 * i;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int n = n0 + lane + 32 * h;
          old[i][h] = (beta != 0.0 && m < M && n < N) ? Cb[(int64_t)m * ldc + n] : 0.0;
        }
      }
#pragma unroll
      for (int i = 0; i < IM / 4; ++i) {
        const int m = m0 + q + 4 * i;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int n = n0 + lane + 32 * h;
          if (m < M && n < N) {
            double xv = tile[(q + 4 * i) * kPitch + lane + 32 * h] * fn[h];
            if (beta != 0.0) xv = fma(beta, old[i][h], xv);
            Cb[(int64_t)m * ldc + n] = xv;
          }
        }
      }
      if (C2) {
        double* C2b = C2 + bz * strideC2;
        for (int j = q; j < IN; j += 4) {
          const int n = n0 + j;
          if (n >= N) break;
          const double f = scalbn(1.0, eB[bz * N + n]);
#pragma unroll
          for (int h = 0; h < IM / 32; ++h) {
            const int m = m0 + lane + 32 * h;
            if (m < M) C2b[(int64_t)n * ldc2 + m] = tile[(lane + 32 * h) * kPitch + j] * f;
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kITmemCols);
  }
}

// 3-D map of the slices: (K bytes, batch * rows, S), box {64, box_rows, S}.
bool encode_slices(CUtensorMap* map, const int8_t* base, int64_t K, int64_t total_rows,
                   int64_t kp, int64_t plane, int box_rows) {
  const uint64_t dims[3] = {(uint64_t)K, (uint64_t)total_rows, (uint64_t)S};
  const uint64_t strides[2] = {(uint64_t)kp, (uint64_t)plane};
  const uint32_t box[3] = {(uint32_t)KC, (uint32_t)box_rows, (uint32_t)S};
  return encode_tmap_nd(map, base, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, dims, strides, box,
                        CU_TENSOR_MAP_SWIZZLE_64B);
}

nvfp4_status slice(const double* X, int64_t rows, int64_t K, int64_t ld, int64_t stride,
                   int batch, int8_t* out, int* e, int64_t kp, int64_t plane, cudaStream_t st) {
  const dim3 grid((unsigned)((rows + 7) / 8), (unsigned)batch);
  NVFP4_CUDA_TRY(launch_chained(slice_rows_kernel, grid, dim3(256), 0, st, X, rows, K, ld, stride,
                                kp, plane, out, e));
  count_launches(1);
  return NVFP4_OK;
}

}  // namespace

size_t dgemm_i8_scratch_bytes(int64_t M, int64_t N, int64_t K, int batch) {
  const int64_t kp = (K + 15) / 16 * 16;
  return align256((size_t)S * batch * M * kp) + align256((size_t)S * batch * N * kp) +
         align256(sizeof(int) * batch * (M + N));
}

nvfp4_status dgemm_i8(int M, int N, int K, double alpha, const double* P, int64_t ldp,
                      int64_t strideP, const double* Q, int64_t ldq, int64_t strideQ,
                      double beta, double* C, int64_t ldc, int64_t strideC, double* C2,
                      int64_t ldc2, int64_t strideC2, int batch, int lower, int ktri,
                      void* scratch, size_t scratch_bytes, int* status, cudaStream_t st) {
  if (M <= 0 || N <= 0 || batch <= 0) return NVFP4_OK;
  // K < 2^16 keeps a level's int32 sum exact: S pairs x K x 64 x 64 < 2^31
  if ((C2 && beta != 0.0) || (lower && M != N) || ktri < 0 || ktri > 2 || !status || K <= 0 ||
      K >= (1 << 16) || (K % 16) != 0 || batch > 65535)
    return NVFP4_ERR_INVALID_ARG;
  if (scratch_bytes < dgemm_i8_scratch_bytes(M, N, K, batch)) return NVFP4_ERR_WORKSPACE;
  ProfileScope ps(kPhaseFactorGemm, st);
  {
    double f = 2.0 * M * N * K;
    if (lower) f = 2.0 * ((double)N * (N + 1) / 2) * K;
    if (ktri != 0 && M <= K)
      f = 2.0 * N * ((double)M * (M + 1) / 2 + (double)M * (K - M) * (ktri == 1));
    add_phase_work(f * batch);
  }
  const int64_t kp = (K + 15) / 16 * 16;
  const int64_t planeA = (int64_t)batch * M * kp, planeB = (int64_t)batch * N * kp;
  char* p = static_cast<char*>(scratch);
  int8_t* A = reinterpret_cast<int8_t*>(p);
  p += align256((size_t)S * planeA);
  int8_t* Bs = reinterpret_cast<int8_t*>(p);
  p += align256((size_t)S * planeB);
  int* eA = reinterpret_cast<int*>(p);
  int* eB = eA + (int64_t)batch * M;
  // P and Q are the same matrix in a symmetric update: slice it once
  const bool same = (P == Q && ldp == ldq && strideP == strideQ && M == N);
  nvfp4_status s = slice(P, M, K, ldp, strideP, batch, A, eA, kp, planeA, st);
  if (s != NVFP4_OK) return s;
  const int8_t* Bsrc = same ? A : Bs;
  const int* eBsrc = same ? eA : eB;
  if (!same) {
    s = slice(Q, N, K, ldq, strideQ, batch, Bs, eB, kp, planeB, st);
    if (s != NVFP4_OK) return s;
  }
  CUtensorMap ma, mb;
  if (!encode_slices(&ma, A, K, (int64_t)batch * M, kp, planeA, IM) ||
      !encode_slices(&mb, Bsrc, K, (int64_t)batch * N, kp, same ? planeA : planeB, IN))
    return NVFP4_ERR_CUDA;
  const ITiles ts{(M + IM - 1) / IM, (N + IN - 1) / IN, lower, ktri};
  const dim3 grid((unsigned)ts.nt, (unsigned)ts.mt, (unsigned)batch);
  if (grid.y > 65535) return NVFP4_ERR_SHAPE;
  NVFP4_CUDA_TRY(cudaFuncSetAttribute(dgemm_i8_kernel,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kISmem));
  NVFP4_CUDA_TRY(launch_chained(dgemm_i8_kernel, grid, dim3(kIThreads), kISmem, st, ma, mb, eA,
                                eBsrc, M, N, K, alpha, beta, C, ldc, strideC, C2, ldc2, strideC2,
                                ts, status));
  count_launches(1);
  return NVFP4_OK;
}

}  // namespace nvfp4
