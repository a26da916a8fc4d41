// a1 on the 5th-generation tensor cores: H (+)= X^T X for bf16 calibration
// activations, fp32 accumulation in tensor memory.
//
// "Replay the Curvature" (arXiv 2609.36654v1), Abstract: the second-order
// state of a layer is accumulated from its calibration activations; here
// H = sum over tokens t of x_t x_t^T, no 1/N factor.
//
// X is tokens x d, row-major, so for C[i][j] = sum_t X[t][i] X[t][j] both MMA
// operands are "MN-major": a TMA box of 64 channels (128 B) x 64 tokens lands
// in shared memory as 64 rows of 128 B with the 128-byte swizzle, which is the
// canonical MN-major layout tcgen05 reads directly -- no transpose pass.
//
// Persistent, warp-specialised CTA (one per SM):
//   warp 0      TMA producer: 4-stage ring of (128 + 256 channels) x 64 tokens
//   warp 1      MMA issuer: tcgen05.mma kind::f16, M=128 N=256 K=16, into one
//               of two 256-column TMEM accumulators (double buffered)
//   warps 2-9   epilogue: each thread owns one accumulator row (TMEM lane)
//               and 128 of its columns
// Accuracy: the tensor cores' fp32 accumulation drops low bits (measured on
// the 4096-token workload: a 1.3e-5 relative, one-sided error in H when all
// tokens go into one accumulator).  So each accumulator only sums a chunk of
// 256 tokens; the epilogue adds the chunk sums into fp32 registers with
// round-to-nearest adds (H within 4e-7 relative Frobenius of the exact sum on
// 16384 lognormal-scaled tokens; 128-token chunks give 2.4e-7 but drain the
// accumulators twice as often and are 11% slower), then stores the upper
// part H[i][j>=i] and its mirror H[j][i].  Only 128x256 tiles that touch the
// upper triangle are computed (J >= I/2); each H element is produced by
// exactly one tile.
#include <cuda.h>

#include "common.cuh"
#include "sm100.cuh"

namespace nvfp4 {
namespace {

using namespace sm100;

constexpr int BM = 128;                       // tile rows (channel i)
constexpr int BN = 256;                       // tile columns (channel j)
constexpr int BK = 64;                        // tokens per stage
constexpr int kStages = 4;
constexpr int kBox = 64;                      // channels per TMA box (128 B)
constexpr uint32_t kRowBytes = 128;           // one token row of a box
constexpr uint32_t kBoxBytes = BK * kRowBytes;  // 8 KB
constexpr uint32_t kABytes = BM / kBox * kBoxBytes;
constexpr uint32_t kBBytes = BN / kBox * kBoxBytes;
constexpr uint32_t kStageBytes = kABytes + kBBytes;  // 48 KB
constexpr int kThreads = 320;
constexpr int kChunkStages = 4;              // 256 tokens per accumulator
constexpr uint32_t kTmemCols = 2 * BN;
constexpr size_t kSmem = kStages * kStageBytes + 1024 + 256;

__device__ int g_hessian_status;

// Up to kHessGroup problems of the same dimension d in one launch: their
// token maps, outputs and token counts (a kernel parameter, 18 KB).  Tile t
// of the launch is band tile t % per of problem t / per; the host orders the
// problems by decreasing token count, so the longest tiles come first.
constexpr int kHessGroup = 128;
struct HessGroup {
  CUtensorMap map[kHessGroup];
  float* H[kHessGroup];
  int n_tok[kHessGroup];
  int P;
};

// 128 x 256 tiles (I, J) with J >= I / 2 (I.e. I <= 2 J + 1), in groups of
// kGroupRows tile rows: group by group, inside a group column by column, and
// inside a column row by row.  The CTAs of one wave then hold a few A slabs
// (the group's rows) and a short run of B slabs, which the L2 keeps for all
// of them while they walk the tokens at the same pace; a row-major order
// would read every B slab of the layer from DRAM once per wave.
constexpr int kGroupRows = 16;
constexpr int kMaxBandGroups = 64;          // d up to 64 * 16 * 128 = 131072
struct BandTiles {
  int nI, nJ, n_groups, per;
  int start[kMaxBandGroups + 1];             // first tile of each group
  // tile rows of group g present in column J
  __host__ __device__ int col_rows(int g, int J) const {
    const int i0 = g * kGroupRows;
    int i1 = i0 + kGroupRows - 1;
    if (i1 > nI - 1) i1 = nI - 1;
    if (i1 > 2 * J + 1) i1 = 2 * J + 1;
    return i1 >= i0 ? i1 - i0 + 1 : 0;
  }
  __host__ bool init(int64_t d) {
    nI = (int)((d + BM - 1) / BM);
    nJ = (int)((d + BN - 1) / BN);
    n_groups = (nI + kGroupRows - 1) / kGroupRows;
    if (n_groups > kMaxBandGroups) return false;
    per = 0;
    for (int g = 0; g < n_groups; ++g) {
      start[g] = per;
      for (int J = (g * kGroupRows) >> 1; J < nJ; ++J) per += col_rows(g, J);
    }
    start[n_groups] = per;
    return true;
  }
  // the first columns of a group are short (rows I <= 2 J + 1); the rest
  // hold all of the group's rows
  __device__ void get(int t, int& I, int& J) const {
    int g = 0;
    while (t >= start[g + 1]) ++g;
    t -= start[g];
    J = (g * kGroupRows) >> 1;
    const int full = col_rows(g, nJ - 1);
    int c = col_rows(g, J);
    while (c < full && t >= c) {
      t -= c;
      c = col_rows(g, ++J);
    }
    J += t / full;
    I = g * kGroupRows + t % full;
  }
};

struct Smem {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  uint64_t accfull[2];
  uint64_t accempty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ void give_up(Smem* sm) {
  atomicExch(&sm->abort, 1);
  atomicCAS(&g_hessian_status, 0, (int)NVFP4_ERR_TIMEOUT);
}

__device__ __forceinline__ bool aborted(Smem* sm) {
  return *reinterpret_cast<volatile int*>(&sm->abort) != 0;
}

#ifdef NVFP4_DEBUG
// debug build: the band tile a loop is about to take lies inside H
__device__ bool band_tile_in_bounds(const BandTiles& band, int per, int P, int t) {
  const int pb = t / per;
  int I, J;
  band.get(t - pb * per, I, J);
  return NVFP4_DCHECK(pb < P && I >= 0 && I < band.nI && J < band.nJ && J >= (I >> 1),
                      &g_hessian_status);
}
#define NVFP4_TILE_CHECK(t) \
  if (!band_tile_in_bounds(band, per, grp.P, (t))) continue;
#else
#define NVFP4_TILE_CHECK(t)
#endif

__global__ void __launch_bounds__(kThreads, 1)
    hessian_tc_kernel(const __grid_constant__ HessGroup grp, int d, int beta, BandTiles band) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* tiles = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~uintptr_t(1023));
  Smem* sm = reinterpret_cast<Smem*>(tiles + kStages * kStageBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per = band.per;
  const int n_tiles = per * grp.P;
  auto nk_of = [&](int pb) { return (grp.n_tok[pb] + BK - 1) / BK; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm->full[s], 1);
      mbar_init(&sm->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&sm->accfull[a], 1);
      mbar_init(&sm->accempty[a], 256);
    }
    mbar_init(&sm->drain, 1);
    sm->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) tmem_alloc(&sm->tmem_base, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm->tmem_base;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ producer
    int s = 0;
    uint32_t ph = 0;
    int issued = 0;
    for (int t = blockIdx.x; t < n_tiles && !aborted(sm); t += gridDim.x) {
      NVFP4_TILE_CHECK(t)
      const int pb = t / per;
      const CUtensorMap* tmX = &grp.map[pb];
      const int nk = nk_of(pb);
      int I, J;
      band.get(t - pb * per, I, J);
      for (int kb = 0; kb < nk; ++kb) {
        if (!mbar_wait(&sm->empty[s], ph ^ 1)) {
          give_up(sm);
          break;
        }
        mbar_arrive_expect_tx(&sm->full[s], kStageBytes);
        uint8_t* a = tiles + s * kStageBytes;
        uint8_t* b = a + kABytes;
        for (int x = 0; x < BM / kBox; ++x)
          tma_load_2d(a + x * kBoxBytes, tmX, &sm->full[s], I * BM + x * kBox, kb * BK);
        for (int x = 0; x < BN / kBox; ++x)
          tma_load_2d(b + x * kBoxBytes, tmX, &sm->full[s], J * BN + x * kBox, kb * BK);
        ++issued;
        if (++s == kStages) {
          s = 0;
          ph ^= 1;
        }
      }
    }
    if (aborted(sm)) {
      // let the copies already issued land before the CTA exits
      for (int k = 0; k < kStages && k < issued; ++k) {
        if (--s < 0) {
          s = kStages - 1;
          ph ^= 1;
        }
        mbar_wait_drain(&sm->full[s], ph);
      }
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc = instr_desc(1 /*bf16*/, 1, 1, BM, BN);
    int s = 0;
    uint32_t ph = 0;
    int g = 0;   // chunks issued by this CTA
    bool ok = true;
    for (int t = blockIdx.x; ok && t < n_tiles && !aborted(sm); t += gridDim.x) {
      NVFP4_TILE_CHECK(t)
      const int nk = nk_of(t / per);
      for (int kb0 = 0; ok && kb0 < nk; kb0 += kChunkStages, ++g) {
        const int acc = g & 1;
        if (!mbar_wait(&sm->accempty[acc], ((g >> 1) & 1) ^ 1)) {
          give_up(sm);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t dt = tmem + acc * BN;
        const int kb1 = kb0 + kChunkStages < nk ? kb0 + kChunkStages : nk;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&sm->full[s], ph)) {
            give_up(sm);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(tiles + s * kStageBytes);
          const uint32_t b0 = a0 + kABytes;
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t ad =
                smem_desc_sw128(a0 + k * 16 * kRowBytes, kBoxBytes, 8 * kRowBytes);
            const uint64_t bd =
                smem_desc_sw128(b0 + k * 16 * kRowBytes, kBoxBytes, 8 * kRowBytes);
            mma_f16(dt, ad, bd, idesc, (kb != kb0) | (k != 0));
          }
          mma_commit(&sm->empty[s]);
          if (++s == kStages) {
            s = 0;
            ph ^= 1;
          }
        }
        if (ok) mma_commit(&sm->accfull[acc]);
      }
    }
    // every MMA issued above completes before TMEM is released
    mma_commit(&sm->drain);
    mbar_wait_drain(&sm->drain, 0);
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;            // TMEM lane quarter this warp may read
    const int r = q * 32 + lane;       // accumulator row = TMEM lane
    const int half = (warp - 2) >> 2;  // which 128 of the tile's 256 columns
    int g = 0;
    // loop exits and wait outcomes are made warp-uniform: tcgen05.ld is a
    // warp-collective instruction
    bool ok = true;
    for (int t = blockIdx.x; ok && t < n_tiles && !__any_sync(0xffffffffu, aborted(sm));
         t += gridDim.x) {
      NVFP4_TILE_CHECK(t)
      const int pb = t / per;
      const int nk = nk_of(pb);
      float* __restrict__ H = grp.H[pb];
      float sum[128];
#pragma unroll
      for (int k = 0; k < 128; ++k) sum[k] = 0.f;
      for (int kb0 = 0; kb0 < nk; kb0 += kChunkStages, ++g) {
        const int acc = g & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(&sm->accfull[acc], (g >> 1) & 1))) {
          give_up(sm);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t ta = tmem + ((uint32_t)(q * 32) << 16) + acc * BN + half * 128;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float v[32];
          tmem_ld32(ta + c * 32, v);
#pragma unroll
          for (int k = 0; k < 32; ++k) sum[c * 32 + k] = __fadd_rn(sum[c * 32 + k], v[k]);
        }
        tc_fence_before();
        mbar_arrive(&sm->accempty[acc]);
      }
      if (!ok) break;
      int I, J;
      band.get(t - pb * per, I, J);
      const int i = I * BM + r;
      const bool row_ok = i < d;
      float* hrow = H + (size_t)i * d;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        float* v = sum + c * 32;
        const int j0 = J * BN + half * 128 + c * 32;
        if (row_ok && j0 >= i && j0 + 32 <= d) {   // whole chunk in the upper part
          float4* dst = reinterpret_cast<float4*>(hrow + j0);
#pragma unroll
          for (int k = 0; k < 8; ++k) {
            float4 x = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
            if (beta) {
              const float4 o = dst[k];
              x.x += o.x; x.y += o.y; x.z += o.z; x.w += o.w;
              v[4 * k] = x.x; v[4 * k + 1] = x.y; v[4 * k + 2] = x.z; v[4 * k + 3] = x.w;
            }
            dst[k] = x;
          }
        } else if (row_ok) {
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            const int j = j0 + k;
            if (j >= i && j < d) {
              float x = v[k];
              if (beta) x += hrow[j];
              v[k] = x;
              hrow[j] = x;
            }
          }
        }
        // mirror: for a fixed k the warp writes 32 consecutive floats
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          const int j = j0 + k;
          if (row_ok && j > i && j < d) H[(size_t)j * d + i] = v[k];
        }
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

bool hessian_tc_supported(const float* H, const void* X, nvfp4_dtype xt, int64_t n_tok,
                          int64_t d) {
  return xt == NVFP4_BF16 && d >= 256 && n_tok >= BK && n_tok < (int64_t(1) << 31) &&
         (reinterpret_cast<uintptr_t>(X) & 15) == 0 && (reinterpret_cast<uintptr_t>(H) & 15) == 0;
}

// H_p (+)= X_p^T X_p for P problems of dimension d (bf16 tokens, each
// hessian_tc_supported), up to kHessGroup per launch.
nvfp4_status launch_hessian_tc_group(int P, float* const* H, const void* const* X,
                                     const int64_t* n_tok, int64_t d, int beta,
                                     cudaStream_t st) {
  // heaviest problems first
  int order[kMaxGroup];
  if (P < 1 || P > kMaxGroup) return NVFP4_ERR_INVALID_ARG;
  for (int i = 0; i < P; ++i) order[i] = i;
  for (int i = 1; i < P; ++i)   // stable insertion sort by decreasing n_tok
    for (int j = i; j > 0 && n_tok[order[j]] > n_tok[order[j - 1]]; --j) {
      const int t = order[j];
      order[j] = order[j - 1];
      order[j - 1] = t;
    }
  BandTiles band;
  if (!band.init(d)) return NVFP4_ERR_SHAPE;
  const int per = band.per;
  const int sms = num_sms();
  NVFP4_CUDA_TRY(cudaFuncSetAttribute(hessian_tc_kernel,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem));
  static thread_local HessGroup grp;   // 18 KB: kept off the stack
  for (int c0 = 0; c0 < P; c0 += kHessGroup) {
    const int n = (P - c0) < kHessGroup ? (P - c0) : kHessGroup;
    grp.P = n;
    for (int i = 0; i < n; ++i) {
      const int q = order[c0 + i];
      const uint64_t dims[2] = {(uint64_t)d, (uint64_t)n_tok[q]};
      const uint64_t strides[1] = {(uint64_t)d * 2};
      const uint32_t box[2] = {(uint32_t)kBox, (uint32_t)BK};
      if (!encode_tmap_2d(&grp.map[i], X[q], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, dims, strides,
                          box, CU_TENSOR_MAP_SWIZZLE_128B))
        return NVFP4_ERR_CUDA;
      grp.H[i] = H[q];
      grp.n_tok[i] = (int)n_tok[q];
    }
    const int n_tiles = per * n;
    hessian_tc_kernel<<<n_tiles < sms ? n_tiles : sms, kThreads, kSmem, st>>>(grp, (int)d,
                                                                              beta, band);
    NVFP4_LAUNCH_CHECK();
    count_launches(1);
  }
  return NVFP4_OK;
}

nvfp4_status launch_hessian_tc(float* H, const void* X, int64_t n_tok, int64_t d, int beta,
                               cudaStream_t st) {
  return launch_hessian_tc_group(1, &H, &X, &n_tok, d, beta, st);
}

int hessian_tc_take_status(cudaStream_t st) {
  int v = 0, zero = 0;
  if (cudaMemcpyFromSymbolAsync(&v, g_hessian_status, sizeof(int), 0, cudaMemcpyDeviceToHost,
                                st) != cudaSuccess ||
      cudaMemcpyToSymbolAsync(g_hessian_status, &zero, sizeof(int), 0, cudaMemcpyHostToDevice,
                              st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess) {
    cudaGetLastError();
    return (int)NVFP4_ERR_CUDA;
  }
  return v;
}

}  // namespace nvfp4
