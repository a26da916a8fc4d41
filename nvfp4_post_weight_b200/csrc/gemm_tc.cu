// fp32 GEMM on the tensor cores, 3xTF32:  C = beta C + alpha P Q^T
// (P: M x K, Q: N x K, both row-major, i.e. K-contiguous; C: M x N row-major),
// optionally batched (third TMA dimension) and optionally restricted to the
// tiles on or below the diagonal.  Used by the factorisation (Cholesky
// trailing update, triangular-inverse doubling) and the layer error.
//
// Pipeline per 128 x 128 output tile, K in chunks of 32 (128 B of fp32):
//   warp 0      TMA producer: raw fp32 tiles of P and Q into a 3-stage ring,
//               128-byte swizzled (the canonical K-major layout)
//   warps 2-5   split: each element x becomes hi = tf32(x) (rounded in place)
//               and lo = x - hi (written to a twin buffer at the same offset,
//               so the swizzle is kept); then fence.proxy.async.  When the
//               caller gives the operands already split (hi and lo arrays,
//               gemm_nt_tc_split), the producer loads all four tiles and
//               these warps stay idle: an operand that many tiles read is
//               then split once instead of once per tile, and the shared
//               memory traffic of the split is gone.
//   warp 1      MMA issuer: per K step of 8, main += Ph Qh and
//               cross += Ph Ql + Pl Qh (kind::tf32, M=128): Qh and Ql lie
//               next to each other in the stage and the cross accumulator
//               next to main in TMEM, so Ph [Qh; Ql] is one N=256 MMA (Ph is
//               read once for both), then Pl Qh an N=128 one
//   warps 6-13  epilogue (two warps per TMEM lane quarter, 64 columns each):
//               every 128 K values the two accumulators are read out of TMEM
//               and added, with round-to-nearest fp32 adds, into register sums
//               (the tensor cores' own fp32
//               accumulation drops low bits, so it is only trusted over short
//               runs); at the end C is written.
#include <cuda.h>

#include "common.cuh"
#include "sm100.cuh"

namespace nvfp4 {
namespace {

using namespace sm100;

constexpr int GM = 128, GN = 128, GK = 32;
constexpr int kStages = 3;
constexpr int kChunkSteps = 4;                     // K = 128 per accumulator
constexpr uint32_t kTile = GM * GK * 4;            // 16 KB (P or Q, raw/hi or lo)
constexpr uint32_t kStageBytes = 4 * kTile;        // Ph, Pl, Qh, Ql
constexpr int kThreads = 448;                      // 14 warps
constexpr int kEpiCols = GN / 2;                   // columns per epilogue thread
constexpr uint32_t kBufCols = 2 * GN;              // main + cross
constexpr uint32_t kTmemCols = 512;
constexpr int kEpiPitch = 33;                      // per-warp 32 x 33 transpose buffer
constexpr size_t kEpiBytes = 8 * 32 * kEpiPitch * sizeof(float);
constexpr size_t kSmem = kStages * kStageBytes + kEpiBytes + 1024 + 256;

struct Smem {
  uint64_t full[kStages], ready[kStages], empty[kStages];
  uint64_t acc_full[2], acc_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ void give_up(Smem* sm, int* status) {
  atomicExch(&sm->abort, 1);
  atomicCAS(status, 0, (int)NVFP4_ERR_TIMEOUT);
}
__device__ __forceinline__ bool aborted(Smem* sm) {
  return *reinterpret_cast<volatile int*>(&sm->abort) != 0;
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar,
                                            int c0, int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(map), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// Output tiles.  A full result goes in groups of kGroupTiles tile rows: group
// by group, inside a group column by column, so that the CTAs of a wave read
// a few A row slabs and a short run of B slabs, which stay in L2 while they
// walk K at the same pace (row-major order re-reads every B slab of a wide
// output from DRAM once per wave).  A lower result (the Gram product) is
// taken row-major over the tiles on or below the diagonal.
constexpr int kGroupTiles = 16;
struct TileSpace {
  int mt, nt, batch, lower;
  __device__ int per() const { return lower ? mt * (mt + 1) / 2 : mt * nt; }
  __device__ int count() const { return per() * batch; }
  __device__ void get(int t, int& tm, int& tn, int& b) const {
    const int p = per();
    b = t / p;
    t -= b * p;
    if (lower) {
      tm = 0;
      while (t > tm) {
        t -= tm + 1;
        ++tm;
      }
      tn = t;
      return;
    }
    constexpr int G = kGroupTiles;
    const int g = t / (G * nt);
    t -= g * G * nt;
    const int r = (mt - g * G) < G ? (mt - g * G) : G;
    tn = t / r;
    tm = g * G + t % r;
  }
};

#ifdef NVFP4_DEBUG
// debug build: the tile a loop is about to take lies inside the output
__device__ bool tile_in_bounds(const TileSpace& ts, int t, int* status) {
  int tm, tn, b;
  ts.get(t, tm, tn, b);
  return NVFP4_DCHECK(b >= 0 && b < ts.batch && tm >= 0 && tm < ts.mt && tn >= 0 &&
                          tn < ts.nt && (!ts.lower || tn <= tm),
                      status);
}
#define NVFP4_TILE_CHECK(t) \
  if (!tile_in_bounds(ts, (t), status)) continue;
#else
#define NVFP4_TILE_CHECK(t)
#endif

__global__ void __launch_bounds__(kThreads, 1)
    gemm_nt_tc_kernel(const __grid_constant__ CUtensorMap tmP,
                      const __grid_constant__ CUtensorMap tmQ,
                      const __grid_constant__ CUtensorMap tmPl,
                      const __grid_constant__ CUtensorMap tmQl, int presplit, float* __restrict__ C,
                      int64_t ldc, int64_t strideC, float* __restrict__ C2, int64_t ldc2,
                      int64_t strideC2, int M, int N, int K, float alpha, float beta,
                      TileSpace ts, int* status, double* __restrict__ C64) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* ring = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  float* epi = reinterpret_cast<float*>(ring + kStages * kStageBytes);
  Smem* sm = reinterpret_cast<Smem*>(ring + kStages * kStageBytes + kEpiBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = ts.count();
  const int nk = (K + GK - 1) / GK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm->full[s], 1);
      mbar_init(&sm->ready[s], 128);
      mbar_init(&sm->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&sm->acc_full[a], 1);
      mbar_init(&sm->acc_empty[a], 256);
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
    tma_prefetch(&tmP);
    tma_prefetch(&tmQ);
    if (presplit) {
      tma_prefetch(&tmPl);
      tma_prefetch(&tmQl);
    }
    int s = 0, issued = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < n_tiles && !aborted(sm); t += gridDim.x) {
      NVFP4_TILE_CHECK(t)
      int tm, tn, b;
      ts.get(t, tm, tn, b);
      for (int kb = 0; kb < nk; ++kb) {
        if (!mbar_wait(&sm->empty[s], ph ^ 1)) {
          give_up(sm, status);
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&sm->full[s], (presplit ? 4 : 2) * kTile);
        // stage: Ph, Pl, Qh, Ql (Qh and Ql adjacent: one 256-row B operand)
        uint8_t* st = ring + s * kStageBytes;
        tma_load_3d(st, &tmP, &sm->full[s], kb * GK, tm * GM, b);
        tma_load_3d(st + 2 * kTile, &tmQ, &sm->full[s], kb * GK, tn * GN, b);
        if (presplit) {
          tma_load_3d(st + kTile, &tmPl, &sm->full[s], kb * GK, tm * GM, b);
          tma_load_3d(st + 3 * kTile, &tmQl, &sm->full[s], kb * GK, tn * GN, b);
        }
        ++issued;
        if (++s == kStages) {
          s = 0;
          ph ^= 1;
        }
      }
    }
    if (aborted(sm)) {
      for (int k = 0; k < kStages && k < issued; ++k) {
        if (--s < 0) {
          s = kStages - 1;
          ph ^= 1;
        }
        mbar_wait_drain(&sm->full[s], ph);
      }
    }
  } else if (warp >= 2 && warp < 6 && !presplit) {
    // ------------------------------------------------------------ split
    const int tid = threadIdx.x - 64;   // 0..127
    int s = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < n_tiles && !aborted(sm); t += gridDim.x) {
      NVFP4_TILE_CHECK(t)
      for (int kb = 0; kb < nk; ++kb) {
        if (!mbar_wait(&sm->full[s], ph)) {
          give_up(sm, status);
          ok = false;
          break;
        }
        // raw P at Ph and raw Q at Qh; each tile's lo part goes kTile after it
        uint8_t* stg = ring + s * kStageBytes;
#pragma unroll 4
        for (int e = tid; e < (int)(2 * kTile / 16); e += 128) {
          const int i = e & (int)(kTile / 16 - 1);
          float4* hi = reinterpret_cast<float4*>(stg + (e >= (int)(kTile / 16) ? 2 * kTile : 0));
          float4* lo = reinterpret_cast<float4*>(reinterpret_cast<uint8_t*>(hi) + kTile);
          float4 x = hi[i];
          float4 h = make_float4(tf32_rn(x.x), tf32_rn(x.y), tf32_rn(x.z),
                                 tf32_rn(x.w));
          hi[i] = h;
          lo[i] = make_float4(x.x - h.x, x.y - h.y, x.z - h.z, x.w - h.w);
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        mbar_arrive(&sm->ready[s]);
        if (++s == kStages) {
          s = 0;
          ph ^= 1;
        }
      }
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc = instr_desc(2 /*tf32*/, 0, 0, GM, GN);
    constexpr uint32_t idesc2 = instr_desc(2 /*tf32*/, 0, 0, GM, 2 * GN);
    int s = 0, g = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < n_tiles && !aborted(sm); t += gridDim.x) {
      NVFP4_TILE_CHECK(t)
      for (int kb0 = 0; ok && kb0 < nk; kb0 += kChunkSteps, ++g) {
        const int buf = g & 1;
        if (!mbar_wait(&sm->acc_empty[buf], ((g >> 1) & 1) ^ 1)) {
          give_up(sm, status);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t mainc = tmem + buf * kBufCols, cross = mainc + GN;
        const int kb1 = kb0 + kChunkSteps < nk ? kb0 + kChunkSteps : nk;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(presplit ? &sm->full[s] : &sm->ready[s], ph)) {
            give_up(sm, status);
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t ph_ = smem_u32(ring + s * kStageBytes);
          const uint32_t pl = ph_ + kTile, qh = ph_ + 2 * kTile;
#pragma unroll
          for (int k = 0; k < GK / 8; ++k) {
            const uint64_t dph = smem_desc_sw128(ph_ + 32 * k, 16, 1024);
            const uint64_t dpl = smem_desc_sw128(pl + 32 * k, 16, 1024);
            const uint64_t dq = smem_desc_sw128(qh + 32 * k, 16, 1024);   // Qh then Ql rows
            const uint32_t first = (kb != kb0) | (k != 0);
            // Ph [Qh; Ql]^T: main += Ph Qh^T in columns 0..127 and cross +=
            // Ph Ql^T in 128..255 (the cross accumulator sits right after
            // main), one operand read of Ph; then cross += Pl Qh^T
            mma_tf32(mainc, dph, dq, idesc2, first);
            mma_tf32(cross, dpl, dq, idesc, 1);
          }
          mma_commit(&sm->empty[s]);
          if (++s == kStages) {
            s = 0;
            ph ^= 1;
          }
        }
        if (ok) mma_commit(&sm->acc_full[buf]);
      }
    }
    mma_commit(&sm->drain);
    mbar_wait_drain(&sm->drain, 0);
  } else if (warp >= 6) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const int h = (warp - 6) >> 2;      // column half of the tile
    int g = 0;
    bool ok = true;
    for (int t = blockIdx.x; ok && t < n_tiles && !__any_sync(0xffffffffu, aborted(sm));
         t += gridDim.x) {
      NVFP4_TILE_CHECK(t)
      float sum[kEpiCols];
#pragma unroll
      for (int k = 0; k < kEpiCols; ++k) sum[k] = 0.f;
      for (int kb0 = 0; kb0 < nk; kb0 += kChunkSteps, ++g) {
        const int buf = g & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(&sm->acc_full[buf], (g >> 1) & 1))) {
          give_up(sm, status);
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t ta =
            tmem + ((uint32_t)(q * 32) << 16) + buf * kBufCols + h * kEpiCols;
#pragma unroll
        for (int c = 0; c < kEpiCols / 32; ++c) {
          float v[32];
          tmem_ld32(ta + c * 32, v);
#pragma unroll
          for (int k = 0; k < 32; ++k) sum[c * 32 + k] = __fadd_rn(sum[c * 32 + k], v[k]);
          tmem_ld32(ta + GN + c * 32, v);
#pragma unroll
          for (int k = 0; k < 32; ++k) sum[c * 32 + k] = __fadd_rn(sum[c * 32 + k], v[k]);
        }
        tc_fence_before();
        mbar_arrive(&sm->acc_empty[buf]);
      }
      if (!ok) break;
      int tm, tn, b;
      ts.get(t, tm, tn, b);
      // C: through a per-warp transpose in shared memory, so that each store
      // instruction writes 32 consecutive floats of one row (and the beta
      // loads are issued together); C2 (= C^T, beta == 0) straight from the
      // row-per-thread layout, which is already coalesced for the transpose.
      float* wb = epi + (warp - 6) * 32 * kEpiPitch;
      float* Cb = C + b * strideC;
      const int row0 = tm * GM + q * 32;
#pragma unroll
      for (int c = 0; c < kEpiCols / 32; ++c) {
#pragma unroll
        for (int k = 0; k < 32; ++k) wb[lane * kEpiPitch + k] = sum[c * 32 + k];
        __syncwarp();
        const int col = tn * GN + h * kEpiCols + c * 32 + lane;
        if (C64 && col < N) {
          // fp64 destination: C64 += alpha (P Q^T), the fp32 result added in fp64
          double* Cd = C64 + b * strideC;
#pragma unroll
          for (int r0 = 0; r0 < 32; r0 += 16) {
            double old[16];
#pragma unroll
            for (int rr = 0; rr < 16; ++rr)
              old[rr] = (row0 + r0 + rr < M) ? Cd[(int64_t)(row0 + r0 + rr) * ldc + col] : 0.0;
#pragma unroll
            for (int rr = 0; rr < 16; ++rr)
              if (row0 + r0 + rr < M)
                Cd[(int64_t)(row0 + r0 + rr) * ldc + col] =
                    old[rr] + (double)(alpha * wb[(r0 + rr) * kEpiPitch + lane]);
          }
        } else if (col < N) {
#pragma unroll
          for (int r0 = 0; r0 < 32; r0 += 16) {
            float old[16];
            if (beta != 0.f) {
#pragma unroll
              for (int rr = 0; rr < 16; ++rr)
                old[rr] = (row0 + r0 + rr < M) ? Cb[(int64_t)(row0 + r0 + rr) * ldc + col] : 0.f;
            }
#pragma unroll
            for (int rr = 0; rr < 16; ++rr) {
              if (row0 + r0 + rr < M) {
                float x = alpha * wb[(r0 + rr) * kEpiPitch + lane];
                if (beta != 0.f) x = fmaf(beta, old[rr], x);
                Cb[(int64_t)(row0 + r0 + rr) * ldc + col] = x;
              }
            }
          }
        }
        __syncwarp();
        if (C2) {
          const int i = row0 + lane;
#pragma unroll
          for (int k = 0; k < 32; ++k) {
            const int j = tn * GN + h * kEpiCols + c * 32 + k;
            if (i < M && j < N) C2[b * strideC2 + (int64_t)j * ldc2 + i] = alpha * sum[c * 32 + k];
          }
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

bool encode_tmap_3d(CUtensorMap* map, const float* base, int64_t cols, int64_t rows,
                    int64_t ld, int64_t batch, int64_t stride) {
  const uint64_t dims[3] = {(uint64_t)cols, (uint64_t)rows, (uint64_t)(batch < 1 ? 1 : batch)};
  const uint64_t strides[2] = {(uint64_t)ld * 4, (uint64_t)(batch > 1 ? stride : rows * ld) * 4};
  const uint32_t box[3] = {(uint32_t)GK, (uint32_t)GM, 1u};
  return encode_tmap_nd(map, base, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, dims, strides, box,
                        CU_TENSOR_MAP_SWIZZLE_128B);
}

}  // namespace

namespace {

nvfp4_status launch_gemm(int M, int N, int K, float alpha, const float* P, const float* Pl,
                         int64_t ldp, int64_t strideP, const float* Q, const float* Ql,
                         int64_t ldq, int64_t strideQ, float beta, float* C, int64_t ldc,
                         int64_t strideC, float* C2, int64_t ldc2, int64_t strideC2, int batch,
                         int lower, int* status, cudaStream_t st, double* C64) {
  if (M <= 0 || N <= 0 || batch <= 0) return NVFP4_OK;
  if (C2 && beta != 0.f) return NVFP4_ERR_INVALID_ARG;   // the transposed copy is alpha P Q^T
  if (C64 && (C2 || beta != 0.f)) return NVFP4_ERR_INVALID_ARG;
  const int presplit = Pl != nullptr;
  if (presplit != (Ql != nullptr)) return NVFP4_ERR_INVALID_ARG;
  if (((ldp | ldq | strideP | strideQ) & 3) != 0 ||
      ((reinterpret_cast<uintptr_t>(P) | reinterpret_cast<uintptr_t>(Q) |
        reinterpret_cast<uintptr_t>(Pl) | reinterpret_cast<uintptr_t>(Ql)) & 15) != 0)
    return NVFP4_ERR_INVALID_ARG;   // TMA: 16-byte aligned rows
  CUtensorMap mp, mq, mpl, mql;
  if (!encode_tmap_3d(&mp, P, K, M, ldp, batch, strideP) ||
      !encode_tmap_3d(&mq, Q, K, N, ldq, batch, strideQ))
    return NVFP4_ERR_CUDA;
  if (presplit) {
    if (!encode_tmap_3d(&mpl, Pl, K, M, ldp, batch, strideP) ||
        !encode_tmap_3d(&mql, Ql, K, N, ldq, batch, strideQ))
      return NVFP4_ERR_CUDA;
  } else {
    mpl = mp;   // not read
    mql = mq;
  }
  TileSpace ts{(M + GM - 1) / GM, (N + GN - 1) / GN, batch, lower};
  const int64_t per = lower ? (int64_t)ts.mt * (ts.mt + 1) / 2 : (int64_t)ts.mt * ts.nt;
  if (per * batch > (1ll << 30) || (lower && M != N)) return NVFP4_ERR_INVALID_ARG;
  const int n_tiles = (int)(per * batch);
  const int sms = num_sms();
  NVFP4_CUDA_TRY(cudaFuncSetAttribute(gemm_nt_tc_kernel,
                                      cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem));
  gemm_nt_tc_kernel<<<n_tiles < sms ? n_tiles : sms, kThreads, kSmem, st>>>(
      mp, mq, mpl, mql, presplit, C, ldc, strideC, C2, ldc2, strideC2, M, N, K, alpha, beta, ts,
      status, C64);
  NVFP4_LAUNCH_CHECK();
  count_launches(1);
  return NVFP4_OK;
}

}  // namespace

nvfp4_status gemm_nt_tc(int M, int N, int K, float alpha, const float* P, int64_t ldp,
                        int64_t strideP, const float* Q, int64_t ldq, int64_t strideQ,
                        float beta, float* C, int64_t ldc, int64_t strideC, float* C2,
                        int64_t ldc2, int64_t strideC2, int batch, int lower, int* status,
                        cudaStream_t st, double* C64) {
  return launch_gemm(M, N, K, alpha, P, nullptr, ldp, strideP, Q, nullptr, ldq, strideQ, beta, C,
                     ldc, strideC, C2, ldc2, strideC2, batch, lower, status, st, C64);
}

nvfp4_status gemm_nt_tc_split(int M, int N, int K, float alpha, const float* Ph,
                              const float* Pl, int64_t ldp, int64_t strideP, const float* Qh,
                              const float* Ql, int64_t ldq, int64_t strideQ, float beta,
                              float* C, int64_t ldc, int64_t strideC, float* C2, int64_t ldc2,
                              int64_t strideC2, int batch, int lower, int* status,
                              cudaStream_t st, double* C64) {
  if (!Pl || !Ql) return NVFP4_ERR_INVALID_ARG;
  return launch_gemm(M, N, K, alpha, Ph, Pl, ldp, strideP, Qh, Ql, ldq, strideQ, beta, C, ldc,
                     strideC, C2, ldc2, strideC2, batch, lower, status, st, C64);
}

}  // namespace nvfp4
